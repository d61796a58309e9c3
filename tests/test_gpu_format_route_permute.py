"""GPU parity of the int4 format kernels, routing, permutation and combine.

All of it is integer, byte or index work (bit-exact) except the routing
weights (fp32 exp and division, compared within a few ulp).
"""
import numpy as np
import pytest
import torch

import oracle
import synth
import quantized_moe_route_b200 as moe
from moe_testlib import u16, to_u16

pytestmark = pytest.mark.gpu


# ------------------------------------------------------------------ int4 format
@pytest.mark.parametrize("N,K,seed", [(128, 128, 0), (1024, 2048, 1), (2048, 512, 2), (32, 64, 3)])
def test_quantize_matches_oracle_bit_exact(N, K, seed):
    w = synth.expert_weights(seed, 0, 0, 0, N, K)
    w[0, :64] = 0.125          # a constant group
    w[1, 64:128] = np.float32(-3.0) if K >= 128 else w[1, 64:128]
    codes, s, m = oracle.quantize_w4(w)
    wd = torch.from_numpy(w).cuda()
    gc = torch.empty((N, K), dtype=torch.uint8, device="cuda")
    gs = torch.empty((N, K // 64), dtype=torch.int16, device="cuda")
    gm = torch.empty((N, K // 64), dtype=torch.int16, device="cuda")
    moe.moe_quantize_w4(wd, gc, gs, gm)
    assert np.array_equal(gc.cpu().numpy(), codes)
    assert np.array_equal(to_u16(gs), s)
    assert np.array_equal(to_u16(gm), m)


@pytest.mark.parametrize("kind", [moe.MOE_W4_PLAIN, moe.MOE_W4_GATE_UP])
@pytest.mark.parametrize("pattern", ["random", "zeros", "fifteen", "alternate"])
def test_pack_unpack_round_trip_and_dequant_bit_exact(kind, pattern):
    N, K = 128, 256
    rng = np.random.default_rng(5)
    codes = {"random": rng.integers(0, 16, (N, K)), "zeros": np.zeros((N, K)),
             "fifteen": np.full((N, K), 15), "alternate": np.tile([0, 15], (N, K // 2))}[pattern].astype(np.uint8)
    s = rng.integers(0, 0x7BFF, (N, K // 64)).astype(np.uint16)
    m = (rng.integers(0, 0x7BFF, (N, K // 64)) | (rng.integers(0, 2, (N, K // 64)) << 15)).astype(np.uint16)
    s[0, 0], m[0, 0] = 0x0001, 0x8001  # subnormal scale and min
    packed = torch.empty(moe.moe_w4_packed_bytes(N, K), dtype=torch.uint8, device="cuda")
    moe.moe_pack_w4(torch.from_numpy(codes).cuda(), u16(s), u16(m), kind, packed)
    c2 = torch.empty((N, K), dtype=torch.uint8, device="cuda")
    s2 = torch.empty((N, K // 64), dtype=torch.int16, device="cuda")
    m2 = torch.empty((N, K // 64), dtype=torch.int16, device="cuda")
    moe.moe_unpack_w4(packed, N, K, kind, c2, s2, m2)
    assert np.array_equal(c2.cpu().numpy(), codes)
    assert np.array_equal(to_u16(s2), s) and np.array_equal(to_u16(m2), m)
    deq = torch.empty((N, K), dtype=torch.float32, device="cuda")
    moe.moe_dequant_w4(packed, N, K, kind, deq)
    want = oracle.dequant_w4(codes, s, m)
    got = deq.cpu().numpy()
    fin = np.isfinite(want)
    assert np.array_equal(got[fin].view(np.uint32), want[fin].view(np.uint32))


def test_packed_size_and_gate_up_strip_interleave():
    assert moe.moe_w4_packed_bytes(1024, 2048) == 1024 * 2048 * 9 // 16
    assert moe.moe_w4_packed_bytes(2048, 512) + moe.moe_w4_packed_bytes(1024, 2048) == 1769472
    # gate strip i and up strip i sit next to each other: the first 576 bytes
    # of strip 1 hold the up rows [F, F + 16)
    N, K = 64, 64
    codes = np.zeros((N, K), np.uint8)
    codes[N // 2:] = 7
    ones = np.full((N, 1), 0x3C00, np.uint16)
    packed = torch.empty(moe.moe_w4_packed_bytes(N, K), dtype=torch.uint8, device="cuda")
    moe.moe_pack_w4(torch.from_numpy(codes).cuda(), u16(ones), u16(np.zeros((N, 1), np.uint16)),
                    moe.MOE_W4_GATE_UP, packed)
    p = packed.cpu().numpy()
    assert p[:512].max() == 0 and p[576:576 + 512].min() == 0x77


# ------------------------------------------------------------------ routing
def _route_gpu(logits, k):
    T, E = logits.shape
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, k), dtype=torch.float32, device="cuda")
    moe.moe_route(torch.from_numpy(np.ascontiguousarray(logits)).cuda(), k, idx, w)
    return idx.cpu().numpy(), w.cpu().numpy()


@pytest.mark.parametrize("T,E,k,variant", [
    (4, 8, 2, "plain"), (1, 256, 8, "plain"), (16, 256, 8, "plain"), (2048, 256, 8, "zipf"),
    (64, 256, 8, "ties"), (33, 1024, 32, "plain"), (5, 256, 1, "plain"), (3, 32, 32, "plain"),
    (7, 100, 5, "ties")])
def test_route_matches_oracle(T, E, k, variant):
    l = synth.router_logits(17, T, T, E, bf16_rounded=(variant == "ties"))
    if variant == "ties":
        l = (np.round(l * 4) / 4).astype(np.float32)
    if variant == "zipf":
        l = (l + synth.zipf_bias(3, E)[None, :]).astype(np.float32)
    idx, w = _route_gpu(l, k)
    oidx, ow = oracle.route(l, k)
    assert np.array_equal(idx, oidx)
    np.testing.assert_allclose(w, ow, rtol=1e-6, atol=1e-7)
    np.testing.assert_allclose(w.sum(1), 1.0, rtol=4e-6)


def test_route_all_equal_and_empty():
    idx, w = _route_gpu(np.zeros((3, 16), np.float32), 4)
    assert idx.tolist() == [[0, 1, 2, 3]] * 3 and np.allclose(w, 0.25)
    idx = torch.empty((0, 8), dtype=torch.int32, device="cuda")
    moe.moe_route(torch.empty((0, 256), device="cuda"), 8, idx, torch.empty((0, 8), device="cuda"))


# ------------------------------------------------------------------ permutation
def _idx_for(T, k, E, mode, seed):
    if T == 0:
        return np.zeros((0, k), np.int32)
    if mode == "one_expert":  # k == 1: every row to the same expert
        return np.full((T, k), 5, np.int32)
    l = synth.router_logits(seed, 0, T, E)
    if mode == "zipf":
        l = l + synth.zipf_bias(seed, E)[None, :]
    return oracle.route(l.astype(np.float32), k)[0]


@pytest.mark.parametrize("T,k,E,mode", [
    (4, 2, 8, "plain"), (1, 8, 256, "plain"), (3, 8, 256, "plain"), (17, 8, 256, "plain"),
    (2048, 8, 256, "zipf"), (512, 8, 256, "zipf"), (100, 1, 256, "one_expert"), (0, 8, 256, "plain"),
    (33, 2, 8, "plain"),
    # the scan splits each expert's chunks among 8 threads here, and needs two passes over E here
    (1024, 4, 64, "zipf"), (256, 8, 2048, "plain")])
def test_permute_matches_oracle_bit_exact(T, k, E, mode):
    H = 128
    idx = _idx_for(T, k, E, mode, 3)
    counts, offsets, sorted_rows, inv = oracle.permute(idx, E)
    x = synth.activations_bf16(9, 0, max(T, 1), H)[:T]
    d = dict(counts=torch.empty(E, dtype=torch.int32, device="cuda"),
             offsets=torch.empty(E + 1, dtype=torch.int32, device="cuda"),
             sorted_rows=torch.empty(T * k, dtype=torch.int32, device="cuda"),
             inv=torch.empty(T * k, dtype=torch.int32, device="cuda"))
    ws = torch.empty(max(1, moe.moe_permute_workspace_bytes(T, k, E)), dtype=torch.uint8, device="cuda")
    xg = u16(x) if T else torch.empty((0, H), dtype=torch.int16, device="cuda")
    x_perm = torch.empty((T * k, H), dtype=torch.int16, device="cuda")
    moe.moe_permute(torch.from_numpy(idx).cuda(), E, d["counts"], d["offsets"], d["sorted_rows"],
                    d["inv"], ws, x=xg, x_perm=x_perm)
    assert np.array_equal(d["counts"].cpu().numpy(), counts)
    assert np.array_equal(d["offsets"].cpu().numpy(), offsets)
    if T:
        assert np.array_equal(d["sorted_rows"].cpu().numpy(), sorted_rows)
        assert np.array_equal(d["inv"].cpu().numpy(), inv)
        assert np.array_equal(to_u16(x_perm), x[sorted_rows // k])


# ------------------------------------------------------------------ combine
@pytest.mark.parametrize("T,k,H,dtype,use_inv", [(4, 2, 128, "f32", False), (16, 8, 2048, "f32", False),
                                                 (2048, 8, 2048, "bf16", True), (3, 8, 64, "bf16", True)])
def test_combine_matches_oracle_bit_exact(T, k, H, dtype, use_inv):
    rows = synth.normal_f32(4, 2, T, T * k * H, 0.5).reshape(T * k, H)
    if dtype == "bf16":
        rows = synth.bf16_bits_to_f32(synth.f32_to_bf16_bits(rows)).reshape(T * k, H)
    l = synth.router_logits(4, 1, T, 64)
    idx, w = oracle.route(l, k)
    inv = np.random.default_rng(T).permutation(T * k).astype(np.int32) if use_inv else None
    stored = rows if inv is None else np.empty_like(rows)
    if inv is not None:
        stored[inv] = rows  # Y[inv[r]] = row r
    if dtype == "f32":
        Y = torch.from_numpy(np.ascontiguousarray(stored)).cuda()
    else:
        Y = u16(synth.f32_to_bf16_bits(stored).reshape(T * k, H))
    y = torch.empty((T, H), dtype=torch.int16, device="cuda")
    moe.moe_unpermute_combine(Y, torch.from_numpy(w).cuda(), y,
                              inv=None if inv is None else torch.from_numpy(inv).cuda())
    assert np.array_equal(to_u16(y), oracle.combine(rows, w))


# ------------------------------------------------------------------ argument errors (no launch)
def test_argument_errors_return_status():
    L = moe.lib()
    assert L.moe_route(None, 4, 8, 9, None, None, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_route(None, 4, 2048, 8, None, None, None) == moe.MOE_ERR_UNSUPPORTED_SHAPE
    assert L.moe_pack_w4(None, None, None, 100, 64, 0, None, 0, None) == moe.MOE_ERR_UNSUPPORTED_SHAPE
    assert L.moe_unpermute_combine(None, 0, None, None, 2, 2, 12, None, None) == moe.MOE_ERR_UNSUPPORTED_SHAPE
    buf = torch.empty(16, dtype=torch.uint8, device="cuda")
    assert L.moe_pack_w4(buf.data_ptr(), buf.data_ptr(), buf.data_ptr(), 16, 64, 0, buf.data_ptr(), 16,
                         None) == moe.MOE_ERR_WORKSPACE
    assert moe.moe_device_error() == 0
