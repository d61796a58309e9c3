"""GPU parity of the NVFP4 format kernels against the CPU oracle: global
scale, matrix quantiser, per-row activation quantiser (all bit-exact: the
same fp32 operations decide every code), and the packed layout round trip."""
import numpy as np
import pytest
import torch

import oracle
import synth
import quantized_moe_route_b200 as moe

pytestmark = pytest.mark.gpu

# E2M1 magnitudes and the midpoints between neighbours (ties to the even code)
E2M1 = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
MIDS = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]


def _global(v):
    G = torch.empty(1, device="cuda")
    moe.moe_nvfp4_global(torch.from_numpy(np.ascontiguousarray(v, np.float32)).cuda(), G)
    return float(G.item())


def test_global_matches_oracle_and_zero_case():
    rng = np.random.default_rng(0)
    for n in (1, 17, 4096, 1 << 20):
        v = (rng.standard_normal(n) * rng.uniform(1e-3, 10)).astype(np.float32)
        assert np.float32(_global(v)) == np.float32(oracle.nvfp4_global(v))
    assert _global(np.zeros(64, np.float32)) == 1.0


def _quantize_gpu(v, G):
    N, K = v.shape
    vd = torch.from_numpy(np.ascontiguousarray(v, np.float32)).cuda()
    Gd = torch.tensor([G], dtype=torch.float32, device="cuda")
    codes = torch.empty((N, K), dtype=torch.uint8, device="cuda")
    sf = torch.empty((N, K // 16), dtype=torch.uint8, device="cuda")
    moe.moe_quantize_nvfp4(vd, Gd, codes, sf)
    return codes.cpu().numpy(), sf.cpu().numpy()


def test_quantize_matrix_bit_exact():
    w = synth.expert_weights(5, 0, 3, synth.PROJ_GATE_UP, 256, 512)
    G = oracle.nvfp4_global(w)
    c, s = _quantize_gpu(w, G)
    oc, os_ = oracle.nvfp4_quantize(w, G)
    assert np.array_equal(s, os_)
    assert np.array_equal(c, oc)


def test_quantize_ties_saturation_signs_and_zero_blocks():
    """Row with amax 2688 (G = 1, denominator 6): a block with amax 6 has
    scale 1, so its values sit exactly on E2M1 points and midpoints."""
    K = 128
    row = np.zeros(K, np.float32)
    row[0] = 2688.0                                   # block 0: scale 448
    blk = np.array(MIDS + [6.0] + [-m for m in MIDS] + [-0.0], np.float32)
    row[16:32] = blk                                  # block 1: ties
    row[32:48] = np.array(E2M1 + [-e for e in E2M1], np.float32)  # exact points
    row[48:64] = 1e-12                                # tiny: scale rounds to 0 -> zero codes
    row[64:80] = np.linspace(-2688, 2688, 16)          # saturating scale
    v = np.stack([row, -row, row * 0.001])
    for r in range(3):
        G = oracle.nvfp4_global(v[r])
        c, s = _quantize_gpu(v[r:r + 1], G)
        oc, os_ = oracle.nvfp4_quantize(v[r:r + 1], G)
        assert np.array_equal(s, os_), r
        assert np.array_equal(c, oc), r
    # the tie block really exercised ties to even: 0.25 -> 0, 0.75 -> 1.0, 2.5 -> 2, 5 -> 4
    oc, _ = oracle.nvfp4_quantize(v[:1], 1.0)
    assert [oracle.e2m1_to_f32(np.array([q], np.uint8))[0] for q in oc[0, 16:23]] == [0, 1, 1, 2, 2, 4, 4]


@pytest.mark.parametrize("N,K,kind", [(64, 256, moe.MOE_W4_GATE_UP), (48, 512, moe.MOE_W4_PLAIN),
                                      (1024, 2048, moe.MOE_W4_GATE_UP)])
def test_pack_unpack_round_trip(N, K, kind):
    rng = np.random.default_rng(N + K)
    codes = rng.integers(0, 16, size=(N, K), dtype=np.uint8)
    sf = rng.integers(0, 256, size=(N, K // 16), dtype=np.uint8)
    packed = torch.empty(moe.moe_nvfp4_packed_bytes(N, K), dtype=torch.uint8, device="cuda")
    assert packed.numel() == N * K * 9 // 16
    moe.moe_pack_nvfp4(torch.from_numpy(codes).cuda(), torch.from_numpy(sf).cuda(), kind, packed)
    c2 = torch.empty((N, K), dtype=torch.uint8, device="cuda")
    s2 = torch.empty((N, K // 16), dtype=torch.uint8, device="cuda")
    moe.moe_unpack_nvfp4(packed, N, K, kind, c2, s2)
    assert np.array_equal(c2.cpu().numpy(), codes)
    assert np.array_equal(s2.cpu().numpy(), sf)
    # the documented layout: logical byte b of row r = codes[2b] | codes[2b+1] << 4,
    # its 16-byte piece XOR-permuted by r & 7 inside each 128-byte run
    p = packed.cpu().numpy()
    byte = lambda n: codes[n, 0::2] | (codes[n, 1::2] << 4)  # noqa: E731
    assert np.array_equal(p[:K // 2], byte(0))  # row 0: identity permutation
    r1 = p[K // 2:K].reshape(-1, 8, 16)[:, [1, 0, 3, 2, 5, 4, 7, 6], :].ravel()
    assert np.array_equal(r1, byte(1))
    # scales: [K/64][16 rows][4]
    sc = p[8 * K:9 * K].reshape(K // 64, 16, 4)
    assert np.array_equal(sc.transpose(1, 0, 2).reshape(16, K // 16), sf[:16])
    if kind == moe.MOE_W4_GATE_UP:  # strip 1 is the first up strip (canonical row F)
        F = N // 2
        sb = 9 * K
        assert np.array_equal(p[sb:sb + K // 2], byte(F))
        sc1 = p[sb + 8 * K:sb + 9 * K].reshape(K // 64, 16, 4)
        assert np.array_equal(sc1.transpose(1, 0, 2).reshape(16, K // 16), sf[F:F + 16])


def _oracle_rows(xf):
    """Per-row oracle quantisation: codes (packed two per byte), sf, G."""
    R, K = xf.shape
    codes = np.empty((R, K // 2), np.uint8)
    sf = np.empty((R, K // 16), np.uint8)
    G = np.empty(R, np.float32)
    for r in range(R):
        G[r] = oracle.nvfp4_global(xf[r])
        c, s = oracle.nvfp4_quantize(xf[r:r + 1], G[r])
        codes[r] = c[0, 0::2] | (c[0, 1::2] << 4)
        sf[r] = s[0]
    return codes, sf, G


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_quantize_rows_bit_exact_with_row_map(dtype):
    T, K, k = 37, 2048, 3
    x = synth.activations_bf16(6, 0, T, K)
    x[5] = 0  # all-zero token: G = 1, zero codes
    xf = synth.bf16_bits_to_f32(x)
    rng = np.random.default_rng(6)
    src_rows = rng.permutation(T * k).astype(np.int32)
    R = T * k
    if dtype == "bf16":
        xd = torch.from_numpy(x.view(np.int16)).cuda()
    else:
        xf = (xf * rng.uniform(0.5, 2.0, size=(T, 1))).astype(np.float32)
        xd = torch.from_numpy(xf).cuda()
    codes = torch.empty((R, K // 2), dtype=torch.uint8, device="cuda")
    sf = torch.empty((R, K // 16), dtype=torch.uint8, device="cuda")
    G = torch.empty(R, dtype=torch.float32, device="cuda")
    moe.moe_quantize_nvfp4_rows(xd, codes, sf, G, src_rows=torch.from_numpy(src_rows).cuda(), src_div=k,
                                rows=R)
    oc, os_, oG = _oracle_rows(xf[src_rows // k])
    assert np.array_equal(G.cpu().numpy(), oG)
    assert np.array_equal(sf.cpu().numpy(), os_)
    assert np.array_equal(codes.cpu().numpy(), oc)
