"""GPU parity of the prefill path: route -> permute -> grouped tcgen05 FFN ->
combine, against the CPU oracle."""
import numpy as np
import pytest
import torch

import oracle
import synth
import quantized_moe_route_b200 as moe
from moe_testlib import Layer, ffn_close, u16, to_u16

pytestmark = pytest.mark.gpu


def _prefill(layer, x, logits, k):
    """Device pipeline; returns idx, inv, y_perm (bf16 bits), y (bf16 bits),
    offsets, sorted_rows and the bf16 h rows the gate/up launch left at the
    start of the workspace (permuted row order)."""
    T, H = x.shape
    E = logits.shape[1]
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, k), dtype=torch.float32, device="cuda")
    moe.moe_route(torch.from_numpy(np.ascontiguousarray(logits)).cuda(), k, idx, w)
    counts = torch.empty(E, dtype=torch.int32, device="cuda")
    offsets = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    sorted_rows = torch.empty(T * k, dtype=torch.int32, device="cuda")
    inv = torch.empty(T * k, dtype=torch.int32, device="cuda")
    ws = torch.empty(moe.moe_permute_workspace_bytes(T, k, E), dtype=torch.uint8, device="cuda")
    x_perm = torch.empty((T * k, H), dtype=torch.int16, device="cuda")
    moe.moe_permute(idx, E, counts, offsets, sorted_rows, inv, ws, x=u16(x), x_perm=x_perm)
    y_perm = torch.full((T * k, H), -1, dtype=torch.int16, device="cuda")
    pws = torch.empty(moe.moe_prefill_workspace_bytes(T * k, layer.F), dtype=torch.uint8, device="cuda")
    moe.moe_ffn_grouped_prefill(layer.desc, x_perm, offsets, y_perm, pws)
    y = torch.empty((T, H), dtype=torch.int16, device="cuda")
    moe.moe_unpermute_combine(y_perm, w, y, inv=inv)
    torch.cuda.synchronize()
    assert moe.moe_device_error() == 0
    h = pws[:T * k * layer.F * 2].view(torch.int16).view(T * k, layer.F)
    return (idx.cpu().numpy(), inv.cpu().numpy(), to_u16(y_perm), to_u16(y), offsets.cpu().numpy(),
            sorted_rows.cpu().numpy(), to_u16(h))


def _check(seed, E, H, F, T, k, bias=None, logits=None):
    x = synth.activations_bf16(seed, 0, T, H)
    if logits is None:
        logits = synth.router_logits(seed, 0, T, E)
        if bias is not None:
            logits = (logits + bias[None, :]).astype(np.float32)
    oidx, _ = oracle.route(logits, k)
    layer = Layer(seed, 0, E, H, F, oidx.ravel())
    idx, inv, y_perm, y, offsets, sorted_rows, h = _prefill(layer, x, logits, k)
    assert np.array_equal(idx, oidx)
    _, _, oy_rows, oy = oracle.moe_forward_w4(x, logits, k, layer.canon)
    got_rows = synth.bf16_bits_to_f32(y_perm[inv])  # back to row order r = t*k + j
    ffn_close(got_rows, oy_rows, "y_perm")
    ffn_close(synth.bf16_bits_to_f32(y), synth.bf16_bits_to_f32(oy), "y")
    # stage-wise: the gate/up launch's h of sampled rows against the oracle's h
    rng = np.random.default_rng(seed)
    ps = rng.choice(T * k, min(16, T * k), replace=False)
    got_h, want_h = [], []
    for p in ps:
        r = int(sorted_rows[p])
        e = int(oidx[r // k, r % k])
        _, h_o = oracle.expert_ffn_w4(x[r // k], *layer.canon[e], return_h=True)
        got_h.append(synth.bf16_bits_to_f32(h[p]))
        want_h.append(h_o)
    ffn_close(np.array(got_h), np.array(want_h), "h (gate/up stage)")
    return offsets


def test_prefill_small():
    _check(0, 8, 256, 128, 64, 2)


def test_prefill_skewed_multi_chunk_and_empty_experts():
    bias = synth.zipf_bias(1, 16)
    bias[[3, 7, 11]] = -100.0  # never selected
    offsets = _check(1, 16, 512, 256, 300, 4, bias=bias)
    counts = np.diff(offsets)
    assert counts.max() > 128 and (counts == 0).any()  # several chunks, empty experts


def test_prefill_all_rows_one_expert():
    T, E, k = 200, 8, 1
    logits = synth.router_logits(2, 0, T, E)
    logits[:, 5] += 100.0
    _check(2, E, 256, 128, T, k, logits=logits.astype(np.float32))


def test_prefill_ragged_single_rows():
    _check(3, 32, 256, 128, 7, 3)


def test_prefill_chunk_boundaries():
    """Experts whose row counts sit on either side of the 128-row (one or two
    MMAs per k step) and 256-row (chunk) boundaries, in one batch: the tile
    schedule numbers the chunks of more than 128 rows first."""
    counts = [0, 1, 127, 128, 129, 255, 256, 257, 384, 385, 513, 16]
    E, k = len(counts), 1
    owner = np.repeat(np.arange(E), counts)
    owner = owner[np.random.default_rng(5).permutation(owner.size)]  # rows of an expert interleaved
    logits = synth.router_logits(5, 0, owner.size, E)
    logits[np.arange(owner.size), owner] += 100.0
    offsets = _check(5, E, 256, 128, owner.size, k, logits=logits.astype(np.float32))
    assert np.array_equal(np.diff(offsets), counts)


def test_prefill_full_shape_sampled_tokens():
    """2048 tokens, 256 experts (Zipf-skewed), top-8, hidden 2048, width 512:
    every routing/permutation output exact, 64 sampled tokens against the oracle."""
    E, H, F, T, k, seed = 256, 2048, 512, 2048, 8, 4
    x = synth.activations_bf16(seed, 0, T, H)
    logits = (synth.router_logits(seed, 0, T, E) + synth.zipf_bias(seed, E)[None, :]).astype(np.float32)
    oidx, ow = oracle.route(logits, k)
    # device weights of all experts: generated on the GPU by the seeded
    # generator's CUDA twin, quantised and packed by the library
    gu_b, d_b = moe.moe_w4_packed_bytes(2 * F, H), moe.moe_w4_packed_bytes(H, F)
    gu = torch.empty(E * gu_b, dtype=torch.uint8, device="cuda")
    dn = torch.empty(E * d_b, dtype=torch.uint8, device="cuda")
    for proj, buf, nb, (N, K), kind in ((0, gu, gu_b, (2 * F, H), moe.MOE_W4_GATE_UP),
                                         (1, dn, d_b, (H, F), moe.MOE_W4_PLAIN)):
        w = torch.empty((16, N, K), device="cuda")
        c = torch.empty((16 * N, K), dtype=torch.uint8, device="cuda")
        s = torch.empty((16 * N, K // 64), dtype=torch.int16, device="cuda")
        m = torch.empty_like(s)
        for e0 in range(0, E, 16):
            synth.cuda_expert_weights(w, seed, 0, e0, proj)
            moe.moe_quantize_w4(w.view(16 * N, K), c, s, m)
            for i in range(16):
                moe.moe_pack_w4(c[i * N:(i + 1) * N], s[i * N:(i + 1) * N], m[i * N:(i + 1) * N], kind,
                                buf[(e0 + i) * nb:(e0 + i + 1) * nb])

    class L:
        pass
    layer = L()
    layer.F = F
    layer.desc = moe.make_layer(E, H, F, gu, dn)
    idx, inv, y_perm, y, offsets, sorted_rows, h = _prefill(layer, x, logits, k)
    assert np.array_equal(idx, oidx)
    counts = np.bincount(oidx.ravel(), minlength=E)
    assert np.array_equal(np.diff(offsets), counts)
    rng = np.random.default_rng(seed)
    toks = rng.choice(T, 64, replace=False)
    need = sorted(set(oidx[toks].ravel().tolist()))
    experts = {e: (oracle.quantize_w4(synth.expert_weights(seed, 0, e, 0, 2 * F, H)),
                   oracle.quantize_w4(synth.expert_weights(seed, 0, e, 1, H, F))) for e in need}
    got_rows, want_rows, got_y, want_y, got_h, want_h = [], [], [], [], [], []
    for t in toks:
        Yh = [oracle.expert_ffn_w4(x[t], *experts[int(e)], return_h=True) for e in oidx[t]]
        Yt = [yh[0] for yh in Yh]
        want_h.append(np.stack([yh[1] for yh in Yh]))
        got_h.append(synth.bf16_bits_to_f32(h[inv[t * k:(t + 1) * k]]))
        want_rows.append(np.stack(Yt))
        got_rows.append(synth.bf16_bits_to_f32(y_perm[inv[t * k:(t + 1) * k]]))
        want_y.append(synth.bf16_bits_to_f32(oracle.combine(np.stack(Yt), ow[t:t + 1])[0]))
        got_y.append(synth.bf16_bits_to_f32(y[t]))
    ffn_close(np.stack(got_h), np.stack(want_h), "sampled h rows (gate/up stage)")
    ffn_close(np.stack(got_rows), np.stack(want_rows), "sampled y_perm rows")
    ffn_close(np.stack(got_y), np.stack(want_y), "sampled y")


def test_prefill_argument_errors():
    L_ = moe.lib()
    d = moe.moe_w4_layer(8, 128, 64, 16, 16)  # F % 128 != 0
    import ctypes
    assert L_.moe_ffn_grouped_prefill(ctypes.byref(d), 16, 16, 4, 16, 16, 1 << 20, None) == \
        moe.MOE_ERR_UNSUPPORTED_SHAPE
