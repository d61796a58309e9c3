"""GPU parity of the NVFP4 prefill path: route -> permute -> per-row NVFP4
quantisation of the grouped rows -> block-scaled tcgen05 grouped FFN ->
combine, against the CPU oracle; plus stage-wise checks of h."""
import numpy as np
import pytest
import torch

import oracle
import synth
import quantized_moe_route_b200 as moe
from moe_testlib import NvLayer, ffn_close, u16, to_u16

pytestmark = pytest.mark.gpu


def _ws_sections(rows, F):
    up = lambda v: (v + 255) // 256 * 256  # noqa: E731
    h = 0
    hc = up(h + rows * F * 4)
    hs = up(hc + rows * F // 2)
    hg = up(hs + rows * F // 16)
    return h, hc, hs, hg


def _prefill(layer, x, logits, k):
    T, H = x.shape
    E, F = layer.E, layer.F
    R = T * k
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, k), dtype=torch.float32, device="cuda")
    moe.moe_route(torch.from_numpy(np.ascontiguousarray(logits)).cuda(), k, idx, w)
    counts = torch.empty(E, dtype=torch.int32, device="cuda")
    offsets = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    sorted_rows = torch.empty(R, dtype=torch.int32, device="cuda")
    inv = torch.empty(R, dtype=torch.int32, device="cuda")
    pws = torch.empty(moe.moe_permute_workspace_bytes(T, k, E), dtype=torch.uint8, device="cuda")
    moe.moe_permute(idx, E, counts, offsets, sorted_rows, inv, pws)
    xc = torch.empty((R, H // 2), dtype=torch.uint8, device="cuda")
    xs = torch.empty((R, H // 16), dtype=torch.uint8, device="cuda")
    xg = torch.empty(R, dtype=torch.float32, device="cuda")
    moe.moe_quantize_nvfp4_rows(u16(x), xc, xs, xg, src_rows=sorted_rows, src_div=k, rows=R)
    y_perm = torch.full((R, H), -1, dtype=torch.int16, device="cuda")
    ws = torch.zeros(moe.moe_prefill_nvfp4_workspace_bytes(R, F), dtype=torch.uint8, device="cuda")
    moe.moe_ffn_grouped_prefill_nvfp4(layer.desc, xc, xs, xg, offsets, y_perm, ws)
    y = torch.empty((T, H), dtype=torch.int16, device="cuda")
    moe.moe_unpermute_combine(y_perm, w, y, inv=inv)
    torch.cuda.synchronize()
    assert moe.moe_device_error() == 0
    out = dict(idx=idx.cpu().numpy(), inv=inv.cpu().numpy(), sorted_rows=sorted_rows.cpu().numpy(),
               y_perm=to_u16(y_perm), y=to_u16(y), offsets=offsets.cpu().numpy())
    wsn = ws.cpu().numpy()
    h0, hc, hs, hg = _ws_sections(R, F)
    out["h"] = wsn[h0:h0 + R * F * 4].view(np.float32).reshape(R, F)
    out["h_codes"] = wsn[hc:hc + R * F // 2].reshape(R, F // 2)
    out["h_sf"] = wsn[hs:hs + R * F // 16].reshape(R, F // 16)
    out["h_G"] = wsn[hg:hg + R * 4].view(np.float32)
    return out


def _check(seed, E, H, F, T, k, bias=None, logits=None, stagewise_rows=16):
    x = synth.activations_bf16(seed, 0, T, H)
    if logits is None:
        logits = synth.router_logits(seed, 0, T, E)
        if bias is not None:
            logits = (logits + bias[None, :]).astype(np.float32)
    oidx, _ = oracle.route(logits, k)
    layer = NvLayer(seed, 0, E, H, F, oidx.ravel())
    g = _prefill(layer, x, logits, k)
    assert np.array_equal(g["idx"], oidx)
    _, _, oY, oy = layer.oracle_forward(x, logits, k)
    got_rows = synth.bf16_bits_to_f32(g["y_perm"][g["inv"]]).reshape(T, k, H)
    ffn_close(got_rows, oY, "y_perm")
    ffn_close(synth.bf16_bits_to_f32(g["y"]), synth.bf16_bits_to_f32(oy), "y")
    # stage-wise: the GPU's fp32 h against the oracle's h, and the GPU's own
    # quantised h through the oracle's down projection against the GPU's y
    # rows (isolates the down GEMM from h code flips at decision boundaries)
    rng = np.random.default_rng(seed)
    for p in rng.choice(T * k, min(stagewise_rows, T * k), replace=False):
        r = int(g["sorted_rows"][p])
        t, e = r // k, int(oidx[r // k, r % k])
        Yo, (h_o, _, _, _) = oracle.expert_ffn_nvfp4(x[t], *layer.canon[e], stages=True)
        np.testing.assert_allclose(g["h"][p], h_o, rtol=2e-5, atol=2e-5 * np.abs(h_o).max())
        hcodes = np.empty(F, np.uint8)
        hcodes[0::2] = g["h_codes"][p] & 15
        hcodes[1::2] = g["h_codes"][p] >> 4
        Yd = oracle.down_nvfp4(hcodes, g["h_sf"][p], g["h_G"][p], layer.canon[e][1])
        ffn_close(synth.bf16_bits_to_f32(g["y_perm"][p]), Yd, f"down of row {p}")
    return g


def test_nvfp4_prefill_small():
    _check(10, 8, 256, 256, 64, 2)


def test_nvfp4_prefill_skewed_multi_chunk_and_empty_experts():
    bias = synth.zipf_bias(11, 16)
    bias[[2, 9]] = -100.0  # never selected
    g = _check(11, 16, 512, 256, 200, 4, bias=bias)
    counts = np.diff(g["offsets"])
    assert counts.max() > 128 and (counts == 0).any()  # several 128-row chunks, empty experts


def test_nvfp4_prefill_ragged_rows():
    _check(12, 32, 256, 512, 7, 3)


def test_nvfp4_prefill_tile_boundaries():
    """Experts whose row counts sit on either side of the 80-row gate/up and
    128-row down tile sizes (and of the 32-row activation boxes), in one batch."""
    counts = [0, 1, 31, 33, 79, 80, 81, 127, 128, 129, 159, 160, 161, 200, 3]
    E, k = len(counts), 1
    owner = np.repeat(np.arange(E), counts)
    owner = owner[np.random.default_rng(6).permutation(owner.size)]
    logits = synth.router_logits(6, 0, owner.size, E)
    logits[np.arange(owner.size), owner] += 100.0
    g = _check(6, E, 256, 256, owner.size, k, logits=logits.astype(np.float32))
    assert np.array_equal(np.diff(g["offsets"]), counts)


def test_nvfp4_prefill_one_expert_all_rows():
    T, E, k = 300, 8, 1
    logits = synth.router_logits(13, 0, T, E)
    logits[:, 6] += 100.0
    _check(13, E, 256, 256, T, k, logits=logits.astype(np.float32))


def test_nvfp4_prefill_512_tokens_full_shape_sampled():
    """512 tokens, 256 experts (Zipf-skewed), top-8, hidden 2048, width 512;
    weights generated, quantised and packed on the GPU; routing exact, 24
    sampled tokens against the oracle."""
    E, H, F, T, k, seed = 256, 2048, 512, 512, 8, 14
    x = synth.activations_bf16(seed, 0, T, H)
    logits = (synth.router_logits(seed, 0, T, E) + synth.zipf_bias(seed, E)[None, :]).astype(np.float32)
    oidx, ow = oracle.route(logits, k)
    gu_b, d_b = moe.moe_nvfp4_packed_bytes(2 * F, H), moe.moe_nvfp4_packed_bytes(H, F)
    gu = torch.empty(E * gu_b, dtype=torch.uint8, device="cuda")
    dn = torch.empty(E * d_b, dtype=torch.uint8, device="cuda")
    g_gu = torch.empty(E, dtype=torch.float32, device="cuda")
    g_d = torch.empty(E, dtype=torch.float32, device="cuda")
    for proj, buf, nb, (N, K), kind, gl in ((0, gu, gu_b, (2 * F, H), moe.MOE_W4_GATE_UP, g_gu),
                                            (1, dn, d_b, (H, F), moe.MOE_W4_PLAIN, g_d)):
        wbuf = torch.empty((16, N, K), device="cuda")
        c = torch.empty((N, K), dtype=torch.uint8, device="cuda")
        s = torch.empty((N, K // 16), dtype=torch.uint8, device="cuda")
        for e0 in range(0, E, 16):
            synth.cuda_expert_weights(wbuf, seed, 0, e0, proj)
            for i in range(16):
                moe.moe_nvfp4_global(wbuf[i], gl[e0 + i:e0 + i + 1])
                moe.moe_quantize_nvfp4(wbuf[i], gl[e0 + i:e0 + i + 1], c, s)
                moe.moe_pack_nvfp4(c, s, kind, buf[(e0 + i) * nb:(e0 + i + 1) * nb])

    class L:
        pass
    layer = L()
    layer.E, layer.F = E, F
    layer.desc = moe.make_nvfp4_layer(E, H, F, gu, dn, g_gu, g_d)
    g = _prefill(layer, x, logits, k)
    assert np.array_equal(g["idx"], oidx)
    assert np.array_equal(np.diff(g["offsets"]), np.bincount(oidx.ravel(), minlength=E))
    rng = np.random.default_rng(seed)
    toks = rng.choice(T, 24, replace=False)
    need = sorted(set(oidx[toks].ravel().tolist()))
    canon = {}
    for e in need:
        mats = []
        for proj, (N, K) in ((synth.PROJ_GATE_UP, (2 * F, H)), (synth.PROJ_DOWN, (H, F))):
            wv = synth.expert_weights(seed, 0, e, proj, N, K)
            G = oracle.nvfp4_global(wv)
            mats.append((*oracle.nvfp4_quantize(wv, G), G))
        canon[e] = mats
    got_rows, want_rows, got_y, want_y = [], [], [], []
    for t in toks:
        Yt = np.stack([oracle.expert_ffn_nvfp4(x[t], *canon[int(e)]) for e in oidx[t]])
        want_rows.append(Yt)
        got_rows.append(synth.bf16_bits_to_f32(g["y_perm"][g["inv"][t * k:(t + 1) * k]]))
        want_y.append(synth.bf16_bits_to_f32(oracle.combine(Yt, ow[t:t + 1])[0]))
        got_y.append(synth.bf16_bits_to_f32(g["y"][t]))
    ffn_close(np.stack(got_rows), np.stack(want_rows), "sampled y_perm rows")
    ffn_close(np.stack(got_y), np.stack(want_y), "sampled y")


def test_nvfp4_prefill_argument_errors():
    import ctypes
    L_ = moe.lib()
    d = moe.moe_nvfp4_layer(8, 256, 128, 16, 16, 16, 16)  # F % 256 != 0
    assert L_.moe_ffn_grouped_prefill_nvfp4(ctypes.byref(d), 16, 16, 16, 16, 4, 16, 256, 1 << 20, None) == \
        moe.MOE_ERR_UNSUPPORTED_SHAPE
