"""GPU parity of the clip-search quantisers and of the symmetric group-128
int4 format run through the int4 kernels.

- moe_quantize_w4_clip / moe_quantize_w4_sym128: codes, scales and mins
  bit-exact with the oracle's quantisers (the clip search takes every
  decision in the same fp32 operations).
- moe_pack_w4_sym128: the packed matrix dequantises (moe_dequant_w4) to
  (q - 8) * s bit for bit.
- Decode (fused layer) and grouped prefill on symmetric group-128 experts
  against the oracle's symmetric group-128 FFN and combine.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
import quantized_moe_route_b200 as moe
from moe_testlib import ffn_close, u16, to_u16

pytestmark = pytest.mark.gpu


def _weights_with_edge_groups(seed, N, K):
    w = synth.expert_weights(seed, 0, 0, synth.PROJ_GATE_UP, N, K).copy()
    w[0, :128] = 0.0                                        # all-zero group
    w[1, :128] = 0.0125                                     # constant group
    w[2, :64] = np.tile(np.arange(16), 4) * np.float32(2.0 ** -8) - np.float32(0.03125)  # exact asym group
    w[3, :128] = synth.expert_weights(seed, 0, 1, 0, 1, 128)[0] * 40  # wide-range group
    # quotients exactly on half-integers at ratio 1.0 (ties to even): asymmetric
    # m = -0.5, s = 0.0625; symmetric amax = 0.46875, s = 2 amax / 15 = 0.0625
    k = np.arange(64) % 15
    w[4, :64] = np.float32(-0.5) + (k + np.float32(0.5)) * np.float32(0.0625)
    w[4, 0], w[4, 63] = np.float32(-0.5), np.float32(0.4375)
    j = np.arange(128) % 8
    w[5, :128] = np.where(np.arange(128) % 2 == 0, 1, -1) * (j + np.float32(0.5)) * np.float32(0.0625)
    w[5, 0] = np.float32(0.46875)
    return w


def _on_device(w, offset):
    """w on the device starting `offset` floats into a buffer (offset 1: not 16-byte aligned)."""
    buf = torch.empty(w.size + 4, dtype=torch.float32, device="cuda")
    d = buf[offset:offset + w.size].view(*w.shape)
    d.copy_(torch.from_numpy(w))
    return d


@pytest.mark.parametrize("offset", [0, 1])
def test_clip_quantiser_bit_exact_with_oracle(offset):
    w = _weights_with_edge_groups(61, 64, 1024)
    c, s, m = oracle.quantize_w4_clip(w)
    dw = _on_device(w, offset)
    gc = torch.empty((64, 1024), dtype=torch.uint8, device="cuda")
    gs = torch.empty((64, 16), dtype=torch.int16, device="cuda")
    gm = torch.empty((64, 16), dtype=torch.int16, device="cuda")
    moe.moe_quantize_w4_clip(dw, gc, gs, gm)
    torch.cuda.synchronize()
    assert np.array_equal(gc.cpu().numpy(), c)
    assert np.array_equal(to_u16(gs), s) and np.array_equal(to_u16(gm), m)


@pytest.mark.parametrize("offset", [0, 1])
def test_sym128_quantiser_bit_exact_with_oracle(offset):
    w = _weights_with_edge_groups(62, 64, 1024)
    c, s = oracle.quantize_sym128(w)
    dw = _on_device(w, offset)
    gc = torch.empty((64, 1024), dtype=torch.uint8, device="cuda")
    gs = torch.empty((64, 8), dtype=torch.int16, device="cuda")
    moe.moe_quantize_w4_sym128(dw, gc, gs)
    torch.cuda.synchronize()
    assert np.array_equal(gc.cpu().numpy(), c)
    assert np.array_equal(to_u16(gs), s)


@pytest.mark.parametrize("kind", [0, 1])
def test_sym128_pack_dequantises_exactly(kind):
    N, K = 64, 512
    w = synth.expert_weights(63, 0, 0, synth.PROJ_DOWN, N, K)
    c, s = oracle.quantize_sym128(w)
    packed = torch.zeros(moe.moe_w4_packed_bytes(N, K), dtype=torch.uint8, device="cuda")
    ws = torch.empty(moe.moe_pack_w4_sym128_workspace_bytes(N, K), dtype=torch.uint8, device="cuda")
    moe.moe_pack_w4_sym128(torch.from_numpy(c).cuda(), u16(s), kind, packed, ws)
    out = torch.empty((N, K), dtype=torch.float32, device="cuda")
    moe.moe_dequant_w4(packed, N, K, kind, out)
    torch.cuda.synchronize()
    got = out.cpu().numpy()
    want = ((c.astype(np.float32) - 8) * np.repeat(s.view(np.float16).astype(np.float32), 128, 1))
    assert np.array_equal(got, want)
    L = oracle.lib()
    for n, k in [(0, 0), (5, 130), (63, 511)]:
        assert got[n, k] == L.orc_dequant_sym128(int(c[n, k]), int(s[n, k // 128]))


class Sym128Layer:
    """A layer whose routed experts are symmetric group-128 int4, packed for
    the int4 kernels (unused experts stay zero)."""

    def __init__(self, seed, E, H, F, experts):
        self.E, self.H, self.F = E, H, F
        self.canon = {}
        gu_b, d_b = moe.moe_w4_packed_bytes(2 * F, H), moe.moe_w4_packed_bytes(H, F)
        self.gu = torch.zeros(E * gu_b, dtype=torch.uint8, device="cuda")
        self.dn = torch.zeros(E * d_b, dtype=torch.uint8, device="cuda")
        ws = torch.empty(moe.moe_pack_w4_sym128_workspace_bytes(H, 2 * max(H, F)), dtype=torch.uint8, device="cuda")
        for e in sorted(set(int(v) for v in experts)):
            gu = oracle.quantize_sym128(synth.expert_weights(seed, 0, e, synth.PROJ_GATE_UP, 2 * F, H))
            d = oracle.quantize_sym128(synth.expert_weights(seed, 0, e, synth.PROJ_DOWN, H, F))
            self.canon[e] = (gu, d)
            moe.moe_pack_w4_sym128(torch.from_numpy(gu[0]).cuda(), u16(gu[1]), moe.MOE_W4_GATE_UP,
                                   self.gu[e * gu_b:(e + 1) * gu_b], ws)
            moe.moe_pack_w4_sym128(torch.from_numpy(d[0]).cuda(), u16(d[1]), moe.MOE_W4_PLAIN,
                                   self.dn[e * d_b:(e + 1) * d_b], ws)
        torch.cuda.synchronize()
        self.desc = moe.make_layer(E, H, F, self.gu, self.dn)

    def oracle_rows(self, x, idx):
        T, k = idx.shape
        return np.stack([oracle.expert_ffn_sym128(x[t], *self.canon[int(idx[t, j])])
                         for t in range(T) for j in range(k)])


def test_fused_decode_with_sym128_experts():
    E, H, F, T, k, seed = 256, 2048, 512, 4, 8, 64
    x = synth.activations_bf16(seed, 0, T, H)
    logits = synth.router_logits(seed, 0, T, E)
    oidx, ow = oracle.route(logits, k)
    layer = Sym128Layer(seed, E, H, F, oidx.ravel())
    y = torch.empty((T, H), dtype=torch.int16, device="cuda")
    ws = torch.zeros(moe.moe_decode_layer_workspace_bytes(T, k, H, F), dtype=torch.uint8, device="cuda")
    moe.moe_decode_layer_w4a16(layer.desc, u16(x), torch.from_numpy(logits).cuda(), k, y, ws)
    torch.cuda.synchronize()
    assert moe.moe_device_error() == 0
    rows = layer.oracle_rows(x, oidx)
    oy = np.stack([oracle.combine(rows[t * k:(t + 1) * k], ow[t:t + 1])[0] for t in range(T)])
    ffn_close(synth.bf16_bits_to_f32(to_u16(y)), synth.bf16_bits_to_f32(oy), "y")


def test_grouped_prefill_with_sym128_experts():
    E, H, F, T, k, seed = 16, 512, 256, 96, 4, 65
    x = synth.activations_bf16(seed, 0, T, H)
    logits = synth.router_logits(seed, 0, T, E)
    oidx, _ = oracle.route(logits, k)
    counts, offsets, sorted_rows, inv = oracle.permute(oidx, E)
    layer = Sym128Layer(seed, E, H, F, oidx.ravel())
    R = T * k
    xp = x[sorted_rows // k]
    y_perm = torch.empty((R, H), dtype=torch.int16, device="cuda")
    ws = torch.empty(moe.moe_prefill_workspace_bytes(R, F), dtype=torch.uint8, device="cuda")
    moe.moe_ffn_grouped_prefill(layer.desc, u16(xp), torch.from_numpy(offsets).cuda(), y_perm, ws)
    torch.cuda.synchronize()
    assert moe.moe_device_error() == 0
    rows = layer.oracle_rows(x, oidx)  # row order r = t*k + j
    ffn_close(synth.bf16_bits_to_f32(to_u16(y_perm))[inv], rows, "y_perm")
