"""Shared helpers of the GPU tests: seeded layers, oracle references, tolerances.

Only synth (inputs) and oracle (expected values) are used on the CPU side;
the GPU side goes through the quantized_moe_route_b200 binding (C ABI).
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
import synth
import quantized_moe_route_b200 as moe

# FFN acceptance bar (fp32 accumulate, bf16 out): relative L2 error and the
# largest absolute error relative to the largest output magnitude.
REL_L2 = 5e-3
MAX_ABS_FRAC = 2e-2


def ffn_close(got, want, what=""):
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    denom = np.linalg.norm(want)
    rel = np.linalg.norm(got - want) / max(denom, 1e-30)
    mx = np.abs(got - want).max() if got.size else 0.0
    scale = np.abs(want).max() if want.size else 0.0
    assert rel <= REL_L2, f"{what}: rel-L2 {rel:.3e} > {REL_L2}"
    assert mx <= MAX_ABS_FRAC * max(scale, 1e-30), f"{what}: max-abs {mx:.3e} > {MAX_ABS_FRAC}*{scale:.3e}"
    return rel, mx


def u16(a: np.ndarray, device="cuda") -> torch.Tensor:
    """uint16 numpy bits -> int16 torch tensor with the same bits."""
    return torch.from_numpy(np.ascontiguousarray(a, np.uint16).view(np.int16)).to(device)


def to_u16(t: torch.Tensor) -> np.ndarray:
    return t.cpu().numpy().view(np.uint16)


class Layer:
    """One MoE layer: canonical oracle weights for the experts that matter and
    the packed device buffers for all E experts (unused experts stay zero)."""

    def __init__(self, seed, layer, E, H, F, experts, weights=None):
        self.E, self.H, self.F = E, H, F
        self.canon = {}
        gu_b = moe.moe_w4_packed_bytes(2 * F, H)
        d_b = moe.moe_w4_packed_bytes(H, F)
        self.gu = torch.zeros(E * gu_b, dtype=torch.uint8, device="cuda")
        self.dn = torch.zeros(E * d_b, dtype=torch.uint8, device="cuda")
        for e in sorted(set(int(v) for v in experts)):
            if weights is not None:
                gu, d = weights[e]
            else:
                gu = oracle.quantize_w4(synth.expert_weights(seed, layer, e, synth.PROJ_GATE_UP, 2 * F, H))
                d = oracle.quantize_w4(synth.expert_weights(seed, layer, e, synth.PROJ_DOWN, H, F))
            self.canon[e] = (gu, d)
            for (codes, s, m), buf, nb, kind in ((gu, self.gu, gu_b, moe.MOE_W4_GATE_UP),
                                                 (d, self.dn, d_b, moe.MOE_W4_PLAIN)):
                moe.moe_pack_w4(torch.from_numpy(codes).cuda(), u16(s), u16(m), kind,
                                buf[e * nb:(e + 1) * nb])
        self.desc = moe.make_layer(E, H, F, self.gu, self.dn)


class NvLayer:
    """One NVFP4 MoE layer: canonical oracle weights (codes, sf, G) for the
    experts that matter, packed device buffers and globals for all E."""

    def __init__(self, seed, layer, E, H, F, experts):
        self.E, self.H, self.F = E, H, F
        self.canon = {}
        gu_b = moe.moe_nvfp4_packed_bytes(2 * F, H)
        d_b = moe.moe_nvfp4_packed_bytes(H, F)
        self.gu = torch.zeros(E * gu_b, dtype=torch.uint8, device="cuda")
        self.dn = torch.zeros(E * d_b, dtype=torch.uint8, device="cuda")
        g_gu = np.ones(E, np.float32)
        g_d = np.ones(E, np.float32)
        for e in sorted(set(int(v) for v in experts)):
            mats = []
            for proj, (N, K) in ((synth.PROJ_GATE_UP, (2 * F, H)), (synth.PROJ_DOWN, (H, F))):
                w = synth.expert_weights(seed, layer, e, proj, N, K)
                G = oracle.nvfp4_global(w)
                mats.append((*oracle.nvfp4_quantize(w, G), G))
            self.canon[e] = tuple(mats)
            g_gu[e], g_d[e] = mats[0][2], mats[1][2]
            for (codes, sf, _), buf, nb, kind in ((mats[0], self.gu, gu_b, moe.MOE_W4_GATE_UP),
                                                  (mats[1], self.dn, d_b, moe.MOE_W4_PLAIN)):
                moe.moe_pack_nvfp4(torch.from_numpy(codes).cuda(), torch.from_numpy(sf).cuda(), kind,
                                   buf[e * nb:(e + 1) * nb])
        self.g_gu = torch.from_numpy(g_gu).cuda()
        self.g_d = torch.from_numpy(g_d).cuda()
        self.desc = moe.make_nvfp4_layer(E, H, F, self.gu, self.dn, self.g_gu, self.g_d)

    def oracle_forward(self, x, logits, k):
        """Oracle: route, per-row NVFP4 expert FFN, combine -> (idx, w, Y rows, y bf16 bits)."""
        idx, w = oracle.route(logits, k)
        T = x.shape[0]
        Y = np.stack([oracle.expert_ffn_nvfp4(x[t], *self.canon[int(idx[t, j])])
                      for t in range(T) for j in range(k)]).reshape(T, k, self.H)
        y = np.stack([oracle.combine(Y[t], w[t:t + 1])[0] for t in range(T)])
        return idx, w, Y, y


def decode_workspace(T, k, F):
    n = moe.moe_decode_workspace_bytes(T, k, F)
    return torch.zeros(n, dtype=torch.uint8, device="cuda")
