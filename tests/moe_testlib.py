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


def decode_workspace(T, k, F):
    n = moe.moe_decode_workspace_bytes(T, k, F)
    return torch.zeros(n, dtype=torch.uint8, device="cuda")
