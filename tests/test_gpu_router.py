"""GPU parity of the router linear fused with routing (moe_router_route).

- logits within the fp32 summation bound of the oracle's (the tensor cores
  sum in their own order);
- the selection and weights are exactly the oracle's routing of the logits
  the call computed (the decision is taken on one set of logits);
- against the oracle's own logits, the selection agrees wherever the k-th and
  (k+1)-th logits are not within that bound of each other;
- a second call on the same workspace gives the same bits.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
import quantized_moe_route_b200 as moe
from moe_testlib import u16

pytestmark = pytest.mark.gpu


def _router(x, wr, k):
    T, H = x.shape
    E = wr.shape[0]
    dx, dw = u16(x), u16(wr)
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, k), dtype=torch.float32, device="cuda")
    lg = torch.empty((T, E), dtype=torch.float32, device="cuda")
    ws = torch.zeros(moe.moe_router_route_workspace_bytes(T, E), dtype=torch.uint8, device="cuda")
    moe.moe_router_route(dx, dw, k, idx, w, ws, logits=lg)
    torch.cuda.synchronize()
    out = (lg.cpu().numpy(), idx.cpu().numpy(), w.cpu().numpy())
    idx2 = torch.empty_like(idx)
    w2 = torch.empty_like(w)
    moe.moe_router_route(dx, dw, k, idx2, w2, ws)  # logits kept in the workspace this time
    torch.cuda.synchronize()
    assert np.array_equal(idx2.cpu().numpy(), out[1]) and np.array_equal(w2.cpu().numpy(), out[2])
    return out


@pytest.mark.parametrize("T,E,H,k", [(1, 256, 2048, 8), (16, 256, 2048, 8), (17, 256, 2048, 8), (37, 64, 512, 4),
                                     (2048, 256, 2048, 8), (5, 1024, 256, 8), (3, 16, 64, 2), (70, 48, 128, 3),
                                     (65, 128, 4096, 4), (300, 1024, 128, 16), (9, 1024, 64, 1)])
def test_router_route_matches_oracle(T, E, H, k):
    seed = 300 + T + E
    x = synth.activations_bf16(seed, 0, T, H)
    wr = synth.f32_to_bf16_bits(synth.expert_weights(seed, 0, 0, 0, E, H, sigma=1.0 / np.sqrt(H)))
    lg, idx, w = _router(x, wr, k)
    want = oracle.router_logits(x, wr)
    xf = synth.bf16_bits_to_f32(x).astype(np.float64)
    wf = synth.bf16_bits_to_f32(wr).astype(np.float64)
    bound = 2 * (H + 1) * 2.0 ** -24 * (np.abs(xf) @ np.abs(wf).T)
    assert np.all(np.abs(lg - want) <= bound)
    # the decision on the call's own logits
    oidx, ow = oracle.route(lg, k)
    assert np.array_equal(idx, oidx)
    np.testing.assert_allclose(w, ow, rtol=1e-6, atol=0)
    # against the oracle's logits, away from near-ties at the k-th place
    ridx, _ = oracle.route(want, k)
    srt = -np.sort(-want, axis=1)
    gap = srt[:, k - 1] - (srt[:, k] if k < E else -np.inf)
    clear = gap > 2 * bound.max(axis=1)
    assert np.array_equal(idx[clear], ridx[clear])
    # the comparison is not vacuous: with the worst-case bound about 15% of
    # tokens have the k-th gap inside it (order-statistics spacing of the
    # logits), so most tokens are clear at large T and a quarter at least at
    # T = 16 (16 samples of that fraction)
    if T >= 256:
        assert clear.mean() > 0.75
    elif T >= 16:
        assert clear.sum() >= T // 4
