"""GPU parity of the decode layer with the router linear in the same launch
(moe_decode_layer_w4a16_router), with and without a shared expert.

- the logits it computes are within the fp32 summation bound of the
  oracle's router_logits (the kernel sums in its own fixed order);
- its selection and weights are exactly the oracle's routing of those logits;
- y equals, bit for bit, the decode layer given those logits as input (whose
  parity against the oracle's forward is pinned elsewhere), and the oracle's
  forward within the FFN tolerance;
- a second call on the same workspace gives the same bits.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
import quantized_moe_route_b200 as moe
from moe_testlib import Layer, ffn_close, u16, to_u16

pytestmark = pytest.mark.gpu


def _router_weights(seed, Er, H):
    return synth.f32_to_bf16_bits(synth.expert_weights(seed, 0, 0, 2, Er, H, sigma=1.0 / np.sqrt(H)))


@pytest.mark.parametrize("seed,E,H,F,T,k,shared", [(100, 256, 2048, 512, 1, 8, 0), (101, 256, 2048, 512, 16, 8, 0),
                                                   (102, 64, 512, 128, 5, 4, 1), (103, 1024, 256, 128, 3, 8, 0),
                                                   (104, 8, 128, 64, 4, 2, 0), (105, 255, 512, 128, 2, 3, 1),
                                                   (106, 256, 2048, 512, 1, 8, 1)])
def test_decode_with_router_matches_oracle_and_the_given_logits_path(seed, E, H, F, T, k, shared):
    x = synth.activations_bf16(seed, 0, T, H)
    wr = _router_weights(seed, E, H)
    want_lg = oracle.router_logits(x, wr)
    # experts that can be selected: every token's top k + 4 by the oracle's
    # logits (a near-tie at the k-th place can only swap neighbours)
    cand = np.argsort(-want_lg, axis=1, kind="stable")[:, :min(E, k + 4)]
    layer = Layer(seed, 0, E + shared, H, F, list(cand.ravel()) + ([E] if shared else []))
    ws = torch.zeros(moe.moe_decode_layer_router_workspace_bytes(T, k, shared, E + shared, H, F), dtype=torch.uint8,
                     device="cuda")
    xd, wd = u16(x), u16(wr)
    y = torch.empty((T, H), dtype=torch.int16, device="cuda")
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, k), dtype=torch.float32, device="cuda")
    lg = torch.empty((T, E), dtype=torch.float32, device="cuda")
    moe.moe_decode_layer_w4a16_router(layer.desc, xd, wd, k, y, ws, shared=shared, idx=idx, w=w, logits=lg)
    torch.cuda.synchronize()
    assert moe.moe_device_error() == 0
    lg_n, idx_n, w_n, y_n = lg.cpu().numpy(), idx.cpu().numpy(), w.cpu().numpy(), to_u16(y)
    xf = synth.bf16_bits_to_f32(x).astype(np.float64)
    wf = synth.bf16_bits_to_f32(wr).astype(np.float64)
    bound = 2 * (H + 1) * 2.0 ** -24 * (np.abs(xf) @ np.abs(wf).T)
    assert np.all(np.abs(lg_n - want_lg) <= bound)
    oidx, ow = oracle.route(lg_n, k)
    assert np.array_equal(idx_n, oidx)
    np.testing.assert_allclose(w_n, ow, rtol=1e-6, atol=0)
    assert set(int(e) for e in idx_n.ravel()) <= set(layer.canon), "selected an expert outside the candidates"
    # the same layer given the computed logits
    ws2 = torch.zeros(moe.moe_decode_layer_workspace_bytes(T, k + shared, H, F), dtype=torch.uint8, device="cuda")
    y2 = torch.empty((T, H), dtype=torch.int16, device="cuda")
    call = moe.moe_decode_layer_w4a16_shared if shared else moe.moe_decode_layer_w4a16
    call(layer.desc, xd, lg, k, y2, ws2)
    torch.cuda.synchronize()
    assert np.array_equal(y_n, to_u16(y2))
    if shared:
        routed = {e: v for e, v in layer.canon.items() if e != E}
        _, _, _, oy = oracle.moe_forward_w4_shared(x, lg_n, k, routed, layer.canon[E])
    else:
        _, _, _, oy = oracle.moe_forward_w4(x, lg_n, k, layer.canon)
    ffn_close(synth.bf16_bits_to_f32(y_n), synth.bf16_bits_to_f32(oy), "decode with router y")
    # the workspace carries over to the next call
    moe.moe_decode_layer_w4a16_router(layer.desc, xd, wd, k, y, ws, shared=shared)
    torch.cuda.synchronize()
    assert np.array_equal(to_u16(y), y_n)


def test_decode_with_router_argument_checks():
    T, H, F, E, k = 2, 128, 64, 8, 2
    gu = torch.zeros(E * moe.moe_w4_packed_bytes(2 * F, H), dtype=torch.uint8, device="cuda")
    dn = torch.zeros(E * moe.moe_w4_packed_bytes(H, F), dtype=torch.uint8, device="cuda")
    layer = moe.make_layer(E, H, F, gu, dn)
    x = u16(synth.activations_bf16(107, 0, T, H))
    y = torch.empty((T, H), dtype=torch.int16, device="cuda")
    wr = torch.zeros((E, H), dtype=torch.int16, device="cuda")
    small = torch.zeros(moe.moe_decode_layer_workspace_bytes(T, k, H, F), dtype=torch.uint8, device="cuda")
    with pytest.raises(moe.MoeError) as ei:  # the logit words need room beyond the plain layer's workspace
        moe.moe_decode_layer_w4a16_router(layer, x, wr, k, y, small)
    assert ei.value.status == moe.MOE_ERR_WORKSPACE
    ws = torch.zeros(moe.moe_decode_layer_router_workspace_bytes(T, k, 0, E, H, F), dtype=torch.uint8, device="cuda")
    with pytest.raises(moe.MoeError) as ei:
        moe.moe_decode_layer_w4a16_router(layer, x, wr, k, y, ws, shared=2)
    assert ei.value.status == moe.MOE_ERR_INVALID_ARG
    with pytest.raises(moe.MoeError) as ei:  # misaligned router weights
        moe.moe_decode_layer_w4a16_router(layer, x, wr.view(-1)[1:1 + E * H - 8], k, y, ws)
    assert ei.value.status == moe.MOE_ERR_INVALID_ARG
