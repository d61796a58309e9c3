"""GPU parity of the shared expert: routing with the shared column, the fused
one-launch decode layer with a shared expert, and the prefill composition
route_shared -> permute (E + 1 experts) -> grouped FFN -> combine (k + 1 rows),
against the oracle's moe_forward_w4_shared.

The reading (a shared expert beside the routed ones: "Drama 3 int4 (drama-rs
format)", table "What's quantized"; "Drama 3 - NVFP4 routed experts",
"Quantization"): every token runs the shared expert with weight 1, its row
added after the routed sum.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
import quantized_moe_route_b200 as moe
from moe_testlib import Layer, decode_workspace, ffn_close, u16, to_u16

pytestmark = pytest.mark.gpu


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


@pytest.mark.parametrize("T,E,k", [(1, 256, 8), (37, 64, 4), (5, 1023, 31), (3, 16, 16), (130, 300, 3)])
def test_route_shared_is_route_plus_the_shared_column(T, E, k):
    logits = synth.router_logits(80 + T, 0, T, E)
    ld = _dev(logits)
    idx = torch.empty((T, k + 1), dtype=torch.int32, device="cuda")
    w = torch.empty((T, k + 1), dtype=torch.float32, device="cuda")
    moe.moe_route_shared(ld, k, idx, w)
    ri = torch.empty((T, k), dtype=torch.int32, device="cuda")
    rw = torch.empty((T, k), dtype=torch.float32, device="cuda")
    moe.moe_route(ld, k, ri, rw)
    torch.cuda.synchronize()
    idx, w, ri, rw = idx.cpu().numpy(), w.cpu().numpy(), ri.cpu().numpy(), rw.cpu().numpy()
    assert np.array_equal(idx[:, :k], ri) and np.array_equal(w[:, :k], rw)  # the same routing, bit for bit
    assert (idx[:, k] == E).all() and (w[:, k] == 1.0).all()
    oidx, ow = oracle.route(logits, k)
    assert np.array_equal(ri, oidx)
    np.testing.assert_allclose(rw, ow, rtol=1e-6, atol=1e-7)


def _shared_layer(seed, E, H, F, logits, k):
    """E routed experts + the shared one (id E); canonical weights of the
    selected experts and of the shared expert."""
    oidx, _ = oracle.route(logits, k)
    layer = Layer(seed, 0, E + 1, H, F, list(oidx.ravel()) + [E])
    routed = {e: v for e, v in layer.canon.items() if e != E}
    return layer, routed, layer.canon[E]


def _unfused_shared(layer, x, logits, k):
    """route_shared -> decode FFN of k + 1 rows per token -> combine."""
    T = x.shape[0]
    idx = torch.empty((T, k + 1), dtype=torch.int32, device="cuda")
    w = torch.empty((T, k + 1), dtype=torch.float32, device="cuda")
    moe.moe_route_shared(_dev(logits), k, idx, w)
    y_rows = torch.full((T * (k + 1), layer.H), float("nan"), device="cuda")
    moe.moe_ffn_w4a16_decode(layer.desc, u16(x), idx, y_rows, decode_workspace(T, k + 1, layer.F))
    y = torch.empty((T, layer.H), dtype=torch.int16, device="cuda")
    moe.moe_unpermute_combine(y_rows, w, y)
    torch.cuda.synchronize()
    assert moe.moe_device_error() == 0
    return y_rows.cpu().numpy().reshape(T, k + 1, layer.H), to_u16(y)


def _fused_shared(layer, x, logits, k, ws=None):
    T = x.shape[0]
    if ws is None:
        ws = torch.zeros(moe.moe_decode_layer_workspace_bytes(T, k + 1, layer.H, layer.F), dtype=torch.uint8,
                         device="cuda")
    y = torch.empty((T, layer.H), dtype=torch.int16, device="cuda")
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, k), dtype=torch.float32, device="cuda")
    moe.moe_decode_layer_w4a16_shared(layer.desc, u16(x), _dev(logits), k, y, ws, idx=idx, w=w)
    torch.cuda.synchronize()
    assert moe.moe_device_error() == 0
    return to_u16(y), idx.cpu().numpy(), w.cpu().numpy(), ws


@pytest.mark.parametrize("seed,E,H,F,T,k", [(90, 8, 128, 64, 4, 2), (91, 256, 2048, 512, 1, 8),
                                            (92, 64, 1024, 256, 16, 8), (93, 255, 512, 128, 5, 3),
                                            (94, 1023, 256, 128, 2, 8)])
def test_fused_shared_layer_matches_oracle_and_the_composed_calls(seed, E, H, F, T, k):
    x = synth.activations_bf16(seed, 0, T, H)
    logits = synth.router_logits(seed, 0, T, E)
    layer, routed, shared = _shared_layer(seed, E, H, F, logits, k)
    y, idx, w, ws = _fused_shared(layer, x, logits, k)
    oidx, ow, orows, oy = oracle.moe_forward_w4_shared(x, logits, k, routed, shared)
    assert np.array_equal(idx, oidx)
    np.testing.assert_allclose(w, ow, rtol=1e-6, atol=1e-7)
    rows, y_unfused = _unfused_shared(layer, x, logits, k)
    assert np.array_equal(y, y_unfused)  # one launch == route_shared -> decode -> combine, bit for bit
    ffn_close(rows, orows, "rows incl. the shared expert's")
    ffn_close(synth.bf16_bits_to_f32(y), synth.bf16_bits_to_f32(oy), "fused shared y")
    y2, _, _, _ = _fused_shared(layer, x, logits, k, ws)  # the workspace carries over
    assert np.array_equal(y2, y)


def test_fused_shared_with_zero_shared_weights_is_the_routed_layer():
    """A zero shared expert adds exact zeros: the fused shared layer gives the
    plain fused layer's bits."""
    E, H, F, T, k, seed = 32, 256, 128, 6, 4, 95
    x = synth.activations_bf16(seed, 0, T, H)
    logits = synth.router_logits(seed, 0, T, E)
    layer, _, _ = _shared_layer(seed, E, H, F, logits, k)
    gu_b = moe.moe_w4_packed_bytes(2 * F, H)
    d_b = moe.moe_w4_packed_bytes(H, F)
    layer.gu[E * gu_b:].zero_()
    layer.dn[E * d_b:].zero_()
    y, _, _, _ = _fused_shared(layer, x, logits, k)
    plain = moe.make_layer(E, H, F, layer.gu, layer.dn)  # the first E experts alone
    ws = torch.zeros(moe.moe_decode_layer_workspace_bytes(T, k, H, F), dtype=torch.uint8, device="cuda")
    y0 = torch.empty((T, H), dtype=torch.int16, device="cuda")
    moe.moe_decode_layer_w4a16(plain, u16(x), _dev(logits), k, y0, ws)
    torch.cuda.synchronize()
    assert np.array_equal(y, to_u16(y0))


def test_prefill_with_shared_expert_matches_oracle():
    E, H, F, T, k, seed = 16, 512, 256, 200, 4, 96
    x = synth.activations_bf16(seed, 0, T, H)
    logits = synth.router_logits(seed, 0, T, E)
    layer, routed, shared = _shared_layer(seed, E, H, F, logits, k)
    k1, E1 = k + 1, E + 1
    idx = torch.empty((T, k1), dtype=torch.int32, device="cuda")
    w = torch.empty((T, k1), dtype=torch.float32, device="cuda")
    moe.moe_route_shared(_dev(logits), k, idx, w)
    counts = torch.empty(E1, dtype=torch.int32, device="cuda")
    offsets = torch.empty(E1 + 1, dtype=torch.int32, device="cuda")
    sorted_rows = torch.empty(T * k1, dtype=torch.int32, device="cuda")
    inv = torch.empty(T * k1, dtype=torch.int32, device="cuda")
    pws = torch.empty(moe.moe_permute_workspace_bytes(T, k1, E1), dtype=torch.uint8, device="cuda")
    x_perm = torch.empty((T * k1, H), dtype=torch.int16, device="cuda")
    moe.moe_permute(idx, E1, counts, offsets, sorted_rows, inv, pws, x=u16(x), x_perm=x_perm)
    y_perm = torch.empty((T * k1, H), dtype=torch.int16, device="cuda")
    fws = torch.empty(moe.moe_prefill_workspace_bytes(T * k1, F), dtype=torch.uint8, device="cuda")
    moe.moe_ffn_grouped_prefill(layer.desc, x_perm, offsets, y_perm, fws)
    y = torch.empty((T, H), dtype=torch.int16, device="cuda")
    moe.moe_unpermute_combine(y_perm, w, y, inv=inv)
    torch.cuda.synchronize()
    assert moe.moe_device_error() == 0
    assert counts.cpu().numpy()[E] == T  # every token visits the shared expert
    _, _, orows, oy = oracle.moe_forward_w4_shared(x, logits, k, routed, shared)
    got_rows = synth.bf16_bits_to_f32(to_u16(y_perm)[inv.cpu().numpy()]).reshape(T, k1, H)
    ffn_close(got_rows, orows, "prefill rows incl. the shared expert's")
    ffn_close(synth.bf16_bits_to_f32(to_u16(y)), synth.bf16_bits_to_f32(oy), "prefill shared y")


def test_shared_argument_limits():
    T, H, F = 2, 128, 64
    x = u16(synth.activations_bf16(97, 0, T, H))
    with pytest.raises(moe.MoeError) as ei:  # 1024 routed experts + the shared id do not fit
        moe.moe_route_shared(torch.zeros((T, 1024), device="cuda"), 2,
                             torch.empty((T, 3), dtype=torch.int32, device="cuda"),
                             torch.empty((T, 3), device="cuda"))
    assert ei.value.status == moe.MOE_ERR_UNSUPPORTED_SHAPE
    gu = torch.zeros(2 * moe.moe_w4_packed_bytes(2 * F, H), dtype=torch.uint8, device="cuda")
    dn = torch.zeros(2 * moe.moe_w4_packed_bytes(H, F), dtype=torch.uint8, device="cuda")
    y = torch.empty((T, H), dtype=torch.int16, device="cuda")
    ws = torch.zeros(moe.moe_decode_layer_workspace_bytes(T, 32, H, F), dtype=torch.uint8, device="cuda")
    one = moe.make_layer(1, H, F, gu, dn)  # the shared expert and no routed one
    with pytest.raises(moe.MoeError) as ei:
        moe.moe_decode_layer_w4a16_shared(one, x, torch.zeros((T, 1), device="cuda"), 1, y, ws)
    assert ei.value.status == moe.MOE_ERR_INVALID_ARG
    two = moe.make_layer(2, H, F, gu, dn)
    with pytest.raises(moe.MoeError) as ei:  # k = 2 of one routed expert
        moe.moe_decode_layer_w4a16_shared(two, x, torch.zeros((T, 1), device="cuda"), 2, y, ws)
    assert ei.value.status == moe.MOE_ERR_INVALID_ARG
    small = torch.zeros(moe.moe_decode_layer_workspace_bytes(T, 1, H, F), dtype=torch.uint8, device="cuda")
    with pytest.raises(moe.MoeError) as ei:  # the workspace must hold k + 1 rows per token
        moe.moe_decode_layer_w4a16_shared(two, x, torch.zeros((T, 1), device="cuda"), 1, y, small)
    assert ei.value.status == moe.MOE_ERR_WORKSPACE
