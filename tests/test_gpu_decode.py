"""GPU parity of the decode path (route -> weight-streaming FFN -> combine)."""
import time

import numpy as np
import pytest
import torch

import oracle
import synth
import quantized_moe_route_b200 as moe
from moe_testlib import Layer, decode_workspace, ffn_close, u16, to_u16

pytestmark = pytest.mark.gpu


def _run_decode(layer, x, logits, k, ws=None):
    T = x.shape[0]
    xd = u16(x)
    ld = torch.from_numpy(np.ascontiguousarray(logits)).cuda()
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, k), dtype=torch.float32, device="cuda")
    moe.moe_route(ld, k, idx, w)
    y_rows = torch.full((T * k, layer.H), float("nan"), device="cuda")
    ws = decode_workspace(T, k, layer.F) if ws is None else ws
    moe.moe_ffn_w4a16_decode(layer.desc, xd, idx, y_rows, ws)
    y = torch.empty((T, layer.H), dtype=torch.int16, device="cuda")
    moe.moe_unpermute_combine(y_rows, w, y)
    torch.cuda.synchronize()
    assert moe.moe_device_error() == 0
    return idx.cpu().numpy(), y_rows.cpu().numpy(), to_u16(y), ws


def _check_layer(seed, E, H, F, T, k, logits=None, repeat=1):
    x = synth.activations_bf16(seed, 0, T, H)
    if logits is None:
        logits = synth.router_logits(seed, 0, T, E)
    oidx, _ = oracle.route(logits, k)
    layer = Layer(seed, 0, E, H, F, oidx.ravel())
    idx, y_rows, y, ws = _run_decode(layer, x, logits, k)
    assert np.array_equal(idx, oidx)
    _, _, oy_rows, oy = oracle.moe_forward_w4(x, logits, k, layer.canon)
    ffn_close(y_rows, oy_rows, "y_rows")
    ffn_close(synth.bf16_bits_to_f32(y), synth.bf16_bits_to_f32(oy), "y")
    for _ in range(repeat - 1):  # the workspace is left ready for the next call
        _, y_rows2, y2, ws = _run_decode(layer, x, logits, k, ws)
        assert np.array_equal(y_rows2, y_rows) and np.array_equal(y2, y)


def test_decode_tiny_layer():
    """1 layer, 8 experts, top-2, hidden 128, width 64, 4 tokens."""
    _check_layer(0, 8, 128, 64, 4, 2, repeat=3)


def test_decode_single_token_full_shape():
    """256 experts, top-8, hidden 2048, width 512, 1 token."""
    _check_layer(1, 256, 2048, 512, 1, 8, repeat=2)


@pytest.mark.parametrize("T", [3, 16])
def test_decode_batches(T):
    _check_layer(2 + T, 64, 1024, 256, T, 8)


def test_decode_all_tokens_on_one_expert():
    """16 tokens all routed to expert 3 first: one expert serves 16 rows (two n8 blocks)."""
    T, E, k = 16, 32, 4
    logits = synth.router_logits(7, 0, T, E)
    logits[:, 3] += 50.0
    _check_layer(7, E, 512, 128, T, k, logits=logits.astype(np.float32))


def test_decode_hand_set_constant_codes_closed_form():
    """All codes 2, scale 0.5, min -0.5: every weight 0.5; closed-form output."""
    E, H, F, T, k = 8, 128, 64, 2, 2
    s = np.full((2 * F, H // 64), np.float16(0.5).view(np.uint16), np.uint16)
    m = np.full((2 * F, H // 64), np.float16(-0.5).view(np.uint16), np.uint16)
    gu = (np.full((2 * F, H), 2, np.uint8), s, m)
    d = (np.full((H, F), 2, np.uint8), s[:H, :1].copy(), m[:H, :1].copy())
    wts = {e: (gu, d) for e in range(E)}
    layer = Layer(0, 0, E, H, F, range(E), weights=wts)
    x = synth.f32_to_bf16_bits(np.full((T, H), 1.0 / 64, np.float32))
    logits = synth.router_logits(3, 0, T, E)
    _, y_rows, y, _ = _run_decode(layer, x, logits, k)
    g = 0.5 * H / 64  # = sum of weights * x
    h = g / (1 + np.exp(-g)) * g
    h_bf16 = float(synth.bf16_bits_to_f32(synth.f32_to_bf16_bits(np.array([h], np.float32)))[0])
    np.testing.assert_allclose(y_rows, 0.5 * F * h_bf16, rtol=1e-6)


def test_decode_workspace_reuse_across_batch_sizes():
    """One workspace serves calls of different batch sizes in a row: stale h
    words of earlier calls never pass for the current call's."""
    E, H, F, k = 64, 512, 128, 8
    ws = decode_workspace(16, k, F)
    for T, seed in [(16, 40), (1, 41), (16, 42), (3, 43)]:
        x = synth.activations_bf16(seed, 0, T, H)
        logits = synth.router_logits(seed, 0, T, E)
        oidx, _ = oracle.route(logits, k)
        layer = Layer(seed, 0, E, H, F, oidx.ravel())
        idx, y_rows, y, ws = _run_decode(layer, x, logits, k, ws)
        _, _, oy_rows, oy = oracle.moe_forward_w4(x, logits, k, layer.canon)
        ffn_close(y_rows, oy_rows, f"y_rows T={T}")


def _fused(layer, x, logits, k, ws=None):
    T = x.shape[0]
    ws = torch.zeros(moe.moe_decode_layer_workspace_bytes(T, k, layer.H, layer.F), dtype=torch.uint8,
                     device="cuda") if ws is None else ws
    y = torch.empty((T, layer.H), dtype=torch.int16, device="cuda")
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, k), dtype=torch.float32, device="cuda")
    moe.moe_decode_layer_w4a16(layer.desc, u16(x), torch.from_numpy(np.ascontiguousarray(logits)).cuda(), k, y, ws,
                               idx=idx, w=w)
    torch.cuda.synchronize()
    assert moe.moe_device_error() == 0
    return to_u16(y), idx.cpu().numpy(), w.cpu().numpy(), ws


@pytest.mark.parametrize("seed,E,H,F,T,k", [(50, 8, 128, 64, 4, 2), (51, 256, 2048, 512, 1, 8),
                                            (52, 64, 1024, 256, 16, 8), (53, 300, 512, 128, 5, 3)])
def test_fused_layer_matches_oracle_and_unfused_path(seed, E, H, F, T, k):
    """One launch (route + FFN + combine) equals route -> decode -> combine
    bit for bit, and the oracle within the FFN tolerance."""
    x = synth.activations_bf16(seed, 0, T, H)
    logits = synth.router_logits(seed, 0, T, E)
    oidx, ow = oracle.route(logits, k)
    layer = Layer(seed, 0, E, H, F, oidx.ravel())
    y, idx, w, _ = _fused(layer, x, logits, k)
    assert np.array_equal(idx, oidx)
    np.testing.assert_allclose(w, ow, rtol=1e-6, atol=1e-7)
    y_unfused = _run_decode(layer, x, logits, k)[2]
    assert np.array_equal(y, y_unfused)
    _, _, _, oy = oracle.moe_forward_w4(x, logits, k, layer.canon)
    ffn_close(synth.bf16_bits_to_f32(y), synth.bf16_bits_to_f32(oy), "fused y")


def test_fused_layer_one_expert_for_all_tokens_and_reuse():
    T, E, k = 16, 32, 4
    logits = synth.router_logits(54, 0, T, E)
    logits[:, 7] += 50.0
    logits = logits.astype(np.float32)
    x = synth.activations_bf16(54, 0, T, 512)
    oidx, _ = oracle.route(logits, k)
    layer = Layer(54, 0, E, 512, 128, oidx.ravel())
    y1, _, _, ws = _fused(layer, x, logits, k)
    y2, _, _, ws = _fused(layer, x, logits, k, ws)  # the workspace carries over
    assert np.array_equal(y1, y2)
    _, _, _, oy = oracle.moe_forward_w4(x, logits, k, layer.canon)
    ffn_close(synth.bf16_bits_to_f32(y1), synth.bf16_bits_to_f32(oy), "fused y")


def test_decode_with_an_sm_held_by_another_stream():
    """The unfused decode kernel's down items wait on gate/up items of other
    CTAs of the same grid, so every CTA must run at once: its launch is
    cooperative, and while a kernel on another stream holds one SM (and all
    its shared memory) for about a second, the grid waits for the SM, runs
    whole, and gives the oracle's result with no device error.  The fused
    layer kernel is launched the same way and gives the oracle's result
    too."""
    import gpu_hold
    E, H, F, T, k, seed = 256, 2048, 512, 1, 8, 91
    x = synth.activations_bf16(seed, 0, T, H)
    logits = synth.router_logits(seed, 0, T, E)
    oidx, _ = oracle.route(logits, k)
    layer = Layer(seed, 0, E, H, F, oidx.ravel())
    xd, ld, idx = u16(x), torch.from_numpy(logits).cuda(), torch.from_numpy(oidx).cuda()
    y_rows = torch.empty((T * k, H), device="cuda")
    ws = decode_workspace(T, k, F)
    y = torch.empty((T, H), dtype=torch.int16, device="cuda")
    lws = torch.zeros(moe.moe_decode_layer_workspace_bytes(T, k, H, F), dtype=torch.uint8, device="cuda")
    done = torch.zeros(2, dtype=torch.int32, device="cuda")
    smem = torch.cuda.get_device_properties(0).shared_memory_per_block_optin
    side, main = torch.cuda.Stream(), torch.cuda.Stream()
    _, _, oy_rows, oy = oracle.moe_forward_w4(x, logits, k, layer.canon)
    torch.cuda.synchronize()
    gpu_hold.hold_sm(2_000_000_000, smem, done[0:1], side)  # about one second at 1.9 GHz
    time.sleep(0.05)  # the holding CTA is resident before the decode is launched
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(main):
        e0.record(main)
        moe.moe_ffn_w4a16_decode(layer.desc, xd, idx, y_rows, ws, stream=main)
        e1.record(main)
    torch.cuda.synchronize()
    assert done[0].item() == 1
    assert moe.moe_device_error() == 0
    ffn_close(y_rows.cpu().numpy(), oy_rows, "y_rows")
    assert e0.elapsed_time(e1) > 300.0  # the grid did wait for the held SM (it needs every SM)
    gpu_hold.hold_sm(2_000_000_000, smem, done[1:2], side)
    time.sleep(0.05)
    with torch.cuda.stream(main):
        moe.moe_decode_layer_w4a16(layer.desc, xd, ld, k, y, lws, stream=main)
    main.synchronize()
    assert moe.moe_device_error() == 0
    ffn_close(synth.bf16_bits_to_f32(to_u16(y)), synth.bf16_bits_to_f32(oy), "fused y")
    torch.cuda.synchronize()
    assert done[1].item() == 1


@pytest.mark.parametrize("T", [1, 16])
def test_fused_decode_chain_of_two_full_size_layers(T):
    """The 40-layer stream's launch configuration: full-size layers (256
    experts, hidden 2048, width 512, top-8), one fused launch per layer, the
    second layer reading the first one's y; each layer's rows are checked
    against the oracle on that layer's own input."""
    E, H, F, k, seed = 256, 2048, 512, 8, 92
    x = synth.activations_bf16(seed, 0, T, H)
    ws = torch.zeros(moe.moe_decode_layer_workspace_bytes(T, k, H, F), dtype=torch.uint8, device="cuda")
    xin = x
    d_in = u16(x)
    for l in range(2):
        logits = synth.router_logits(seed, l, T, E)
        oidx, _ = oracle.route(logits, k)
        layer = Layer(seed, l, E, H, F, oidx.ravel())
        y = torch.empty((T, H), dtype=torch.int16, device="cuda")
        moe.moe_decode_layer_w4a16(layer.desc, d_in, torch.from_numpy(logits).cuda(), k, y, ws)
        torch.cuda.synchronize()
        assert moe.moe_device_error() == 0
        _, _, _, oy = oracle.moe_forward_w4(xin, logits, k, layer.canon)
        got = to_u16(y)
        ffn_close(synth.bf16_bits_to_f32(got), synth.bf16_bits_to_f32(oy), f"layer {l} y")
        xin, d_in = got, y  # the next layer reads this layer's output
