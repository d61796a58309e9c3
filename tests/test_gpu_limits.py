"""Edge cases at the documented limits: the fused decode at its row limit
(T*k = 256) and expert limit (E = 1024), the prefill at E = 960, the
no-op T = 0 / rows = 0 calls, the rejections just past each limit, and a
prefill group table that claims more rows than the call has."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import synth
import quantized_moe_route_b200 as moe
from moe_testlib import Layer, NvLayer, ffn_close, u16, to_u16

pytestmark = pytest.mark.gpu


def _fused(layer, x, logits, k, nvfp4=False):
    T = x.shape[0]
    ws = torch.zeros(moe.moe_decode_layer_workspace_bytes(T, k, layer.H, layer.F), dtype=torch.uint8,
                     device="cuda")
    y = torch.empty((T, layer.H), dtype=torch.int16, device="cuda")
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, k), dtype=torch.float32, device="cuda")
    call = moe.moe_decode_layer_nvfp4 if nvfp4 else moe.moe_decode_layer_w4a16
    call(layer.desc, u16(x), torch.from_numpy(np.ascontiguousarray(logits)).cuda(), k, y, ws, idx=idx, w=w)
    torch.cuda.synchronize()
    assert moe.moe_device_error() == 0
    return to_u16(y), idx.cpu().numpy()


@pytest.mark.parametrize("E,T,k", [(64, 16, 16), (1024, 2, 8)])
def test_fused_int4_decode_at_row_and_expert_limits(E, T, k):
    H, F, seed = 256, 128, 70 + E
    x = synth.activations_bf16(seed, 0, T, H)
    logits = synth.router_logits(seed, 0, T, E)
    oidx, _ = oracle.route(logits, k)
    layer = Layer(seed, 0, E, H, F, oidx.ravel())
    y, idx = _fused(layer, x, logits, k)
    assert np.array_equal(idx, oidx)
    _, _, _, oy = oracle.moe_forward_w4(x, logits, k, layer.canon)
    ffn_close(synth.bf16_bits_to_f32(y), synth.bf16_bits_to_f32(oy), "y")


def test_fused_nvfp4_decode_at_row_limit():
    E, T, k, H, F, seed = 64, 16, 16, 256, 256, 75
    x = synth.activations_bf16(seed, 0, T, H)
    logits = synth.router_logits(seed, 0, T, E)
    oidx, _ = oracle.route(logits, k)
    layer = NvLayer(seed, 0, E, H, F, oidx.ravel())
    y, idx = _fused(layer, x, logits, k, nvfp4=True)
    assert np.array_equal(idx, oidx)
    _, _, _, oy = layer.oracle_forward(x, logits, k)
    ffn_close(synth.bf16_bits_to_f32(y), synth.bf16_bits_to_f32(oy), "y")


def test_no_op_calls_leave_outputs_untouched():
    layer = Layer(76, 0, 8, 128, 64, [0])
    y = torch.full((1, 128), 123, dtype=torch.int16, device="cuda")
    x = torch.zeros((1, 128), dtype=torch.int16, device="cuda")
    lg = torch.zeros((1, 8), dtype=torch.float32, device="cuda")
    ws = torch.zeros(1 << 16, dtype=torch.uint8, device="cuda")
    L = moe.lib()
    st = L.moe_decode_layer_w4a16(ctypes.byref(layer.desc), moe._p(x), moe._p(lg), 0, 2, moe._p(y), None, None,
                                  moe._p(ws), ws.numel(), None)
    assert st == moe.MOE_OK
    assert L.moe_route(moe._p(lg), 0, 8, 2, None, None, None) == moe.MOE_OK
    pf = moe.moe_w4_layer(8, 256, 128, 16, 16)  # a shape the prefill tiles (H % 256, F % 128)
    assert L.moe_ffn_grouped_prefill(ctypes.byref(pf), None, None, 0, None, None, 0, None) == moe.MOE_OK
    assert L.moe_unpermute_combine(None, 0, None, None, 0, 2, 128, None, None) == moe.MOE_OK
    torch.cuda.synchronize()
    assert (y == 123).all()


def test_rejections_just_past_the_limits():
    layer = Layer(77, 0, 8, 128, 64, [0])
    L = moe.lib()
    p = ctypes.c_void_p(16)
    big = 1 << 30
    # 17 tokens (limit 16); 16 tokens x k 17 = 272 rows (limit 256)
    assert L.moe_decode_layer_w4a16(ctypes.byref(layer.desc), p, p, 17, 2, p, None, None, p, big, None) == \
        moe.MOE_ERR_UNSUPPORTED_SHAPE
    d = moe.moe_w4_layer(64, 128, 64, 16, 16)
    assert L.moe_decode_layer_w4a16(ctypes.byref(d), p, p, 16, 17, p, None, None, p, big, None) == \
        moe.MOE_ERR_UNSUPPORTED_SHAPE
    # k > E is an argument error; E = 961 is past the prefill's expert limit
    assert L.moe_decode_layer_w4a16(ctypes.byref(layer.desc), p, p, 1, 9, p, None, None, p, big, None) == \
        moe.MOE_ERR_INVALID_ARG
    d = moe.moe_w4_layer(961, 128, 128, 16, 16)
    assert L.moe_ffn_grouped_prefill(ctypes.byref(d), p, p, 4, p, p, big, None) == moe.MOE_ERR_UNSUPPORTED_SHAPE
    # a workspace one byte short
    n = moe.moe_decode_layer_workspace_bytes(1, 2, 128, 64)
    assert L.moe_decode_layer_w4a16(ctypes.byref(layer.desc), p, p, 1, 2, p, None, None, p, n - 1, None) == \
        moe.MOE_ERR_WORKSPACE


def test_int4_prefill_at_expert_limit():
    """960 experts (the prefill's limit), 512 rows: most experts empty."""
    from test_gpu_prefill import _check
    offsets = _check(78, 960, 256, 128, 128, 4)
    assert (np.diff(offsets) == 0).sum() > 400


def test_nvfp4_prefill_at_expert_limit():
    from test_gpu_prefill_nvfp4 import _check as nv_check
    g = nv_check(79, 960, 256, 256, 128, 4, stagewise_rows=4)
    assert (np.diff(g["offsets"]) == 0).sum() > 400


def test_prefill_offsets_past_rows_write_nothing_past_rows():
    """A group table that breaks its contract (offsets[E] = 160 > rows = 100)
    is clamped to the rows the caller passed: the rows below 100 still get
    their experts' outputs, and nothing at or past row 100 (of y_perm or of
    the h workspace) is written."""
    E, H, F, rows, pad, seed = 4, 256, 128, 100, 96, 81
    offsets = np.array([0, 30, 60, 100, 160], np.int32)
    layer = Layer(seed, 0, E, H, F, range(E))
    xp = synth.activations_bf16(seed, 0, rows + pad, H)
    x_perm = u16(xp)
    sentinel = 0x5A5A
    y_perm = torch.full((rows + pad, H), sentinel, dtype=torch.int16, device="cuda")
    hbytes = moe.moe_prefill_workspace_bytes(rows, F)
    ws = torch.full((hbytes + pad * F * 2,), 0x5A, dtype=torch.uint8, device="cuda")
    d_off = torch.from_numpy(offsets).cuda()
    L = moe.lib()
    st = L.moe_ffn_grouped_prefill(ctypes.byref(layer.desc), moe._p(x_perm), moe._p(d_off), rows, moe._p(y_perm),
                                   moe._p(ws), hbytes, None)
    assert st == moe.MOE_OK
    torch.cuda.synchronize()
    assert moe.moe_device_error() == 0
    y = to_u16(y_perm)
    assert np.all(y[rows:] == sentinel)
    assert np.all(ws[rows * F * 2:].cpu().numpy() == 0x5A)
    want = np.stack([oracle.expert_ffn_w4(xp[p], *layer.canon[int(np.searchsorted(offsets, p, side="right") - 1)])
                     for p in range(rows)])
    ffn_close(synth.bf16_bits_to_f32(y[:rows]), want, "y_perm (valid rows)")
