"""The allocation-free decode entry point.

moe_ffn_w4a16_decode_static serves callers that cannot allocate device
memory (plugins whose host owns all device memory, fixed memory plans): it
keeps its scratch in a fixed library-owned array instead of a caller
workspace.  Here it is called through the C ABI and compared with the
workspace form, moe_ffn_w4a16_decode, on two calls in a row, and with the
CPU oracle's per-row expert outputs.  This file is
collected last so that a run stopping at the first failure has run every
other test already.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import synth
import quantized_moe_route_b200 as moe
from moe_testlib import Layer, decode_workspace, ffn_close, u16

pytestmark = pytest.mark.gpu


def _decode_both(layer, x, idx, k):
    T = x.shape[0]
    L = moe.lib()
    s = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    ref = torch.full((T * k, layer.H), float("nan"), device="cuda")
    ws = decode_workspace(T, k, layer.F)
    st = L.moe_ffn_w4a16_decode(ctypes.byref(layer.desc), x.data_ptr(), idx.data_ptr(), T, k,
                                ref.data_ptr(), ws.data_ptr(), ws.numel(), s)
    assert st == moe.MOE_OK
    outs = []
    for _ in range(2):  # two calls in a row share the fixed scratch
        y = torch.full((T * k, layer.H), float("nan"), device="cuda")
        st = L.moe_ffn_w4a16_decode_static(ctypes.byref(layer.desc), x.data_ptr(), idx.data_ptr(),
                                           T, k, y.data_ptr(), s)
        assert st == moe.MOE_OK, L.moe_status_string(st)
        outs.append(y)
    torch.cuda.synchronize()
    assert moe.moe_device_error() == 0
    return ref.cpu().numpy(), [o.cpu().numpy() for o in outs]


@pytest.mark.parametrize("E,H,F,T,k", [(8, 128, 64, 4, 2), (256, 2048, 512, 1, 8), (64, 1024, 256, 16, 8)])
def test_static_scratch_decode_matches_workspace_decode(E, H, F, T, k):
    x = synth.activations_bf16(31, 0, T, H)
    logits = synth.router_logits(31, 0, T, E)
    idx_np, _ = oracle.route(logits, k)
    layer = Layer(31, 0, E, H, F, idx_np.ravel())
    idx = torch.from_numpy(idx_np).cuda()
    ref, outs = _decode_both(layer, u16(x), idx, k)
    _, _, oracle_rows, _ = oracle.moe_forward_w4(x, logits, k, layer.canon)
    for y in outs:
        ffn_close(y, ref, "static-scratch decode vs workspace decode")
        ffn_close(y, oracle_rows, "static-scratch decode vs oracle")


def test_static_scratch_rejects_sizes_over_its_limit():
    L = moe.lib()
    buf = torch.zeros(64, dtype=torch.uint8, device="cuda")
    desc = moe.moe_w4_layer(256, 2048, 4096, buf.data_ptr(), buf.data_ptr())
    # 16 tokens x 8 rows x F=4096 x 8 B = 4 MiB of h words > 512 KiB
    st = L.moe_ffn_w4a16_decode_static(ctypes.byref(desc), buf.data_ptr(), buf.data_ptr(), 16, 8,
                                       buf.data_ptr(), None)
    assert st == moe.MOE_ERR_WORKSPACE
