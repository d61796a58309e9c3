"""Failure detection without a GPU fault.

Every spin-wait in the kernels is bounded; when a bound runs out the kernel
records a code in the device error word, lets its own copies in flight land,
and returns, so the context stays usable.  The test hooks
moe_debug_starve_decode / moe_debug_starve_prefill switch one producer role
off (a flag nothing sets) and shorten the bound, so the wait runs out in
milliseconds.  Each test checks that the call returns, that the error word
names the wait, that reading the word clears it, and that the next normal
call on a re-zeroed workspace matches the oracle.
"""
import time

import numpy as np
import pytest
import torch

import oracle
import synth
import quantized_moe_route_b200 as moe
from moe_testlib import Layer, decode_workspace, ffn_close, u16, to_u16

pytestmark = pytest.mark.gpu


def test_decode_h_wait_runs_out_then_next_call_is_correct():
    E, H, F, T, k, seed = 256, 2048, 512, 2, 8, 101
    x = synth.activations_bf16(seed, 0, T, H)
    logits = synth.router_logits(seed, 0, T, E)
    oidx, _ = oracle.route(logits, k)
    layer = Layer(seed, 0, E, H, F, oidx.ravel())
    xd, idx = u16(x), torch.from_numpy(oidx).cuda()
    y_rows = torch.zeros((T * k, H), device="cuda")
    ws = decode_workspace(T, k, F)
    assert moe.moe_device_error() == 0
    t0 = time.time()
    moe.moe_debug_starve_decode(layer.desc, xd, idx, y_rows, ws, polls=2000)
    torch.cuda.synchronize()
    assert time.time() - t0 < 10.0
    assert moe.moe_device_error() == moe.MOE_DEVERR_DECODE_H_WAIT
    assert moe.moe_device_error() == 0  # cleared on read
    ws.zero_()
    moe.moe_ffn_w4a16_decode(layer.desc, xd, idx, y_rows, ws)
    torch.cuda.synchronize()
    assert moe.moe_device_error() == 0
    _, _, oy_rows, _ = oracle.moe_forward_w4(x, logits, k, layer.canon)
    ffn_close(y_rows.cpu().numpy(), oy_rows, "y_rows after the starved call")


def test_prefill_pipeline_wait_runs_out_then_next_call_is_correct():
    E, H, F, T, k, seed = 16, 512, 256, 96, 4, 102
    x = synth.activations_bf16(seed, 0, T, H)
    logits = synth.router_logits(seed, 0, T, E)
    oidx, _ = oracle.route(logits, k)
    counts, offsets, sorted_rows, inv = oracle.permute(oidx, E)
    layer = Layer(seed, 0, E, H, F, oidx.ravel())
    R = T * k
    xp = x[sorted_rows // k]
    x_perm = u16(xp)
    d_off = torch.from_numpy(offsets.astype(np.int32)).cuda()
    ws = torch.zeros(moe.moe_prefill_workspace_bytes(R, F), dtype=torch.uint8, device="cuda")
    assert moe.moe_device_error() == 0
    t0 = time.time()
    moe.moe_debug_starve_prefill(layer.desc, x_perm, d_off, ws, polls=256)
    torch.cuda.synchronize()
    assert time.time() - t0 < 10.0
    assert moe.moe_device_error() == moe.MOE_DEVERR_PREFILL_WAIT
    assert moe.moe_device_error() == 0
    ws.zero_()
    y_perm = torch.empty((R, H), dtype=torch.int16, device="cuda")
    moe.moe_ffn_grouped_prefill(layer.desc, x_perm, d_off, y_perm, ws)
    torch.cuda.synchronize()
    assert moe.moe_device_error() == 0
    want = np.stack([oracle.expert_ffn_w4(xp[p], *layer.canon[int(oidx.ravel()[sorted_rows[p]])])
                     for p in range(R)])
    ffn_close(synth.bf16_bits_to_f32(to_u16(y_perm)), want, "y_perm after the starved call")
