"""GPU parity of the NVFP4 single-launch decode layer against the CPU oracle
(route, per-token x quantisation, NVFP4 expert FFN with per-row h
re-quantisation, combine)."""
import numpy as np
import pytest
import torch

import oracle
import synth
import quantized_moe_route_b200 as moe
from moe_testlib import NvLayer, ffn_close, u16, to_u16

pytestmark = pytest.mark.gpu


def _run(layer, x, logits, k, ws=None):
    T = x.shape[0]
    if ws is None:
        ws = torch.zeros(moe.moe_decode_layer_workspace_bytes(T, k, layer.H, layer.F), dtype=torch.uint8,
                         device="cuda")
    y = torch.empty((T, layer.H), dtype=torch.int16, device="cuda")
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, k), dtype=torch.float32, device="cuda")
    moe.moe_decode_layer_nvfp4(layer.desc, u16(x), torch.from_numpy(np.ascontiguousarray(logits)).cuda(), k, y,
                               ws, idx=idx, w=w)
    torch.cuda.synchronize()
    assert moe.moe_device_error() == 0
    return to_u16(y), idx.cpu().numpy(), w.cpu().numpy(), ws


@pytest.mark.parametrize("seed,E,H,F,T,k", [(60, 8, 256, 256, 4, 2), (61, 256, 2048, 512, 1, 8),
                                            (62, 64, 1024, 256, 16, 8), (63, 300, 512, 512, 5, 3)])
def test_nvfp4_decode_layer_matches_oracle(seed, E, H, F, T, k):
    x = synth.activations_bf16(seed, 0, T, H)
    logits = synth.router_logits(seed, 0, T, E)
    oidx, ow = oracle.route(logits, k)
    layer = NvLayer(seed, 0, E, H, F, oidx.ravel())
    y, idx, w, _ = _run(layer, x, logits, k)
    assert np.array_equal(idx, oidx)
    np.testing.assert_allclose(w, ow, rtol=1e-6, atol=1e-7)
    _, _, _, oy = layer.oracle_forward(x, logits, k)
    ffn_close(synth.bf16_bits_to_f32(y), synth.bf16_bits_to_f32(oy), "nvfp4 decode y")


def test_nvfp4_decode_one_expert_all_tokens_zero_token_and_reuse():
    T, E, k, H, F = 16, 32, 4, 512, 256
    logits = synth.router_logits(64, 0, T, E)
    logits[:, 9] += 50.0
    logits = logits.astype(np.float32)
    x = synth.activations_bf16(64, 0, T, H)
    x[3] = 0  # a zero token: global 1, zero codes, zero output
    oidx, _ = oracle.route(logits, k)
    layer = NvLayer(64, 0, E, H, F, oidx.ravel())
    y1, _, _, ws = _run(layer, x, logits, k)
    y2, _, _, ws = _run(layer, x, logits, k, ws)  # the workspace carries over
    assert np.array_equal(y1, y2)
    assert not synth.bf16_bits_to_f32(y1[3]).any()
    _, _, _, oy = layer.oracle_forward(x, logits, k)
    ffn_close(synth.bf16_bits_to_f32(y1), synth.bf16_bits_to_f32(oy), "nvfp4 decode y")


def test_nvfp4_decode_rejects_shapes():
    L = moe.lib()
    import ctypes
    d = moe.moe_nvfp4_layer(8, 256, 128, 16, 16, 16, 16)  # F % 256 != 0
    assert L.moe_decode_layer_nvfp4(ctypes.byref(d), 16, 16, 1, 2, 16, None, None, 16, 1 << 20, None) == \
        moe.MOE_ERR_UNSUPPORTED_SHAPE
