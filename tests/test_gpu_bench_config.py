"""Parity in the benchmark's own configuration: layers built exactly as
bench.py builds them (weights generated on the GPU by the CUDA twin of the
seeded generator, quantised and packed on the GPU, 256 experts + the shared
slot), inputs from the bench's seeds, and the same calls the timed legs make,
against the oracle on the CPU twin's weights.  Full sizes: hidden 2048,
expert width 512, top-8."""
import numpy as np
import pytest
import torch

import bench
import oracle
import synth
import quantized_moe_route_b200 as moe
from moe_testlib import ffn_close, to_u16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def w4_layers():
    return bench.build_layers(2, bench.SEED_W4, lambda m: None)


def _decode(call, desc, x, lg, k, kk):
    T = x.shape[0]
    y = torch.empty((T, bench.H), dtype=torch.int16, device="cuda")
    ws = torch.zeros(moe.moe_decode_layer_workspace_bytes(T, kk, bench.H, bench.F), dtype=torch.uint8,
                     device="cuda")
    call(desc, torch.from_numpy(x.view(np.int16)).cuda(), torch.from_numpy(lg).cuda(), k, y, ws)
    torch.cuda.synchronize()
    assert moe.moe_device_error() == 0
    return to_u16(y)


@pytest.mark.parametrize("layer,T,seed", [(0, 1, bench.SEED_DECODE), (1, 1, bench.SEED_DECODE),
                                          (1, 16, bench.SEED_STREAM)])
def test_bench_decode_layer_matches_oracle(w4_layers, layer, T, seed):
    k = bench.TOPK
    x, lg = bench.layer_inputs(seed, layer, T)
    y = _decode(moe.moe_decode_layer_w4a16, w4_layers[layer][2], x, lg, k, k)
    idx, _ = oracle.route(lg, k)
    ex = bench.oracle_experts(bench.SEED_W4, layer, idx.ravel(), "w4")
    _, _, _, oy = oracle.moe_forward_w4(x, lg, k, ex)
    ffn_close(synth.bf16_bits_to_f32(y), synth.bf16_bits_to_f32(oy), f"bench decode layer {layer} T={T}")


def test_bench_shared_decode_matches_oracle(w4_layers):
    k, layer = bench.TOPK, 0
    x, lg = bench.layer_inputs(bench.SEED_SHARED, layer, 1)
    y = _decode(moe.moe_decode_layer_w4a16_shared, w4_layers[layer][3], x, lg, k, k + 1)
    idx, _ = oracle.route(lg, k)
    ex = bench.oracle_experts(bench.SEED_W4, layer, list(idx.ravel()) + [bench.E], "w4")
    sh = ex.pop(bench.E)
    _, _, _, oy = oracle.moe_forward_w4_shared(x, lg, k, ex, sh)
    ffn_close(synth.bf16_bits_to_f32(y), synth.bf16_bits_to_f32(oy), "bench shared decode")


def test_bench_nvfp4_decode_matches_oracle():
    k, layer = bench.TOPK, 1
    layers = bench.build_layers_nvfp4(2, bench.SEED_NV, lambda m: None)
    x, lg = bench.layer_inputs(bench.SEED_NVD, layer, 1)
    y = _decode(moe.moe_decode_layer_nvfp4, layers[layer][2], x, lg, k, k)
    idx, _ = oracle.route(lg, k)
    ex = bench.oracle_experts(bench.SEED_NV, layer, idx.ravel(), "nvfp4")
    oy = bench.oracle_forward(x, lg, ex, "nvfp4")
    ffn_close(synth.bf16_bits_to_f32(y), synth.bf16_bits_to_f32(oy), "bench nvfp4 decode")
