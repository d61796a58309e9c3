"""Pins of the oracle's router linear (CPU only).

Source: "Drama 3 int4 (drama-rs format)", table "What's quantized" (the
router stays bf16) and "DRAMA-3 MLX expert-only 4-bit", section
"Quantization and provenance" (routers retain source BF16).  The reading:
logits = Wr x with bf16 operands, fp32 products and sums, no bias.

- One-hot router rows make every logit one channel of x, exactly.
- A float64 matmul of the bf16 values agrees within the fp32 summation bound.
- Scaling x by a power of two scales the logits by it exactly.
- Routing the oracle's logits gives what the pinned route gives.
"""
import numpy as np

import oracle
import synth


def _bf16(a):
    return synth.f32_to_bf16_bits(np.asarray(a, np.float32))


def test_one_hot_rows_select_channels():
    T, E, H = 5, 32, 256
    x = synth.activations_bf16(51, 0, T, H)
    pick = np.random.default_rng(1).integers(0, H, E)
    wr = np.zeros((E, H), np.float32)
    wr[np.arange(E), pick] = 1.0
    got = oracle.router_logits(x, _bf16(wr))
    want = synth.bf16_bits_to_f32(x)[:, pick]
    assert np.array_equal(got, want)


def test_float64_cross_check_within_the_fp32_bound():
    T, E, H = 8, 64, 2048
    x = synth.activations_bf16(52, 0, T, H)
    wr = _bf16(synth.expert_weights(52, 0, 0, 0, E, H))
    got = oracle.router_logits(x, wr).astype(np.float64)
    xf = synth.bf16_bits_to_f32(x).astype(np.float64)
    wf = synth.bf16_bits_to_f32(wr).astype(np.float64)
    ref = xf @ wf.T
    mag = np.abs(xf) @ np.abs(wf).T
    assert np.all(np.abs(got - ref) <= (H + 1) * 2.0 ** -24 * mag)


def test_power_of_two_scaling_is_exact():
    T, E, H = 3, 16, 512
    x = synth.activations_bf16(53, 0, T, H)
    wr = _bf16(synth.expert_weights(53, 0, 0, 0, E, H))
    x4 = _bf16(synth.bf16_bits_to_f32(x) * 4.0)
    assert np.array_equal(oracle.router_logits(x4, wr), 4.0 * oracle.router_logits(x, wr))


def test_routing_of_router_logits():
    T, E, H, k = 6, 256, 2048, 8
    x = synth.activations_bf16(54, 0, T, H)
    wr = _bf16(synth.expert_weights(54, 0, 0, 0, E, H, sigma=1.0 / 32))
    lg = oracle.router_logits(x, wr)
    idx, w = oracle.route(lg, k)
    order = np.argsort(-lg, axis=1, kind="stable")[:, :k]
    assert np.array_equal(idx, order)
    np.testing.assert_allclose(w.sum(1), 1.0, rtol=1e-6)
