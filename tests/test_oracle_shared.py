"""Pins of the oracle's shared expert (CPU only).

Source: a shared expert sits beside the routed ones ("Drama 3 int4
(drama-rs format)", table "What's quantized"; "Drama 3 - NVFP4 routed
experts", section "Quantization").  The reading: one more SwiGLU expert on
every token, weight 1, added after the routed sum (the combine of k + 1
rows), stored in the routed experts' int4 format.

- Zero shared weights give the routed-only result, bit for bit.
- Zero routed experts give the shared expert alone (rounded to bf16).
- The rows are the pinned per-expert FFN, and y the pinned combine of the
  k + 1 rows with the shared row's weight 1.
"""
import numpy as np

import oracle
import synth


def _experts(seed, E, H, F, which):
    return {e: (oracle.quantize_w4(synth.expert_weights(seed, 0, e, synth.PROJ_GATE_UP, 2 * F, H)),
                oracle.quantize_w4(synth.expert_weights(seed, 0, e, synth.PROJ_DOWN, H, F))) for e in which}


def _zero(N, K):
    return (np.zeros((N, K), np.uint8), np.zeros((N, K // 64), np.uint16), np.zeros((N, K // 64), np.uint16))


def test_zero_shared_expert_gives_the_routed_result():
    E, H, F, T, k = 8, 128, 64, 4, 2
    x = synth.activations_bf16(61, 0, T, H)
    lg = synth.router_logits(61, 0, T, E)
    ex = _experts(61, E, H, F, range(E))
    _, _, _, y0 = oracle.moe_forward_w4(x, lg, k, ex)
    _, _, _, y1 = oracle.moe_forward_w4_shared(x, lg, k, ex, (_zero(2 * F, H), _zero(H, F)))
    assert np.array_equal(y0, y1)


def test_zero_routed_experts_give_the_shared_expert():
    E, H, F, T, k = 8, 128, 64, 3, 2
    x = synth.activations_bf16(62, 0, T, H)
    lg = synth.router_logits(62, 0, T, E)
    ex = {e: (_zero(2 * F, H), _zero(H, F)) for e in range(E)}
    sh = _experts(62, 1, H, F, [0])[0]
    _, _, rows, y = oracle.moe_forward_w4_shared(x, lg, k, ex, sh)
    for t in range(T):
        Ys = oracle.expert_ffn_w4(x[t], *sh)
        assert np.array_equal(rows[t, k], Ys)
        assert np.array_equal(y[t], synth.f32_to_bf16_bits(Ys))


def test_rows_and_combine_compose_the_pinned_pieces():
    E, H, F, T, k = 16, 256, 128, 5, 4
    x = synth.activations_bf16(63, 0, T, H)
    lg = synth.router_logits(63, 0, T, E)
    ex = _experts(63, E, H, F, range(E))
    sh = _experts(64, 1, H, F, [0])[0]
    idx, w, rows, y = oracle.moe_forward_w4_shared(x, lg, k, ex, sh)
    ridx, rw = oracle.route(lg, k)
    assert np.array_equal(idx, ridx) and np.array_equal(w, rw)
    for t in range(T):
        for j in range(k):
            assert np.array_equal(rows[t, j], oracle.expert_ffn_w4(x[t], *ex[int(idx[t, j])]))
        assert np.array_equal(rows[t, k], oracle.expert_ffn_w4(x[t], *sh))
        w1 = np.concatenate([w[t], [1.0]]).astype(np.float32)[None, :]
        assert np.array_equal(y[t], oracle.combine(rows[t], w1)[0])
