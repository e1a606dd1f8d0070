"""Pins for the oracle's KV compression (softmax-gated per-channel pooling).

Compression rule: blog.nickys.cn/?p=150 section "1. CSA" (m tokens -> one entry)
with the gate weights exp(Z[i] + B[i mod m]) of the method's specification.
"""
import json
import math
import os

import numpy as np
import pytest

import oracle

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def words(x):
    return oracle.to_bf16_words(np.asarray(x, np.float64))


def test_bf16_rounding_helper_is_rne():
    # 1 + 2^-8 is a tie between 1 and 1 + 2^-7: even mantissa wins (1.0).
    assert oracle.bf16_words_to_f64(words([1 + 2 ** -8]))[0] == 1.0
    # 1 + 3*2^-8 ties between 1+2^-7 (odd) and 1+2^-6 (even): rounds up.
    assert oracle.bf16_words_to_f64(words([1 + 3 * 2 ** -8]))[0] == 1 + 2 ** -6
    assert oracle.bf16_words_to_f64(words([-2.5]))[0] == -2.5


def test_hand_example_equal_weights():
    g = json.load(open(os.path.join(GOLD, "hand_compress_attention.json")))
    K = words(np.array(g["K"]).reshape(4, 1))
    V = words(np.array(g["V"]).reshape(4, 1))
    Z = words(np.zeros((4, 1)))
    Kc, Vc = oracle.compress(K, V, Z, np.zeros((2, 1), np.float32), 2)
    np.testing.assert_array_equal(Kc[:, 0], g["Z_zero"]["Kc"])
    np.testing.assert_array_equal(Vc[:, 0], g["Z_zero"]["Vc"])


def test_hand_example_bias_by_position_in_block():
    g = json.load(open(os.path.join(GOLD, "hand_compress_attention.json")))
    K = words(np.array(g["K"]).reshape(4, 1))
    V = words(np.array(g["V"]).reshape(4, 1))
    Z = words(np.zeros((4, 1)))
    B = np.array(g["B_ln3"]["B"], np.float32).reshape(2, 1)
    Kc, Vc = oracle.compress(K, V, Z, B, 2)
    # B is float32(ln 3): weights 3/4, 1/4 up to float32 rounding of ln 3.
    np.testing.assert_allclose(Kc[:, 0], g["B_ln3"]["Kc"], rtol=1e-7)
    np.testing.assert_allclose(Vc[:, 0], g["B_ln3"]["Vc"], rtol=1e-7)


def test_m1_is_identity():
    rng = np.random.default_rng(0)
    K = words(rng.standard_normal((37, 8)))
    V = words(rng.standard_normal((37, 8)))
    Z = words(rng.standard_normal((37, 8)))
    B = rng.standard_normal((1, 8)).astype(np.float32)
    Kc, Vc = oracle.compress(K, V, Z, B, 1)
    np.testing.assert_array_equal(Kc, oracle.bf16_words_to_f64(K))
    np.testing.assert_array_equal(Vc, oracle.bf16_words_to_f64(V))


def test_constant_gate_gives_block_mean():
    rng = np.random.default_rng(1)
    T, d, m = 64, 16, 8
    K = words(rng.standard_normal((T, d)))
    V = words(rng.standard_normal((T, d)))
    Z = words(np.full((T, d), 0.75))
    Kc, Vc = oracle.compress(K, V, Z, np.zeros((m, d), np.float32), m)
    Kf = oracle.bf16_words_to_f64(K).reshape(T // m, m, d).mean(axis=1)
    Vf = oracle.bf16_words_to_f64(V).reshape(T // m, m, d).mean(axis=1)
    np.testing.assert_allclose(Kc, Kf, rtol=0, atol=1e-14)
    np.testing.assert_allclose(Vc, Vf, rtol=0, atol=1e-14)


def test_weights_are_a_per_channel_softmax_over_the_block():
    """Against the two-point closed form: with m=2 the weight of the first token
    is the logistic function of the gate difference, per channel."""
    rng = np.random.default_rng(2)
    T, d = 16, 4
    K = words(rng.standard_normal((T, d)))
    V = words(rng.standard_normal((T, d)))
    Z = words(rng.standard_normal((T, d)))
    B = rng.standard_normal((2, d)).astype(np.float32) * 0.5
    Kc, Vc = oracle.compress(K, V, Z, B, 2)
    Kf, Vf, Zf = (oracle.bf16_words_to_f64(a) for a in (K, V, Z))
    for j in range(T // 2):
        for c in range(d):
            g0 = Zf[2 * j, c] + B[0, c]
            g1 = Zf[2 * j + 1, c] + B[1, c]
            a0 = 1.0 / (1.0 + math.exp(g1 - g0))
            assert Kc[j, c] == pytest.approx(a0 * Kf[2 * j, c] + (1 - a0) * Kf[2 * j + 1, c], abs=1e-14)
            assert Vc[j, c] == pytest.approx(a0 * Vf[2 * j, c] + (1 - a0) * Vf[2 * j + 1, c], abs=1e-14)


def test_shift_invariance_and_large_logits():
    rng = np.random.default_rng(3)
    T, d, m = 32, 8, 4
    K = words(rng.standard_normal((T, d)))
    V = words(rng.standard_normal((T, d)))
    Zs = rng.integers(-4, 5, (T, d)).astype(np.float64)  # small integers: still exact in bf16 after +64
    B = np.zeros((m, d), np.float32)
    Kc0, Vc0 = oracle.compress(K, V, words(Zs), B, m)
    # a common shift of the gate logits leaves the pooled values unchanged
    Kc1, Vc1 = oracle.compress(K, V, words(Zs + 64.0), B, m)
    np.testing.assert_allclose(Kc1, Kc0, atol=1e-13)
    np.testing.assert_allclose(Vc1, Vc0, atol=1e-13)
    # logits of 4096 overflow exp() unless the block maximum is subtracted first
    Kc2, _ = oracle.compress(K, V, words(np.full((T, d), 4096.0)), B, m)
    np.testing.assert_allclose(Kc2, oracle.bf16_words_to_f64(K).reshape(T // m, m, d).mean(axis=1), atol=1e-14)


def test_convex_combination_bounds_and_trailing_block():
    rng = np.random.default_rng(4)
    T, d, m = 45, 8, 4       # 11 full blocks, 1 trailing token not compressed
    K = words(rng.standard_normal((T, d)) * 3)
    V = words(rng.standard_normal((T, d)))
    Z = words(rng.standard_normal((T, d)) * 2)
    B = (rng.standard_normal((m, d)) * 0.5).astype(np.float32)
    Kc, Vc = oracle.compress(K, V, Z, B, m)
    assert Kc.shape == (11, d)
    Kf = oracle.bf16_words_to_f64(K)[: 44].reshape(11, m, d)
    assert np.all(Kc >= Kf.min(axis=1) - 1e-12) and np.all(Kc <= Kf.max(axis=1) + 1e-12)


def test_gates_shared_by_k_and_v():
    """K and V are pooled with the same weights: pooling V = K returns Kc."""
    rng = np.random.default_rng(5)
    T, d, m = 24, 8, 6
    K = words(rng.standard_normal((T, d)))
    Z = words(rng.standard_normal((T, d)))
    B = (rng.standard_normal((m, d)) * 0.5).astype(np.float32)
    Kc, Vc = oracle.compress(K, K, Z, B, m)
    np.testing.assert_array_equal(Kc, Vc)
