"""Pins of the fp64 oracle's primitives against closed forms, hand-worked
values, invariants and independent library routines (CPU only).

Each test is chosen so that a plausible slip in the oracle (a dropped term,
a wrong sign or index, a transposed operand, a wrong order of update and
readout) fails it.
"""
import json
import math
import os

import numpy as np
import pytest

import oracle
from attention_decode_megakernel_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# ---------------------------------------------------------------- bf16 ----

def test_bf16_rounding_hand_values():
    for x, bits in _golden("bf16_rounding.json")["cases"]:
        assert oracle.bf16_round(x) == int(bits, 16), (x, bits)


def test_bf16_roundtrip_exact():
    rng = np.random.default_rng(0)
    b = rng.integers(0, 0x7F00, size=2000).astype(np.uint16)
    b = b[(b & 0x7F80) != 0]                  # normal numbers only
    for v in b[:500]:
        assert oracle.bf16_round(oracle.bf16_value(v)) == v


# ------------------------------------------------------------- scalars ----

def test_scalar_functions_closed_forms():
    assert oracle.sigmoid(0.0) == 0.5
    assert oracle.softplus(0.0) == pytest.approx(math.log(2.0), rel=1e-15)
    assert oracle.silu(0.0) == 0.0
    for x in (-7.5, -1.0, 0.3, 2.0, 11.0):
        assert oracle.sigmoid(x) + oracle.sigmoid(-x) == pytest.approx(1.0, abs=1e-15)
        assert oracle.softplus(x) - oracle.softplus(-x) == pytest.approx(x, abs=1e-12)
        assert oracle.silu(x) == pytest.approx(x / (1.0 + math.exp(-x)), rel=1e-14)
    assert oracle.softplus(40.0) == pytest.approx(40.0, rel=1e-15)
    assert oracle.silu(40.0) == pytest.approx(40.0, rel=1e-15)


# ---------------------------------------------------------------- gemv ----

def test_gemv_matches_numpy_matmul():
    rng = np.random.default_rng(1)
    W = synth.f32_to_bf16_bits(rng.standard_normal((37, 300), dtype=np.float32))
    x = rng.standard_normal(300)
    ref = synth.bf16_bits_to_f32(W).astype(np.float64) @ x
    np.testing.assert_allclose(oracle.gemv(W, x), ref, rtol=1e-12, atol=1e-12)


def test_gemv_is_row_times_vector_not_transposed():
    # W = [[1, 2, 0], [0, 0, 4]] -> W x for x = e_1 is the first column (1, 0)
    W = synth.f32_to_bf16_bits(np.array([[1, 2, 0], [0, 0, 4]], np.float32))
    np.testing.assert_array_equal(oracle.gemv(W, np.array([1.0, 0, 0])), [1.0, 0.0])
    np.testing.assert_array_equal(oracle.gemv(W, np.array([0, 0, 1.0])), [0.0, 4.0])


# ------------------------------------------------------------- norms ------

def test_rmsnorm_closed_form_and_gain():
    y = oracle.rmsnorm([3.0, 4.0], eps=0.0)
    np.testing.assert_allclose(y, np.array([3.0, 4.0]) / math.sqrt(12.5), rtol=1e-15)
    y = oracle.rmsnorm([3.0, 4.0], eps=1e-6)
    np.testing.assert_allclose(y, np.array([3.0, 4.0]) / math.sqrt(12.5 + 1e-6), rtol=1e-15)
    g = synth.f32_to_bf16_bits(np.array([2.0, -0.5], np.float32))
    y = oracle.rmsnorm([3.0, 4.0], g, eps=0.0)
    np.testing.assert_allclose(y, np.array([6.0, -2.0]) / math.sqrt(12.5), rtol=1e-15)


def test_rmsnorm_unit_rms_and_scale_invariance():
    x = np.random.default_rng(2).standard_normal(1024) * 3.0
    y = oracle.rmsnorm(x, eps=0.0)
    assert math.sqrt(np.mean(y * y)) == pytest.approx(1.0, rel=1e-14)
    np.testing.assert_allclose(oracle.rmsnorm(17.0 * x, eps=0.0), y, rtol=1e-13)


def test_l2norm_unit_length_same_direction():
    x = np.random.default_rng(3).standard_normal(128)
    y = oracle.l2norm(x, eps=0.0)
    assert np.linalg.norm(y) == pytest.approx(1.0, rel=1e-14)
    assert np.dot(x, y) == pytest.approx(np.linalg.norm(x), rel=1e-14)
    y = oracle.l2norm([3.0, 4.0], eps=1e-6)
    np.testing.assert_allclose(y, np.array([3.0, 4.0]) / math.sqrt(25.0 + 1e-6), rtol=1e-15)


# ---------------------------------------------------------------- conv ----

def _bf(a):
    return synth.f32_to_bf16_bits(np.asarray(a, np.float32))


def test_conv_hand_values_taps_1234():
    # one channel, taps (1,2,3,4); input u_t = t+1.  Tap K-1 multiplies the
    # current input, tap 0 the input three steps back; zeros before t=0.
    w = _bf([[1.0, 2.0, 3.0, 4.0]])
    st = np.zeros((1, 3))
    expect_pre = [4.0, 3 + 8.0, 2 + 6 + 12.0, 1 + 4 + 9 + 16.0, 2 + 6 + 12 + 20.0]
    for t, e in enumerate(expect_pre):
        out = oracle.conv_step(w, st, [t + 1.0])
        assert out[0] == pytest.approx(oracle.silu(e), rel=1e-15)
    np.testing.assert_array_equal(st[0], [3.0, 4.0, 5.0])


def test_conv_one_hot_tap_is_pure_delay():
    rng = np.random.default_rng(4)
    ch = 5
    w = np.zeros((ch, 4), np.float32)
    w[:, 0] = 1.0                        # oldest tap only: delay of 3 steps
    w = _bf(w)
    st = np.zeros((ch, 3))
    us = rng.standard_normal((9, ch))
    for t in range(9):
        out = oracle.conv_step(w, st, us[t])
        expect = np.zeros(ch) if t < 3 else us[t - 3]
        np.testing.assert_allclose(out, [oracle.silu(e) for e in expect], rtol=1e-15)


# ---------------------------------------------------------- delta rule ----

def _rand_state(rng, dv, dk, scale=0.3):
    return rng.standard_normal((dv, dk)) * scale


def test_delta_rule_golden_2x2():
    g = _golden("delta_rule_2x2.json")
    S = np.array(g["S"], dtype=np.float64)
    o = oracle.delta_step(S, g["q"], g["k"], g["v"], g["alpha"], g["beta"])
    np.testing.assert_array_equal(S, np.array(g["S_next"]))
    np.testing.assert_array_equal(o, np.array(g["o"]))


def test_delta_rule_beta0_alpha1_keeps_state_bitwise():
    rng = np.random.default_rng(5)
    S = _rand_state(rng, 16, 16)
    S0 = S.copy()
    q = rng.standard_normal(16)
    o = oracle.delta_step(S, q, oracle.l2norm(rng.standard_normal(16)),
                          rng.standard_normal(16), 1.0, 0.0)
    np.testing.assert_array_equal(S, S0)
    np.testing.assert_allclose(o, S0 @ q, rtol=1e-13, atol=1e-15)


@pytest.mark.parametrize("alpha,beta", [(1.0, 1.0), (0.7, 0.25), (0.93, 0.6)])
def test_delta_rule_action_on_k_and_its_complement(alpha, beta):
    """For unit k the update is fixed by its action on k and on k-perp:
    S_t k = alpha (1-beta) S k + beta v  and  S_t x = alpha S x for x . k = 0."""
    rng = np.random.default_rng(6)
    dk, dv = 12, 9
    S = _rand_state(rng, dv, dk)
    S_old = S.copy()
    k = oracle.l2norm(rng.standard_normal(dk), eps=0.0)
    v = rng.standard_normal(dv)
    x = rng.standard_normal(dk)
    x -= np.dot(x, k) * k                       # x orthogonal to k
    oracle.delta_step(S, x, k, v, alpha, beta)
    np.testing.assert_allclose(S @ k, alpha * (1 - beta) * (S_old @ k) + beta * v,
                               rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(S @ x, alpha * (S_old @ x), rtol=1e-12, atol=1e-13)


def test_delta_rule_readout_uses_updated_state():
    rng = np.random.default_rng(7)
    dk = dv = 8
    S = _rand_state(rng, dv, dk)
    S_old = S.copy()
    k = oracle.l2norm(rng.standard_normal(dk), eps=0.0)
    v = rng.standard_normal(dv)
    o = oracle.delta_step(S, k, k, v, 0.8, 0.4)          # q = k
    np.testing.assert_allclose(o, 0.8 * 0.6 * (S_old @ k) + 0.4 * v,
                               rtol=1e-12, atol=1e-13)


def test_delta_rule_orthonormal_writes_are_recalled_exactly():
    """alpha=1, beta=1 with orthonormal keys: after writing (k_i, v_i) for all
    i, S k_i = v_i for every i (later writes do not disturb earlier keys)."""
    rng = np.random.default_rng(8)
    dk, dv, m = 32, 16, 20
    Q, _ = np.linalg.qr(rng.standard_normal((dk, dk)))
    keys = Q[:, :m].T
    vals = rng.standard_normal((m, dv))
    S = _rand_state(rng, dv, dk)
    for i in range(m):
        oracle.delta_step(S, keys[i], keys[i], vals[i], 1.0, 1.0)
    for i in range(m):
        np.testing.assert_allclose(S @ keys[i], vals[i], rtol=0, atol=1e-12)


def test_delta_rule_pure_decay_closed_form():
    rng = np.random.default_rng(9)
    S = _rand_state(rng, 6, 6)
    S0 = S.copy()
    k = oracle.l2norm(rng.standard_normal(6), eps=0.0)
    for _ in range(10):
        oracle.delta_step(S, k, k, rng.standard_normal(6), 0.9, 0.0)
    np.testing.assert_allclose(S, 0.9 ** 10 * S0, rtol=1e-13)


def test_delta_sequence_matches_unrolled_matrix_product_form():
    """Brute force in matrix form: S_T = S_0 prod_t A_t + sum_t beta_t v_t k_t^T
    prod_{r>t} A_r with A_t = alpha_t (I - beta_t k_t k_t^T)."""
    rng = np.random.default_rng(10)
    dk, dv, T = 5, 4, 7
    S0 = _rand_state(rng, dv, dk)
    ks = np.stack([oracle.l2norm(rng.standard_normal(dk), eps=0.0) for _ in range(T)])
    qs = rng.standard_normal((T, dk))
    vs = rng.standard_normal((T, dv))
    al = rng.uniform(0.5, 1.0, T)
    be = rng.uniform(0.0, 1.0, T)
    A = [al[t] * (np.eye(dk) - be[t] * np.outer(ks[t], ks[t])) for t in range(T)]
    S = S0.copy()
    o = oracle.delta_sequence(S, qs, ks, vs, al, be)
    ref = S0.copy()
    for t in range(T):
        ref = ref @ A[t] + be[t] * np.outer(vs[t], ks[t])
        np.testing.assert_allclose(o[t], ref @ qs[t], rtol=1e-11, atol=1e-12)
    # the same S_T written as one sum of products
    total = S0.copy()
    for t in range(T):
        total = total @ A[t]
    for t in range(T):
        P = np.eye(dk)
        for r in range(t + 1, T):
            P = P @ A[r]
        total += be[t] * np.outer(vs[t], ks[t]) @ P
    np.testing.assert_allclose(S, total, rtol=1e-11, atol=1e-12)


# ---------------------------------------------------------------- rope ----

def test_rope_hand_values():
    env = {"cos": math.cos, "sin": math.sin}
    for case in _golden("rope_hand_values.json")["cases"]:
        y = oracle.rope(case["x"], case["pos"], case["theta"])
        expect = [eval(e, env) for e in case["expect"]]
        np.testing.assert_allclose(y, expect, rtol=1e-14, atol=1e-15)


def test_rope_identity_at_zero_and_norm_preserving():
    x = np.random.default_rng(11).standard_normal(256)
    np.testing.assert_array_equal(oracle.rope(x, 0, 1e7), x)
    for pos in (1, 17, 4095, 32767):
        assert np.linalg.norm(oracle.rope(x, pos, 1e7)) == pytest.approx(
            np.linalg.norm(x), rel=1e-13)


def test_rope_scores_depend_only_on_relative_position():
    rng = np.random.default_rng(12)
    q, k = rng.standard_normal(64), rng.standard_normal(64)
    d1 = np.dot(oracle.rope(q, 5, 1e4), oracle.rope(k, 2, 1e4))
    d2 = np.dot(oracle.rope(q, 133, 1e4), oracle.rope(k, 130, 1e4))
    assert d1 == pytest.approx(d2, rel=1e-11)


# ------------------------------------------------------------ softmax -----

def test_softmax_sum_shift_and_two_point_form():
    s = np.random.default_rng(13).standard_normal(50) * 5
    p = oracle.softmax(s)
    assert p.sum() == pytest.approx(1.0, abs=1e-15)
    np.testing.assert_allclose(oracle.softmax(s + 123.0), p, rtol=1e-12)
    p2 = oracle.softmax([0.3, -1.1])
    assert p2[0] == pytest.approx(oracle.sigmoid(1.4), rel=1e-15)


# ---------------------------------------------------------- attention -----

def test_attention_single_key_returns_its_value():
    rng = np.random.default_rng(14)
    V = rng.standard_normal((1, 16))
    o = oracle.attention_head(rng.standard_normal(16), rng.standard_normal((1, 16)), V)
    np.testing.assert_allclose(o, V[0], rtol=1e-15)


def test_attention_zero_query_is_mean_of_values():
    rng = np.random.default_rng(15)
    V = rng.standard_normal((9, 16))
    o = oracle.attention_head(np.zeros(16), rng.standard_normal((9, 16)), V)
    np.testing.assert_allclose(o, V.mean(axis=0), rtol=1e-13)


def test_attention_two_keys_closed_form_with_scale():
    rng = np.random.default_rng(16)
    hd = 16
    q, K, V = rng.standard_normal(hd), rng.standard_normal((2, hd)), rng.standard_normal((2, hd))
    s = K @ q / math.sqrt(hd)
    w0 = 1.0 / (1.0 + math.exp(-(s[0] - s[1])))
    np.testing.assert_allclose(oracle.attention_head(q, K, V), w0 * V[0] + (1 - w0) * V[1],
                               rtol=1e-13)
