"""Pins of the oracle's gate delta = exp(softplus(v Delta) * A).

Source: "Trainable Dynamic Mask Sparse Attention" (HF blog), section "Dynamic
Sparse Mask Generation", equation for delta; tau read as softplus, v_j read as
the concatenation of the Hkv value heads.  None of these checks re-types the
oracle's expression: they use library routines (numpy.logaddexp,
scipy.special.expit), closed forms of special cases and brute-force sums.
"""
import math

import numpy as np
import pytest
import scipy.special

import oracle
from workloads import get, make_inputs


def test_softplus_matches_logaddexp():
    x = np.linspace(-60, 60, 2001)
    np.testing.assert_allclose(oracle.softplus(x), np.logaddexp(0.0, x), rtol=1e-15, atol=0)
    assert oracle.softplus(np.array([0.0]))[0] == pytest.approx(math.log(2.0), rel=1e-16)


def test_sigmoid_matches_expit():
    x = np.linspace(-700, 700, 4001)
    np.testing.assert_allclose(oracle.sigmoid(x), scipy.special.expit(x), rtol=1e-14, atol=1e-300)


def _tiny_gate_inputs(seed=0, B=2, Hkv=2, N=5, d=3, H=4):
    rng = np.random.default_rng(seed)
    V = rng.standard_normal((B, Hkv, N, d))
    Delta = rng.standard_normal((Hkv * d, H)) * 0.5
    A = rng.uniform(-1, 0, size=H)
    return V, Delta, A


def test_x_is_brute_force_sum_over_concatenated_heads():
    """x[b,h,j] = sum_g sum_c V[b,g,j,c] * Delta[g*d+c, h], by explicit loops."""
    V, Delta, A = _tiny_gate_inputs()
    B, Hkv, N, d = V.shape
    H = Delta.shape[1]
    x, _ = oracle.gate(V, Delta, A)
    for b in range(B):
        for h in range(H):
            for j in range(N):
                acc = 0.0
                for g in range(Hkv):
                    for c in range(d):
                        acc += V[b, g, j, c] * Delta[g * d + c, h]
                assert x[b, h, j] == pytest.approx(acc, rel=1e-13, abs=1e-15)


def test_zero_delta_weights_give_two_to_the_A():
    """Delta = 0 -> x = 0 -> softplus(0) = ln 2 -> delta = exp(A ln 2) = 2^A."""
    V, Delta, A = _tiny_gate_inputs()
    _, delta = oracle.gate(V, np.zeros_like(Delta), A)
    np.testing.assert_allclose(delta, np.broadcast_to((2.0 ** A)[None, :, None], delta.shape), rtol=1e-15)


def test_A_zero_gives_one():
    V, Delta, A = _tiny_gate_inputs()
    _, delta = oracle.gate(V, Delta, np.zeros_like(A))
    assert np.all(delta == 1.0)


def test_A_minus_one_is_logistic():
    """exp(-ln(1+e^x)) = 1/(1+e^x) = expit(-x)."""
    V, Delta, A = _tiny_gate_inputs(seed=3)
    x, delta = oracle.gate(V, Delta, -np.ones_like(A))
    np.testing.assert_allclose(delta, scipy.special.expit(-x), rtol=1e-14)


def test_A_minus_two_is_squared_logistic():
    V, Delta, A = _tiny_gate_inputs(seed=4)
    x, delta = oracle.gate(V, Delta, -2.0 * np.ones_like(A))
    np.testing.assert_allclose(delta, scipy.special.expit(-x) ** 2, rtol=1e-13)


def test_large_x_limit():
    """For x >> 0 softplus(x) -> x, so delta -> exp(A x)."""
    V = np.zeros((1, 1, 1, 1))
    V[0, 0, 0, 0] = 1.0
    Delta = np.array([[50.0, 80.0]])
    A = np.array([-0.25, -0.5])
    x, delta = oracle.gate(V, Delta, A)
    np.testing.assert_allclose(delta[0, :, 0], np.exp(A * np.array([50.0, 80.0])), rtol=1e-15)


def test_head_concatenation_and_index_roles():
    """A single non-zero value entry V[b,g,j,c] = 1 makes x[b,h,j] equal to the
    Delta row g*d+c and leaves every other position at 0 (catches a transposed
    Delta or a wrong head/channel pairing)."""
    B, Hkv, N, d, H = 2, 3, 4, 5, 6
    rng = np.random.default_rng(7)
    Delta = rng.standard_normal((Hkv * d, H))
    A = -np.ones(H)
    for (b, g, j, c) in [(0, 0, 0, 0), (1, 2, 3, 4), (0, 1, 2, 3), (1, 0, 1, 2)]:
        V = np.zeros((B, Hkv, N, d))
        V[b, g, j, c] = 1.0
        x, _ = oracle.gate(V, Delta, A)
        expect = np.zeros((B, H, N))
        expect[b, :, j] = Delta[g * d + c, :]
        np.testing.assert_array_equal(x, expect)


def test_range_for_nonpositive_A_on_workloads():
    """A in [-1, 0] and softplus >= 0 give delta in (0, 1]."""
    for name in ("tiny", "prefill"):
        I = make_inputs(get(name))
        _, delta = oracle.gate(I.V, I.Delta, I.A)
        assert np.all(delta > 0) and np.all(delta <= 1)


def test_float32_gemm_close_to_float64():
    I = make_inputs(get("tiny"))
    _, d64 = oracle.gate(I.V, I.Delta, I.A)
    _, d32 = oracle.gate(I.V, I.Delta, I.A, gemm_dtype=np.float32)
    np.testing.assert_allclose(d32, d64, rtol=1e-6)
