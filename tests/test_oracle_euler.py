"""Pins of the oracle's Euler rule (the delta rule, DeltaNet), which the pages name as the explicit
Euler step of the ODE they integrate exactly.

"Exact Flow Linear Attention: Exact Solution from Continuous-Time Dynamics", technical summary:
Methodology 1 (dS/dt = -A_t S + b_t with A_t = k_t k_t^T and b_t = k_t v_t^T), Key Contributions
("Reinterpretation of Delta-Rule": the delta rule is that ODE's explicit Euler step;
"Theoretical Stability": the exact flow contracts the key direction by e^{-beta lambda}).

Each check uses arithmetic of its own (full matrices, closed forms, a brute-force loop), not the
oracle's.
"""
import math

import numpy as np
import pytest


def _rand(rng, *shape):
    return rng.standard_normal(shape)


def test_euler_coefficient_is_beta(oracle_mod):
    for lam in (0.0, 1e-300, 1e-8, 0.3, 1.0, 7.5, 1e3):
        for beta in (0.0, 1e-6, 0.25, 0.9, 3.0):
            assert oracle_mod.alpha(lam, beta, "euler") == beta


def test_euler_step_is_the_explicit_euler_step_of_the_ode(oracle_mod):
    """S_t = S + beta (b - A S), with A = k k^T and b = k v^T built as full matrices."""
    rng = np.random.default_rng(11)
    for dk, dv in ((5, 3), (8, 8), (1, 4)):
        S = _rand(rng, dk, dv)
        q, k, v = _rand(rng, dk), _rand(rng, dk), _rand(rng, dv)
        beta = 0.37
        A = np.outer(k, k)
        b = np.outer(k, v)
        S_ref = S + beta * (b - A @ S)
        S_t, o_t, a = oracle_mod.step(S, q, k, v, beta, rule="euler")
        assert a == beta
        np.testing.assert_allclose(S_t, S_ref, rtol=0, atol=1e-13)
        np.testing.assert_allclose(o_t, S_ref.T @ q, rtol=0, atol=1e-12)


def test_rules_differ_by_the_coefficient_gap_times_the_residual(oracle_mod):
    """Both rules are S - x (A S - b) with x = alpha or beta, so their difference is exactly
    (beta - alpha)(A S - b) for any inputs, and beta - alpha = beta^2 lambda / 2 + O(beta^3 lambda^2)."""
    rng = np.random.default_rng(12)
    dk, dv = 6, 4
    S = _rand(rng, dk, dv)
    q, k, v = _rand(rng, dk), _rand(rng, dk), _rand(rng, dv)
    lam = float(k @ k)
    for beta in (1e-4, 0.05, 0.8, 2.5):
        S_e, _, a_e = oracle_mod.step(S, q, k, v, beta, rule="exact")
        S_u, _, a_u = oracle_mod.step(S, q, k, v, beta, rule="euler")
        resid = np.outer(k, k) @ S - np.outer(k, v)
        np.testing.assert_allclose(S_e - S_u, (a_u - a_e) * resid, rtol=0,
                                   atol=1e-12 * max(1.0, np.abs(resid).max()))
    beta = 1e-4 / lam  # beta * lambda = 1e-4
    gap = beta - oracle_mod.alpha(lam, beta)
    assert abs(gap / (beta * beta * lam / 2) - 1) < 1e-4


def test_euler_retrieves_the_value_exactly_at_unit_step(oracle_mod):
    """With beta ||k||^2 = 1 the delta rule overwrites the key direction: S_t^T k = v.  The exact
    flow instead moves S^T k a fraction 1 - e^{-1} of the way to v."""
    rng = np.random.default_rng(13)
    dk, dv = 7, 5
    S = _rand(rng, dk, dv)
    q, k, v = _rand(rng, dk), _rand(rng, dk), _rand(rng, dv)
    beta = 1.0 / float(k @ k)
    S_u, _, _ = oracle_mod.step(S, q, k, v, beta, rule="euler")
    np.testing.assert_allclose(S_u.T @ k, v, rtol=0, atol=1e-12)
    S_e, _, _ = oracle_mod.step(S, q, k, v, beta, rule="exact")
    expect = math.exp(-1.0) * (S.T @ k) + (1 - math.exp(-1.0)) * v
    np.testing.assert_allclose(S_e.T @ k, expect, rtol=0, atol=1e-12)


def test_stiff_steps_grow_under_euler_and_contract_under_the_exact_flow(oracle_mod):
    """v = 0 and the same key every token with beta lambda = 3: the key component of the state
    is multiplied by 1 - 3 = -2 per Euler step and by e^{-3} per exact step."""
    rng = np.random.default_rng(14)
    dk, dv, n = 4, 3, 6
    k = _rand(rng, dk)
    lam = float(k @ k)
    beta = 3.0 / lam
    S0 = _rand(rng, dk, dv)
    q = _rand(rng, dk)
    v = np.zeros(dv)
    for rule, factor in (("euler", -2.0), ("exact", math.exp(-3.0))):
        S = S0.copy()
        for _ in range(n):
            S, _, _ = oracle_mod.step(S, q, k, v, beta, rule=rule)
        np.testing.assert_allclose(S.T @ k, factor ** n * (S0.T @ k), rtol=1e-10,
                                   atol=1e-13 * float(np.abs(S0.T @ k).max()))


def test_euler_forward_matches_a_brute_force_delta_rule_loop(oracle_mod):
    rng = np.random.default_rng(15)
    B, H, L, dk, dv = 1, 2, 9, 4, 3
    q, k = _rand(rng, B, H, L, dk), _rand(rng, B, H, L, dk) / 2
    v, beta = _rand(rng, B, H, L, dv), rng.uniform(0.0, 1.0, (B, H, L))
    S0 = _rand(rng, B, H, dk, dv) * 0.1
    o, S = oracle_mod.fwd(q, k, v, beta, S0, rule="euler")
    for b in range(B):
        for h in range(H):
            St = S0[b, h].copy()
            for t in range(L):
                kt, vt = k[b, h, t], v[b, h, t]
                St = St - beta[b, h, t] * np.outer(kt, kt @ St) + beta[b, h, t] * np.outer(kt, vt)
                np.testing.assert_allclose(o[b, h, t], St.T @ q[b, h, t], rtol=0, atol=1e-12)
            np.testing.assert_allclose(S[b, h], St, rtol=0, atol=1e-12)


def test_exact_is_still_the_default(oracle_mod):
    rng = np.random.default_rng(16)
    q, k, v = _rand(rng, 1, 1, 5, 3), _rand(rng, 1, 1, 5, 3), _rand(rng, 1, 1, 5, 2)
    beta = rng.uniform(0.5, 2.0, (1, 1, 5))
    o1, S1 = oracle_mod.fwd(q, k, v, beta)
    o2, S2 = oracle_mod.fwd(q, k, v, beta, rule="exact")
    assert np.array_equal(o1, o2) and np.array_equal(S1, S2)
    with pytest.raises(KeyError):
        oracle_mod.fwd(q, k, v, beta, rule="midpoint")
