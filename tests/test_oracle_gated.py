"""Pins of the oracle's gated form, S_t = g_t (I - alpha_t k_t k_t^T) S_{t-1} + alpha_t k_t v_t^T.

The pages name Gated DeltaNet among the baselines ("Exact Flow Linear Attention", technical
summary, Experimental Results) without printing its equations; the reading is Gated DeltaNet's
gate placement, a per-token decay g_t in (0, 1] on the previous state's transition, with EFLA's
coefficient alpha_t (Methodology 3).  What fixes it, independently of the oracle's code:

  - g = 1 is EFLA itself (bit for bit, both rules);
  - a literal matrix loop of the formula (numpy, the matrices built in full);
  - k = 0 is a pure decay, S_t = g_t S_{t-1}, o_t = S_t^T q_t;
  - the gate then the exact flow: the step equals an RK4 integration of the EFLA ODE
    dS/dtau = -beta (k k^T S - k v^T) over unit time started from g S_{t-1} (Methodology 1);
  - the contraction invariants: k^T S_t = g e^{-beta lambda} k^T S_{t-1} + (1 - e^{-beta lambda})
    v^T and u^T S_t = g u^T S_{t-1} for u orthogonal to k (Key Contributions, the memory along
    k contracts by e^{-beta lambda});
  - the scalar case's fixed point under constant inputs;
  - the chunkwise (WY/UT) restatement with cumulative decays, which the kernels evaluate,
    against the token loop to 1e-12.
Mutations of the gate's placement each fail one of these.
"""
import math

import numpy as np
import pytest

import oracle


def _rand(seed, B=1, H=2, L=40, dk=6, dv=5, gmin=0.3):
    rng = np.random.default_rng(seed)
    q = rng.normal(size=(B, H, L, dk))
    k = rng.normal(size=(B, H, L, dk)) * rng.uniform(0.2, 1.5, size=(B, H, L, 1))
    v = rng.normal(size=(B, H, L, dv))
    beta = rng.uniform(0.05, 1.0, size=(B, H, L))
    g = rng.uniform(gmin, 1.0, size=(B, H, L))
    S0 = rng.normal(size=(B, H, dk, dv)) * 0.3
    return q, k, v, beta, g, S0


def _alpha(lam, beta):
    return beta if lam == 0.0 else -math.expm1(-beta * lam) / lam


def _literal(q, k, v, beta, g, S0, gate_on_input=False, drop_gate=False):
    """The formula with the matrices built in full (test-side, independent of the oracle)."""
    L, dk = k.shape
    S = S0.copy()
    o = np.zeros((L, v.shape[1]))
    for t in range(L):
        lam = float(k[t] @ k[t])
        a = _alpha(lam, beta[t])
        M = np.eye(dk) - a * np.outer(k[t], k[t])
        gt = 1.0 if drop_gate else g[t]
        if gate_on_input:
            S = gt * (M @ S + a * np.outer(k[t], v[t]))
        else:
            S = gt * (M @ S) + a * np.outer(k[t], v[t])
        o[t] = S.T @ q[t]
    return o, S


@pytest.mark.parametrize("rule", ["exact", "euler"])
def test_gate_one_is_efla_bit_for_bit(rule):
    q, k, v, beta, g, S0 = _rand(1)
    o1, S1 = oracle.fwd(q, k, v, beta, S0, rule=rule)
    o2, S2 = oracle.fwd(q, k, v, beta, S0, rule=rule, g=np.ones_like(beta))
    assert np.array_equal(o1, o2) and np.array_equal(S1, S2)


def test_matches_literal_matrix_loop():
    q, k, v, beta, g, S0 = _rand(2, B=1, H=3, L=60)
    o, S = oracle.fwd(q, k, v, beta, S0, g=g)
    for h in range(3):
        ol, Sl = _literal(q[0, h], k[0, h], v[0, h], beta[0, h], g[0, h], S0[0, h])
        assert np.abs(o[0, h] - ol).max() <= 1e-12 * max(1.0, np.abs(ol).max())
        assert np.abs(S[0, h] - Sl).max() <= 1e-12 * max(1.0, np.abs(Sl).max())


def test_zero_keys_are_a_pure_decay():
    q, k, v, beta, g, S0 = _rand(3, L=30)
    k = np.zeros_like(k)
    o, S = oracle.fwd(q, k, v, beta, S0, g=g)
    cum = np.cumprod(g, axis=-1)  # [B, H, L]
    for h in range(2):
        for t in range(30):
            St = cum[0, h, t] * S0[0, h]
            assert np.allclose(o[0, h, t], St.T @ q[0, h, t], rtol=1e-13, atol=1e-15)
        assert np.allclose(S[0, h], cum[0, h, -1] * S0[0, h], rtol=1e-13, atol=1e-15)


def _rk4_flow(S, k, v, beta, n=2000):
    """dS/dtau = -beta (k k^T S - k v^T) over tau in [0, 1] (test-side integrator)."""
    A = np.outer(k, k)
    b = np.outer(k, v)
    f = lambda X: -beta * (A @ X - b)
    h = 1.0 / n
    for _ in range(n):
        k1 = f(S); k2 = f(S + 0.5 * h * k1); k3 = f(S + 0.5 * h * k2); k4 = f(S + h * k3)
        S = S + h / 6.0 * (k1 + 2 * k2 + 2 * k3 + k4)
    return S


def test_step_is_the_decay_then_the_exact_flow():
    rng = np.random.default_rng(4)
    for trial in range(5):
        dk, dv = 5, 4
        S = rng.normal(size=(dk, dv))
        k, v, q = rng.normal(size=dk), rng.normal(size=dv), rng.normal(size=dk)
        beta, g = rng.uniform(0.1, 1.2), rng.uniform(0.2, 1.0)
        St, o, _ = oracle.step(S, q, k, v, beta, g=g)
        ref = _rk4_flow(g * S, k, v, beta)
        assert np.abs(St - ref).max() <= 1e-10 * max(1.0, np.abs(ref).max())
        assert np.allclose(o, St.T @ q, rtol=1e-13, atol=1e-14)


def test_contraction_invariants():
    rng = np.random.default_rng(5)
    dk, dv = 7, 3
    for trial in range(10):
        S = rng.normal(size=(dk, dv))
        k, v, q = rng.normal(size=dk), rng.normal(size=dv), rng.normal(size=dk)
        beta, g = rng.uniform(0.05, 2.0), rng.uniform(0.1, 1.0)
        St, _, _ = oracle.step(S, q, k, v, beta, g=g)
        lam = float(k @ k)
        e = math.exp(-beta * lam)
        assert np.allclose(k @ St, g * e * (k @ S) + (1 - e) * v, rtol=1e-12, atol=1e-12)
        u = rng.normal(size=dk)
        u -= (u @ k) / lam * k
        assert np.allclose(u @ St, g * (u @ S), rtol=1e-12, atol=1e-12)


def test_scalar_fixed_point():
    """d = 1 with constant inputs: s_t = g (1 - alpha k^2) s_{t-1} + alpha k v converges to
    s* = alpha k v / (1 - g (1 - alpha k^2))."""
    L = 400
    k, v, beta, g = 1.3, 0.7, 0.4, 0.9
    q = np.ones((1, 1, L, 1))
    o, S = oracle.fwd(q, np.full((1, 1, L, 1), k), np.full((1, 1, L, 1), v), np.full((1, 1, L), beta),
                      None, g=np.full((1, 1, L), g))
    a = _alpha(k * k, beta)
    s_star = a * k * v / (1 - g * (1 - a * k * k))
    assert abs(S[0, 0, 0, 0] - s_star) <= 1e-12
    assert abs(o[0, 0, -1, 0] - s_star) <= 1e-12


def chunk_gated(q, k, v, beta, g, S0, C):
    """The chunkwise (WY/UT) form of the gated recurrence on one head, fp64 (test-side
    restatement of the algebra the kernels evaluate).  Within a chunk entered with state S, with
    l_t the cumulative log-decay to token t (l_0 = 0 at the chunk start) and Gam_ts = e^{l_t - l_s}:
        A    = strictly-lower(diag(alpha) (Gam o K K^T))          T = (I + A)^{-1}
        U'   = T diag(alpha) V - T diag(alpha e^{l}) K S
        O    = diag(e^{l}) Q S + (lower-incl(Gam) o Q K^T) U'
        S   <- e^{l_C} S + K^T diag(e^{l_C - l}) U'
    """
    L = k.shape[0]
    S = S0.copy()
    o = np.zeros((L, v.shape[1]))
    for c0 in range(0, L, C):
        sl = slice(c0, min(L, c0 + C))
        Q, K, V, b, gg = q[sl], k[sl], v[sl], beta[sl], g[sl]
        n = K.shape[0]
        a = np.array([_alpha(float(K[t] @ K[t]), b[t]) for t in range(n)])
        lcum = np.cumsum(np.log(gg))
        Gam = np.exp(lcum[:, None] - lcum[None, :])
        A = np.tril(a[:, None] * Gam * (K @ K.T), -1)
        T = np.linalg.inv(np.eye(n) + A)
        U = T @ (a[:, None] * V) - T @ ((a * np.exp(lcum))[:, None] * K) @ S
        O = np.exp(lcum)[:, None] * (Q @ S) + (np.tril(Gam) * (Q @ K.T)) @ U
        S = np.exp(lcum[-1]) * S + K.T @ (np.exp(lcum[-1] - lcum)[:, None] * U)
        o[sl] = O
    return o, S


@pytest.mark.parametrize("C", [4, 8, 16])
@pytest.mark.parametrize("gmin", [0.9, 0.3, 0.01])
def test_chunk_form_matches_token_loop(C, gmin):
    q, k, v, beta, g, S0 = _rand(6 + C, B=1, H=2, L=53, dk=8, dv=6, gmin=gmin)
    k[0, 1, 10] = 0.0  # a zero key
    k[0, 1, 20] *= 6.0  # a stiff one
    o, S = oracle.fwd(q, k, v, beta, S0, g=g)
    for h in range(2):
        oc, Sc = chunk_gated(q[0, h], k[0, h], v[0, h], beta[0, h], g[0, h], S0[0, h], C)
        assert np.abs(oc - o[0, h]).max() <= 1e-12 * max(1.0, np.abs(o[0, h]).max())
        assert np.abs(Sc - S[0, h]).max() <= 1e-12 * max(1.0, np.abs(S[0, h]).max())


def test_gate_placement_mutations_fail_a_pin():
    """The gate on the input term too, or no gate at all, breaks the contraction invariant or
    the literal loop's agreement with the oracle."""
    rng = np.random.default_rng(7)
    dk, dv = 6, 4
    S = rng.normal(size=(dk, dv))
    k, v, q = rng.normal(size=dk), rng.normal(size=dv), rng.normal(size=dk)
    beta, g = 0.7, 0.6
    lam = float(k @ k)
    e = math.exp(-beta * lam)
    for mut in (dict(gate_on_input=True), dict(drop_gate=True)):
        _, Sm = _literal(q[None], k[None], v[None], [beta], [g], S, **mut)
        assert not np.allclose(k @ Sm, g * e * (k @ S) + (1 - e) * v, rtol=1e-6, atol=1e-6)
