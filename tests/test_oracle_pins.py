"""Pins for the fp64 oracle: checks against what the method and the mathematics
fix, independent of the oracle's own code.

Source: "Exact Flow Linear Attention: Exact Solution from Continuous-Time
Dynamics" (technical summary): Methodology 1 (the ZOH ODE dS/dt = -A S + b with
A = k k^T, b = k v^T), Methodology 2 (A^n = lambda^(n-1) A and the closed-form
exponential), Methodology 3 (the update rule and alpha), Key Contributions
("Theoretical Stability": contraction along k by exp(-beta lambda);
"Reinterpretation": the delta rule is the explicit Euler step).

The pages print no worked numeric example, so every pin is a closed form, an
independent integration, a limit, an invariant or brute force.  Each pin is a
function of a `step` callable so that the mutation tests at the bottom can
show that plausible mistakes (Euler alpha, readout before the update, a sign
error, a transposed state) fail at least one pin.
"""
import math
from decimal import Decimal, getcontext

import numpy as np
import pytest

from conftest import rel_err

RNG = np.random.default_rng(20251214)


# --------------------------------------------------------------------------
# independent helpers (no oracle code)
# --------------------------------------------------------------------------
def expm_taylor(M: np.ndarray) -> np.ndarray:
    """exp(M) by scaling-and-squaring around a Taylor series summed to convergence."""
    nrm = np.abs(M).sum(axis=1).max()
    s = max(0, int(math.ceil(math.log2(nrm))) + 1) if nrm > 0.5 else 0
    X = M / (2.0 ** s)
    E = np.eye(M.shape[0])
    term = np.eye(M.shape[0])
    for n in range(1, 60):
        term = term @ X / n
        E = E + term
        if np.abs(term).max() < 1e-18:
            break
    for _ in range(s):
        E = E @ E
    return E


def rk4_token(S, k, v, beta, steps=2000):
    """Integrate dS/dtau = -beta (k k^T S - k v^T) over tau in [0, 1] with RK4.

    This is the ODE dS/dt = -A S + b held for a duration beta (zero-order hold),
    rescaled to unit time."""
    A = np.outer(k, k)
    b = np.outer(k, v)
    f = lambda X: -beta * (A @ X - b)
    h = 1.0 / steps
    X = S.copy()
    for _ in range(steps):
        k1 = f(X)
        k2 = f(X + 0.5 * h * k1)
        k3 = f(X + 0.5 * h * k2)
        k4 = f(X + h * k3)
        X = X + (h / 6.0) * (k1 + 2 * k2 + 2 * k3 + k4)
    return X


def alpha_decimal(lam: float, beta: float) -> float:
    """alpha = (1 - e^{-beta lam})/lam in 800-digit decimal arithmetic (beta at lam = 0).

    800 digits keep 1 - e^{-x} exact to double precision down to x ~ 1e-700."""
    getcontext().prec = 800
    L, Bt = Decimal(lam), Decimal(beta)
    if L == 0:
        return float(Bt)
    return float((1 - (-(Bt * L)).exp()) / L)


# --------------------------------------------------------------------------
# the pins, as functions of a step(S, q, k, v, beta) -> (S_t, o_t, alpha)
# --------------------------------------------------------------------------
def pin_closed_form_exponential(alpha_fn):
    """(a) e^{-beta k k^T} = I - alpha k k^T, checked against scaling-and-squaring Taylor."""
    worst = 0.0
    for d in (1, 2, 3, 5, 8):
        for scale in (1e-3, 0.3, 1.0, 3.0):
            k = RNG.standard_normal(d) * scale
            beta = float(RNG.uniform(0.05, 2.0))
            A = np.outer(k, k)
            lam = float(k @ k)
            E = expm_taylor(-beta * A)
            C = np.eye(d) - alpha_fn(lam, beta) * A
            worst = max(worst, float(np.abs(E - C).max()))
    return worst


def pin_ode(step):
    """(b) one token equals the exact flow of the ODE over the hold interval; o = S_t^T q."""
    worst = 0.0
    for dk, dv in ((1, 1), (3, 2), (8, 5)):
        for knorm in (0.2, 1.0, 2.0):
            S = RNG.standard_normal((dk, dv))
            k = RNG.standard_normal(dk)
            k *= knorm / np.linalg.norm(k)
            v = RNG.standard_normal(dv)
            q = RNG.standard_normal(dk)
            beta = float(RNG.uniform(0.1, 1.0))
            St, o, _ = step(S, q, k, v, beta)
            X = rk4_token(S, k, v, beta)
            worst = max(worst, rel_err(St, X), rel_err(o, X.T @ q))
    return worst


def pin_contraction(step):
    """(d) k^T S_t = e^{-bl} k^T S_{t-1} + (1 - e^{-bl}) v^T, and u^T S_t = u^T S_{t-1} for u _|_ k."""
    worst = 0.0
    for _ in range(20):
        dk, dv = 6, 4
        S = RNG.standard_normal((dk, dv))
        k = RNG.standard_normal(dk) * RNG.uniform(0.1, 2.0)
        v = RNG.standard_normal(dv)
        q = RNG.standard_normal(dk)
        beta = float(RNG.uniform(0.05, 3.0))
        lam = float(k @ k)
        St, _, _ = step(S, q, k, v, beta)
        e = math.exp(-beta * lam)
        worst = max(worst, float(np.abs(k @ St - (e * (k @ S) + (1 - e) * v)).max()))
        u = RNG.standard_normal(dk)
        u -= (u @ k) / lam * k
        worst = max(worst, float(np.abs(u @ St - u @ S).max()))
    return worst


def pin_scalar(step):
    """(g) dk = dv = 1: s' = e^{-b k^2} s + (1 - e^{-b k^2}) v / k, o = s' q (textbook linear ODE)."""
    worst = 0.0
    for _ in range(50):
        s, k, v, q = RNG.standard_normal(4)
        beta = float(RNG.uniform(0.01, 4.0))
        e = math.exp(-beta * k * k)
        ref = e * s + (1 - e) * v / k
        St, o, _ = step(np.array([[s]]), np.array([q]), np.array([k]), np.array([v]), beta)
        worst = max(worst, abs(St[0, 0] - ref) / max(1.0, abs(ref)), abs(o[0] - ref * q) / max(1.0, abs(ref * q)))
    return worst


def pin_euler_limit(step):
    """(c) as beta*lambda -> 0 the exact step approaches the explicit Euler (DeltaNet) step
    S + beta k (v - S^T k)^T, with a gap of second order in beta*lambda."""
    ratios = []
    dk, dv = 5, 3
    S = RNG.standard_normal((dk, dv))
    k0 = RNG.standard_normal(dk)
    k0 /= np.linalg.norm(k0)
    v = RNG.standard_normal(dv)
    q = RNG.standard_normal(dk)
    beta = 0.7
    for eps in (1e-1, 1e-2, 1e-3):
        k = k0 * math.sqrt(eps / beta)  # beta * lambda = eps
        St, _, _ = step(S, q, k, v, beta)
        euler = S + beta * np.outer(k, v - S.T @ k)
        # the difference is (beta - alpha) k (v - S^T k)^T with beta - alpha ~ beta^2 lambda / 2
        gap = np.abs(St - euler).max() / (np.abs(np.outer(k, v - S.T @ k)).max() * beta)
        ratios.append(gap / eps)
    return ratios


def pin_stiff(step):
    """(f) beta*lambda >> 1: alpha -> 1/lambda, and the new value is written exactly along k."""
    worst = 0.0
    for _ in range(10):
        dk, dv = 4, 3
        S = RNG.standard_normal((dk, dv))
        k = RNG.standard_normal(dk)
        k *= 3.0 / np.linalg.norm(k)  # lambda = 9
        v = RNG.standard_normal(dv)
        beta = 8.0  # beta*lambda = 72
        St, _, a = step(S, np.zeros(dk), k, v, beta)
        worst = max(worst, abs(a * 9.0 - 1.0), float(np.abs(k @ St - v).max()))
    return worst


# --------------------------------------------------------------------------
# tests of the oracle against the pins
# --------------------------------------------------------------------------
def _oracle_step(oracle_mod):
    return lambda S, q, k, v, beta: oracle_mod.step(S, q, k, v, beta)


def test_alpha_closed_form_decimal(oracle_mod):
    """alpha against a 60-digit evaluation of (1 - e^{-beta lambda})/lambda, including
    the lambda -> 0 limit, tiny lambda and large beta*lambda.  (Subnormal lambda, below
    ~2e-308, is outside every input here: keys are bf16 or fp32, so lambda >= ~1e-90.)"""
    cases = [(0.0, 0.5), (1e-300, 0.3), (1e-90, 0.9), (1e-12, 0.7), (1e-4, 0.98),
             (0.25, 0.5), (1.0, 1.0), (4.0, 0.73), (100.0, 0.99), (1e4, 0.6), (3.0, 0.0)]
    for lam, beta in cases:
        ref = alpha_decimal(lam, beta)
        got = oracle_mod.alpha(lam, beta)
        assert abs(got - ref) <= 4e-16 * abs(ref) + 1e-300, (lam, beta, got, ref)


def test_power_identity():
    """A^n = lambda^(n-1) A for A = k k^T (Methodology 2), the identity the closed form rests on."""
    for d in (2, 5, 8):
        k = RNG.standard_normal(d)
        A = np.outer(k, k)
        lam = float(k @ k)
        P = A.copy()
        for n in range(2, 7):
            P = P @ A
            assert np.allclose(P, lam ** (n - 1) * A, rtol=1e-12, atol=0)


def test_pin_a_closed_form(oracle_mod):
    assert pin_closed_form_exponential(oracle_mod.alpha) < 1e-13


def test_pin_b_ode(oracle_mod):
    assert pin_ode(_oracle_step(oracle_mod)) < 1e-10


def test_pin_c_euler_limit(oracle_mod):
    ratios = pin_euler_limit(_oracle_step(oracle_mod))
    # gap / (beta lambda) tends to 1/2 (beta - alpha = beta (beta lambda)/2 + O((beta lambda)^2))
    for r, eps in zip(ratios, (1e-1, 1e-2, 1e-3)):
        assert abs(r - 0.5) < eps, ratios
    assert oracle_mod.alpha(1e-9, 0.7) / 0.7 == pytest.approx(1.0, abs=1e-9)


def test_pin_d_contraction(oracle_mod):
    assert pin_contraction(_oracle_step(oracle_mod)) < 1e-12


def test_pin_d_nonexpansive(oracle_mod):
    """||I - alpha k k^T||_2 = 1 for beta >= 0: the eigenvalues are 1 (on k's complement)
    and e^{-beta lambda} (along k)."""
    for _ in range(10):
        k = RNG.standard_normal(6) * RNG.uniform(0.1, 3)
        beta = float(RNG.uniform(0, 5))
        lam = float(k @ k)
        M = np.eye(6) - oracle_mod.alpha(lam, beta) * np.outer(k, k)
        ev = np.sort(np.linalg.eigvalsh(M))
        assert ev[0] == pytest.approx(math.exp(-beta * lam), rel=1e-12, abs=1e-15)
        assert np.allclose(ev[1:], 1.0, atol=1e-13)


def test_pin_f_stiff(oracle_mod):
    assert pin_stiff(_oracle_step(oracle_mod)) < 1e-12


def test_pin_g_scalar(oracle_mod):
    assert pin_scalar(_oracle_step(oracle_mod)) < 1e-13


def test_pin_h_linearity(oracle_mod):
    """o and S_final are jointly linear in (V, S0) for fixed q, k, beta."""
    B, H, L, dk, dv = 1, 2, 23, 6, 5
    q = RNG.standard_normal((B, H, L, dk))
    k = RNG.standard_normal((B, H, L, dk)) * 0.5
    beta = RNG.uniform(0, 1, (B, H, L))
    V1, V2 = RNG.standard_normal((2, B, H, L, dv))
    S1, S2 = RNG.standard_normal((2, B, H, dk, dv))
    a, b = 0.7, -1.3
    o1, F1 = oracle_mod.fwd(q, k, V1, beta, S1)
    o2, F2 = oracle_mod.fwd(q, k, V2, beta, S2)
    o3, F3 = oracle_mod.fwd(q, k, a * V1 + b * V2, beta, a * S1 + b * S2)
    assert rel_err(o3, a * o1 + b * o2) < 1e-12
    assert rel_err(F3, a * F1 + b * F2) < 1e-12


def test_pin_i_padding_and_resume(oracle_mod):
    """Tokens with k = 0 or beta = 0 leave the state unchanged; a split run with the
    state carried across equals one run (the state is the whole memory)."""
    B, H, L, dk, dv = 2, 1, 40, 4, 3
    q = RNG.standard_normal((B, H, L, dk))
    k = RNG.standard_normal((B, H, L, dk))
    v = RNG.standard_normal((B, H, L, dv))
    beta = RNG.uniform(0, 1, (B, H, L))
    S0 = RNG.standard_normal((B, H, dk, dv))
    o, F = oracle_mod.fwd(q, k, v, beta, S0)
    # resume
    oa, Fa = oracle_mod.fwd(q[:, :, :17], k[:, :, :17], v[:, :, :17], beta[:, :, :17], S0)
    ob, Fb = oracle_mod.fwd(q[:, :, 17:], k[:, :, 17:], v[:, :, 17:], beta[:, :, 17:], Fa)
    assert np.array_equal(np.concatenate([oa, ob], axis=2), o)
    assert np.array_equal(Fb, F)
    # padding: insert no-op tokens
    for kill in ("k", "beta"):
        k2, b2 = k.copy(), beta.copy()
        if kill == "k":
            k2[:, :, 5] = 0.0
        else:
            b2[:, :, 5] = 0.0
        _, Fp = oracle_mod.fwd(q[:, :, :6], k2[:, :, :6], v[:, :, :6], b2[:, :, :6], S0)
        _, Fq = oracle_mod.fwd(q[:, :, :5], k[:, :, :5], v[:, :, :5], beta[:, :, :5], S0)
        assert np.array_equal(Fp, Fq)


def test_readout_after_update(oracle_mod):
    """o_t is read from the state that includes token t: o_t = S_t^T q_t, with S_t the
    final state of the prefix run of length t (pins the readout's time index)."""
    B, H, L, dk, dv = 1, 1, 12, 5, 4
    q = RNG.standard_normal((B, H, L, dk))
    k = RNG.standard_normal((B, H, L, dk))
    v = RNG.standard_normal((B, H, L, dv))
    beta = RNG.uniform(0.2, 1, (B, H, L))
    o, _ = oracle_mod.fwd(q, k, v, beta)
    for t in (0, 5, 11):
        _, St = oracle_mod.fwd(q[:, :, :t + 1], k[:, :, :t + 1], v[:, :, :t + 1], beta[:, :, :t + 1])
        assert np.allclose(o[0, 0, t], St[0, 0].T @ q[0, 0, t], rtol=1e-13, atol=1e-14)


def test_fwd_matches_literal_update(oracle_mod):
    """Brute force on tiny inputs: the literal matrix form (I - a k k^T) S + a k v^T with the
    decimal alpha, token by token, equals the oracle's forward pass."""
    B, H, L, dk, dv = 1, 2, 9, 3, 4
    q = RNG.standard_normal((B, H, L, dk))
    k = RNG.standard_normal((B, H, L, dk))
    v = RNG.standard_normal((B, H, L, dv))
    beta = RNG.uniform(0, 1, (B, H, L))
    o, F = oracle_mod.fwd(q, k, v, beta)
    for h in range(H):
        S = np.zeros((dk, dv))
        for t in range(L):
            kt = k[0, h, t]
            a = alpha_decimal(float(kt @ kt), float(beta[0, h, t]))
            S = (np.eye(dk) - a * np.outer(kt, kt)) @ S + a * np.outer(kt, v[0, h, t])
            assert np.allclose(o[0, h, t], S.T @ q[0, h, t], rtol=1e-12, atol=1e-13)
        assert np.allclose(F[0, h], S, rtol=1e-12, atol=1e-13)


# --------------------------------------------------------------------------
# mutation tests: plausible mistakes must fail at least one pin
# --------------------------------------------------------------------------
def _mut_step(kind):
    def step(S, q, k, v, beta):
        lam = float(k @ k)
        a = beta if kind == "euler" else (-math.expm1(-beta * lam) / lam if lam else beta)
        if kind == "alpha_no_lambda":
            a = -math.expm1(-beta * lam)
        x = S.T @ k
        if kind == "sign":
            St = S + a * np.outer(k, -v - x)
        elif kind == "drop_forcing":
            St = S - a * np.outer(k, x)
        else:
            St = S + a * np.outer(k, v - x)
        o = St.T @ q
        if kind == "readout_before":
            o = S.T @ q
        elif kind == "readout_with_k":
            o = St.T @ k
        return St, o, a
    return step


@pytest.mark.parametrize("kind", ["euler", "alpha_no_lambda", "sign", "drop_forcing",
                                  "readout_before", "readout_with_k"])
def test_pins_reject_mutants(kind):
    step = _mut_step(kind)
    caught = (pin_ode(step) > 1e-6 or pin_contraction(step) > 1e-6
              or pin_scalar(step) > 1e-6 or pin_stiff(step) > 1e-6)
    assert caught, kind


def test_pins_accept_reference_python_step():
    """The mutation harness itself: its unmutated step passes every pin."""
    step = _mut_step("none")
    assert pin_ode(step) < 1e-10
    assert pin_contraction(step) < 1e-12
    assert pin_scalar(step) < 1e-13
    assert pin_stiff(step) < 1e-12
