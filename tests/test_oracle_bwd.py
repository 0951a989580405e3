"""Pins of the oracle's backward pass (reverse mode through the token recurrence of "Exact Flow
Linear Attention", technical summary, Methodology 3, and through the delta rule's Euler step).

The loss is L = sum(o * Wo) + sum(S_final * WS) with fixed random weights, so dO = Wo and
dS_final = WS.  Each gradient is checked against (a) central finite differences of the forward
oracle -- arithmetic that shares nothing with the backward's -- and (b) torch autograd through an
independent fp64 torch loop of the recurrence.
"""
import numpy as np
import pytest
import torch


def _problem(seed, L=6, dk=3, dv=2, k_scale=1.0, beta_lo=0.2, beta_hi=1.5):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((1, 1, L, dk))
    k = rng.standard_normal((1, 1, L, dk)) * k_scale
    v = rng.standard_normal((1, 1, L, dv))
    beta = rng.uniform(beta_lo, beta_hi, (1, 1, L))
    S0 = rng.standard_normal((1, 1, dk, dv)) * 0.3
    Wo = rng.standard_normal((1, 1, L, dv))
    WS = rng.standard_normal((1, 1, dk, dv))
    return q, k, v, beta, S0, Wo, WS


def _loss(oracle_mod, q, k, v, beta, S0, Wo, WS, rule):
    o, S = oracle_mod.fwd(q, k, v, beta, S0, nthreads=1, rule=rule)
    return float((o * Wo).sum() + (S * WS).sum())


def _fd(oracle_mod, args, idx, rule, h=1e-6):
    """Central differences of the loss with respect to args[idx], element by element."""
    base = [a.copy() for a in args]
    g = np.zeros_like(base[idx])
    it = np.nditer(base[idx], flags=["multi_index"])
    for _ in it:
        mi = it.multi_index
        plus = [a.copy() for a in base]
        minus = [a.copy() for a in base]
        plus[idx][mi] += h
        minus[idx][mi] -= h
        g[mi] = (_loss(oracle_mod, *plus, rule) - _loss(oracle_mod, *minus, rule)) / (2 * h)
    return g


@pytest.mark.parametrize("rule", ["exact", "euler"])
@pytest.mark.parametrize("seed,k_scale", [(1, 1.0), (2, 2.0), (3, 3e-3)])
def test_backward_matches_finite_differences(oracle_mod, rule, seed, k_scale):
    """k_scale 3e-3 puts beta*lambda below 1e-4, where df/dlambda takes its series branch."""
    q, k, v, beta, S0, Wo, WS = _problem(seed, k_scale=k_scale)
    dq, dk, dv, db, dS0 = oracle_mod.bwd(q, k, v, beta, Wo, S0, WS, rule=rule)
    args = [q, k, v, beta, S0, Wo, WS]
    for idx, g in ((0, dq), (1, dk), (2, dv), (3, db), (4, dS0)):
        ref = _fd(oracle_mod, args, idx, rule)
        scale = max(1e-3, float(np.abs(ref).max()))
        assert np.abs(g - ref).max() <= 2e-6 * scale, (idx, np.abs(g - ref).max(), scale)


def _torch_forward(q, k, v, beta, S0, rule):
    L = q.shape[2]
    S = S0[0, 0]
    outs = []
    for t in range(L):
        kt, vt, qt = k[0, 0, t], v[0, 0, t], q[0, 0, t]
        lam = (kt * kt).sum()
        if rule == "euler":
            a = beta[0, 0, t]
        else:
            a = -torch.expm1(-beta[0, 0, t] * lam) / lam
        S = S + a * torch.outer(kt, vt - S.T @ kt)
        outs.append(S.T @ qt)
    return torch.stack(outs)[None, None], S[None, None]


@pytest.mark.parametrize("rule", ["exact", "euler"])
def test_backward_matches_torch_autograd_of_an_independent_loop(oracle_mod, rule):
    q, k, v, beta, S0, Wo, WS = _problem(7, L=12, dk=5, dv=4)
    ts = [torch.tensor(a, dtype=torch.float64, requires_grad=True) for a in (q, k, v, beta, S0)]
    o, S = _torch_forward(*ts, rule)
    ((o * torch.tensor(Wo)).sum() + (S * torch.tensor(WS)).sum()).backward()
    got = oracle_mod.bwd(q, k, v, beta, Wo, S0, WS, rule=rule)
    for t, g in zip(ts, got):
        np.testing.assert_allclose(g, t.grad.numpy(), rtol=0,
                                   atol=1e-11 * max(1.0, float(t.grad.abs().max())))


def test_zero_upstream_gradient_gives_zero(oracle_mod):
    q, k, v, beta, S0, Wo, WS = _problem(9)
    for g in oracle_mod.bwd(q, k, v, beta, np.zeros_like(Wo), S0, None):
        assert not np.any(g)
