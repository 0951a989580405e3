"""Pin (e): the recurrent oracle equals the chunkwise (WY/UT) form on tiny inputs.

The technical summary ("Exact Flow Linear Attention: Exact Solution from
Continuous-Time Dynamics", Methodology 3) states that the EFLA update keeps
the rank-1 algebra of the delta rule and therefore the WY/UT chunkwise
parallel form.  This file restates that form in plain numpy fp64 (test code,
independent of both the oracle and the CUDA library) and checks that it
reaches the oracle's result, which is exact in exact arithmetic:

  per chunk, with S the state entering it,
    A  = strictly-lower(diag(alpha) K K^T)        T = (I + A)^{-1}
    W  = T diag(alpha) K                          U = T diag(alpha) V
    U' = U - W S
    O  = Q S + lower-incl-diagonal(Q K^T) U'
    S  <- S + K^T U'
"""
import math

import numpy as np
import pytest

from conftest import rel_err

RNG = np.random.default_rng(7)


def chunkwise_numpy(q, k, v, beta, S0, C):
    B, H, L, dk = q.shape
    dv = v.shape[-1]
    o = np.zeros((B, H, L, dv))
    S_out = np.zeros((B, H, dk, dv))
    for b in range(B):
        for h in range(H):
            S = np.zeros((dk, dv)) if S0 is None else S0[b, h].copy()
            for c0 in range(0, L, C):
                c1 = min(L, c0 + C)
                Q, K, V = q[b, h, c0:c1], k[b, h, c0:c1], v[b, h, c0:c1]
                lam = np.einsum("td,td->t", K, K)
                al = np.array([(-math.expm1(-bt * lm) / lm) if lm > 0 else bt
                               for lm, bt in zip(lam, beta[b, h, c0:c1])])
                A = np.tril(al[:, None] * (K @ K.T), -1)
                T = np.linalg.solve(np.eye(c1 - c0) + A, np.eye(c1 - c0))
                W = T @ (al[:, None] * K)
                U = T @ (al[:, None] * V)
                Up = U - W @ S
                o[b, h, c0:c1] = Q @ S + np.tril(Q @ K.T) @ Up
                S = S + K.T @ Up
            S_out[b, h] = S
    return o, S_out


@pytest.mark.parametrize("C", [4, 8, 16])
@pytest.mark.parametrize("L", [16, 37])
def test_chunkwise_equals_recurrent(oracle_mod, C, L):
    B, H, dk, dv = 2, 2, 8, 6
    q = RNG.standard_normal((B, H, L, dk)) / math.sqrt(dk)
    k = RNG.standard_normal((B, H, L, dk)) * RNG.uniform(0.2, 1.5, (B, H, L, 1)) / math.sqrt(dk) * 2
    v = RNG.standard_normal((B, H, L, dv))
    beta = 1 / (1 + np.exp(-RNG.standard_normal((B, H, L))))
    S0 = 0.1 * RNG.standard_normal((B, H, dk, dv))
    o_ref, S_ref = oracle_mod.fwd(q, k, v, beta, S0)
    o_chk, S_chk = chunkwise_numpy(q, k, v, beta, S0, C)
    assert rel_err(o_chk, o_ref) < 1e-12
    assert rel_err(S_chk, S_ref) < 1e-12


def test_chunkwise_stiff_and_zero_keys(oracle_mod):
    """Keys spanning 1e-4..100 in squared norm (T gets large entries) and exact-zero keys."""
    B, H, L, dk, dv, C = 1, 1, 48, 8, 8, 16
    d = RNG.standard_normal((B, H, L, dk))
    d /= np.linalg.norm(d, axis=-1, keepdims=True)
    k = d * np.sqrt(np.exp(RNG.uniform(math.log(1e-4), math.log(100), (B, H, L, 1))))
    k[0, 0, 5] = 0.0
    q = RNG.standard_normal((B, H, L, dk)) / math.sqrt(dk)
    v = RNG.standard_normal((B, H, L, dv))
    beta = 1 / (1 + np.exp(-2 * RNG.standard_normal((B, H, L))))
    o_ref, S_ref = oracle_mod.fwd(q, k, v, beta, None)
    o_chk, S_chk = chunkwise_numpy(q, k, v, beta, None, C)
    assert rel_err(o_chk, o_ref) < 1e-9
    assert rel_err(S_chk, S_ref) < 1e-9
