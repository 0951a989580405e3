"""The backward pass in the chunkwise (WY/UT) form, restated in numpy fp64, equals the oracle's
token-by-token backward.

The forward per chunk of C tokens ("Exact Flow Linear Attention", technical summary,
Methodology 3, in the chunk form the method shares with DeltaNet), from the state S at the
chunk's start:
    A = strictly_lower(diag(a) K K^T),  T = (I + A)^{-1},  R = V - K S,  U' = T diag(a) R,
    O = Q S + (M o Q K^T) U'   (M: lower triangle with the diagonal),   S' = S + K^T U'.
Reverse mode through those lines, given dO and dS' (the state gradient from the later chunks):
    dU' = K dS' + (M o Q K^T)^T dO,        dK = U' dS'^T + (M o dO U'^T)^T Q - dR S^T + ...
    dQ = dO S^T + (M o dO U'^T) K,
    d(diag(a) R) = T^T dU',   dT = dU' (diag(a) R)^T,   dR = diag(a) T^T dU',   dV = dR,
    dA = strictly_lower(-T^T dT T^T),   da += rowsum(dA o K K^T) + rowsum(T^T dU' o R),
    dK += B K + B^T K with B = diag(a) dA,   dK_t += 2 da_t (df/dlambda)_t k_t,
    dbeta = da df/dbeta,   and the state gradient carried to the previous chunk
    dS = dS' + Q^T dO - K^T dR   ( = dS' + Q^T dO - W^T dU' with W = T diag(a) K ).
The last line is a chain over chunks of the same shape as the forward's state pass; everything
else is per chunk.  This file pins that algebra against the token-level oracle; nothing here is
used by the library.
"""
import numpy as np
import pytest


def coeff(lam, beta, rule):
    """a = f(lambda, beta) and its partial derivatives, written out from the definition."""
    if rule == "euler":
        return beta.copy(), np.ones_like(beta), np.zeros_like(beta)
    x = beta * lam
    a = np.where(lam > 0, -np.expm1(-x) / np.where(lam > 0, lam, 1.0), beta)
    fb = np.exp(-x)
    # df/dlambda = (beta e^{-x} - a) / lambda; near x = 0 its series beta^2 (-1/2 + x/3 - x^2/8 ...)
    series = beta * beta * (-0.5 + x * (1 / 3 + x * (-1 / 8 + x * (1 / 30 - x / 144))))
    fl = np.where(np.abs(x) < 1e-3, series, (beta * fb - a) / np.where(lam > 0, lam, 1.0))
    return a, fb, fl


def chunk_bwd_head(q, k, v, beta, dO, S0, dSF, C, rule):
    L, dk = q.shape
    dv = v.shape[1]
    S = S0.copy()
    starts = []
    for c0 in range(0, L, C):  # forward, keeping the state at every chunk start
        starts.append(S.copy())
        K, V, bt = k[c0:c0 + C], v[c0:c0 + C], beta[c0:c0 + C]
        a, _, _ = coeff((K * K).sum(1), bt, rule)
        A = np.tril(a[:, None] * (K @ K.T), -1)
        T = np.linalg.inv(np.eye(len(a)) + A)
        S = S + K.T @ (T @ (a[:, None] * (V - K @ S)))
    dq, dkk, dvv, db = (np.zeros_like(q), np.zeros_like(k), np.zeros_like(v), np.zeros_like(beta))
    dS = dSF.copy()
    for ci in reversed(range(len(starts))):
        c0 = ci * C
        Q, K, V, bt, dOc = q[c0:c0 + C], k[c0:c0 + C], v[c0:c0 + C], beta[c0:c0 + C], dO[c0:c0 + C]
        S = starts[ci]
        lam = (K * K).sum(1)
        a, fb, fl = coeff(lam, bt, rule)
        Gm = K @ K.T
        A = np.tril(a[:, None] * Gm, -1)
        T = np.linalg.inv(np.eye(len(a)) + A)
        R = V - K @ S
        DR = a[:, None] * R
        U = T @ DR
        P = np.tril(Q @ K.T)
        # S' = S + K^T U
        dU = K @ dS
        dK = U @ dS.T
        # O = Q S + P U
        dQ = dOc @ S.T
        dSp = dS + Q.T @ dOc
        dP = np.tril(dOc @ U.T)
        dU = dU + P.T @ dOc
        dQ = dQ + dP @ K
        dK = dK + dP.T @ Q
        # U = T (diag(a) R)
        dDR = T.T @ dU
        dT = dU @ DR.T
        da = (dDR * R).sum(1)
        dR = a[:, None] * dDR
        # R = V - K S
        dV = dR
        dK = dK - dR @ S.T
        dSp = dSp - K.T @ dR
        # T = (I + A)^{-1}, A = strictly_lower(diag(a) K K^T)
        dA = np.tril(-T.T @ dT @ T.T, -1)
        da = da + (dA * Gm).sum(1)
        B = a[:, None] * dA
        dK = dK + B @ K + B.T @ K
        # a = f(lambda, beta)
        dK = dK + 2.0 * (da * fl)[:, None] * K
        dq[c0:c0 + C], dkk[c0:c0 + C], dvv[c0:c0 + C] = dQ, dK, dV
        db[c0:c0 + C] = da * fb
        dS = dSp
    return dq, dkk, dvv, db, dS


def _problem(seed, L, dk, dv, k_scale=1.0):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((1, 1, L, dk)) / np.sqrt(dk)
    k = rng.standard_normal((1, 1, L, dk)) / np.sqrt(dk) * k_scale * rng.uniform(0.5, 2.0, (1, 1, L, 1))
    v = rng.standard_normal((1, 1, L, dv))
    beta = rng.uniform(0.05, 1.5, (1, 1, L))
    S0 = rng.standard_normal((1, 1, dk, dv)) * 0.3
    dO = rng.standard_normal((1, 1, L, dv))
    dSF = rng.standard_normal((1, 1, dk, dv)) * 0.5
    return q, k, v, beta, S0, dO, dSF


@pytest.mark.parametrize("rule", ["exact", "euler"])
@pytest.mark.parametrize("L,C,dk,dv", [(70, 16, 6, 5), (64, 64, 8, 8), (33, 8, 4, 7), (1, 16, 3, 2)])
def test_chunk_backward_equals_token_backward(oracle_mod, rule, L, C, dk, dv):
    q, k, v, beta, S0, dO, dSF = _problem(L * 7 + dk, L, dk, dv, k_scale=1.0 if rule == "exact" else 0.7)
    ref = oracle_mod.bwd(q, k, v, beta, dO, S0, dSF, rule=rule)
    got = chunk_bwd_head(q[0, 0], k[0, 0], v[0, 0], beta[0, 0], dO[0, 0], S0[0, 0], dSF[0, 0], C, rule)
    for name, g, r in zip(("dq", "dk", "dv", "dbeta", "dS0"), got, ref):
        r = np.asarray(r)[0, 0]
        scale = max(1.0, float(np.abs(r).max()))
        assert np.abs(g - r).max() <= 1e-10 * scale, (name, float(np.abs(g - r).max()))


def test_chunk_backward_with_stiff_and_zero_keys(oracle_mod):
    """Keys of norm up to ~10 (beta lambda up to ~100) and exact zero keys in the same chunk."""
    q, k, v, beta, S0, dO, dSF = _problem(5, 48, 6, 4, k_scale=4.0)
    k[0, 0, 5] = 0.0
    k[0, 0, 20] = 0.0
    ref = oracle_mod.bwd(q, k, v, beta, dO, S0, dSF)
    got = chunk_bwd_head(q[0, 0], k[0, 0], v[0, 0], beta[0, 0], dO[0, 0], S0[0, 0], dSF[0, 0], 16, "exact")
    for name, g, r in zip(("dq", "dk", "dv", "dbeta", "dS0"), got, ref):
        r = np.asarray(r)[0, 0]
        scale = max(1.0, float(np.abs(r).max()))
        assert np.abs(g - r).max() <= 1e-9 * scale, (name, float(np.abs(g - r).max()))
