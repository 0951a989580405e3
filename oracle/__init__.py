"""fp64 CPU oracle for the EFLA forward pass -- TEST INFRASTRUCTURE ONLY.

Only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA library and its Python binding
never import it, and it imports nothing from them.

The arithmetic lives in ``efla_oracle.c`` (plain C, fp64, one token at a time,
libm ``expm1``, built with ``-O2`` and no fast-math).  This module only
compiles it with gcc and marshals numpy arrays through ctypes.

Source of the recurrence: "Exact Flow Linear Attention: Exact Solution from
Continuous-Time Dynamics", technical summary, Methodology 2 (lambda = ||k||^2)
and Methodology 3 (alpha and the update rule); readout o_t = S_t^T q_t.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "efla_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile efla_oracle.c into liboracle.so with gcc (no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp.%d" % os.getpid()
        subprocess.check_call(
            ["gcc", "-O2", "-std=c99", "-D_POSIX_C_SOURCE=200809L", "-fPIC", "-shared",
             "-fno-fast-math", "-ffp-contract=off", "-o", tmp, _SRC, "-lm", "-lpthread"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        dp = ctypes.POINTER(ctypes.c_double)
        lib.efla_oracle_alpha.restype = ctypes.c_double
        lib.efla_oracle_alpha.argtypes = [ctypes.c_double, ctypes.c_double]
        lib.efla_oracle_step.restype = ctypes.c_double
        lib.efla_oracle_step.argtypes = [ctypes.c_int, ctypes.c_int, dp, dp, dp, dp,
                                         ctypes.c_double, dp]
        lib.efla_oracle_fwd.restype = ctypes.c_int
        lib.efla_oracle_fwd.argtypes = [ctypes.c_int] * 5 + [dp] * 7 + [ctypes.c_int]
        lib.efla_oracle_coeff.restype = ctypes.c_double
        lib.efla_oracle_coeff.argtypes = [ctypes.c_double, ctypes.c_double, ctypes.c_int]
        lib.efla_oracle_step_rule.restype = ctypes.c_double
        lib.efla_oracle_step_rule.argtypes = [ctypes.c_int, ctypes.c_int, dp, dp, dp, dp,
                                              ctypes.c_double, dp, ctypes.c_int]
        lib.efla_oracle_bwd.restype = None
        lib.efla_oracle_bwd.argtypes = [ctypes.c_int] * 5 + [dp] * 12 + [ctypes.c_int]
        lib.efla_oracle_fwd_rule.restype = ctypes.c_int
        lib.efla_oracle_fwd_rule.argtypes = [ctypes.c_int] * 5 + [dp] * 7 + [ctypes.c_int] * 2
        lib.efla_oracle_fwd_gated.restype = ctypes.c_int
        lib.efla_oracle_fwd_gated.argtypes = [ctypes.c_int] * 5 + [dp] * 8 + [ctypes.c_int] * 2
        lib.efla_oracle_step_gated.restype = ctypes.c_double
        lib.efla_oracle_step_gated.argtypes = [ctypes.c_int, ctypes.c_int, dp, dp, dp, dp,
                                               ctypes.c_double, ctypes.c_double, dp, ctypes.c_int]
        _lib = lib
    return _lib


def _f64(a) -> np.ndarray:
    """Contiguous fp64 numpy copy of a numpy array or a (CPU) torch tensor."""
    if hasattr(a, "detach"):
        a = a.detach().to("cpu")
        import torch  # local: only when given torch tensors

        a = a.to(torch.float64).numpy()
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


RULES = {"exact": 0, "euler": 1}


def alpha(lam: float, beta: float, rule: str = "exact") -> float:
    """alpha = (1 - exp(-beta*lam))/lam, evaluated as -expm1(-beta*lam)/lam; beta at lam == 0.
    rule="euler": the delta rule's coefficient, beta."""
    if rule == "exact":
        return float(_load().efla_oracle_alpha(float(lam), float(beta)))
    return float(_load().efla_oracle_coeff(float(lam), float(beta), RULES[rule]))


def step(S, q, k, v, beta: float, rule: str = "exact", g: float | None = None):
    """One recurrent token on one head.  Returns (S_t, o_t, alpha_t); S is not modified.
    g: the gated form's decay of this token (None: no decay)."""
    S = _f64(S).copy()
    q, k, v = _f64(q), _f64(k), _f64(v)
    dk, dv = S.shape
    o = np.zeros(dv)
    if g is None:
        a = _load().efla_oracle_step_rule(dk, dv, _ptr(S), _ptr(q), _ptr(k), _ptr(v), float(beta),
                                          _ptr(o), RULES[rule])
    else:
        a = _load().efla_oracle_step_gated(dk, dv, _ptr(S), _ptr(q), _ptr(k), _ptr(v), float(beta),
                                           float(g), _ptr(o), RULES[rule])
    return S, o, float(a)


def fwd(q, k, v, beta, S0=None, nthreads: int | None = None, want_o: bool = True,
        rule: str = "exact", g=None):
    """Token-by-token forward over [B,H,L,d] inputs.  Returns (o, S_final) in fp64.

    q, k: [B,H,L,dk]; v: [B,H,L,dv]; beta: [B,H,L]; S0: [B,H,dk,dv] or None (zeros).
    rule="euler" takes the delta rule's explicit Euler step (alpha = beta) instead.
    g: [B,H,L] per-token decay of the gated form S_t = g_t (I - alpha_t k_t k_t^T) S_{t-1}
    + alpha_t k_t v_t^T, or None (no decay).
    """
    q, k, v, beta = _f64(q), _f64(k), _f64(v), _f64(beta)
    gg = None if g is None else _f64(g)
    B, H, L, dk = q.shape
    dv = v.shape[-1]
    assert k.shape == (B, H, L, dk) and v.shape == (B, H, L, dv) and beta.shape == (B, H, L)
    s0 = None
    if S0 is not None:
        s0 = _f64(S0)
        assert s0.shape == (B, H, dk, dv)
    o = np.zeros((B, H, L, dv)) if want_o else None
    S = np.zeros((B, H, dk, dv))
    if nthreads is None:
        nthreads = os.cpu_count() or 1
    if gg is not None:
        assert gg.shape == (B, H, L)
    rc = _load().efla_oracle_fwd_gated(B, H, L, dk, dv, _ptr(q), _ptr(k), _ptr(v), _ptr(beta),
                                       _ptr(gg) if gg is not None else None,
                                       _ptr(s0) if s0 is not None else None,
                                       _ptr(o) if o is not None else None, _ptr(S), int(nthreads),
                                       RULES[rule])
    if rc != 0:
        raise MemoryError("oracle forward failed to allocate")
    return o, S


def bwd(q, k, v, beta, dO, S0=None, dS_final=None, rule: str = "exact"):
    """Gradients (dq, dk, dv, dbeta, dS0) of a loss through fwd(), given dO = dL/do and
    dS_final = dL/dS_final (None = 0).  fp64, token by token, heads in sequence."""
    q, k, v, beta, dO = _f64(q), _f64(k), _f64(v), _f64(beta), _f64(dO)
    B, H, L, dk = q.shape
    dv = v.shape[-1]
    assert dO.shape == (B, H, L, dv)
    s0 = _f64(S0) if S0 is not None else None
    dsf = _f64(dS_final) if dS_final is not None else None
    dq, dkk, dvv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    db, dS0 = np.zeros_like(beta), np.zeros((B, H, dk, dv))
    _load().efla_oracle_bwd(B, H, L, dk, dv, _ptr(q), _ptr(k), _ptr(v), _ptr(beta),
                            _ptr(s0) if s0 is not None else None, _ptr(dO),
                            _ptr(dsf) if dsf is not None else None, _ptr(dq), _ptr(dkk), _ptr(dvv),
                            _ptr(db), _ptr(dS0), RULES[rule])
    return dq, dkk, dvv, db, dS0
