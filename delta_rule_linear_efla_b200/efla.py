"""Python binding of the C-ABI library libefla.so (include/efla.h).

Argument marshalling only: this module checks tensor dtypes, shapes and
devices, allocates outputs and workspace with torch, and passes raw device
pointers plus the current CUDA stream to the library.  Every step of the
computation runs in the library's CUDA kernels.  There is no CPU fallback: if
the library is missing or no CUDA device is present, every call raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libefla.so")

EFLA_F32, EFLA_BF16 = 0, 1
# Update rules: the exact flow (the method) and the delta rule's explicit Euler step.
RULES = {"exact": 0, "euler": 1}

# Every extern "C" symbol declared in include/efla.h.
ABI_SYMBOLS = (
    "efla_status_str", "efla_version", "efla_alpha", "efla_chunk_fwd_workspace_size",
    "efla_chunk_fwd", "efla_recurrent_step", "efla_last_device_error", "efla_chunk_fwd_path",
    "efla_kernel_launches", "efla_chunk_fwd_noalloc", "efla_alpha_rule", "efla_chunk_fwd_rule",
    "efla_recurrent_step_rule", "efla_state_affine", "efla_bwd_workspace_size", "efla_bwd",
    "efla_selftest_bounded_wait", "efla_chunk_fwd_gated", "efla_recurrent_step_gated",
    "efla_bwd_kept_size", "efla_chunk_fwd_keep", "efla_bwd_kept",
)

_lib = None


class EflaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__("%s failed: %s (status %d)" % (where, status_str(status), status))


def load_library(path: str | None = None) -> ctypes.CDLL:
    """Load libefla.so (raises if it has not been built)."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise RuntimeError("libefla.so is not built (%s); run `python -m "
                           "delta_rule_linear_efla_b200.build` on a machine with nvcc" % p)
    L = ctypes.CDLL(p)
    vp, i, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    L.efla_status_str.restype = ctypes.c_char_p
    L.efla_status_str.argtypes = [i]
    L.efla_version.restype = i
    L.efla_version.argtypes = []
    L.efla_alpha.restype = i
    L.efla_alpha.argtypes = [vp, vp, vp, i, i, i, i, i, vp]
    L.efla_chunk_fwd_workspace_size.restype = sz
    L.efla_chunk_fwd_workspace_size.argtypes = [i, i, i, i, i, i, i, i]
    L.efla_chunk_fwd.restype = i
    L.efla_chunk_fwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, i, i, vp, sz, vp]
    L.efla_recurrent_step.restype = i
    L.efla_recurrent_step.argtypes = [vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, vp]
    L.efla_last_device_error.restype = i
    L.efla_last_device_error.argtypes = [vp]
    L.efla_chunk_fwd_path.restype = i
    L.efla_chunk_fwd_path.argtypes = [i, i, i, i, i, i, i, i]
    L.efla_kernel_launches.restype = ctypes.c_ulonglong
    L.efla_kernel_launches.argtypes = []
    L.efla_chunk_fwd_noalloc.restype = i
    L.efla_chunk_fwd_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, i, i, vp]
    L.efla_alpha_rule.restype = i
    L.efla_alpha_rule.argtypes = [vp, vp, vp, i, i, i, i, i, i, vp]
    L.efla_chunk_fwd_rule.restype = i
    L.efla_chunk_fwd_rule.argtypes = [vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, i, i, i, vp, sz, vp]
    L.efla_bwd_workspace_size.restype = sz
    L.efla_bwd_workspace_size.argtypes = [i, i, i, i, i]
    L.efla_bwd.restype = i
    L.efla_bwd.argtypes = [vp] * 12 + [i] * 7 + [vp, sz, vp]
    L.efla_selftest_bounded_wait.restype = i
    L.efla_selftest_bounded_wait.argtypes = [ctypes.c_longlong, vp]
    L.efla_state_affine.restype = i
    L.efla_state_affine.argtypes = [vp, vp, vp, vp, i, i, i, i, vp]
    L.efla_recurrent_step_rule.restype = i
    L.efla_recurrent_step_rule.argtypes = [vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, i, vp]
    L.efla_chunk_fwd_gated.restype = i
    L.efla_chunk_fwd_gated.argtypes = [vp] * 8 + [i] * 9 + [vp, sz, vp]
    L.efla_recurrent_step_gated.restype = i
    L.efla_recurrent_step_gated.argtypes = [vp] * 7 + [i] * 7 + [vp]
    L.efla_chunk_fwd_keep.restype = i
    L.efla_chunk_fwd_keep.argtypes = [vp] * 7 + [i] * 8 + [vp, sz, vp]
    L.efla_bwd_kept.restype = i
    L.efla_bwd_kept.argtypes = [vp] * 12 + [i] * 7 + [vp, sz, vp, sz, vp]
    L.efla_bwd_kept_size.restype = sz
    L.efla_bwd_kept_size.argtypes = [i, i, i, i, i]
    if path is None:
        _lib = L
    return L


def status_str(status: int) -> str:
    return load_library().efla_status_str(int(status)).decode()


def _check(status: int, where: str) -> None:
    if status != 0:
        raise EflaError(status, where)


def _code(dtype) -> int:
    if dtype == torch.float32:
        return EFLA_F32
    if dtype == torch.bfloat16:
        return EFLA_BF16
    raise TypeError("EFLA tensors must be float32 or bfloat16, got %s" % dtype)


def _dtype_code(t: torch.Tensor) -> int:
    return _code(t.dtype)


def _rule(rule: str) -> int:
    if rule not in RULES:
        raise ValueError("rule must be one of %s, got %r" % (sorted(RULES), rule))
    return RULES[rule]


def _dev(t: torch.Tensor, name: str, dtype=None) -> int:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError("%s must be a CUDA tensor" % name)
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    if dtype is not None and t.dtype != dtype:
        raise TypeError("%s must be %s, got %s" % (name, dtype, t.dtype))
    return t.data_ptr()


def _stream_handle(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def alpha(k: torch.Tensor, beta: torch.Tensor, out: torch.Tensor | None = None, stream=None,
          rule: str = "exact"):
    """alpha_t = -expm1(-beta_t ||k_t||^2)/||k_t||^2 (beta_t at ||k_t|| = 0); [B,H,L] fp32.
    rule="euler" gives the delta rule's coefficient, alpha_t = beta_t."""
    B, H, L, dk = k.shape
    if beta.shape != (B, H, L) or beta.dtype != k.dtype:
        raise ValueError("beta must be [B,H,L] with k's dtype")
    if out is None:
        out = torch.empty((B, H, L), dtype=torch.float32, device=k.device)
    _check(load_library().efla_alpha_rule(_dev(k, "k"), _dev(beta, "beta"),
                                           _dev(out, "alpha", torch.float32), B, H, L, dk,
                                           _dtype_code(k), _rule(rule), _stream_handle(stream)),
           "efla_alpha_rule")
    return out


def workspace_size(B: int, H: int, L: int, dk: int, dv: int, chunk: int, dtype,
                   o_dtype=torch.float32) -> int:
    return int(load_library().efla_chunk_fwd_workspace_size(B, H, L, dk, dv, chunk, _code(dtype),
                                                            _code(o_dtype)))


def chunk_fwd_path(B, H, L, dk, dv, chunk, dtype, o_dtype=torch.float32) -> str:
    p = load_library().efla_chunk_fwd_path(B, H, L, dk, dv, chunk, _code(dtype), _code(o_dtype))
    return {0: "simt", 1: "tcgen05", 2: "tcgen05-segments"}[p]


def chunk_fwd(q, k, v, beta, S0=None, chunk: int = 64, o=None, S_final=None,
              want_state: bool = True, workspace=None, o_dtype=torch.float32, stream=None,
              rule: str = "exact", g=None):
    """EFLA forward in the WY/UT chunkwise form.  Returns (o, S_final or None).
    rule="euler" runs the same kernels with the delta rule's coefficient alpha = beta.
    g: [B,H,L] per-token decay of the gated form S_t = g_t (I - alpha_t k_t k_t^T) S_{t-1}
    + alpha_t k_t v_t^T (efla_chunk_fwd_gated), or None.

    q, k: [B,H,L,dk]; v: [B,H,L,dv]; beta: [B,H,L], all float32 or all bfloat16 on one
    CUDA device; S0: [B,H,dk,dv] float32 or None.  o is float32 by default (the fp32
    accumulator) or bfloat16 with o_dtype=torch.bfloat16; S_final is float32 and may be S0
    (in-place carry)."""
    B, H, L, dk = q.shape
    dv = v.shape[-1]
    if k.shape != q.shape or v.shape[:3] != (B, H, L) or beta.shape != (B, H, L):
        raise ValueError("shape mismatch: q,k [B,H,L,dk], v [B,H,L,dv], beta [B,H,L]")
    if g is not None and g.shape != (B, H, L):
        raise ValueError("g must be [B,H,L]")
    code = _dtype_code(q)
    for name, t in (("k", k), ("v", v), ("beta", beta), ("g", g)):
        if t is not None and t.dtype != q.dtype:
            raise TypeError("%s must have q's dtype %s" % (name, q.dtype))
    if o is not None:
        o_dtype = o.dtype
    o_code = _code(o_dtype)
    if o is None:
        o = torch.empty((B, H, L, dv), dtype=o_dtype, device=q.device)
    if S_final is None and want_state:
        S_final = torch.empty((B, H, dk, dv), dtype=torch.float32, device=q.device)
    need = workspace_size(B, H, L, dk, dv, chunk, q.dtype, o_dtype)
    if need and (workspace is None or workspace.numel() * workspace.element_size() < need):
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_ptr = _dev(workspace, "workspace") if (need and workspace is not None) else None
    ws_bytes = workspace.numel() * workspace.element_size() if ws_ptr else 0
    S0p = _dev(S0, "S0", torch.float32) if S0 is not None else None
    Sfp = _dev(S_final, "S_final", torch.float32) if S_final is not None else None
    if g is None:
        st = load_library().efla_chunk_fwd_rule(
            _dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _dev(beta, "beta"), S0p, _dev(o, "o", o_dtype),
            Sfp, B, H, L, dk, dv, int(chunk), code, o_code, _rule(rule), ws_ptr, ws_bytes,
            _stream_handle(stream))
        _check(st, "efla_chunk_fwd_rule")
    else:
        st = load_library().efla_chunk_fwd_gated(
            _dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _dev(beta, "beta"), _dev(g, "g"), S0p,
            _dev(o, "o", o_dtype), Sfp, B, H, L, dk, dv, int(chunk), code, o_code, _rule(rule),
            ws_ptr, ws_bytes, _stream_handle(stream))
        _check(st, "efla_chunk_fwd_gated")
    return o, S_final


def chunk_fwd_noalloc(q, k, v, beta, o, S_final=None, S0=None, chunk: int = 64, stream=None):
    """chunk_fwd for callers that cannot allocate device memory: the caller passes every
    output buffer and the library uses its own fixed scratch (efla_chunk_fwd_noalloc)."""
    B, H, L, dk = q.shape
    dv = v.shape[-1]
    st = load_library().efla_chunk_fwd_noalloc(
        _dev(q, "q"), _dev(k, "k", q.dtype), _dev(v, "v", q.dtype), _dev(beta, "beta", q.dtype),
        _dev(S0, "S0", torch.float32) if S0 is not None else None, _dev(o, "o"),
        _dev(S_final, "S_final", torch.float32) if S_final is not None else None,
        B, H, L, dk, dv, int(chunk), _dtype_code(q), _dtype_code(o), _stream_handle(stream))
    _check(st, "efla_chunk_fwd_noalloc")
    return o, S_final


def recurrent_step(q, k, v, beta, S, o=None, o_dtype=torch.float32, stream=None,
                   rule: str = "exact", g=None):
    """One decode token per head; S ([B,H,dk,dv] float32) is updated in place.  Returns o
    (float32 by default, or bfloat16 with o_dtype=torch.bfloat16).  rule="euler" takes the
    delta rule's step (alpha = beta).  g: [B,H] decay of the gated form, or None."""
    B, H, dk = q.shape
    dv = v.shape[-1]
    if k.shape != q.shape or v.shape[:2] != (B, H) or beta.shape != (B, H) or \
            S.shape != (B, H, dk, dv):
        raise ValueError("shape mismatch: q,k [B,H,dk], v [B,H,dv], beta [B,H], S [B,H,dk,dv]")
    code = _dtype_code(q)
    if o is not None:
        o_dtype = o.dtype
    if o is None:
        o = torch.empty((B, H, dv), dtype=o_dtype, device=q.device)
    if g is None:
        st = load_library().efla_recurrent_step_rule(
            _dev(q, "q"), _dev(k, "k", q.dtype), _dev(v, "v", q.dtype), _dev(beta, "beta", q.dtype),
            _dev(S, "S", torch.float32), _dev(o, "o", o_dtype), B, H, dk, dv, code, _code(o_dtype),
            _rule(rule), _stream_handle(stream))
        _check(st, "efla_recurrent_step_rule")
    else:
        if g.shape != (B, H):
            raise ValueError("g must be [B,H]")
        st = load_library().efla_recurrent_step_gated(
            _dev(q, "q"), _dev(k, "k", q.dtype), _dev(v, "v", q.dtype), _dev(beta, "beta", q.dtype),
            _dev(g, "g", q.dtype), _dev(S, "S", torch.float32), _dev(o, "o", o_dtype), B, H, dk, dv,
            code, _code(o_dtype), _rule(rule), _stream_handle(stream))
        _check(st, "efla_recurrent_step_gated")
    return o


def state_affine(P, S_in=None, H=None, out=None, stream=None):
    """S_out = P S_in + H per head in fp32 (P [B,H,dk,dk]; S_in, H, out [B,H,dk,dv]; S_in or H
    None means zero; out may be S_in).  Chains the affine state maps of sequence stretches."""
    B, Hh, dk, dk2 = P.shape
    if dk2 != dk:
        raise ValueError("P must be [B,H,dk,dk]")
    ref = S_in if S_in is not None else (H if H is not None else out)
    if ref is None:
        raise ValueError("one of S_in, H or out must give the value dimension")
    dv = ref.shape[-1]
    for name, t in (("S_in", S_in), ("H", H), ("out", out)):
        if t is not None and t.shape != (B, Hh, dk, dv):
            raise ValueError("%s must be [B,H,dk,dv]" % name)
    if out is None:
        out = torch.empty((B, Hh, dk, dv), dtype=torch.float32, device=P.device)
    st = load_library().efla_state_affine(
        _dev(P, "P", torch.float32), _dev(S_in, "S_in", torch.float32) if S_in is not None else None,
        _dev(H, "H", torch.float32) if H is not None else None, _dev(out, "out", torch.float32),
        B, Hh, dk, dv, _stream_handle(stream))
    _check(st, "efla_state_affine")
    return out


def bwd(q, k, v, beta, dO, S0=None, dS_final=None, want_dS0: bool = True, rule: str = "exact",
        workspace=None, stream=None, kept=None):
    """Gradients of chunk_fwd: returns (dq, dk, dv, dbeta, dS0 or None), all float32, given
    dO = dL/do (float32 [B,H,L,dv]) and dS_final = dL/dS_final (float32 or None = 0).
    kept: the buffer chunk_fwd_keep filled for the same inputs (efla_bwd_kept), or None."""
    B, H, L, dk = q.shape
    dv = v.shape[-1]
    if k.shape != q.shape or v.shape[:3] != (B, H, L) or beta.shape != (B, H, L) or \
            dO.shape != (B, H, L, dv):
        raise ValueError("shape mismatch: q,k [B,H,L,dk], v,dO [B,H,L,dv], beta [B,H,L]")
    code = _dtype_code(q)
    for name, t in (("k", k), ("v", v), ("beta", beta)):
        if t.dtype != q.dtype:
            raise TypeError("%s must have q's dtype %s" % (name, q.dtype))
    f32 = dict(dtype=torch.float32, device=q.device)
    dq, dkey, dval = torch.empty((B, H, L, dk), **f32), torch.empty((B, H, L, dk), **f32), \
        torch.empty((B, H, L, dv), **f32)
    dbeta = torch.empty((B, H, L), **f32)
    dS0 = torch.empty((B, H, dk, dv), **f32) if want_dS0 else None
    need = int(load_library().efla_bwd_workspace_size(B, H, L, dk, dv))
    if need and (workspace is None or workspace.numel() * workspace.element_size() < need):
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_ptr = _dev(workspace, "workspace") if need else None
    kargs = ()
    if kept is not None:
        kargs = (_dev(kept, "kept"), kept.numel() * kept.element_size())
    entry = load_library().efla_bwd_kept if kept is not None else load_library().efla_bwd
    st = entry(
        _dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _dev(beta, "beta"),
        _dev(S0, "S0", torch.float32) if S0 is not None else None, _dev(dO, "dO", torch.float32),
        _dev(dS_final, "dS_final", torch.float32) if dS_final is not None else None,
        _dev(dq, "dq"), _dev(dkey, "dk"), _dev(dval, "dv"), _dev(dbeta, "dbeta"),
        _dev(dS0, "dS0") if dS0 is not None else None, B, H, L, dk, dv, code, _rule(rule),
        *kargs, ws_ptr, need if ws_ptr else 0, _stream_handle(stream))
    _check(st, "efla_bwd_kept" if kept is not None else "efla_bwd")
    return dq, dkey, dval, dbeta, dS0


def keeps_for_bwd(q, v, chunk: int = 64, rule: str = "exact") -> bool:
    """Whether chunk_fwd_keep takes these inputs: bf16 at the tensor-core backward's sizes."""
    B, H, L, dk = q.shape
    return (q.dtype == torch.bfloat16 and chunk == 64 and L > 0 and dk in (64, 128) and
            v.shape[-1] in (64, 128) and rule in RULES)


def chunk_fwd_keep(q, k, v, beta, S0=None, o_dtype=torch.float32, rule: str = "exact", stream=None):
    """The forward of a training step (efla_chunk_fwd_keep): (o, S_final, kept), where o and
    S_final are chunk_fwd's bit for bit and kept (efla_bwd_kept_size bytes) holds what
    bwd(..., kept=kept) reads instead of running the forward again.  bf16 inputs at the
    tensor-core sizes only (keeps_for_bwd)."""
    B, H, L, dk = q.shape
    dv = v.shape[-1]
    if k.shape != q.shape or v.shape[:3] != (B, H, L) or beta.shape != (B, H, L):
        raise ValueError("shape mismatch: q,k [B,H,L,dk], v [B,H,L,dv], beta [B,H,L]")
    code = _dtype_code(q)
    o = torch.empty((B, H, L, dv), dtype=o_dtype, device=q.device)
    S_final = torch.empty((B, H, dk, dv), dtype=torch.float32, device=q.device)
    need = int(load_library().efla_bwd_kept_size(B, H, L, dk, dv))
    kept = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    st = load_library().efla_chunk_fwd_keep(
        _dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _dev(beta, "beta"),
        _dev(S0, "S0", torch.float32) if S0 is not None else None, _dev(o, "o", o_dtype),
        _dev(S_final, "S_final", torch.float32), B, H, L, dk, dv, code, _code(o_dtype), _rule(rule),
        _dev(kept, "kept"), need, _stream_handle(stream))
    _check(st, "efla_chunk_fwd_keep")
    return o, S_final, kept


class EflaFunction(torch.autograd.Function):
    """(o, S_final) = EFLA forward with autograd: the forward is chunk_fwd and the backward is
    efla_bwd.  Gradients flow to q, k, v, beta (in their dtype) and to S0 when given."""

    @staticmethod
    def forward(ctx, q, k, v, beta, S0, rule="exact", chunk=64):
        kept = None
        if keeps_for_bwd(q, v, chunk, rule):  # the backward will read what this forward keeps
            o, S, kept = chunk_fwd_keep(q, k, v, beta, S0, rule=rule)
        else:
            o, S = chunk_fwd(q, k, v, beta, S0, chunk=chunk, rule=rule)
        ctx.save_for_backward(q, k, v, beta, S0 if S0 is not None else torch.empty(0))
        ctx.has_S0, ctx.rule, ctx.kept = S0 is not None, rule, kept
        return o, S

    @staticmethod
    def backward(ctx, dO, dS):
        q, k, v, beta, S0 = ctx.saved_tensors
        dO = dO.float().contiguous() if dO is not None else torch.zeros(
            q.shape[:3] + v.shape[-1:], dtype=torch.float32, device=q.device)
        dS = dS.float().contiguous() if dS is not None else None
        dq, dk, dv, db, dS0 = bwd(q, k, v, beta, dO, S0 if ctx.has_S0 else None, dS,
                                  want_dS0=ctx.has_S0, rule=ctx.rule, kept=ctx.kept)
        ctx.kept = None
        return (dq.to(q.dtype), dk.to(k.dtype), dv.to(v.dtype), db.to(beta.dtype),
                dS0 if ctx.has_S0 else None, None, None)


def efla_attention(q, k, v, beta, S0=None, rule: str = "exact", chunk: int = 64):
    """Differentiable EFLA forward: (o, S_final) with gradients through efla_bwd."""
    return EflaFunction.apply(q, k, v, beta, S0, rule, chunk)


def selftest_bounded_wait(budget_cycles: int = 1_000_000, stream=None) -> None:
    """Launch the bounded-wait self-test kernel (its wait runs out by design); read the
    outcome with last_device_error()."""
    _check(load_library().efla_selftest_bounded_wait(int(budget_cycles), _stream_handle(stream)),
           "efla_selftest_bounded_wait")


def kernel_launches() -> int:
    """Kernels the library has enqueued since it was loaded (host-side counter)."""
    return int(load_library().efla_kernel_launches())


def last_device_error(stream=None) -> int:
    """Synchronise and return (and clear) the device error word's status code."""
    return int(load_library().efla_last_device_error(_stream_handle(stream)))
