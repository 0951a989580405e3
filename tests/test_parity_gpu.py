"""GPU parity: the CUDA chunkwise forward (through the C ABI) against the fp64
oracle, element by element on the same seeded inputs.

Bounds: max|x_gpu - x_oracle| / RMS(x_oracle) <= 1e-4 for fp32 inputs and
<= 2e-2 for bf16 inputs with fp32 accumulation, for o and for S_final; o is
the fp32 accumulator (the library's default output type).  The oracle sees the
exact dtype-rounded values the GPU sees.  The optional bf16 output adds its own
rounding, at most half a bf16 ulp (2^-8 relative) per element, so it is checked
against 2e-2 + 2^-8 max|o| / RMS(o).

Sizes: every workload at its full size, every head,
plus smaller cases that span several chunks and end in a ragged tail, and the
edge cases (L = 0, L = 1, L < chunk, dk != dv, S_final aliasing S0, zero keys,
beta = 0).
"""
import numpy as np
import pytest
import torch

from conftest import rel_err
from delta_rule_linear_efla_b200 import efla, inputs

pytestmark = pytest.mark.gpu

TOL = {"fp32": 1e-4, "bf16": 2e-2}


def _to_dev(x):
    return {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in x.items()}


def _run_gpu(x, chunk=None):
    d = _to_dev(x)
    o, S = efla.chunk_fwd(d["q"], d["k"], d["v"], d["beta"], d["S0"], chunk=chunk or x["chunk"])
    torch.cuda.synchronize()
    assert efla.last_device_error() == 0
    return o.float().cpu(), S.cpu()


def _oracle(oracle_mod, x, heads=None):
    """Oracle on all heads, or on a list of (b, h) heads."""
    if heads is None:
        return oracle_mod.fwd(x["q"], x["k"], x["v"], x["beta"], x["S0"])
    os_, Ss = [], []
    for b, h in heads:
        sl = lambda t: t[b:b + 1, h:h + 1]
        o, S = oracle_mod.fwd(sl(x["q"]), sl(x["k"]), sl(x["v"]), sl(x["beta"]),
                              None if x["S0"] is None else sl(x["S0"]))
        os_.append(o[0, 0])
        Ss.append(S[0, 0])
    return np.stack(os_), np.stack(Ss)


def _check(x, o_gpu, S_gpu, o_ref, S_ref, heads=None):
    tol = TOL[x["workload"].dtype]
    if heads is not None:
        o_gpu = torch.stack([o_gpu[b, h] for b, h in heads])
        S_gpu = torch.stack([S_gpu[b, h] for b, h in heads])
    eo, es = rel_err(o_gpu.numpy(), o_ref), rel_err(S_gpu.numpy(), S_ref)
    assert eo <= tol and es <= tol, (eo, es, tol)
    return eo, es


@pytest.mark.parametrize("wid", [1, 2, 3, 4])
def test_workload_full_size(oracle_mod, wid):
    x = inputs.make_inputs(wid)
    o, S = _run_gpu(x)
    o_ref, S_ref = _oracle(oracle_mod, x)
    _check(x, o, S, o_ref, S_ref)


def test_workload5_full_size_all_heads(oracle_mod):
    """The long stiff workload at full size (16 heads x 65536 tokens, sequence segments on the
    GPU), every head against the oracle (about 1e11 fp64 flop, threaded over the heads)."""
    x = inputs.make_inputs(5)
    o, S = _run_gpu(x)
    assert torch.isfinite(o).all() and torch.isfinite(S).all()
    o_ref, S_ref = _oracle(oracle_mod, x)
    _check(x, o, S, o_ref, S_ref)


@pytest.mark.parametrize("wid,L,B,H", [(2, 333, 1, 3), (3, 200, 2, 2), (4, 130, 1, 4),
                                       (5, 1000, 1, 3), (1, 37, 2, 2)])
def test_ragged_tail(oracle_mod, wid, L, B, H):
    x = inputs.make_inputs(inputs.workload(wid, L=L, B=B, H=H))
    o, S = _run_gpu(x)
    o_ref, S_ref = _oracle(oracle_mod, x)
    _check(x, o, S, o_ref, S_ref)


@pytest.mark.parametrize("chunk", [16, 32, 64])
@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_chunk_sizes(oracle_mod, chunk, dtype):
    x = inputs.make_inputs(inputs.workload(3, L=150, B=1, H=2, dk=64, dv=64, dtype=dtype))
    o, S = _run_gpu(x, chunk=chunk)
    o_ref, S_ref = _oracle(oracle_mod, x)
    _check(x, o, S, o_ref, S_ref)


@pytest.mark.parametrize("dk,dv", [(64, 128), (128, 64), (32, 16), (96, 80), (128, 128)])
def test_rectangular_and_odd_heads(oracle_mod, dk, dv):
    x = inputs.make_inputs(inputs.workload(2, L=100, B=1, H=2, dk=dk, dv=dv))
    o, S = _run_gpu(x)
    o_ref, S_ref = _oracle(oracle_mod, x)
    _check(x, o, S, o_ref, S_ref)


@pytest.mark.parametrize("L", [1, 5, 63, 64, 65])
def test_short_sequences(oracle_mod, L):
    x = inputs.make_inputs(inputs.workload(2, L=L, B=1, H=2))
    o, S = _run_gpu(x)
    o_ref, S_ref = _oracle(oracle_mod, x)
    _check(x, o, S, o_ref, S_ref)


def test_empty_sequence_copies_state():
    x = inputs.make_inputs(inputs.workload(2, L=0, B=1, H=2))
    d = _to_dev(x)
    o, S = efla.chunk_fwd(d["q"], d["k"], d["v"], d["beta"], d["S0"], chunk=64)
    assert o.numel() == 0
    assert torch.equal(S.cpu(), x["S0"])
    o, S = efla.chunk_fwd(d["q"], d["k"], d["v"], d["beta"], None, chunk=64)
    assert torch.count_nonzero(S) == 0


def test_zero_keys_and_zero_beta_are_noops(oracle_mod):
    w = inputs.workload(3, L=192, B=1, H=2)
    x = inputs.make_inputs(w)
    x["k"][:, :, 10:20] = 0
    x["beta"][:, :, 70:90] = 0
    o, S = _run_gpu(x)
    o_ref, S_ref = _oracle(oracle_mod, x)
    _check(x, o, S, o_ref, S_ref)


def test_state_aliasing_and_resume(oracle_mod):
    """S_final may alias S0; running L in two calls with the state carried equals one
    call (bit-exact when the split falls on a chunk boundary)."""
    x = inputs.make_inputs(inputs.workload(2, L=256, B=1, H=2))
    d = _to_dev(x)
    o_full, S_full = efla.chunk_fwd(d["q"], d["k"], d["v"], d["beta"], d["S0"], chunk=64)
    S = d["S0"].clone()
    sl = lambda t, a, b: t[:, :, a:b].contiguous()
    o1, _ = efla.chunk_fwd(sl(d["q"], 0, 128), sl(d["k"], 0, 128), sl(d["v"], 0, 128),
                           sl(d["beta"], 0, 128), S, chunk=64, S_final=S)
    o2, _ = efla.chunk_fwd(sl(d["q"], 128, 256), sl(d["k"], 128, 256), sl(d["v"], 128, 256),
                           sl(d["beta"], 128, 256), S, chunk=64, S_final=S)
    torch.cuda.synchronize()
    assert torch.equal(torch.cat([o1, o2], dim=2), o_full)
    assert torch.equal(S, S_full)


@pytest.mark.parametrize("wid", [3, 5])
def test_bf16_output_option(oracle_mod, wid):
    x = inputs.make_inputs(inputs.workload(wid, L=300, B=1, H=2))
    d = _to_dev(x)
    o, S = efla.chunk_fwd(d["q"], d["k"], d["v"], d["beta"], d["S0"], chunk=64,
                          o_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    assert o.dtype == torch.bfloat16
    o_ref, S_ref = _oracle(oracle_mod, x)
    rms = float(np.sqrt(np.mean(o_ref ** 2)))
    bound = 2e-2 + 2.0 ** -8 * float(np.abs(o_ref).max()) / rms
    assert rel_err(o.float().cpu().numpy(), o_ref) <= bound
    assert rel_err(S.cpu().numpy(), S_ref) <= 2e-2


@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 64), (128, 64), (64, 128)])
def test_tensor_core_path_selected(dk, dv):
    """bf16 inputs with chunk 64 and head sizes 64/128 take the tcgen05 kernels."""
    assert efla.chunk_fwd_path(2, 4, 1000, dk, dv, 64, torch.bfloat16) == "tcgen05"
    assert efla.chunk_fwd_path(2, 4, 1000, dk, dv, 64, torch.float32) == "simt"
    assert efla.chunk_fwd_path(2, 4, 1000, dk, dv, 32, torch.bfloat16) == "simt"


def test_tensor_core_state_carry_across_calls(oracle_mod):
    """Chunk boundaries aligned to calls: two tcgen05 calls with the state carried equal
    one call up to the fp16 rounding of the carried state's operand copy."""
    x = inputs.make_inputs(inputs.workload(4, L=512, B=1, H=2))
    d = _to_dev(x)
    o_full, S_full = efla.chunk_fwd(d["q"], d["k"], d["v"], d["beta"], None, chunk=64)
    sl = lambda t, a, b: t[:, :, a:b].contiguous()
    o1, S1 = efla.chunk_fwd(sl(d["q"], 0, 256), sl(d["k"], 0, 256), sl(d["v"], 0, 256),
                            sl(d["beta"], 0, 256), None, chunk=64)
    o2, S2 = efla.chunk_fwd(sl(d["q"], 256, 512), sl(d["k"], 256, 512), sl(d["v"], 256, 512),
                            sl(d["beta"], 256, 512), S1, chunk=64)
    torch.cuda.synchronize()
    # loading S0 into the tensor-memory state is exact, so the split run is bit-identical
    assert torch.equal(torch.cat([o1, o2], dim=2), o_full)
    assert torch.equal(S2, S_full)
    o_ref, S_ref = _oracle(oracle_mod, x)
    assert rel_err(S2.cpu().numpy(), S_ref) < 2e-2


def test_linearity_in_values_and_state():
    """o and S_final are linear in (V, S0) for fixed q, k, beta (fp32 inputs)."""
    w = inputs.workload(1, L=80, B=1, H=2)
    x = inputs.make_inputs(w)
    d = _to_dev(x)
    g = torch.Generator().manual_seed(3)
    V2 = torch.randn(d["v"].shape, generator=g).cuda()
    S1 = 0.1 * torch.randn((1, 2, 16, 16), generator=g).cuda()
    S2 = 0.1 * torch.randn((1, 2, 16, 16), generator=g).cuda()
    a, b = 0.75, -1.5
    o1, F1 = efla.chunk_fwd(d["q"], d["k"], d["v"], d["beta"], S1, chunk=16)
    o2, F2 = efla.chunk_fwd(d["q"], d["k"], V2, d["beta"], S2, chunk=16)
    o3, F3 = efla.chunk_fwd(d["q"], d["k"], a * d["v"] + b * V2, d["beta"], a * S1 + b * S2, chunk=16)
    assert rel_err(o3.cpu().numpy(), (a * o1 + b * o2).cpu().numpy()) < 1e-5
    assert rel_err(F3.cpu().numpy(), (a * F1 + b * F2).cpu().numpy()) < 1e-5


# ---- sequence segments: few heads and a long sequence run as parallel segments whose affine
# state maps (S_out = P S_in + H) are chained and then rerun from their true starting states


def test_segment_path_selection():
    bf = torch.bfloat16
    assert efla.chunk_fwd_path(1, 16, 65536, 128, 128, 64, bf) == "tcgen05-segments"
    assert efla.chunk_fwd_path(1, 48, 4096, 128, 128, 64, bf) == "tcgen05-segments"
    assert efla.chunk_fwd_path(1, 49, 4096, 128, 128, 64, bf) == "tcgen05"   # too many heads
    assert efla.chunk_fwd_path(1, 2, 47 * 64, 128, 128, 64, bf) == "tcgen05"  # too few chunks
    assert efla.chunk_fwd_path(1, 2, 4096, 128, 64, 64, bf) == "tcgen05"      # dk != dv


@pytest.mark.parametrize("L", [48 * 64 - 10, 48 * 64])
def test_segments_stiff_parity(oracle_mod, L):
    """Workload-5 distributions (key norms over six decades, 5% of values x10) on two heads,
    cut into three segments; the first length ends in a ragged chunk."""
    x = inputs.make_inputs(inputs.workload(5, B=1, H=2, L=L))
    assert efla.chunk_fwd_path(1, 2, L, 128, 128, 64, torch.bfloat16) == "tcgen05-segments"
    o, S = _run_gpu(x)
    o_ref, S_ref = _oracle(oracle_mod, x)
    _check(x, o, S, o_ref, S_ref)


def test_segments_from_nonzero_state(oracle_mod):
    """A nonzero initial state enters through segment 0 and every later segment's start."""
    x = inputs.make_inputs(inputs.workload(2, B=1, H=3, L=64 * 64, dk=128, dv=128))
    assert x["S0"] is not None and float(x["S0"].abs().max()) > 0
    assert efla.chunk_fwd_path(1, 3, 64 * 64, 128, 128, 64, torch.bfloat16) == "tcgen05-segments"
    o, S = _run_gpu(x)
    o_ref, S_ref = _oracle(oracle_mod, x)
    _check(x, o, S, o_ref, S_ref)


def test_segments_in_place_state_carry(oracle_mod):
    """S_final may alias S0 with segments too: the segments read S0 before the last writes it."""
    x = inputs.make_inputs(inputs.workload(2, B=1, H=2, L=64 * 64, dk=128, dv=128))
    d = _to_dev(x)
    S = d["S0"].clone()
    o, S_out = efla.chunk_fwd(d["q"], d["k"], d["v"], d["beta"], S, chunk=64, S_final=S)
    torch.cuda.synchronize()
    assert efla.last_device_error() == 0
    assert S_out.data_ptr() == S.data_ptr()
    o_ref, S_ref = _oracle(oracle_mod, x)
    _check(x, o.float().cpu(), S.cpu(), o_ref, S_ref)


def test_bounded_wait_reports_timeout_and_leaves_the_context_usable(oracle_mod):
    """A wait that nothing completes gives up after its bound, sets the device error word
    (read as EFLA_ERR_TIMEOUT, then cleared) and returns; the next forward runs normally."""
    EFLA_ERR_TIMEOUT = 6
    efla.selftest_bounded_wait(1_000_000)
    assert efla.last_device_error() == EFLA_ERR_TIMEOUT
    assert efla.last_device_error() == 0  # read-and-clear
    x = inputs.make_inputs(inputs.workload(4, B=1, H=2, L=200))
    o, S = _run_gpu(x)  # asserts the error word is clear again
    o_ref, S_ref = _oracle(oracle_mod, x)
    _check(x, o, S, o_ref, S_ref)


def test_bf16_inputs_near_the_fp16_range(oracle_mod):
    """The tensor-core path runs its products on fp16 operands: the bf16 q, k and v tiles are
    converted to fp16, and so are the intermediates U' and the state's operand copy.  fp16's
    largest finite value is 65504, so inputs must keep every such value below it; close to that
    limit the path must still match the oracle.  v is scaled to max |v| = 6e4 with keys of squared
    norm in [1, 4] (so alpha <= 1); the fp64 walk below checks that the largest u_t = alpha_t (v_t -
    S_{t-1}^T k_t), state entry and output each lie between 2e4 and 65504."""
    w = inputs.workload(3, B=1, H=2, L=300)
    x = inputs.make_inputs(w, seed=23)
    g = torch.Generator().manual_seed(24)
    k = x["k"].double()
    k = k / k.norm(dim=-1, keepdim=True)
    n2 = torch.exp(torch.rand(k.shape[:-1] + (1,), generator=g, dtype=torch.float64) * np.log(4.0))
    x["k"] = (k * n2.sqrt()).to(torch.bfloat16)
    v = x["v"].double()
    x["v"] = (v * (6e4 / v.abs().max())).to(torch.bfloat16)
    # fp64 walk of the recurrence: the magnitudes the fp16 operands must hold
    q64, k64, v64, b64 = (x[n].double().numpy() for n in ("q", "k", "v", "beta"))
    big = {"u": 0.0, "S": 0.0, "o": 0.0}
    for h in range(w.H):
        S = np.zeros((w.dk, w.dv))
        for t in range(w.L):
            kt, vt, qt = k64[0, h, t], v64[0, h, t], q64[0, h, t]
            lam = float(kt @ kt)
            a = -np.expm1(-b64[0, h, t] * lam) / lam
            u = a * (vt - S.T @ kt)
            S += np.outer(kt, u)
            big["u"] = max(big["u"], float(np.abs(u).max()))
            big["S"] = max(big["S"], float(np.abs(S).max()))
            big["o"] = max(big["o"], float(np.abs(S.T @ qt).max()))
    assert all(2e4 < m < 65504.0 for m in big.values()), big
    o, S = _run_gpu(x)
    o_ref, S_ref = _oracle(oracle_mod, x)
    _check(x, o, S, o_ref, S_ref)


def test_workspace_alignment_does_not_change_results(oracle_mod):
    """The tensor-core forward drops its Ta tiles from L2 unwritten once the state kernel has read
    them, but only when the workspace is 128-byte aligned. A workspace that is only 16-byte
    aligned keeps them. Both give the same outputs bit for bit. A call that follows a dropping
    call on the same workspace is not affected by the dropped lines, and the result meets the
    oracle's bf16 bound."""
    x = inputs.make_inputs(inputs.workload(4, B=1, H=3, L=300))
    d = _to_dev(x)
    args = (d["q"], d["k"], d["v"], d["beta"], d["S0"])
    B, H, L, dk = x["q"].shape
    need = efla.workspace_size(B, H, L, dk, x["v"].shape[-1], 64, torch.bfloat16, torch.bfloat16)
    buf = torch.empty(need + 256, dtype=torch.uint8, device="cuda")
    assert buf.data_ptr() % 128 == 0 and (buf.data_ptr() + 16) % 128 != 0
    runs = [efla.chunk_fwd(*args, chunk=64, o_dtype=torch.bfloat16, workspace=w)
            for w in (buf[:need], buf[16:16 + need], buf[:need], buf[:need])]
    torch.cuda.synchronize()
    assert efla.last_device_error() == 0
    for o, S in runs[1:]:
        assert torch.equal(o, runs[0][0]) and torch.equal(S, runs[0][1])
    o_ref, S_ref = _oracle(oracle_mod, x)
    rms = float(np.sqrt(np.mean(o_ref ** 2)))
    assert rel_err(runs[1][0].float().cpu().numpy(), o_ref) <= 2e-2 + 2.0 ** -8 * float(np.abs(o_ref).max()) / rms
    assert rel_err(runs[1][1].cpu().numpy(), S_ref) <= 2e-2
