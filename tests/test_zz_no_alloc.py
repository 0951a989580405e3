"""efla_chunk_fwd_noalloc: the chunk forward for callers that cannot allocate
device memory (they receive only their input and output buffers, or must not
call cudaMalloc on their hot path), so they cannot provide the workspace that
efla_chunk_fwd asks for.  The library serves them from one fixed scratch array
in its device code.

The entry point is called through the C ABI on several sizes in a row, and
each result is compared with the workspace entry point's result on the same
inputs.  Both run the same kernels on the same inputs, so the outputs must be
bit-identical; a partial overwrite of the shared scratch by an earlier call
would show as a difference.  The sizes cover the one-pass tensor-core path at
exactly the scratch size (the 1.3B-shaped workload: 4096 chunks x 8 KiB of
T*diag(alpha) tiles), the sequence-segment path (few heads, long sequences),
including a size whose tiles and segment states fill the scratch exactly, a
size whose segment states would not fit, which keeps the one-pass form, and a
size beyond the scratch, which is refused.  This file is named so that pytest
collects it last.
"""
import pytest
import torch

from delta_rule_linear_efla_b200 import efla, inputs

pytestmark = pytest.mark.gpu

EFLA_ERR_TOO_LARGE = 9
SCRATCH_BYTES = 32 * 1024 * 1024


def _dev(x):
    return {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in x.items()}


def _noalloc(d, o, S_final, chunk=64):
    lib = efla.load_library()
    B, H, L, dk = d["q"].shape
    dv = d["v"].shape[-1]
    return lib.efla_chunk_fwd_noalloc(
        d["q"].data_ptr(), d["k"].data_ptr(), d["v"].data_ptr(), d["beta"].data_ptr(),
        d["S0"].data_ptr() if d["S0"] is not None else None, o.data_ptr(), S_final.data_ptr(),
        B, H, L, dk, dv, chunk, efla.EFLA_BF16, efla.EFLA_F32,
        torch.cuda.current_stream().cuda_stream)


CASES = [
    # (workload overrides, path efla_chunk_fwd takes: 1 one pass, 2 segments)
    (dict(wid=4), 1),                                          # 4*16*64 chunks: the full scratch
    (dict(wid=2, B=3, H=5, L=1000, dk=128, dv=128), 1),        # other sizes, S0 != 0, ragged tail
    (dict(wid=3, B=1, H=2, L=4096), 2),                        # segments: 2 heads x 64 chunks
    (dict(wid=3, B=1, H=16, L=4096), 2),                       # segments, tiles + states = 32 MiB
    (dict(wid=5, B=1, H=2, L=4100), 2),                        # segments, ragged tail, stiff inputs
]


@pytest.mark.parametrize("case,path", CASES)
def test_noalloc_equals_workspace_entry_point(case, path):
    case = dict(case)
    w = inputs.workload(case.pop("wid"), **case)
    names = {1: "tcgen05", 2: "tcgen05-segments"}
    assert efla.chunk_fwd_path(w.B, w.H, w.L, w.dk, w.dv, 64, torch.bfloat16) in (names[path], "tcgen05")
    d = _dev(inputs.make_inputs(w, seed=77 + w.id + w.H))
    o_ref, S_ref = efla.chunk_fwd(d["q"], d["k"], d["v"], d["beta"], d["S0"], chunk=64)
    o = torch.full_like(o_ref, float("nan"))
    S = torch.full_like(S_ref, float("nan"))
    assert _noalloc(d, o, S) == 0
    torch.cuda.synchronize()
    assert efla.last_device_error() == 0
    assert torch.equal(o, o_ref) and torch.equal(S, S_ref)


def test_noalloc_two_calls_in_a_row():
    """Two calls back to back on different sizes, each bit-identical to the workspace entry
    point: the second call finds the first call's contents in the scratch."""
    for w in (inputs.workload(4), inputs.workload(3, B=1, H=16, L=4096)):
        d = _dev(inputs.make_inputs(w, seed=5))
        o = torch.empty((w.B, w.H, w.L, w.dv), dtype=torch.float32, device="cuda")
        S = torch.empty((w.B, w.H, w.dk, w.dv), dtype=torch.float32, device="cuda")
        assert _noalloc(d, o, S) == 0
        torch.cuda.synchronize()
        o_ref, S_ref = efla.chunk_fwd(d["q"], d["k"], d["v"], d["beta"], d["S0"], chunk=64)
        torch.cuda.synchronize()
        assert torch.equal(o, o_ref) and torch.equal(S, S_ref)


def test_noalloc_keeps_the_one_pass_form_when_segment_states_do_not_fit(oracle_mod):
    """22 heads of 4096 tokens: efla_chunk_fwd would cut the sequence into segments, whose states
    (22 x 1.5 MiB) do not fit beside the tiles (11 MiB) in the fixed scratch, so this call runs
    the one-pass form instead.
    The rounding then differs from the segmented call's, so both are checked against the oracle
    (bf16 bound), and nothing is refused."""
    from conftest import rel_err

    w = inputs.workload(3, B=1, H=22, L=4096)
    assert efla.chunk_fwd_path(w.B, w.H, w.L, w.dk, w.dv, 64, torch.bfloat16) == "tcgen05-segments"
    assert efla.workspace_size(w.B, w.H, w.L, w.dk, w.dv, 64, torch.bfloat16) > SCRATCH_BYTES
    x = inputs.make_inputs(w, seed=9)
    d = _dev(x)
    o = torch.empty((w.B, w.H, w.L, w.dv), dtype=torch.float32, device="cuda")
    S = torch.empty((w.B, w.H, w.dk, w.dv), dtype=torch.float32, device="cuda")
    assert _noalloc(d, o, S) == 0
    torch.cuda.synchronize()
    assert efla.last_device_error() == 0
    o_ref, S_ref = oracle_mod.fwd(x["q"], x["k"], x["v"], x["beta"], x["S0"])
    assert rel_err(o.cpu().numpy(), o_ref) <= 2e-2
    assert rel_err(S.cpu().numpy(), S_ref) <= 2e-2


def test_noalloc_refuses_sizes_beyond_its_scratch():
    w = inputs.workload(4, L=4096 + 64)  # 4*16*65 chunks of tiles > 32 MiB: refused on the host
    d = _dev(inputs.make_inputs(w))
    o = torch.empty((w.B, w.H, w.L, w.dv), dtype=torch.float32, device="cuda")
    S = torch.empty((w.B, w.H, w.dk, w.dv), dtype=torch.float32, device="cuda")
    before = efla.kernel_launches()
    assert _noalloc(d, o, S) == EFLA_ERR_TOO_LARGE
    assert efla.kernel_launches() == before
    assert "scratch" in efla.status_str(EFLA_ERR_TOO_LARGE)
