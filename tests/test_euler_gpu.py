"""GPU parity of the Euler rule (the delta rule, alpha = beta) against the fp64 oracle's Euler
rule, on every path the exact rule takes.  Keys are scaled to unit norm and beta lies in (0, 1):
the delta rule's stable regime (with beta ||k||^2 > 2 its step grows the state, which the oracle
pins show).  Bounds as for the exact rule: 1e-4 for fp32 inputs, 2e-2 for bf16 inputs.
"""
import numpy as np
import pytest
import torch

from conftest import rel_err
from delta_rule_linear_efla_b200 import efla, inputs

pytestmark = pytest.mark.gpu

TOL = {"fp32": 1e-4, "bf16": 2e-2}


def _unit_keys(x):
    k = x["k"].double()
    k = k / k.norm(dim=-1, keepdim=True).clamp_min(1e-6)
    x["k"] = k.to(x["k"].dtype)
    return x


def _dev(x):
    return {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in x.items()}


def _check_fwd(oracle_mod, x, chunk=64):
    d = _dev(x)
    o, S = efla.chunk_fwd(d["q"], d["k"], d["v"], d["beta"], d["S0"], chunk=chunk, rule="euler")
    torch.cuda.synchronize()
    assert efla.last_device_error() == 0
    o_ref, S_ref = oracle_mod.fwd(x["q"], x["k"], x["v"], x["beta"], x["S0"], rule="euler")
    tol = TOL[x["workload"].dtype]
    eo, es = rel_err(o.float().cpu().numpy(), o_ref), rel_err(S.cpu().numpy(), S_ref)
    assert eo <= tol and es <= tol, (eo, es)
    return o, S


def test_euler_tensor_core_path(oracle_mod):
    x = _unit_keys(inputs.make_inputs(inputs.workload(4, B=1, H=4, L=500)))
    assert efla.chunk_fwd_path(1, 4, 500, 128, 128, 64, torch.bfloat16) == "tcgen05"
    _check_fwd(oracle_mod, x)


def test_euler_sequence_segments(oracle_mod):
    x = _unit_keys(inputs.make_inputs(inputs.workload(2, B=1, H=2, L=48 * 64, dk=128, dv=128)))
    assert efla.chunk_fwd_path(1, 2, 48 * 64, 128, 128, 64, torch.bfloat16) == "tcgen05-segments"
    _check_fwd(oracle_mod, x)


@pytest.mark.parametrize("wid,chunk", [(1, 16), (1, 64), (3, 32)])
def test_euler_simt_path(oracle_mod, wid, chunk):
    w = inputs.workload(3, B=1, H=2, L=150, dk=64, dv=64) if wid == 3 else inputs.workload(1)
    x = _unit_keys(inputs.make_inputs(w))
    _check_fwd(oracle_mod, x, chunk=chunk)


def test_euler_decode_step(oracle_mod):
    x = _unit_keys(inputs.make_inputs(inputs.workload(2, B=2, H=3, L=1, dk=128, dv=128)))
    d = _dev(x)
    S = d["S0"].clone()
    o = efla.recurrent_step(d["q"][:, :, 0].contiguous(), d["k"][:, :, 0].contiguous(),
                            d["v"][:, :, 0].contiguous(), d["beta"][:, :, 0].contiguous(), S,
                            rule="euler")
    torch.cuda.synchronize()
    o_ref, S_ref = oracle_mod.fwd(x["q"], x["k"], x["v"], x["beta"], x["S0"], rule="euler")
    assert rel_err(o.cpu().numpy(), o_ref[:, :, 0]) < 1e-5
    assert rel_err(S.cpu().numpy(), S_ref) < 1e-5


def test_euler_alpha_is_beta():
    x = inputs.make_inputs(inputs.workload(4, B=1, H=2, L=300))
    d = _dev(x)
    a = efla.alpha(d["k"], d["beta"], rule="euler")
    torch.cuda.synchronize()
    assert torch.equal(a.cpu(), x["beta"].float())


def test_rule_changes_the_result():
    x = _unit_keys(inputs.make_inputs(inputs.workload(4, B=1, H=2, L=256)))
    x["beta"] = (x["beta"].float() * 2).to(x["beta"].dtype)  # beta lambda up to 2: rules differ
    d = _dev(x)
    o_e, _ = efla.chunk_fwd(d["q"], d["k"], d["v"], d["beta"], d["S0"], rule="exact")
    o_u, _ = efla.chunk_fwd(d["q"], d["k"], d["v"], d["beta"], d["S0"], rule="euler")
    torch.cuda.synchronize()
    assert rel_err(o_u.cpu().numpy(), o_e.cpu().numpy()) > 0.1
