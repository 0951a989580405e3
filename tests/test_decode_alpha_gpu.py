"""GPU parity of the decode step and of the per-token alpha kernel against the
fp64 oracle.

Decode: workload 4's batch (B=64, H=16, dk=dv=128) starting from the carried
fp32 state, which the oracle computes from the seeded 256-token prefix; both
sides start from that same fp32 state.  Bound 2e-2 (bf16 inputs) / 1e-4 (fp32),
max |delta| / RMS, on o and on the updated state.
"""
import math

import numpy as np
import pytest
import torch

from conftest import rel_err
from delta_rule_linear_efla_b200 import efla, inputs

pytestmark = pytest.mark.gpu


def _oracle_step_batch(oracle_mod, S, q, k, v, beta):
    B, H, dk, dv = S.shape
    S_new = np.zeros((B, H, dk, dv))
    o = np.zeros((B, H, dv))
    for b in range(B):
        for h in range(H):
            S_new[b, h], o[b, h], _ = oracle_mod.step(S[b, h], q[b, h], k[b, h], v[b, h],
                                                      float(beta[b, h]))
    return o, S_new


def test_decode_workload4(oracle_mod):
    d = inputs.make_decode_inputs(4)
    p = d["prefix"]
    _, S_carried = oracle_mod.fwd(p["q"], p["k"], p["v"], p["beta"], None)
    S32 = torch.from_numpy(S_carried).float()  # the carried state is stored in fp32
    o_ref, S_ref = _oracle_step_batch(oracle_mod, S32.double().numpy(), d["q"].double().numpy(),
                                      d["k"].double().numpy(), d["v"].double().numpy(),
                                      d["beta"].double().numpy())
    S = S32.cuda()
    o = efla.recurrent_step(d["q"].cuda(), d["k"].cuda(), d["v"].cuda(), d["beta"].cuda(), S)
    torch.cuda.synchronize()
    assert rel_err(o.float().cpu().numpy(), o_ref) <= 2e-2
    assert rel_err(S.cpu().numpy(), S_ref) <= 2e-2
    # the state update itself is fp32 arithmetic on exact inputs: far inside the bound
    assert rel_err(S.cpu().numpy(), S_ref) <= 1e-5


@pytest.mark.parametrize("dk,dv,dtype", [(16, 16, torch.float32), (64, 64, torch.float32),
                                         (128, 128, torch.float32), (128, 64, torch.bfloat16),
                                         (96, 80, torch.float32), (200, 130, torch.bfloat16),
                                         (32, 128, torch.bfloat16)])
def test_decode_shapes(oracle_mod, dk, dv, dtype):
    g = torch.Generator().manual_seed(dk * 1000 + dv)
    B, H = 3, 5
    q = (torch.randn((B, H, dk), generator=g) / math.sqrt(dk)).to(dtype)
    k = (torch.randn((B, H, dk), generator=g) / math.sqrt(dk)).to(dtype)
    v = torch.randn((B, H, dv), generator=g).to(dtype)
    beta = torch.sigmoid(torch.randn((B, H), generator=g)).to(dtype)
    S0 = 0.3 * torch.randn((B, H, dk, dv), generator=g)
    o_ref, S_ref = _oracle_step_batch(oracle_mod, S0.double().numpy(), q.double().numpy(),
                                      k.double().numpy(), v.double().numpy(), beta.double().numpy())
    S = S0.cuda()
    o = efla.recurrent_step(q.cuda(), k.cuda(), v.cuda(), beta.cuda(), S)
    torch.cuda.synchronize()
    tol = 1e-4 if dtype == torch.float32 else 2e-2
    assert rel_err(o.float().cpu().numpy(), o_ref) <= tol
    assert rel_err(S.cpu().numpy(), S_ref) <= 1e-4


def test_decode_bf16_output():
    g = torch.Generator().manual_seed(5)
    q = (torch.randn((4, 16, 128), generator=g) / 11.3).bfloat16()
    k = (torch.randn((4, 16, 128), generator=g) / 11.3).bfloat16()
    v = torch.randn((4, 16, 128), generator=g).bfloat16()
    beta = torch.sigmoid(torch.randn((4, 16), generator=g)).bfloat16()
    S0 = 0.3 * torch.randn((4, 16, 128, 128), generator=g)
    S1, S2 = S0.cuda(), S0.cuda()
    o32 = efla.recurrent_step(q.cuda(), k.cuda(), v.cuda(), beta.cuda(), S1)
    o16 = efla.recurrent_step(q.cuda(), k.cuda(), v.cuda(), beta.cuda(), S2, o_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    assert o16.dtype == torch.bfloat16 and o32.dtype == torch.float32
    assert torch.equal(o16, o32.bfloat16())
    assert torch.equal(S1, S2)


def test_decode_matches_one_token_chunk_forward():
    """A decode step equals a one-token chunk forward from the same state."""
    x = inputs.make_inputs(inputs.workload(2, L=1, B=2, H=3))
    d = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in x.items()}
    o1, S1 = efla.chunk_fwd(d["q"], d["k"], d["v"], d["beta"], d["S0"], chunk=64)
    S = d["S0"].clone()
    o2 = efla.recurrent_step(d["q"][:, :, 0].contiguous(), d["k"][:, :, 0].contiguous(),
                             d["v"][:, :, 0].contiguous(), d["beta"][:, :, 0].contiguous(), S)
    torch.cuda.synchronize()
    # the chunk forward of bf16 inputs runs on the tensor cores with fp16 operands
    # (relative rounding 2^-11 per operand); the decode step is fp32 throughout
    tc = efla.chunk_fwd_path(2, 3, 1, 64, 64, 64, torch.bfloat16) == "tcgen05"
    tol = 1e-2 if tc else 1e-5
    assert rel_err(o2.float().cpu().numpy(), o1[:, :, 0].float().cpu().numpy()) < 2e-2
    assert rel_err(S.cpu().numpy(), S1.cpu().numpy()) < tol


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_alpha_kernel(oracle_mod, dtype):
    w = inputs.workload(5, H=4, L=3000)
    x = inputs.make_inputs(w)
    k, beta = x["k"].to(dtype), x["beta"].to(dtype)
    k[0, 0, :5] = 0  # the lambda -> 0 limit
    a = efla.alpha(k.cuda(), beta.cuda())
    torch.cuda.synchronize()
    lam = k.double().pow(2).sum(-1).numpy()
    bt = beta.double().numpy()
    ref = np.vectorize(oracle_mod.alpha)(lam, bt)
    got = a.cpu().double().numpy()
    rel = np.abs(got - ref) / np.abs(ref)
    assert rel.max() < 1e-5, rel.max()  # fp32 sum of dk squares + expm1f
    assert np.array_equal(got[0, 0, :5], bt[0, 0, :5].astype(np.float32).astype(np.float64))
