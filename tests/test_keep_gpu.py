"""GPU checks of the training-step pair efla_chunk_fwd_keep / efla_bwd_kept: the forward that keeps
what the backward would recompute gives efla_chunk_fwd's o and S_final bit for bit, and the
backward that reads the kept buffer gives efla_bwd's gradients (the kept u and chunk states come
from the same products, rounded at the same points) and meets the oracle's bf16 bound, with
ragged tails, sequence segments, both rules, S0 and dS_final, a head that walks on CUDA cores,
and through the autograd wrapper."""
import pytest
import torch

from conftest import rel_err
from delta_rule_linear_efla_b200 import efla, inputs

pytestmark = pytest.mark.gpu

BF16_TOL = 2e-2


def _case(wid, rule="exact", seed=9, **kw):
    x = inputs.make_inputs(inputs.workload(wid, **kw), seed=seed)
    if rule == "euler":
        k = x["k"].double()
        x["k"] = (k / k.norm(dim=-1, keepdim=True)).to(x["k"].dtype)
    g = torch.Generator().manual_seed(seed + 1)
    B, H, L, dv = x["v"].shape
    dk = x["k"].shape[-1]
    x["dO"] = torch.randn(B, H, L, dv, generator=g)
    x["dS"] = torch.randn(B, H, dk, dv, generator=g) * 0.1
    if x["S0"] is None:
        x["S0"] = torch.randn(B, H, dk, dv, generator=g) * 0.1
    return x


def _dev(x):
    return {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in x.items()}


@pytest.mark.parametrize("rule", ["exact", "euler"])
@pytest.mark.parametrize("wid,kw", [(4, dict(B=1, H=3, L=300)),                     # ragged tail
                                    (3, dict(B=1, H=2, L=4096)),                    # sequence segments
                                    (2, dict(B=2, H=2, L=200, dk=64, dv=128))])     # rectangular heads
def test_keep_pair_matches_the_plain_calls_and_the_oracle(oracle_mod, rule, wid, kw):
    x = _case(wid, rule, **kw)
    d = _dev(x)
    args = (d["q"], d["k"], d["v"], d["beta"])
    o_ref, S_ref = efla.chunk_fwd(*args, d["S0"], rule=rule)
    o, S, kept = efla.chunk_fwd_keep(*args, d["S0"], rule=rule)
    torch.cuda.synchronize()
    assert efla.last_device_error() == 0
    assert torch.equal(o, o_ref) and torch.equal(S, S_ref)
    plain = efla.bwd(*args, d["dO"], d["S0"], d["dS"], rule=rule)
    got = efla.bwd(*args, d["dO"], d["S0"], d["dS"], rule=rule, kept=kept)
    torch.cuda.synchronize()
    assert efla.last_device_error() == 0
    ref = oracle_mod.bwd(x["q"], x["k"], x["v"], x["beta"], x["dO"], x["S0"], x["dS"], rule=rule)
    for name, g, p, r in zip(("dq", "dk", "dv", "dbeta", "dS0"), got, plain, ref):
        assert rel_err(g.cpu().numpy(), p.cpu().numpy()) <= 1e-5, name
        assert rel_err(g.cpu().numpy(), r) <= BF16_TOL, name


def test_kept_buffer_with_a_head_on_cuda_cores(oracle_mod):
    """A key of squared norm 30 sends head 1 to the fp32 walk, which ignores the kept buffer; the
    other heads read it.  Every head against the oracle."""
    x = _case(4, B=1, H=3, L=200)
    k = x["k"].double()
    k[0, 1, 50] *= (30.0 / k[0, 1, 50].pow(2).sum()).sqrt()
    x["k"] = k.to(torch.bfloat16)
    d = _dev(x)
    args = (d["q"], d["k"], d["v"], d["beta"])
    _, _, kept = efla.chunk_fwd_keep(*args, d["S0"])
    got = efla.bwd(*args, d["dO"], d["S0"], d["dS"], kept=kept)
    torch.cuda.synchronize()
    assert efla.last_device_error() == 0
    ref = oracle_mod.bwd(x["q"], x["k"], x["v"], x["beta"], x["dO"], x["S0"], x["dS"])
    for name, g, r in zip(("dq", "dk", "dv", "dbeta", "dS0"), got, ref):
        for h in range(3):
            assert rel_err(g[0, h].cpu().numpy(), r[0, h]) <= BF16_TOL, (name, h)


def test_autograd_wrapper_keeps_the_forward():
    """efla_attention on bf16 heads of 128 runs chunk_fwd_keep and hands the kept buffer to its
    backward: its outputs and its gradients (rounded to the inputs' dtype) are those of the
    explicit pair, bit for bit (the pair itself is checked against the oracle above)."""
    x = _case(4, B=1, H=2, L=257)
    d = _dev(x)
    assert efla.keeps_for_bwd(d["q"], d["v"])
    leaves = [d[n].clone().requires_grad_(True) for n in ("q", "k", "v", "beta", "S0")]
    o, S = efla.efla_attention(*leaves)
    ((o * d["dO"]).sum() + (S * d["dS"]).sum()).backward()
    args = (d["q"], d["k"], d["v"], d["beta"])
    o2, S2, kept = efla.chunk_fwd_keep(*args, d["S0"])
    grads = efla.bwd(*args, d["dO"], d["S0"], d["dS"], kept=kept)
    torch.cuda.synchronize()
    assert torch.equal(o.detach(), o2) and torch.equal(S.detach(), S2)
    for t, g in zip(leaves, grads):
        assert t.grad is not None and t.grad.dtype == t.dtype
        assert torch.equal(t.grad, g.to(t.dtype))
