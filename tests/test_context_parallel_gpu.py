"""GPU pieces of the context-parallel forward in one process (a run of this suite has one GPU):
the affine chaining kernel against numpy, and the shard protocol -- shard maps from the library's
chunk forward, chained starting states, reruns -- over emulated ranks against one oracle pass."""
import numpy as np
import pytest
import torch

from conftest import rel_err
from delta_rule_linear_efla_b200 import context_parallel as cp
from delta_rule_linear_efla_b200 import efla, inputs

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 128), (16, 8), (200, 33)])
def test_state_affine_kernel(dk, dv):
    g = torch.Generator().manual_seed(dk * 1000 + dv)
    P = torch.randn(2, 3, dk, dk, generator=g) / dk ** 0.5
    S = torch.randn(2, 3, dk, dv, generator=g)
    Hm = torch.randn(2, 3, dk, dv, generator=g)
    ref = np.einsum("bhij,bhjk->bhik", P.double().numpy(), S.double().numpy()) + Hm.double().numpy()
    out = efla.state_affine(P.cuda(), S.cuda(), Hm.cuda())
    assert rel_err(out.cpu().numpy(), ref) < 1e-5
    Sd = S.cuda()
    efla.state_affine(P.cuda(), Sd, Hm.cuda(), out=Sd)  # in place over S_in
    assert rel_err(Sd.cpu().numpy(), ref) < 1e-5
    only_h = efla.state_affine(P.cuda(), None, Hm.cuda())
    assert torch.equal(only_h.cpu(), Hm)


@pytest.mark.parametrize("cuts,rule", [((0, 300, 700, 1000), "exact"), ((0, 64, 128), "exact"),
                                       ((0, 500, 1000), "euler")])
def test_shards_emulated_on_one_gpu(oracle_mod, cuts, rule):
    x = inputs.make_inputs(inputs.workload(4, B=1, H=3, L=cuts[-1]))
    if rule == "euler":
        k = x["k"].double()
        x["k"] = (k / k.norm(dim=-1, keepdim=True)).to(x["k"].dtype)
    d = {k_: (v.cuda() if isinstance(v, torch.Tensor) else v) for k_, v in x.items()}
    sl = lambda t, a, b: t[:, :, a:b].contiguous()
    maps, outs = [], []
    for r in range(len(cuts) - 1):
        a, b = cuts[r], cuts[r + 1]
        q, k, v, beta = (sl(d[n], a, b) for n in ("q", "k", "v", "beta"))
        if r == 0:
            o, S = efla.chunk_fwd(q, k, v, beta, d["S0"], rule=rule)
            maps.append((torch.zeros(1, 3, 128, 128, device="cuda"), S))
        else:
            S_in = cp.chain_start(maps)
            o, S = efla.chunk_fwd(q, k, v, beta, S_in, rule=rule)
            maps.append(cp.shard_map(q, k, v, beta, rule=rule))
        outs.append(o)
    torch.cuda.synchronize()
    assert efla.last_device_error() == 0
    o_ref, S_ref = oracle_mod.fwd(x["q"], x["k"], x["v"], x["beta"], x["S0"], rule=rule)
    assert rel_err(torch.cat(outs, dim=2).cpu().numpy(), o_ref) < 2e-2
    assert rel_err(S.cpu().numpy(), S_ref) < 2e-2
    S_chain = cp.chain_start(maps)  # the maps chained end to end give the final state too
    assert rel_err(S_chain.cpu().numpy(), S_ref) < 2e-2
