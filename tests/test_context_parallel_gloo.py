"""Context-parallel forward on CPU: 2 and 3 ranks over gloo (127.0.0.1), each holding one shard of
the sequence.  The per-shard forward and the affine chaining are injected (the fp64 oracle and a
matmul), so this checks the protocol itself -- the shard maps (P from the identity with v = 0,
H from zero), the all_gather, the chaining in rank order and the rerun -- against one oracle pass
over the whole sequence.  On GPUs the same code runs the library's kernels and NCCL.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir, cuts, rule):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import torch.distributed as dist

    import oracle
    from delta_rule_linear_efla_b200 import context_parallel as cp
    from delta_rule_linear_efla_b200 import inputs

    def ofwd(q, k, v, beta, S0, rule_, chunk):
        o, S = oracle.fwd(q, k, v, beta, S0, nthreads=1, rule=rule_)
        return torch.from_numpy(o), torch.from_numpy(S)

    def affine(P, S, Hm):
        return Hm.clone() if S is None else torch.matmul(P, S) + Hm

    dist.init_process_group("gloo", init_method="env://", timeout=__import__("datetime").timedelta(seconds=60))
    x = inputs.make_inputs(inputs.workload(2, B=1, H=2, L=cuts[-1], dk=8, dv=6))
    if rule == "euler":  # unit keys: the delta rule's stable regime
        k = x["k"].double()
        x["k"] = (k / k.norm(dim=-1, keepdim=True)).to(x["k"].dtype)
    a, b = cuts[rank], cuts[rank + 1]
    sl = lambda t: t[:, :, a:b].contiguous()
    o, S = cp.cp_chunk_fwd(sl(x["q"]), sl(x["k"]), sl(x["v"]), sl(x["beta"]), x["S0"], rule=rule,
                           fwd=ofwd, affine=affine)
    o_ref, S_ref = oracle.fwd(x["q"], x["k"], x["v"], x["beta"], x["S0"], nthreads=1, rule=rule)
    eo = float(np.abs(o.numpy() - o_ref[:, :, a:b]).max())
    es = float(np.abs(S.numpy() - oracle.fwd(x["q"][:, :, :b], x["k"][:, :, :b], x["v"][:, :, :b],
                                             x["beta"][:, :, :b], x["S0"], nthreads=1,
                                             rule=rule)[1]).max())
    with open(os.path.join(out_dir, "rank%d.txt" % rank), "w") as f:
        f.write("%r %r\n" % (eo, es))
    if rank == world - 1:
        assert np.abs(S.numpy() - S_ref).max() < 1e-9
    dist.destroy_process_group()


@pytest.mark.timeout(300)
@pytest.mark.parametrize("cuts,rule", [((0, 40, 97), "exact"), ((0, 30, 31, 100), "exact"),
                                       ((0, 50, 120), "euler")])
def test_context_parallel_matches_one_pass(tmp_path, cuts, rule):
    world = len(cuts) - 1
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path), cuts, rule),
                       nprocs=world, join=True, start_method="spawn")
    for r in range(world):
        eo, es = (float(t) for t in (tmp_path / ("rank%d.txt" % r)).read_text().split())
        assert eo < 1e-9 and es < 1e-9, (r, eo, es)
