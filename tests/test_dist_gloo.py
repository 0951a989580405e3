"""The multi-GPU plumbing of bench.py on CPU: two ranks over gloo (127.0.0.1).

Heads are independent, so N GPUs run N replicas on disjoint heads; the only collectives are
the barrier around the timed region and the max of its duration.  This checks the
environment parsing, the max-over-ranks reduction, the whole-job rate and that the ranks'
seeded inputs are disjoint.
"""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, out_dir: str) -> None:
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import torch.distributed as dist

    from delta_rule_linear_efla_b200 import dist as edist
    from delta_rule_linear_efla_b200 import inputs

    assert edist.world() == (world, rank, rank)
    edist.init("gloo", timeout_s=60)
    edist.barrier()
    local_ms = 10.0 + 5.0 * rank
    slowest = edist.max_over_ranks(local_ms)
    assert slowest == 10.0 + 5.0 * (world - 1)
    rate = edist.aggregate_rate(1000, 4, world, slowest)
    assert abs(rate - 1000 * 4 * world / (slowest / 1e3)) < 1e-6
    # each rank draws its own heads
    w = inputs.workload(3, B=1, H=2, L=64)
    x = inputs.make_inputs(w, seed=edist.replica_seed(1003, rank))
    mine = torch.tensor([float(x["k"].float().sum())], dtype=torch.float64)
    allv = [torch.zeros(1, dtype=torch.float64) for _ in range(world)]
    dist.all_gather(allv, mine)
    assert len({float(v) for v in allv}) == world
    with open(os.path.join(out_dir, "rank%d.ok" % rank), "w") as f:
        f.write("%.3f\n" % slowest)
    dist.destroy_process_group()


@pytest.mark.timeout(300)
def test_two_ranks_gloo(tmp_path):
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    for r in range(world):
        assert (tmp_path / ("rank%d.ok" % r)).read_text().strip() == "15.000"


def test_single_process_defaults(monkeypatch):
    from delta_rule_linear_efla_b200 import dist as edist

    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    assert edist.world() == (1, 0, 0)
    assert edist.max_over_ranks(3.5) == 3.5
    assert edist.replica_seed(1004, 0, 0) != edist.replica_seed(1004, 0, 1)
