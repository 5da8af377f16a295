"""Multi-rank host logic with world size 2 on the gloo backend (CPU only).

The decode step shards by batch item with no data-path collective; the ranks
only agree on timing. These tests run two real processes and check the
whole-job throughput (sum of units over the slowest rank's time), the
max-over-ranks of elapsed times, the per-rank seeds, and that each rank's
independent batch differs from the others.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    from datetime import timedelta

    from gated_delta_rule_recurrent_b200 import distributed as D
    from gated_delta_rule_recurrent_b200 import workloads

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        w, r, lr = D.rank_env()
        assert (w, r, lr) == (world, rank, rank)
        # rank r processed 100 * (r + 1) units in (r + 1) seconds
        tput, slowest = D.throughput(100.0 * (rank + 1), float(rank + 1))
        mx = D.max_over_ranks(10.0 - rank)
        sm = D.sum_over_ranks(1.0)
        x = workloads.make_inputs(0, seed=D.rank_seed(workloads.WORKLOADS[0].seed, rank))
        torch.save({"tput": tput, "slowest": slowest, "max": mx, "sum": sm,
                    "query": x["query"], "seed": D.rank_seed(1000, rank)},
                   os.path.join(out_dir, f"rank{rank}.pt"))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(180)
def test_two_gloo_ranks(tmp_path):
    world = 2
    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    res = [torch.load(tmp_path / f"rank{r}.pt") for r in range(world)]
    for r in res:
        assert r["tput"] == pytest.approx((100.0 + 200.0) / 2.0)
        assert r["slowest"] == 2.0
        assert r["max"] == 10.0
        assert r["sum"] == 2.0
    assert res[0]["seed"] == 1000 and res[1]["seed"] != res[0]["seed"]
    assert not torch.equal(res[0]["query"], res[1]["query"])


def test_single_process_without_group():
    from gated_delta_rule_recurrent_b200 import distributed as D

    assert D.max_over_ranks(3.5) == 3.5
    assert D.sum_over_ranks(2.0) == 2.0
    assert D.throughput(10.0, 2.0) == (5.0, 2.0)
