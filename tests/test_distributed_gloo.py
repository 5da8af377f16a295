"""Multi-rank host logic with world size 2 on the gloo backend (CPU only).

The decode step shards by batch item or by value head with no data-path
collective; the ranks only agree on timing. These tests run two real
processes and check the whole-job throughput (sum of units over the slowest
rank's time), the max-over-ranks of elapsed times, the per-rank seeds, that
each rank's batch differs from the others, and that one call split over the
ranks (each running the oracle on its share) gathers back to the unsharded
oracle's result exactly.
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


def _oracle_call(x, gated):
    """The oracle on a call's arguments (torch tensors), as float64 arrays."""
    import numpy as np

    from oracle.gdr_oracle import recurrent_gated_delta_rule, recurrent_gated_delta_rule_gated

    def f(t):
        return t.to(torch.float64).numpy()

    asl = x["actual_seq_lengths"].numpy()
    idx = x["ssm_state_indices"].numpy()
    nat = x["num_accepted_tokens"].numpy()
    if gated:
        return recurrent_gated_delta_rule_gated(
            f(x["query"]), f(x["key"]), f(x["value"]), f(x["a"]), f(x["b"]), f(x["dt_bias"]),
            f(x["decay_scale"]), f(x["state_pool"]), asl, idx, f(x["gk"]), nat,
            x["scale_value"])
    return recurrent_gated_delta_rule(
        f(x["query"]), f(x["key"]), f(x["value"]), f(x["beta"]), f(x["state_pool"]), asl, idx,
        f(x["g"]), f(x["gk"]), nat, x["scale_value"])


def _sharded_call():
    """A ragged call: grouped heads, an empty item, a slot outside the pool,
    committed counts below the lengths."""
    from gated_delta_rule_recurrent_b200 import workloads

    w = workloads.WORKLOADS[0].replace(name="shard", B=7, H_qk=2, H_v=4, T=3, D_k=8, D_v=8,
                                       pool=10, lengths="uniform", indices="subset", seed=5)
    x = workloads.make_inputs(w)
    x["actual_seq_lengths"][2] = 0
    x["ssm_state_indices"][4] = 99
    x["num_accepted_tokens"] = (x["actual_seq_lengths"] - 1).clamp(min=0)
    return x


def _shard_worker(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    from datetime import timedelta

    from gated_delta_rule_recurrent_b200 import distributed as D

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        x = _sharded_call()
        results = {}
        for by in ("item", "head"):
            for gated in (False, True):
                xs, shard = D.shard_call(x, world, rank, by=by)
                out, pool = _oracle_call(xs, gated)
                parts = [None] * world
                dist.all_gather_object(parts, (torch.from_numpy(out), torch.from_numpy(pool),
                                               shard))
                o, p = D.gather_call([q[0] for q in parts], [q[1] for q in parts],
                                     [q[2] for q in parts],
                                     x["state_pool"].to(torch.float64))
                results[(by, gated)] = (o, p)
        torch.save(results, os.path.join(out_dir, f"shard{rank}.pt"))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(180)
def test_one_call_sharded_over_two_gloo_ranks(tmp_path):
    """Each rank runs the oracle on its share of one call (by item, by value
    head); the gathered out and pool equal the unsharded oracle bit for bit."""
    world = 2
    mp.start_processes(_shard_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    x = _sharded_call()
    for rank in range(world):
        res = torch.load(tmp_path / f"shard{rank}.pt")
        for (by, gated), (o, p) in res.items():
            ref_out, ref_pool = _oracle_call(x, gated)
            assert torch.equal(o, torch.from_numpy(ref_out)), (by, gated)
            assert torch.equal(p, torch.from_numpy(ref_pool)), (by, gated)


@pytest.mark.parametrize("world", [1, 2, 3, 4])
def test_shard_bounds_partition(world):
    from gated_delta_rule_recurrent_b200 import distributed as D

    for n in (0, 1, 5, 7, 64):
        bounds = [D.shard_bounds(n, world, r) for r in range(world)]
        assert bounds[0][0] == 0 and bounds[-1][1] == n
        assert all(bounds[r][1] == bounds[r + 1][0] for r in range(world - 1))
        sizes = [hi - lo for lo, hi in bounds]
        assert max(sizes) - min(sizes) <= 1


def test_head_shard_needs_divisible_heads():
    from gated_delta_rule_recurrent_b200 import distributed as D

    with pytest.raises(ValueError):
        D.shard_call(_sharded_call(), 3, 0, by="head")


def test_single_process_without_group():
    from gated_delta_rule_recurrent_b200 import distributed as D

    assert D.max_over_ranks(3.5) == 3.5
    assert D.sum_over_ranks(2.0) == 2.0
    assert D.throughput(10.0, 2.0) == (5.0, 2.0)
