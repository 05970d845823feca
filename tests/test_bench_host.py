"""Host-side logic of bench.py on the CPU: the max-over-ranks reduction and
the whole-job aggregation, run as two gloo ranks (the same code path that
bench.py takes over NCCL with one process per GPU)."""
import datetime
import json
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp

import bench


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, outdir):
    import torch.distributed as dist

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    my_ms = 1.0 + rank * 0.5  # rank 1 is the slowest
    ms = bench.max_over_ranks(my_ms, dist, "cpu")
    seed = bench.shard_seed(1003, rank)
    seeds = [None] * world
    dist.all_gather_object(seeds, seed)
    ops = 210_453_397_504
    value, t = bench.aggregate([ms] * world, ops)
    json.dump({"ms": ms, "value": value, "seeds": seeds},
              open(os.path.join(outdir, f"r{rank}.json"), "w"))
    dist.destroy_process_group()


def test_two_rank_max_and_aggregate(tmp_path):
    world = 2
    mp.spawn(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    res = [json.load(open(tmp_path / f"r{r}.json")) for r in range(world)]
    for r in res:
        assert r["ms"] == 1.5  # every rank sees the slowest rank's time
        assert r["value"] == pytest.approx(2 * 210_453_397_504 / 1.5e-3)
        assert len(set(r["seeds"])) == world  # independent batches per rank


def test_aggregate_single():
    v, t = bench.aggregate([2.0], 1000)
    assert t == 2.0 and v == pytest.approx(1000 / 2e-3)


def test_peaks_and_traffic_parsing(tmp_path, monkeypatch):
    hbm, bf16, kind = bench.peaks()
    assert hbm > 1000 and bf16 > 100 and kind in ("measured", "fallback")
    sha = bench.kernel_source_sha()
    assert len(sha) == 12
    assert bench.read_traffic("does_not_exist.md", sha) is None


def test_workload_numbers_match_the_plan():
    ops, nbytes = bench.workload_units("3")
    assert ops == 2 * 2048 * 784 * 512 * 128  # 210.45 G int-ops
    assert abs(nbytes / 1e9 - 1.8497) < 0.001  # x + r + out + weights (+ bias, m)
