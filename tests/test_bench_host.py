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


def test_spawned_dry_run_over_two_ranks():
    """`bench.py --gpus 2` started without a launcher spawns two ranks (one
    process per GPU on a GPU machine); --dry-run takes the same rank path on the
    CPU over gloo and rank 0 prints one line with n_gpus = 2."""
    import subprocess
    import sys

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    res = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--gpus", "2",
                          "--dry-run", "--steps", "5", "--warmup", "3"],
                         capture_output=True, text=True, timeout=240, cwd=root)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [ln for ln in res.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, res.stdout
    d = json.loads(lines[0])
    assert d["n_gpus"] == 2 and d["dry_run"] is True and d["steps"] == 5


def test_roofline_takes_the_larger_bound():
    ops, nbytes = bench.workload_units("3")
    r = bench.roofline(ops, nbytes, 350e-6, 6533.5, 1673.6, "measured")
    assert r["bound"] == "hbm" and r["unit"] == "GB/s"
    assert r["frac"] == pytest.approx(nbytes / 350e-6 / 1e9 / 6533.5)
    assert r["int8_tensor"]["peak_tops"] == pytest.approx(2 * 1673.6)
    assert r["roofline_time_us"] == pytest.approx(nbytes / 6533.5e9 * 1e6)
    # the block's 3x3 stage: 1151 ops per byte, above the ridge -> tensor-bound
    conv2 = bench.synth.CONFIGS["5"].stages()[1]
    r2 = bench.roofline(conv2.ops(), conv2.bytes_moved(), 125e-6, 6533.5, 1673.6, "measured")
    assert r2["bound"] == "tensor" and r2["unit"] == "TOPS"
    assert r2["frac"] == pytest.approx(conv2.ops() / 125e-6 / 1e12 / (2 * 1673.6))


def test_rotation_and_metric_per_config():
    assert bench.rotation_sets(2 * 10 ** 9) == 1
    n1 = bench.rotation_sets(bench.workload_units("1")[1])
    assert n1 * bench.workload_units("1")[1] >= 3 * bench.L2_BYTES
    assert bench.metric_for("3") == bench.METRIC
    assert "B=2048" not in bench.metric_for("1") and "B=1" in bench.metric_for("1")


def test_clock_verdict():
    assert not bench.clocks_verdict({"sm_mhz": 1800, "sm_max_mhz": 1965, "reasons": ["sw_power_cap"]})
    assert bench.clocks_verdict({"sm_mhz": 1800, "sm_max_mhz": 1965, "reasons": ["hw_slowdown"]})
    assert bench.clocks_verdict({"sm_mhz": 900, "sm_max_mhz": 1965, "reasons": []})
