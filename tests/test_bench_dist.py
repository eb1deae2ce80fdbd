"""bench.py's multi-rank aggregation (max of step time, sum of bytes) on two
gloo ranks on CPU: the replicas path needs no GPU to check."""

import os

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench

    mx = bench.max_over_ranks(1.0 + rank, "cpu")
    sm = bench.sum_over_ranks(10.0 * (rank + 1), "cpu")
    q.put((rank, mx, sm))
    dist.barrier()
    dist.destroy_process_group()


def test_two_rank_aggregation():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + os.getpid() % 1000
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert res == [(0, 2.0, 30.0), (1, 2.0, 30.0)]


def test_reference_arm_other_ranks_exit_without_work(monkeypatch, capsys):
    import bench

    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    assert bench.main(["--impl", "reference", "--steps", "1", "--warmup", "3"]) == 0
    assert capsys.readouterr().out == ""


def test_single_process_helpers_are_identity():
    import bench

    assert bench.max_over_ranks(3.5, "cpu") == 3.5
    assert bench.sum_over_ranks(2.0, "cpu") == 2.0



def test_recorded_traffic_follows_the_kernel_sources(tmp_path):
    """roofline.traffic is reported only while every source an entry lists
    hashes as it did when the counters were taken."""
    import json

    import bench

    rec = {"config2_fused": {"dram_bytes_per_launch": 123, "kernel_hash": bench.kernel_source_hash()},
           "config5_cascade": {"dram_bytes_per_launch": 456, "sources": ["pa_prefill.cu"],
                               "kernel_hash": "0" * 16}}
    path = tmp_path / "decode_traffic.json"
    path.write_text(json.dumps(rec))
    assert bench.recorded_traffic(2, "fused", str(path)) == 123
    assert bench.recorded_traffic(5, "cascade", str(path)) is None  # the listed source changed
    assert bench.recorded_traffic(3, "fused", str(path)) is None    # no capture
    assert bench.recorded_traffic(2, "fused", str(tmp_path / "missing.json")) is None
