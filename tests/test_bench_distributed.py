"""Multi-rank plumbing of bench.py on CPU: two gloo ranks (replicas only, no
data-path collective; the process group carries timing and byte totals)."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import torch.distributed as dist
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    times, nbytes = bench.combine_ranks(dist, [10.0 + rank, 5.0 * (rank + 1)], [100 * (rank + 1), 7], "cpu")
    dist.barrier()
    dist.destroy_process_group()
    out[rank] = (times, nbytes, bench.replica_seed(rank))


def test_two_gloo_ranks_combine_time_max_and_bytes_sum():
    world, port = 2, _free_port()
    manager = mp.Manager()
    out = manager.dict()
    mp.spawn(_rank_main, args=(world, port, out), nprocs=world, join=True)
    for r in range(world):
        times, nbytes, seed = out[r]
        assert times == [11.0, 10.0]          # max over ranks
        assert nbytes == [300.0, 14.0]        # sum over ranks
    assert out[0][2] != out[1][2]             # each replica draws its own workload


def _Args():
    import bench
    return bench.parse(["--impl", "reference", "--steps", "1", "--warmup", "0"])


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    import bench
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("RANK", "1")
    bench.run_reference(_Args())
    assert capsys.readouterr().out == ""


def test_reference_arm_prints_one_json_line(monkeypatch, capsys):
    import json
    import bench
    monkeypatch.setenv("WORLD_SIZE", "1")
    monkeypatch.setenv("RANK", "0")
    bench.run_reference(_Args())
    lines = [ln for ln in capsys.readouterr().out.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC and d["unit"] == "GB/s"
    assert d["value"] > 0 and d["cpu_baseline"]["kind"] == "oracle"
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]
    # the same config dict the GPU arm prints for the same command line
    from synthetic import workloads as wl
    r = wl.continuous_batch()
    assert d["config"] == bench.arm_config(_Args(), r["shape"], len(r["schedule"].initial), 1)
