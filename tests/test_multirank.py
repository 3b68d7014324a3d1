"""Multi-rank host logic of bench.py on CPU (gloo, world size 2).

The decode batch shards by sequence with no data-path collective: each rank
runs its own batch, and the only cross-rank operations are the barrier around
the timed region and the max over ranks of the elapsed time. These tests run
that logic in two gloo processes.
"""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    import datetime
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world,
                                         timeout=datetime.timedelta(seconds=60))
    import bench
    try:
        bench.barrier(world)
        t_max = bench.dist_max(1.0 + rank, world)         # rank r "took" 1 + r seconds
        value = bench.weak_scaling_value(262144, 10, world, t_max)
        out[rank] = (t_max, value)
        bench.barrier(world)
    finally:
        torch.distributed.destroy_process_group()


def test_two_ranks_time_is_max_and_value_counts_all_ranks():
    world = 2
    out = mp.Manager().dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    for r in range(world):
        t_max, value = out[r]
        assert t_max == 2.0
        assert value == pytest.approx(262144 * 10 * world / 2.0)


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.dist_max(3.5, 1) == 3.5
    bench.barrier(1)
    assert bench.weak_scaling_value(100, 4, 1, 2.0) == 200.0


def _stub_runner(args, world, rank, local):
    """One rank's work with the GPU part left out: the same timing reduction
    and output rule (rank 0 prints) as the benchmark, over gloo on CPU."""
    import json
    import bench
    assert torch.distributed.get_backend() == "gloo"
    assert torch.distributed.get_world_size() == args.gpus == world
    bench.barrier(world)
    t_max = bench.dist_max(1.0 + rank, world)
    value = bench.weak_scaling_value(262144, args.steps, world, t_max)
    bench.barrier(world)
    if rank == 0:
        with open(os.environ["MFA_TEST_OUT"], "w") as f:
            json.dump({"n_gpus": world, "t_max": t_max, "value": value, "rank": rank,
                       "local": local}, f)


def test_bench_launches_its_own_ranks(tmp_path, monkeypatch):
    """`bench.py --gpus 2` outside torchrun spawns two ranks itself; each joins
    the process group and rank 0 reports the job-wide figures."""
    import json
    import bench
    out = tmp_path / "line.json"
    monkeypatch.setenv("MFA_TEST_OUT", str(out))
    monkeypatch.delenv("WORLD_SIZE", raising=False)
    bench.main(["--gpus", "2", "--steps", "10"], runner=_stub_runner)
    line = json.loads(out.read_text())
    assert line["n_gpus"] == 2 and line["t_max"] == 2.0 and line["local"] == 0
    assert line["value"] == pytest.approx(262144 * 10 * 2 / 2.0)


def test_bench_single_gpu_runs_in_process(monkeypatch):
    import bench
    seen = {}

    def runner(args, world, rank, local):
        seen.update(world=world, rank=rank, local=local, gpus=args.gpus)

    monkeypatch.delenv("WORLD_SIZE", raising=False)
    bench.main(["--gpus", "1"], runner=runner)
    assert seen == {"world": 1, "rank": 0, "local": 0, "gpus": 1}
