"""Multi-rank host logic of bench.py, run as world-size-2 gloo process groups on
the CPU.

With --gpus N > 1 each rank runs its own replica of the workload (the path has
no exchange step: every sequence is an independent recurrence), the timed
region is bracketed by barriers, the per-step time is the maximum over ranks
and the reported rate is N replicas' tokens divided by that time.  These tests
cover that logic without a GPU; the CUDA side of each rank is the single-GPU
path the gpu tests already cover.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, values, out_dir):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port),
                      RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    try:
        got_world, got_rank, got_local = bench._dist()
        res = {"dist": [got_world, got_rank, got_local]}
        bench._barrier(world)
        # two collectives in the same order on every rank, as in the bench
        res["max_ms"] = bench._max_over_ranks(values[rank], world)
        res["max_e2e"] = bench._max_over_ranks(10.0 * values[rank], world)
        res["rate"] = bench.weak_scaling_rate(8192, res["max_ms"], world)
        bench._barrier(world)
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump(res, f)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("values", [[0.41, 0.43], [0.52, 0.40]])
def test_max_over_ranks_and_weak_rate(tmp_path, values):
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), values, str(tmp_path)),
                       nprocs=world, join=True, start_method="spawn")
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    for r, x in enumerate(res):
        assert x["dist"] == [world, r, r]
        # every rank sees the slowest rank's time
        assert x["max_ms"] == max(values)
        assert x["max_e2e"] == 10.0 * max(values)
        # whole-job rate: both replicas' tokens over the slowest rank's step
        assert x["rate"] == pytest.approx(2 * 8192 / (max(values) * 1e-3), rel=1e-12)


def test_weak_rate_single_rank_is_plain_throughput():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.weak_scaling_rate(8192, 0.5, 1) == pytest.approx(8192 / 0.5e-3)
    assert bench._max_over_ranks(1.25, 1) == 1.25


def test_reference_arm_under_torchrun_prints_one_line(tmp_path):
    """`bench.py --impl reference` launched on two ranks: rank 0 alone times the
    oracle and prints one JSON line, the other rank exits 0 without work."""
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()),
           os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
           "--steps", "1", "--warmup", "3", "--cpu-seconds", "3"]
    env = dict(os.environ, OMP_NUM_THREADS="1")
    p = subprocess.run(cmd, cwd=str(tmp_path), env=env, capture_output=True, text=True,
                       timeout=600)
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [l for l in p.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, p.stdout
    line = json.loads(lines[0])
    assert line["impl"] == "reference"
    assert line["n_gpus"] == 2
    assert line["value"] > 0 and line["unit"] == "tokens/s/layer"
    assert line["e2e"]["h2d_bytes_per_step"] == 0
    assert line["cpu_baseline"]["kind"] == "oracle"
