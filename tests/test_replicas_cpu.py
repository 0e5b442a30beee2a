"""The multi-GPU path on CPU: replicas with no data-path collective.

The denoise loop does not shard (each GPU runs an independent replica), so the only
collectives are the timing ones: a barrier around the timed region and the maximum of each
rank's time.  Checked here with two `gloo` ranks, and the launch of the reference arm under
torch.distributed.run with two ranks (rank 0 alone prints; the other exits without work).
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


def _rank_main(rank, world, port, out_dir):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        dist.barrier()
        got = bench.reduce_max([1.0 + rank, 10.0 - rank, -3.0 * rank], "cpu")
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump(got, f)
    finally:
        dist.destroy_process_group()


def test_timing_is_the_maximum_over_two_gloo_ranks(tmp_path):
    port = _free_port()
    mp.start_processes(_rank_main, args=(2, port, str(tmp_path)), nprocs=2, join=True, start_method="spawn")
    for rank in range(2):
        got = json.load(open(tmp_path / f"rank{rank}.json"))
        assert got == [2.0, 10.0, 0.0], (rank, got)


def test_reduce_max_without_a_group_returns_the_values():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.reduce_max([1.5, -2.0], "cpu") == [1.5, -2.0]


@pytest.mark.timeout(600)
def test_reference_arm_under_torchrun_prints_once_from_rank_0():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr=127.0.0.1", f"--master-port={port}", os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--workload", "1-view", "--steps", "1", "--warmup", "0", "--gpus", "2"]
    env = dict(os.environ, OMP_NUM_THREADS="4")
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600, env=env)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [json.loads(l) for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout
    line = lines[0]
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["unit"] == "ms"
    assert line["cpu_baseline"]["kind"] == "oracle" and line["value"] > 0
