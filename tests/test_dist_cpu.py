"""bench.py's multi-process plumbing on CPU with the gloo backend, 2 ranks.

The matmul path needs no collective (every rank runs an independent replica),
so what the N > 1 run relies on is the timing plumbing: the process group set
up from the torchrun environment, the barrier around the timed region, and the
max (time) and sum (bytes) over ranks.  These run here without a GPU.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port),
                       "WORLD_SIZE": str(world), "RANK": str(rank), "LOCAL_RANK": str(rank)})
    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist
    r, w, _ = bench.dist_setup(world)
    assert (r, w) == (rank, world)
    bench.barrier(w)
    mx = bench.allreduce_max(1.5 + rank, w)       # e.g. per-rank elapsed ms
    sm = bench.allreduce_sum(1000.0 * (rank + 1), w)  # e.g. per-rank bytes
    bench.barrier(w)
    with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
        json.dump({"max": mx, "sum": sm}, f)
    dist.destroy_process_group()


def test_allreduce_helpers_two_ranks(tmp_path):
    world = 2
    mp.spawn(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    for rank in range(world):
        got = json.load(open(tmp_path / f"rank{rank}.json"))
        assert got["max"] == 2.5                 # max over ranks, seen by every rank
        assert got["sum"] == 3000.0              # sum over ranks, seen by every rank


@pytest.mark.slow
def test_reference_arm_under_torchrun_two_ranks():
    """The launch the driver uses for N > 1, on CPU: rank 0 alone prints one
    JSON line (the oracle arm), rank 1 exits 0 without work."""
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py",
           "--impl", "reference", "--gpus", "2", "--steps", "3", "--warmup", "3",
           "--reference-seconds", "1"]
    p = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [l for l in p.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, p.stdout
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2
    assert line["value"] > 0 and line["cpu_baseline"]["kind"] == "oracle"


def test_reference_arm_json_line_single_process():
    """`bench.py --impl reference` at N = 1 (the oracle on the host cores):
    one JSON line with every key of the bench contract."""
    cmd = [sys.executable, "bench.py", "--impl", "reference", "--steps", "3", "--warmup", "3",
           "--reference-seconds", "1"]
    p = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [l for l in p.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, p.stdout
    line = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "impl", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["n_gpus"] == 1 and line["value"] > 0
    assert line["config"]["workload"] == "llama3_8b_decode_layer_m1"
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["unit"] == line["unit"]
