"""The multi-process plumbing of bench.py on CPU: two ranks over gloo.

bench.py runs one process per GPU under torchrun; on more than one rank it
joins a process group, brackets the timed region with barriers and takes the
maximum of the per-rank times (whole-job throughput is tokens of all ranks over
that time). These tests run the same helpers with two CPU ranks over gloo, and
check that the reference arm under torchrun prints exactly one line (rank 0)
while the other rank exits cleanly.
"""
import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _torchrun(args, timeout):
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes", "1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port())] + args
    env = dict(os.environ, OMP_NUM_THREADS="2")
    return subprocess.run(cmd, capture_output=True, text=True, timeout=timeout, cwd=ROOT, env=env)


def test_barrier_and_max_over_ranks_gloo(tmp_path):
    worker = tmp_path / "worker.py"
    worker.write_text(
        "import datetime, sys\n"
        f"sys.path.insert(0, {ROOT!r})\n"
        "import torch, torch.distributed as dist\n"
        "import bench\n"
        "world, rank, local = bench.dist_env()\n"
        "assert world == 2 and local == rank\n"
        "dist.init_process_group('gloo', timeout=datetime.timedelta(seconds=60))\n"
        "bench.barrier(world)\n"
        "v = bench.max_over_ranks(1.5 + 2.0 * rank, world, torch.device('cpu'))\n"
        "bench.barrier(world)\n"
        f"open({str(tmp_path)!r} + f'/rank{{rank}}.txt', 'w').write(repr(v))\n"
        "dist.destroy_process_group()\n")
    out = _torchrun([str(worker)], timeout=180)
    assert out.returncode == 0, out.stderr[-2000:]
    vals = [float((tmp_path / f"rank{r}.txt").read_text()) for r in range(2)]
    assert vals == [3.5, 3.5]   # both ranks see the slower rank's time


@pytest.mark.slow
def test_reference_arm_prints_once_under_torchrun():
    out = _torchrun([os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                     "--steps", "1", "--warmup", "3"], timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["value"] > 0
    assert rec["e2e"]["h2d_bytes_per_step"] == 0 and rec["cpu_baseline"]["kind"] == "oracle"
