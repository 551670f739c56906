"""The multi-rank plumbing of ssd_fwd_cp on CPU: three ranks over gloo.

ssd_fwd_cp runs ssd_cp_begin on each rank's slice, all-gathers the per-rank
records in rank order and runs ssd_cp_end. Here the two device calls are
replaced by fp64 stand-ins built on the oracle (the record layout is the C
ABI's: state [b,H,P,N], then alpha = prod a_t [b,H], padded to 4 floats), so
the test checks what runs on the host: slicing by rank, the collective, the
rank order of the records, the initial state entering on rank 0 only, and the
fold of earlier ranks into each rank's entering state (Knowl 8: only the
boundary state passes between workers). The device kernels behind the two
calls are checked against the oracle on a GPU (test_gpu_cp.py).
"""
import os
import socket
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

WORKER = r'''
import datetime, sys
sys.path.insert(0, ROOT)
import numpy as np, torch, torch.distributed as dist
import oracle
import structured_state_space_fwd_b200 as m
from ssd_inputs import make_inputs

dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
rank, world = dist.get_rank(), dist.get_world_size()
inp = make_inputs(2, 70, 4, 8, 2, 6, dtype="f32", initial_states=True, seed=11)
cuts = [0, 25, 25, 70]
sl = slice(cuts[rank], cuts[rank + 1])
part = {k: inp[k][:, sl].contiguous() for k in ("x", "dt", "B", "C")}


def fake_begin(x, dt, A, B, chunk_size=256, initial_states=None, record=None, workspace=None,
               stream=None):
    _, s, _ = oracle.recurrence(x, dt, A, B, torch.zeros_like(B), None, initial_states)
    alpha = np.exp(A.double().numpy()[None, :] * dt.double().numpy().sum(axis=1))
    rec = np.concatenate([s.ravel(), alpha.ravel()])
    rec = np.concatenate([rec, np.zeros((-rec.size) % 4)])
    return torch.from_numpy(rec), {"A": A}


def fake_end(x, dt, B, C, D, records, nranks, rank, workspace, chunk_size=256,
             initial_states=None, y=None, final_states=None, stream=None):
    b, H, P, N = x.shape[0], x.shape[2], x.shape[3], B.shape[3]
    nst = b * H * P * N
    R = records.numpy().reshape(nranks, -1)
    if rank == 0:
        h = initial_states.double().numpy() if initial_states is not None else np.zeros((b, H, P, N))
    else:
        h = np.zeros((b, H, P, N))
        for k in range(rank):
            h = R[k, nst:nst + b * H].reshape(b, H, 1, 1) * h + R[k, :nst].reshape(b, H, P, N)
    yv, fin, _ = oracle.recurrence(x, dt, workspace["A"], B, C, D, h)
    return torch.from_numpy(yv), torch.from_numpy(fin)


m.ssd_cp_begin = fake_begin
m.ssd_cp_end = fake_end
y, fin = m.ssd_fwd_cp(part["x"], part["dt"], inp["A"], part["B"], part["C"], inp["D"],
                      chunk_size=64, initial_states=inp["initial_states"],
                      return_final_states=True)
pre = {k: (v[:, :cuts[rank + 1]] if k in ("x", "dt", "B", "C") else v) for k, v in inp.items()}
y_ref, s_ref, _ = oracle.recurrence(**pre)
ey = oracle.rel_err(y, y_ref[:, sl]) if y.shape[1] else 0.0
es = oracle.rel_err(fin, s_ref)
open(OUT + f"/rank{rank}.txt", "w").write(f"{ey!r} {es!r} {tuple(y.shape)!r}")
dist.destroy_process_group()
'''


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_context_parallel_exchange_gloo(tmp_path):
    worker = tmp_path / "cp_worker.py"
    worker.write_text(f"ROOT = {ROOT!r}\nOUT = {str(tmp_path)!r}\n" + WORKER)
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes", "1", "--nproc-per-node", "3",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()), str(worker)]
    env = dict(os.environ, OMP_NUM_THREADS="2")
    out = subprocess.run(cmd, capture_output=True, text=True, timeout=300, cwd=ROOT, env=env)
    assert out.returncode == 0, out.stderr[-3000:]
    shapes = []
    for r in range(3):
        ey, es, shp = (tmp_path / f"rank{r}.txt").read_text().split(" ", 2)
        assert float(ey) <= 1e-12, (r, ey)
        assert float(es) <= 1e-12, (r, es)
        shapes.append(shp)
    assert shapes == ["(2, 25, 4, 8)", "(2, 0, 4, 8)", "(2, 45, 4, 8)"]
