"""Device-side failure detection without a GPU fault.

Every wait inside the single-pass kernel is bounded (about 2 s). The test build
of the library (libssd_testhooks.so; the shipped libssd.so has no such hook)
honours SSD_TEST_STALL_CHAIN=1, which makes each tile-to-tile hand-off wait for
a flag value nobody writes, so the kernel gives up, records the wait in its
status word and ends; the host reads that through ssd_fwd_check / ssd_fwd_host
as SSD_ERR_TIMEOUT, and the CUDA context stays usable for the next call. The
check runs in a child process that loads the test build.
"""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r"""
import os, time, torch
import oracle
from ssd_inputs import make_inputs
import structured_state_space_fwd_b200 as ssd
from structured_state_space_fwd_b200._lib import SSD_ERR_TIMEOUT, SSDError

assert ssd.lib_path.endswith("libssd_testhooks.so"), ssd.lib_path
# 160 chains (head pairs of one batch row), more than the GPU has SMs, so the
# two-tile sequence is split into two segments with one hand-off between them
inp = make_inputs(batch=1, seqlen=256, nheads=320, headdim=64, ngroups=1, dstate=128,
                  dtype="bf16", initial_states=True, seed=5)
d = {k: (v.cuda() if v is not None else None) for k, v in inp.items()}
shape = ssd.make_shape(d["x"], d["B"], 256)
assert ssd.ssd_fwd_plan(shape)[0] == "fused"
# the workspace holds a segment-state buffer only when a sequence has several segments
assert ssd.ssd_fwd_workspace_size(shape) >= 2 * 320 * 64 * 128 * 4
ws = torch.empty(ssd.ssd_fwd_workspace_size(shape), dtype=torch.uint8, device="cuda")

os.environ["SSD_TEST_STALL_CHAIN"] = "1"
t0 = time.perf_counter()
ssd.ssd_fwd(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], chunk_size=256,
            initial_states=d["initial_states"], return_final_states=True, workspace=ws)
try:
    ssd.ssd_fwd_check(shape, ws)
    raise SystemExit("no timeout reported")
except SSDError as e:
    assert e.status == SSD_ERR_TIMEOUT, e
    assert "chain" in str(e), e
elapsed = time.perf_counter() - t0
assert 1.0 < elapsed < 30.0, elapsed

# the host-buffer entry point reports the same status
try:
    ssd.ssd_fwd_host(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], inp["D"], chunk_size=256,
                     initial_states=inp["initial_states"],
                     final_states=torch.empty_like(inp["initial_states"]))
    raise SystemExit("host entry point: no timeout reported")
except SSDError as e:
    assert e.status == SSD_ERR_TIMEOUT, e

# and the no-alloc entry point, through its own status check
import ctypes
p = lambda t: ctypes.c_void_p(t.data_ptr()) if t is not None else None  # noqa: E731
yb = torch.empty_like(d["x"])
fb = torch.empty_like(d["initial_states"])
st = ssd.lib().ssd_fwd_no_alloc(ctypes.byref(shape), p(d["x"]), p(d["dt"]), p(d["A"]), p(d["B"]), p(d["C"]),
                                p(d["D"]), p(d["initial_states"]), p(yb), p(fb), None)
assert st == 0, st
st = ssd.lib().ssd_fwd_no_alloc_check(ctypes.byref(shape), None)
assert st == SSD_ERR_TIMEOUT, st

# the context is still usable: the next call is correct and reports OK
del os.environ["SSD_TEST_STALL_CHAIN"]
y, f = ssd.ssd_fwd(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], chunk_size=256,
                   initial_states=d["initial_states"], return_final_states=True, workspace=ws)
ssd.ssd_fwd_check(shape, ws)
st = ssd.lib().ssd_fwd_no_alloc(ctypes.byref(shape), p(d["x"]), p(d["dt"]), p(d["A"]), p(d["B"]), p(d["C"]),
                                p(d["D"]), p(d["initial_states"]), p(yb), p(fb), None)
assert st == 0 and ssd.lib().ssd_fwd_no_alloc_check(ctypes.byref(shape), None) == 0
torch.cuda.synchronize()
y_ref, f_ref, _ = oracle.recurrence(**inp)
assert oracle.rel_err(y.float().cpu(), y_ref) <= 5e-3
assert oracle.rel_err(f.cpu(), f_ref) <= 5e-3
print("CHILD_OK")
"""


def test_stalled_chain_reports_timeout_and_context_survives(cuda_device):
    from structured_state_space_fwd_b200 import build
    build.build()
    env = dict(os.environ, SSD_LIBRARY=build.TEST_LIB, PYTHONPATH=ROOT)
    env.pop("SSD_PATH", None)
    r = subprocess.run([sys.executable, "-c", CHILD], cwd=ROOT, env=env, capture_output=True,
                       text=True, timeout=300)
    assert r.returncode == 0 and "CHILD_OK" in r.stdout, r.stdout + r.stderr

