"""ssd_fwd_no_alloc: the forward for callers that cannot allocate device memory.

Some callers cannot call cudaMalloc: a host application that owns every
device allocation and passes a library only its inputs and outputs, or a
latency-critical path where an allocation could synchronize the device. The
no-alloc entry point serves them from a static device scratch array. These
tests call it through the C ABI and compare it with the oracle's recurrence and
with ssd_fwd (which takes a caller-provided workspace), on two consecutive
calls with different inputs so that anything left over in the shared scratch
from the first call would show in the second. The file sorts last so a stop-at-first-failure run has already
run every other test.
"""
import ctypes

import pytest
import torch

import oracle
from ssd_inputs import make_inputs

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-5, "bf16": 5e-3}


@pytest.fixture(scope="module")
def ssd(cuda_device):
    from structured_state_space_fwd_b200 import build
    build.build()
    import structured_state_space_fwd_b200 as m
    return m


def no_alloc_call(ssd, d, Q, final=True):
    shp = ssd.make_shape(d["x"], d["B"], Q)
    y = torch.empty_like(d["x"])
    fin = (torch.empty((d["x"].shape[0], d["x"].shape[2], d["x"].shape[3], d["B"].shape[3]),
                       dtype=torch.float32, device=d["x"].device) if final else None)
    p = lambda t: ctypes.c_void_p(t.data_ptr()) if t is not None else None  # noqa: E731
    st = ssd.lib().ssd_fwd_no_alloc(ctypes.byref(shp), p(d["x"]), p(d["dt"]), p(d["A"]),
                                    p(d["B"]), p(d["C"]), p(d["D"]), p(d["initial_states"]),
                                    p(y), p(fin),
                                    ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return st, y, fin


@pytest.mark.parametrize("path", [None, "steps"])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_no_alloc_matches_oracle_and_workspace_entry_point_twice(ssd, monkeypatch, dtype, path):
    # default plan (single-pass kernel for bf16) and the four-kernel step path
    if path is None:
        monkeypatch.delenv("SSD_PATH", raising=False)
    else:
        monkeypatch.setenv("SSD_PATH", path)
    Q = 128
    for seed in (0, 1):   # two calls in a row on the shared scratch
        inp = make_inputs(batch=2, seqlen=700, nheads=4, headdim=64, ngroups=2, dstate=128,
                          dtype=dtype, initial_states=True, seed=seed)
        d = {k: (v.cuda() if v is not None else None) for k, v in inp.items()}
        st, y, fin = no_alloc_call(ssd, d, Q)
        assert st == 0, ssd.status_string(st)
        y_ws, f_ws = ssd.ssd_fwd(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], chunk_size=Q,
                                 initial_states=d["initial_states"], return_final_states=True)
        torch.cuda.synchronize()
        y_ref, f_ref, _ = oracle.recurrence(**inp)
        assert oracle.rel_err(y.float().cpu(), y_ref) <= TOL[dtype]
        assert oracle.rel_err(fin.cpu(), f_ref) <= TOL[dtype]
        # same plan, same workspace layout: the two entry points agree exactly
        assert torch.equal(y, y_ws) and torch.equal(fin, f_ws)


def test_no_alloc_without_final_states(ssd, monkeypatch):
    monkeypatch.delenv("SSD_PATH", raising=False)
    inp = make_inputs(batch=2, seqlen=1000, nheads=8, headdim=64, ngroups=1, dstate=128,
                      dtype="bf16", initial_states=True, seed=7)
    d = {k: (v.cuda() if v is not None else None) for k, v in inp.items()}
    st, y, fin = no_alloc_call(ssd, d, 256, final=False)
    assert st == 0 and fin is None, ssd.status_string(st)
    torch.cuda.synchronize()
    y_ref, _, _ = oracle.recurrence(**inp)
    assert oracle.rel_err(y.float().cpu(), y_ref) <= TOL["bf16"]


@pytest.mark.parametrize("dims", [
    # bf16, one chain (one batch row, one head pair) of 9.8M tokens: the sequence is
    # cut into 1200 segments of 64 tiles whose entering states take 1200*2*64*128*4
    # = 79 MB
    (1, 64 * 128 * 1200, 2, 64, 1, 128, 256, 1),
    # fp32, 64 batch rows of the 2.7B layer shape on the step path: the chunk
    # states alone take 64*8*80*64*128*4 = 671 MB
    (64, 2048, 80, 64, 1, 128, 256, 0),
])
def test_no_alloc_rejects_shape_beyond_scratch(ssd, monkeypatch, dims):
    # only sizes are computed: the pointers below are never dereferenced
    monkeypatch.delenv("SSD_PATH", raising=False)
    from structured_state_space_fwd_b200._lib import ShapeT
    shp = ShapeT(*dims, 0)
    assert ssd.ssd_fwd_workspace_size(shp) > (64 << 20)
    x = torch.empty(16, dtype=torch.uint8, device="cuda")
    p = ctypes.c_void_p(x.data_ptr())
    st = ssd.lib().ssd_fwd_no_alloc(ctypes.byref(shp), p, p, p, p, p, None, None, p, None, None)
    assert st == 2   # SSD_ERR_UNSUPPORTED, nothing enqueued
    assert b"static scratch" in ssd.lib().ssd_last_error_detail()
