"""Device-side failure detection without a GPU fault.

Every wait inside the fused kernel is bounded (about 2 s). The test hook
SSD_TEST_STALL_CHAIN=1 makes each tile-to-tile hand-off wait for a flag value
nobody writes, so the kernel gives up, records the wait in its status word and
ends; the host reads that through ssd_fwd_check / ssd_fwd_host as
SSD_ERR_TIMEOUT, and the CUDA context stays usable for the next call.
"""
import time

import pytest
import torch

import oracle
from ssd_inputs import make_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ssd(cuda_device):
    from structured_state_space_fwd_b200 import build
    build.build()
    import structured_state_space_fwd_b200 as m
    return m


def _inputs():
    # two 128-token tiles per sequence, so every sequence has one hand-off
    return make_inputs(batch=2, seqlen=256, nheads=8, headdim=64, ngroups=2, dstate=128,
                       dtype="bf16", initial_states=True, seed=5)


def test_stalled_chain_reports_timeout_and_context_survives(ssd, monkeypatch):
    from structured_state_space_fwd_b200._lib import SSD_ERR_TIMEOUT, SSDError
    inp = _inputs()
    d = {k: (v.cuda() if v is not None else None) for k, v in inp.items()}
    shape = ssd.make_shape(d["x"], d["B"], 256)
    assert ssd.ssd_fwd_plan(shape)[0] == "fused"
    ws = torch.empty(ssd.ssd_fwd_workspace_size(shape), dtype=torch.uint8, device="cuda")

    monkeypatch.setenv("SSD_TEST_STALL_CHAIN", "1")
    t0 = time.perf_counter()
    ssd.ssd_fwd(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], chunk_size=256,
                initial_states=d["initial_states"], return_final_states=True, workspace=ws)
    with pytest.raises(SSDError) as e:
        ssd.ssd_fwd_check(shape, ws)
    elapsed = time.perf_counter() - t0
    assert e.value.status == SSD_ERR_TIMEOUT
    assert "chain" in str(e.value)
    assert 1.0 < elapsed < 30.0

    # the host-buffer entry point reports the same status
    with pytest.raises(SSDError) as e2:
        ssd.ssd_fwd_host(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], inp["D"], chunk_size=256,
                         initial_states=inp["initial_states"],
                         final_states=torch.empty_like(inp["initial_states"]))
    assert e2.value.status == SSD_ERR_TIMEOUT

    # the context is still usable: the next call is correct and reports OK
    monkeypatch.delenv("SSD_TEST_STALL_CHAIN")
    y, f = ssd.ssd_fwd(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], chunk_size=256,
                       initial_states=d["initial_states"], return_final_states=True, workspace=ws)
    ssd.ssd_fwd_check(shape, ws)
    torch.cuda.synchronize()
    y_ref, f_ref, _ = oracle.recurrence(**inp)
    assert oracle.rel_err(y.float().cpu(), y_ref) <= 5e-3
    assert oracle.rel_err(f.cpu(), f_ref) <= 5e-3
