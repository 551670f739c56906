"""Sequence (context) parallelism on one GPU: R ranks emulated one after another.

Each "rank" runs ssd_cp_begin on its slice of the sequence; the records are
concatenated in rank order (what the all-gather delivers); each rank then runs
ssd_cp_end. The slices' y, put back together, and the state after each slice
must match the fp64 oracle's recurrence over the whole sequence ("Transformers
are SSMs", Knowl 8: only the boundary state passes between workers; Knowl 1 for
the result). No kernel waits on another, so running the ranks in turn on one
device exercises every kernel of the multi-rank path.
"""
import datetime
import socket

import numpy as np
import pytest
import torch

import oracle
import ssd_inputs as W
from ssd_inputs import make_inputs

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-5, "bf16": 5e-3}


@pytest.fixture(scope="module")
def ssd(cuda_device):
    from structured_state_space_fwd_b200 import build
    build.build()
    import structured_state_space_fwd_b200 as m
    return m


def emulate(ssd, inp, cuts, Q):
    d = {k: (v.cuda() if v is not None else None) for k, v in inp.items()}
    R = len(cuts) - 1
    recs, wss, parts = [], [], []
    for r in range(R):
        sl = slice(cuts[r], cuts[r + 1])
        p = {k: d[k][:, sl].contiguous() for k in ("x", "dt", "B", "C")}
        init = d["initial_states"] if r == 0 else None
        rec, ws = ssd.ssd_cp_begin(p["x"], p["dt"], d["A"], p["B"], Q, initial_states=init)
        recs.append(rec)
        wss.append(ws)
        parts.append(p)
    records = torch.cat(recs)
    ys, fins = [], []
    for r in range(R):
        p = parts[r]
        init = d["initial_states"] if r == 0 else None
        y, fin = ssd.ssd_cp_end(p["x"], p["dt"], p["B"], p["C"], d["D"], records, R, r, wss[r], Q,
                                initial_states=init)
        ys.append(y)
        fins.append(fin)
    torch.cuda.synchronize()
    return torch.cat(ys, dim=1), fins


def check(ssd, inp, cuts, Q, dtype):
    y, fins = emulate(ssd, inp, cuts, Q)
    y_ref, _, _ = oracle.recurrence(**inp)
    ey = oracle.rel_err(y.float().cpu(), y_ref)
    assert ey <= TOL[dtype], f"y rel err {ey:.3e}"
    for r in range(len(cuts) - 1):
        pre = {k: (v[:, :cuts[r + 1]] if k in ("x", "dt", "B", "C") else v) for k, v in inp.items()}
        _, s_ref, _ = oracle.recurrence(**pre)
        es = oracle.rel_err(fins[r].cpu(), s_ref)
        assert es <= TOL[dtype], f"state after slice {r}: rel err {es:.3e}"


@pytest.mark.parametrize("cuts,Q", [
    ([0, 300, 300, 555, 700], 256),    # an empty slice, slices off chunk boundaries
    ([0, 256, 512, 700], 256),         # chunk-aligned slices
    ([0, 130, 700], 128),
    ([0, 700], 256),                   # one rank: ssd_fwd
])
def test_cp_tensor_core_steps(ssd, cuts, Q):
    inp = make_inputs(2, 700, 8, 64, 2, 128, dtype="bf16", initial_states=True, seed=21)
    check(ssd, inp, cuts, Q, "bf16")


@pytest.mark.parametrize("cuts", [[0, 64, 130, 200], [0, 1, 2, 200], [0, 199, 200]])
def test_cp_fp32(ssd, cuts):
    inp = make_inputs(1, 200, 2, 16, 1, 16, dtype="f32", dt_dist="softplus", initial_states=True,
                      seed=22)
    check(ssd, inp, cuts, 64, "f32")


def test_cp_no_init_no_D(ssd):
    inp = make_inputs(2, 333, 4, 32, 2, 64, dtype="f32", with_D=False, seed=23)
    check(ssd, inp, [0, 100, 200, 333], 32, "f32")


def test_cp_long_context_eight_ranks(ssd):
    """The long-context workload (65536 tokens, 32 heads, 8 groups, state carried
    in) split over 8 ranks of 8192 tokens, checked on sampled heads."""
    w = W.LONG_CONTEXT
    inp = W.workload_inputs(w)
    cuts = [i * (w.seqlen // 8) for i in range(9)]
    y, fins = emulate(ssd, inp, cuts, w.chunk_size)
    pairs = [(0, 0), (0, 13), (0, 31)]
    y_ref, f_ref, _ = oracle.recurrence(**inp, bh_list=pairs)
    yc, fc = y.float().cpu().numpy(), fins[-1].cpu().numpy()
    assert np.isfinite(yc).all() and np.isfinite(fc).all()
    ey = oracle.rel_err(np.stack([yc[b, :, h] for b, h in pairs]),
                        np.stack([y_ref[b, :, h] for b, h in pairs]))
    ef = oracle.rel_err(np.stack([fc[b, h] for b, h in pairs]),
                        np.stack([f_ref[b, h] for b, h in pairs]))
    assert ey <= TOL["bf16"], f"y rel err {ey:.3e}"
    assert ef <= TOL["bf16"], f"final rel err {ef:.3e}"


def test_cp_single_rank_nccl_group(ssd):
    """ssd_fwd_cp through a one-rank NCCL process group (the real all-gather)."""
    import torch.distributed as dist
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device("cuda", 0))
    try:
        inp = make_inputs(2, 500, 8, 64, 1, 128, dtype="bf16", initial_states=True, seed=24)
        d = {k: (v.cuda() if v is not None else None) for k, v in inp.items()}
        y, fin = ssd.ssd_fwd_cp(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], chunk_size=256,
                                initial_states=d["initial_states"], return_final_states=True)
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    y_ref, f_ref, _ = oracle.recurrence(**inp)
    assert oracle.rel_err(y.float().cpu(), y_ref) <= TOL["bf16"]
    assert oracle.rel_err(fin.cpu(), f_ref) <= TOL["bf16"]
