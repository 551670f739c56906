"""Parity of ssd_fwd_varlen (packed variable-length documents, Knowl 8) with the
fp64 oracle's recurrence_varlen: every document is its own sequence, with its own
initial and final state. Same metric and bars as ssd_fwd (5e-3 bf16, 1e-5 fp32).

bf16 with head dim 64 runs on the single-pass kernel with one unit per (document,
head block); other shapes run document by document on the step path.
"""
import numpy as np
import pytest
import torch

import oracle
import ssd_inputs as W
from ssd_inputs import make_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ssd(cuda_device):
    from structured_state_space_fwd_b200 import build
    build.build()
    import structured_state_space_fwd_b200 as m
    return m


def varlen_case(ssd, cu, seed=0, with_init=True, dtype="bf16", H=8, P=64, G=2, N=128, tol=5e-3,
                final=True, device_cu=False):
    T = cu[-1]
    inp = make_inputs(1, T, H, P, G, N, dtype=dtype, seed=seed)
    inp.pop("initial_states")
    rng = np.random.Generator(np.random.PCG64(seed + 7))
    init = torch.from_numpy(rng.standard_normal((len(cu) - 1, H, P, N)) * 0.1).float() if with_init else None
    d = {k: (v.cuda() if v is not None else None) for k, v in inp.items()}
    cu_arg = torch.tensor(cu, dtype=torch.int32, device="cuda") if device_cu else cu
    out = ssd.ssd_fwd_varlen(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], cu_seqlens=cu_arg,
                             initial_states=init.cuda() if init is not None else None,
                             return_final_states=final)
    torch.cuda.synchronize()
    y, fin = out if final else (out, None)
    y_ref, f_ref = oracle.recurrence_varlen(**inp, cu_seqlens=cu, initial_states=init)
    yc = y.float().cpu()
    assert torch.isfinite(yc).all()
    ey = oracle.rel_err(yc, y_ref)
    assert ey <= tol, f"y rel err {ey:.3e}"
    if final:
        ef = oracle.rel_err(fin.cpu(), f_ref)
        assert ef <= tol, f"final rel err {ef:.3e}"
    return y, fin


@pytest.mark.parametrize("cu", [[0, 300, 301, 700, 1024], [0, 0, 256, 256, 900], [0, 1024],
                                [0, 1, 2, 3, 50], [0, 127, 255, 383, 1000]])
def test_varlen_single_pass(ssd, cu):
    varlen_case(ssd, cu, seed=len(cu) + cu[1])


@pytest.mark.parametrize("N,H,G", [(16, 4, 1), (64, 8, 2), (256, 4, 2), (176, 6, 3), (128, 5, 5)])
def test_varlen_state_sizes_and_head_blocks(ssd, N, H, G):
    # state 128 pairs heads per unit when H/G is even, state 256 runs one head per unit
    varlen_case(ssd, [0, 130, 130, 600, 1100], seed=N + H, H=H, G=G, N=N)


def test_varlen_many_documents_device_offsets(ssd):
    # 300 documents of 0..200 tokens, offsets given as a device tensor; every
    # (document, head pair) is one unit
    rng = np.random.Generator(np.random.PCG64(11))
    lens = rng.integers(0, 201, size=300)
    lens[::37] = 0
    cu = [0] + np.cumsum(lens).tolist()
    varlen_case(ssd, cu, seed=5, H=4, G=1, device_cu=True)


def test_varlen_without_states(ssd):
    varlen_case(ssd, [0, 200, 900, 1500], seed=9, with_init=False, final=False)


def test_varlen_packed_docs_full_size(ssd):
    # the 16-document pack at the 2.7B head shape, every element against the oracle
    w = W.PACKED_DOCS_27B
    cu = W.packed_cu_seqlens()
    inp = W.workload_inputs(w)
    d = {k: (v.cuda() if v is not None else None) for k, v in inp.items()}
    y, fin = ssd.ssd_fwd_varlen(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], cu_seqlens=cu,
                                return_final_states=True)
    torch.cuda.synchronize()
    inp.pop("initial_states")
    y_ref, f_ref = oracle.recurrence_varlen(**inp, cu_seqlens=cu)
    assert oracle.rel_err(y.float().cpu(), y_ref) <= 5e-3
    assert oracle.rel_err(fin.cpu(), f_ref) <= 5e-3
    # repeatable bit for bit, whatever CTA takes which unit
    y2, f2 = ssd.ssd_fwd_varlen(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], cu_seqlens=cu,
                                return_final_states=True)
    torch.cuda.synchronize()
    assert torch.equal(y, y2) and torch.equal(fin, f2)


def test_varlen_matches_batched_forward_on_equal_lengths(ssd):
    # documents of equal length are a batch: the packed call and ssd_fwd agree
    b, L = 3, 700
    inp = make_inputs(b, L, 8, 64, 2, 128, dtype="bf16", initial_states=True, seed=17)
    d = {k: v.cuda() for k, v in inp.items()}
    y_b, f_b = ssd.ssd_fwd(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"],
                           initial_states=d["initial_states"], return_final_states=True)
    pack = lambda t: t.reshape(1, b * L, *t.shape[2:]).contiguous()  # noqa: E731
    y_v, f_v = ssd.ssd_fwd_varlen(pack(d["x"]), pack(d["dt"]), d["A"], pack(d["B"]), pack(d["C"]), d["D"],
                                  cu_seqlens=[0, L, 2 * L, 3 * L], initial_states=d["initial_states"],
                                  return_final_states=True)
    torch.cuda.synchronize()
    assert oracle.rel_err(y_v.reshape(b, L, 8, 64).float().cpu(), y_b.float().cpu()) <= 1e-6
    assert oracle.rel_err(f_v.cpu(), f_b.cpu()) <= 1e-6


def test_varlen_malformed_device_offsets_reported(ssd):
    # a decreasing list on the device: the kernel clamps every document into the
    # pack (no access outside it) and the check reports the list
    T = 512
    inp = make_inputs(1, T, 4, 64, 1, 128, dtype="bf16", seed=3)
    d = {k: (v.cuda() if v is not None else None) for k, v in inp.items()}
    cu = torch.tensor([0, 300, 200, T], dtype=torch.int32, device="cuda")
    shp = ssd.make_shape(d["x"], d["B"], 256)
    ws = torch.empty(ssd.ssd_fwd_varlen_workspace_size(shp, 3), dtype=torch.uint8, device="cuda")
    ssd.ssd_fwd_varlen(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], cu_seqlens=cu, workspace=ws)
    with pytest.raises(ssd.SSDError) as e:
        ssd.ssd_fwd_varlen_check(shp, 3, ws)
    assert e.value.status == 1   # SSD_ERR_INVALID_ARG
    # a good list on the same workspace reports OK
    good = torch.tensor([0, 200, 300, T], dtype=torch.int32, device="cuda")
    ssd.ssd_fwd_varlen(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], cu_seqlens=good, workspace=ws)
    ssd.ssd_fwd_varlen_check(shp, 3, ws)


@pytest.mark.parametrize("cu", [[0, 7, 8, 20, 33], [0, 0, 10, 10, 33]])
def test_varlen_fp32_by_document(ssd, cu):
    varlen_case(ssd, cu, seed=4, dtype="f32", H=4, P=8, G=2, N=8, tol=1e-5)


def test_varlen_bf16_head_dim_32_by_document(ssd):
    varlen_case(ssd, [0, 100, 400, 401, 800], seed=6, H=4, P=32, G=1, N=64)
