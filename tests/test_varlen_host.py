"""Host side of ssd_fwd_varlen (packed variable-length documents, Knowl 8) on the CPU.

The packed forward runs in the library's kernels on the device (test_gpu_varlen.py
checks it against the oracle's recurrence_varlen). What runs without a GPU is the
C entry point's shape checking and workspace query, and the binding's checks of a
host-side cu_seqlens list before it is copied to the device.
"""
import ctypes

import pytest
import torch

from ssd_inputs import make_inputs


@pytest.fixture(scope="module")
def ssd():
    from structured_state_space_fwd_b200 import build
    build.build()
    import structured_state_space_fwd_b200 as m
    return m


def test_varlen_workspace_grows_with_documents(ssd):
    # bf16, head dim 64: the single-pass kernel's layout (status words + document order)
    shp = ssd.ShapeT(1, 16384, 80, 64, 1, 128, 256, ssd.SSD_BF16, 0)
    sizes = [ssd.ssd_fwd_varlen_workspace_size(shp, n) for n in (1, 16, 64, 1000)]
    assert sizes[0] > 0 and sizes == sorted(sizes) and sizes[-1] >= 1000 * 4
    # no documents only with no tokens
    assert ssd.ssd_fwd_varlen_workspace_size(ssd.ShapeT(1, 0, 80, 64, 1, 128, 256, ssd.SSD_BF16, 0), 0) == 0
    with pytest.raises(ssd.SSDError):
        ssd.ssd_fwd_varlen_workspace_size(shp, 0)


def test_varlen_workspace_other_shapes_bounds_every_document(ssd):
    # fp32 runs document by document on the step path: the pack's own ssd_fwd
    # workspace bounds that of any document in it
    shp = ssd.ShapeT(1, 1000, 4, 8, 2, 8, 64, ssd.SSD_F32, 0)
    n = ssd.ssd_fwd_varlen_workspace_size(shp, 5)
    assert n >= ssd.ssd_fwd_workspace_size(shp)
    for T in (1, 64, 999):
        assert n >= ssd.ssd_fwd_workspace_size(ssd.ShapeT(1, T, 4, 8, 2, 8, 64, ssd.SSD_F32, 0))


def test_varlen_rejects_batch_other_than_one(ssd):
    shp = ssd.ShapeT(2, 100, 4, 8, 2, 8, 64, ssd.SSD_F32, 0)
    n = ctypes.c_size_t(0)
    st = ssd.lib().ssd_fwd_varlen_workspace_size(ctypes.byref(shp), ctypes.c_int64(3), ctypes.byref(n))
    assert st == 1   # SSD_ERR_INVALID_ARG
    st = ssd.lib().ssd_fwd_varlen(ctypes.byref(shp), *([None] * 7), ctypes.c_int64(3), *([None] * 4),
                                  ctypes.c_size_t(0), None)
    assert st == 1


def test_varlen_binding_checks_host_offsets(ssd):
    inp = make_inputs(1, 10, 2, 8, 1, 8, dtype="f32", seed=1)
    args = (inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], inp["D"])
    # the binding refuses tensors that are not on the device before anything else
    with pytest.raises(ValueError):
        ssd.ssd_fwd_varlen(*args, cu_seqlens=[0, 10])
    b2 = make_inputs(2, 10, 2, 8, 1, 8, dtype="f32", seed=1)
    with pytest.raises(ValueError):
        ssd.ssd_fwd_varlen(b2["x"], b2["dt"], b2["A"], b2["B"], b2["C"], b2["D"], cu_seqlens=[0, 10])
    for cu in ([0, 5], [1, 10], [0, 6, 5, 10], []):
        with pytest.raises(ValueError):
            ssd.check_cu_seqlens(cu, 10)
    assert ssd.check_cu_seqlens(torch.tensor([0, 0, 4, 10]), 10) == [0, 0, 4, 10]
