"""Parity of ssd_fwd_varlen (packed variable-length documents, Knowl 8) with the
fp64 oracle's recurrence_varlen: every document is its own sequence, with its own
initial and final state. Same metric and bars as ssd_fwd (5e-3 bf16, 1e-5 fp32)."""
import pytest
import torch

from test_varlen_host import varlen_case

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ssd(cuda_device):
    from structured_state_space_fwd_b200 import build
    build.build()
    import structured_state_space_fwd_b200 as m
    return m


@pytest.mark.parametrize("cu", [[0, 300, 301, 700, 1024], [0, 0, 256, 256, 900], [0, 1024]])
def test_varlen_tensor_core_shapes(ssd, cu):
    # bf16, head dim 64, state 128: the fused / step tensor-core paths per document
    varlen_case(torch.cuda.synchronize, ssd, cu, seed=3, dtype="bf16", H=8, P=64, G=2, N=128,
                device="cuda", chunk_size=256, tol=5e-3)


@pytest.mark.parametrize("cu", [[0, 7, 8, 20, 33], [0, 0, 10, 10, 33]])
def test_varlen_fp32(ssd, cu):
    varlen_case(torch.cuda.synchronize, ssd, cu, seed=4, dtype="f32", H=4, P=8, G=2, N=8,
                device="cuda", chunk_size=16, tol=1e-5)
