"""Parity of ssd_gated_rmsnorm (gate and RMSNorm after the layer, Knowl 6) with
the fp64 oracle: max|out - ref| / max|ref| <= 5e-3 for bf16 storage, 1e-5 for
fp32, over all elements (small cases) or sampled tokens (full size)."""
import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu

TOL = {torch.float32: 1e-5, torch.bfloat16: 5e-3}


@pytest.fixture(scope="module")
def ssd(cuda_device):
    from structured_state_space_fwd_b200 import build
    build.build()
    import structured_state_space_fwd_b200 as m
    return m


def inputs(b, T, H, P, dtype, seed=0):
    g = torch.Generator().manual_seed(seed)
    y = torch.randn(b, T, H, P, generator=g).to(dtype)
    z = (torch.randn(b, T, H, P, generator=g) * 2.0).to(dtype)
    w = (torch.rand(H * P, generator=g) + 0.5).float()
    return y, z, w


def check(ssd, y, z, w, gs, eps, dtype):
    out = ssd.ssd_gated_rmsnorm(y.cuda(), z.cuda(), w.cuda(), group_size=gs, eps=eps)
    torch.cuda.synchronize()
    ref = oracle.gated_rmsnorm(y, z, w, gs, eps)
    e = oracle.rel_err(out.float().cpu(), ref)
    assert e <= TOL[dtype], f"rel err {e:.3e}"


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("b,T,H,P,gs", [
    (2, 37, 4, 64, 256),      # one group per token
    (2, 37, 4, 64, 64),       # a group per head
    (1, 5, 80, 64, 5120),     # the 2.7B layer's channels, one group
    (1, 2, 160, 256, 40960),  # a group larger than the threads' registers hold (second pass)
    (3, 7, 2, 3, 3),          # groups not a multiple of 16 bytes: scalar path
    (2, 4, 8, 64, 16),        # many small groups per CTA
])
def test_gated_rmsnorm_shapes(ssd, dtype, b, T, H, P, gs):
    y, z, w = inputs(b, T, H, P, dtype)
    check(ssd, y, z, w, gs, 1e-5, dtype)


def test_gated_rmsnorm_eps_zero_and_closed_gate(ssd):
    y, z, w = inputs(2, 9, 4, 64, torch.float32, seed=3)
    check(ssd, y, z, w, 256, 0.0, torch.float32)
    out = ssd.ssd_gated_rmsnorm(y.cuda(), torch.zeros_like(z).cuda(), w.cuda(), eps=1e-5)
    torch.cuda.synchronize()
    assert torch.count_nonzero(out) == 0


def test_gated_rmsnorm_empty(ssd):
    y, z, w = inputs(0, 4, 4, 64, torch.bfloat16)
    out = ssd.ssd_gated_rmsnorm(y.cuda(), z.cuda(), w.cuda())
    assert out.numel() == 0


def test_gated_rmsnorm_full_layer_shape(ssd):
    """The 2.7B layer shape (b8 T2048 H80 P64, one group of 5120 channels), checked
    on sampled tokens."""
    y, z, w = inputs(8, 2048, 80, 64, torch.bfloat16, seed=5)
    out = ssd.ssd_gated_rmsnorm(y.cuda(), z.cuda(), w.cuda(), group_size=5120)
    torch.cuda.synchronize()
    rows = [(0, 0), (7, 2047), (3, 1000), (5, 17)]
    got = np.stack([out[b, t].float().cpu().numpy() for b, t in rows])
    ref = np.stack([oracle.gated_rmsnorm(y[b, t][None], z[b, t][None], w, 5120, 1e-5)[0]
                    for b, t in rows])
    assert np.isfinite(out.float().cpu().numpy()).all()
    assert oracle.rel_err(got, ref) <= TOL[torch.bfloat16]
