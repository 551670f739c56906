"""Host side of ssd_fwd_varlen on the CPU: the per-document dispatch over ssd_fwd.

ssd_fwd_varlen runs every packed document (Knowl 8) as one ssd_fwd call on views
of the caller's buffers. Here ssd_fwd is replaced by an fp64 stand-in built on the
oracle's recurrence, so the test checks what the binding itself does: the slicing
by cu_seqlens, the per-document initial and final states, empty documents, and
that the results land in the caller's y and final_states. The device kernels
behind ssd_fwd are checked against the oracle on a GPU (test_gpu_varlen.py).
"""
import numpy as np
import pytest
import torch

import oracle
from ssd_inputs import make_inputs


def varlen_case(check_fn, m, cu, seed=0, with_init=True, dtype="f32", H=4, P=8, G=2, N=8,
                device="cpu", chunk_size=64, tol=1e-12):
    T = cu[-1]
    inp = make_inputs(1, T, H, P, G, N, dtype=dtype, seed=seed)
    inp.pop("initial_states")
    rng = np.random.Generator(np.random.PCG64(seed + 7))
    init = torch.from_numpy(rng.standard_normal((len(cu) - 1, H, P, N)) * 0.1).float() if with_init else None
    d = {k: (v.to(device) if v is not None else None) for k, v in inp.items()}
    y, fin = m.ssd_fwd_varlen(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], cu_seqlens=cu,
                              chunk_size=chunk_size,
                              initial_states=init.to(device) if init is not None else None,
                              return_final_states=True)
    check_fn()
    y_ref, f_ref = oracle.recurrence_varlen(**inp, cu_seqlens=cu, initial_states=init)
    ey = oracle.rel_err(y.float().cpu(), y_ref)
    ef = oracle.rel_err(fin.cpu(), f_ref)
    assert ey <= tol, f"y rel err {ey:.3e}"
    assert ef <= tol, f"final rel err {ef:.3e}"


@pytest.fixture
def fake_module(monkeypatch):
    import structured_state_space_fwd_b200 as m

    def fake_fwd(x, dt, A, B, C, D=None, chunk_size=256, initial_states=None,
                 return_final_states=False, y=None, final_states=None, workspace=None, stream=None):
        assert x.is_contiguous() and y.is_contiguous() and final_states.is_contiguous()
        yv, fv, _ = oracle.recurrence(x, dt, A, B, C, D, initial_states)
        y.copy_(torch.from_numpy(yv))
        final_states.copy_(torch.from_numpy(fv))
        return (y, final_states) if return_final_states else y
    monkeypatch.setattr(m, "ssd_fwd", fake_fwd)
    return m


@pytest.mark.parametrize("cu", [[0, 7, 8, 20, 33], [0, 33], [0, 0, 10, 10, 33], [0, 1, 2, 3, 33]])
@pytest.mark.parametrize("with_init", [False, True])
def test_varlen_dispatch(fake_module, cu, with_init):
    # fp64 stand-in results stored in fp32 buffers: fp32 rounding is the bar
    varlen_case(lambda: None, fake_module, cu, seed=len(cu), with_init=with_init, tol=1e-6)


def test_varlen_rejects_bad_cu_seqlens(fake_module):
    inp = make_inputs(1, 10, 2, 8, 1, 8, dtype="f32", seed=1)
    args = (inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], inp["D"])
    for cu in ([0, 5], [1, 10], [0, 6, 5, 10], [0]):
        with pytest.raises(ValueError):
            fake_module.ssd_fwd_varlen(*args, cu_seqlens=cu)
    with pytest.raises(ValueError):
        b2 = make_inputs(2, 10, 2, 8, 1, 8, dtype="f32", seed=1)
        fake_module.ssd_fwd_varlen(b2["x"], b2["dt"], b2["A"], b2["B"], b2["C"], b2["D"],
                                   cu_seqlens=[0, 10])
