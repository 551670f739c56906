"""Parity of ssd_step (the recurrent form, decoding mode) with the fp64 oracle.

The oracle is the recurrence itself run from the same state over the same
tokens ("Transformers are SSMs", Knowl 1, linear form): ssd_step must return
its y and leave its final state in the state buffer. Same metric and bars as
the chunked forward: max|err| / max|ref| <= 5e-3 for bf16 storage, <= 1e-5
for fp32 (the state is fp32 in both, so it is held to 1e-5 throughout).
"""
import numpy as np
import pytest
import torch

import oracle
import ssd_inputs as W
from ssd_inputs import make_inputs

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-5, "bf16": 5e-3}
STATE_TOL = 1e-5


@pytest.fixture(scope="module")
def ssd(cuda_device):
    from structured_state_space_fwd_b200 import build
    build.build()
    import structured_state_space_fwd_b200 as m
    return m


def step_inputs(b, T, H, P, G, N, dtype, seed=0, with_D=True):
    inp = make_inputs(b, T, H, P, G, N, dtype=dtype, initial_states=True, with_D=with_D,
                      seed=seed)
    return inp


def run_step(ssd, inp):
    d = {k: (v.cuda() if v is not None else None) for k, v in inp.items()}
    state = d["initial_states"].clone()
    y = ssd.ssd_step(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], state)
    torch.cuda.synchronize()
    return y, state


def check(ssd, inp, dtype):
    y, state = run_step(ssd, inp)
    y_ref, s_ref, _ = oracle.recurrence(**inp)
    ey = oracle.rel_err(y.float().cpu(), y_ref)
    es = oracle.rel_err(state.cpu(), s_ref)
    assert ey <= TOL[dtype], f"y rel err {ey:.3e}"
    assert es <= STATE_TOL, f"state rel err {es:.3e}"
    return ey, es


@pytest.mark.parametrize("b,T,H,P,G,N,dtype", [
    (2, 1, 4, 64, 1, 128, "bf16"),      # one token, the Mamba-2 head shape
    (2, 1, 4, 64, 1, 128, "f32"),
    (3, 5, 6, 16, 3, 16, "f32"),        # several tokens, grouped heads, 4 lanes per row
    (3, 5, 6, 16, 3, 16, "bf16"),
    (1, 3, 2, 17, 1, 6, "f32"),         # N not a multiple of 4: scalar pieces; ragged rows
    (2, 2, 4, 256, 2, 256, "bf16"),     # largest head and state dims: 2 pieces per lane
    (1, 2, 2, 33, 2, 255, "f32"),       # 8 scalar pieces per lane
    (2, 1, 2, 1, 1, 1, "f32"),          # P = N = 1: a first-order IIR filter per head
    (1, 4, 8, 64, 8, 64, "bf16"),       # one group per head
])
def test_step_shapes(ssd, b, T, H, P, G, N, dtype):
    check(ssd, step_inputs(b, T, H, P, G, N, dtype), dtype)


def test_step_without_D(ssd):
    check(ssd, step_inputs(2, 2, 4, 32, 2, 64, "f32", with_D=False), "f32")


def test_step_zero_tokens_leaves_state(ssd):
    inp = step_inputs(2, 0, 4, 64, 1, 128, "bf16")
    y, state = run_step(ssd, inp)
    assert y.numel() == 0
    assert torch.equal(state.cpu(), inp["initial_states"])


def test_step_empty_batch(ssd):
    inp = step_inputs(0, 1, 4, 64, 1, 128, "bf16")
    y, state = run_step(ssd, inp)
    assert y.numel() == 0 and state.numel() == 0


def test_step_one_token_form(ssd):
    """[b,H,P] inputs (one token) give the same numbers as [b,1,H,P]."""
    inp = step_inputs(2, 1, 4, 64, 1, 128, "bf16", seed=3)
    d = {k: (v.cuda() if v is not None else None) for k, v in inp.items()}
    s1 = d["initial_states"].clone()
    s2 = d["initial_states"].clone()
    y1 = ssd.ssd_step(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], s1)
    y2 = ssd.ssd_step(d["x"][:, 0], d["dt"][:, 0], d["A"], d["B"][:, 0], d["C"][:, 0], d["D"], s2)
    torch.cuda.synchronize()
    assert torch.equal(y1[:, 0], y2) and torch.equal(s1, s2)


def test_prefill_then_decode(ssd):
    """ssd_fwd over a prompt (final states), then ssd_step token by token, equals the
    recurrence over the whole sequence (Knowl 1: both forms compute the same map)."""
    T0, T1 = 300, 4
    inp = make_inputs(2, T0 + T1, 8, 64, 1, 128, dtype="bf16", initial_states=True, seed=5)
    d = {k: (v.cuda() if v is not None else None) for k, v in inp.items()}
    y0, state = ssd.ssd_fwd(d["x"][:, :T0].contiguous(), d["dt"][:, :T0].contiguous(), d["A"],
                            d["B"][:, :T0].contiguous(), d["C"][:, :T0].contiguous(), d["D"],
                            chunk_size=256, initial_states=d["initial_states"],
                            return_final_states=True)
    ys = [y0]
    for t in range(T0, T0 + T1):
        ys.append(ssd.ssd_step(d["x"][:, t].contiguous(), d["dt"][:, t].contiguous(), d["A"],
                               d["B"][:, t].contiguous(), d["C"][:, t].contiguous(), d["D"],
                               state).unsqueeze(1))
    torch.cuda.synchronize()
    y = torch.cat(ys, dim=1)
    y_ref, s_ref, _ = oracle.recurrence(**inp)
    assert oracle.rel_err(y.float().cpu(), y_ref) <= TOL["bf16"]
    # the prompt's state comes from ssd_fwd, held to the bf16 bar like its final_states
    assert oracle.rel_err(state.cpu(), s_ref) <= TOL["bf16"]


def test_step_deterministic(ssd):
    inp = step_inputs(3, 2, 4, 64, 1, 128, "bf16", seed=7)
    ya, sa = run_step(ssd, inp)
    yb, sb = run_step(ssd, inp)
    assert torch.equal(ya, yb) and torch.equal(sa, sb)


def test_full_decode_step(ssd):
    """The benchmarked decoding workload at full size, checked on sampled sequences."""
    w = W.DECODE_STEP_27B
    inp = W.workload_inputs(w)
    y, state = run_step(ssd, inp)
    pairs = [(0, 0), (w.batch - 1, w.nheads - 1), (w.batch // 2, w.nheads // 2), (17, 63)]
    y_ref, s_ref, _ = oracle.recurrence(**inp, bh_list=pairs)
    yc, sc = y.float().cpu().numpy(), state.cpu().numpy()
    assert np.isfinite(yc).all() and np.isfinite(sc).all()
    ey = oracle.rel_err(np.stack([yc[b, :, h] for b, h in pairs]),
                        np.stack([y_ref[b, :, h] for b, h in pairs]))
    es = oracle.rel_err(np.stack([sc[b, h] for b, h in pairs]),
                        np.stack([s_ref[b, h] for b, h in pairs]))
    assert ey <= TOL["bf16"], f"y rel err {ey:.3e}"
    assert es <= STATE_TOL, f"state rel err {es:.3e}"
