"""Pins for the fp64 oracle, checked against what the pages and the mathematics fix.

Every test here runs on the CPU (no GPU). Each one ties the oracle to something
other than itself: a hand-worked example, a closed form, a library routine
(scipy's IIR filter, numpy's convolution), a brute-force dense matrix, or an
identity the pages state ("Transformers are SSMs", Knowls 1, 2, 3 and 8;
"Mamba-2 and State Space Duality (SSD)", dual form).
"""
import json
import math
import os

import numpy as np
import pytest
import scipy.signal

import oracle
from ssd_inputs import make_inputs

HERE = os.path.dirname(os.path.abspath(__file__))


def rnd(b=2, T=40, H=4, P=3, G=2, N=5, seed=0, init=False, dt_dist="loguniform"):
    return make_inputs(batch=b, seqlen=T, nheads=H, headdim=P, ngroups=G, dstate=N,
                       dtype="f32", dt_dist=dt_dist, initial_states=init, seed=seed)


def f64(t):
    return None if t is None else t.double().numpy()


def test_hand_worked_example():
    # One head, N = P = 1, a_t = exp(dt*A) = exp(1 * -ln 2) = 1/2, B = 2, C = 3, D = 1/2,
    # x = (1, 2, -1), h_{-1} = 0 (Knowl 1, linear form, with dt and D):
    #   h0 = 2*1 = 2          y0 = 3*2 + 0.5*1  = 6.5
    #   h1 = 1 + 2*2 = 5      y1 = 15 + 0.5*2   = 16
    #   h2 = 2.5 + 2*-1 = 0.5 y2 = 1.5 - 0.5    = 1
    x = np.array([1.0, 2.0, -1.0]).reshape(1, 3, 1, 1)
    dt = np.ones((1, 3, 1))
    A = np.array([-math.log(2.0)])
    B = np.full((1, 3, 1, 1), 2.0)
    C = np.full((1, 3, 1, 1), 3.0)
    D = np.array([0.5])
    y, final, _ = oracle.recurrence(x, dt, A, B, C, D)
    np.testing.assert_allclose(y.reshape(-1), [6.5, 16.0, 1.0], rtol=0, atol=1e-14)
    np.testing.assert_allclose(final.reshape(-1), [0.5], rtol=0, atol=1e-15)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_recurrence_equals_dual_form(seed):
    # Knowl 1: the linear form and the quadratic masked-attention form are the same map.
    inp = rnd(seed=seed)
    y_rec, _, _ = oracle.recurrence(**{k: v for k, v in inp.items()})
    y_dual = oracle.dual_form(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], inp["D"])
    assert oracle.rel_err(y_rec, y_dual) < 1e-12


def test_zero_decay_is_causal_linear_attention():
    # A = 0 makes every a_t = 1, so L is the all-ones lower triangle and the layer is
    # causal linear attention y_j = sum_{i<=j} (C_j . B_i) dt_i x_i + D x_j.
    inp = rnd(seed=3)
    x, dt, B, C, D = (f64(inp[k]) for k in ("x", "dt", "B", "C", "D"))
    A = np.zeros(inp["A"].shape)
    b, T, H, P = x.shape
    G = B.shape[2]
    ref = np.zeros_like(x)
    for bi in range(b):
        for h in range(H):
            g = h // (H // G)
            for j in range(T):
                acc = np.zeros(P)
                for i in range(j + 1):
                    acc += float(np.dot(C[bi, j, g], B[bi, i, g])) * dt[bi, i, h] * x[bi, i, h]
                ref[bi, j, h] = acc + D[h] * x[bi, j, h]
    y, _, _ = oracle.recurrence(x, dt, A, B, C, D)
    assert oracle.rel_err(y, ref) < 1e-12
    assert oracle.rel_err(oracle.dual_form(x, dt, A, B, C, D), ref) < 1e-12
    yc, _, _, _, _ = oracle.chunked(x, dt, A, B, C, D, chunk_size=16)
    assert oracle.rel_err(yc, ref) < 1e-12


def test_impulse_response_closed_form():
    # x is zero except at t0 and the state starts at 0, so
    #   y_t = 0                                                   for t < t0
    #   y_t0 = (C_t0 . B_t0) dt_t0 x_t0 + D x_t0
    #   y_t  = (C_t . B_t0) dt_t0 exp(A * sum_{s=t0+1}^{t} dt_s) x_t0  for t > t0
    inp = rnd(b=1, T=30, H=2, P=4, G=1, N=6, seed=4)
    x, dt, A, B, C, D = (f64(inp[k]) for k in ("x", "dt", "A", "B", "C", "D"))
    t0 = 11
    xi = np.zeros_like(x)
    xi[:, t0] = x[:, t0]
    y, _, _ = oracle.recurrence(xi, dt, A, B, C, D)
    for h in range(2):
        assert np.all(y[0, :t0, h] == 0.0)
        np.testing.assert_allclose(
            y[0, t0, h], (C[0, t0, 0] @ B[0, t0, 0]) * dt[0, t0, h] * xi[0, t0, h] + D[h] * xi[0, t0, h],
            rtol=1e-13, atol=1e-15)
        for t in range(t0 + 1, 30):
            decay = math.exp(A[h] * dt[0, t0 + 1:t + 1, h].sum())
            want = (C[0, t, 0] @ B[0, t0, 0]) * dt[0, t0, h] * decay * xi[0, t0, h]
            np.testing.assert_allclose(y[0, t, h], want, rtol=1e-12, atol=1e-15)


def test_scalar_time_invariant_is_iir_filter():
    # N = P = 1 with constant dt, B, C: h_t = a h_{t-1} + dt B x_t is a first-order
    # IIR filter, so y = C * lfilter([dt B], [1, -a], x) + D x.
    rng = np.random.default_rng(5)
    T = 200
    x = rng.standard_normal(T)
    dtv, Bv, Cv, Dv, Av = 0.07, 0.8, -1.3, 0.4, -2.5
    a = math.exp(dtv * Av)
    want = Cv * scipy.signal.lfilter([dtv * Bv], [1.0, -a], x) + Dv * x
    y, _, _ = oracle.recurrence(x.reshape(1, T, 1, 1), np.full((1, T, 1), dtv), np.array([Av]),
                                np.full((1, T, 1, 1), Bv), np.full((1, T, 1, 1), Cv),
                                np.array([Dv]))
    np.testing.assert_allclose(y.reshape(-1), want, rtol=1e-12, atol=1e-13)


def test_time_invariant_is_convolution():
    # Constant dt, B, C over time makes the layer a causal convolution of each
    # channel p with the kernel K_k = (C . B) dt a^k.
    rng = np.random.default_rng(6)
    T, P, N = 64, 3, 7
    x = rng.standard_normal((1, T, 1, P))
    Bv = rng.standard_normal(N) / math.sqrt(N)
    Cv = rng.standard_normal(N) / math.sqrt(N)
    dtv, Av, Dv = 0.05, -3.0, -0.7
    a = math.exp(dtv * Av)
    K = float(Cv @ Bv) * dtv * a ** np.arange(T)
    want = np.stack([np.convolve(x[0, :, 0, p], K)[:T] for p in range(P)], axis=-1) + Dv * x[0, :, 0]
    y, _, _ = oracle.recurrence(x, np.full((1, T, 1), dtv), np.array([Av]),
                                np.broadcast_to(Bv, (1, T, 1, N)).copy(),
                                np.broadcast_to(Cv, (1, T, 1, N)).copy(), np.array([Dv]))
    np.testing.assert_allclose(y[0, :, 0], want, rtol=1e-11, atol=1e-12)


@pytest.mark.parametrize("Q", [1, 4, 16, 64, 50])
def test_chunked_algorithm_equals_recurrence(Q):
    # Knowl 2: the block decomposition gives the same Y and h_final as the recurrence for
    # every chunk size, including T not a multiple of Q (T = 50, Q = 4, 16, 64).
    inp = rnd(T=50, seed=7, init=True)
    y, final, entry = oracle.recurrence(**inp, chunk_size=Q)
    yc, fc, cs, S, ec = oracle.chunked(**inp, chunk_size=Q)
    assert oracle.rel_err(yc, y) < 1e-12
    assert oracle.rel_err(fc, final) < 1e-12
    assert oracle.rel_err(ec, entry) < 1e-12
    S_def = oracle.chunk_states(inp["x"], inp["dt"], inp["A"], inp["B"], Q)
    assert oracle.rel_err(S, S_def) < 1e-12


def test_state_passing_identity():
    # Knowl 2, state passing: h_{c+1} = (prod_{t in chunk c} a_t) h_c + S_c, where h_c
    # comes from the recurrence itself and S_c from a zero-state run of chunk c.
    Q = 8
    inp = rnd(T=37, seed=8, init=True)
    _, final, entry = oracle.recurrence(**inp, chunk_size=Q)
    S = oracle.chunk_states(inp["x"], inp["dt"], inp["A"], inp["B"], Q)
    dt, A = f64(inp["dt"]), f64(inp["A"])
    b, T, H = dt.shape
    nc = entry.shape[1]
    for c in range(nc):
        sl = slice(c * Q, min(T, (c + 1) * Q))
        decay = np.exp((dt[:, sl, :] * A[None, None, :]).sum(axis=1))      # [b, H]
        nxt = entry[:, c + 1] if c + 1 < nc else final
        np.testing.assert_allclose(nxt, decay[:, :, None, None] * entry[:, c] + S[:, c],
                                   rtol=1e-12, atol=1e-13)


def test_chunk_cumsum_matches_products_of_a():
    # exp(cs_j - cs_i) is the mask entry prod_{s=i+1}^{j} a_s, the direct products of Knowl 1.
    inp = rnd(b=1, T=20, H=2, seed=9)
    dt, A = f64(inp["dt"]), f64(inp["A"])
    cs = oracle.chunk_cumsum(dt, A, 20)
    for h in range(2):
        a = np.exp(dt[0, :, h] * A[h])
        for j in range(20):
            for i in range(j + 1):
                np.testing.assert_allclose(math.exp(cs[0, h, 0, j] - cs[0, h, 0, i]),
                                           np.prod(a[i + 1:j + 1]), rtol=1e-12)


def test_continuation_equals_whole_sequence():
    # Knowl 8 (sequence parallelism): run [0, T1), hand its final state to [T1, T).
    inp = rnd(T=45, seed=10, init=True)
    y, final, _ = oracle.recurrence(**inp)
    T1 = 17
    first = {k: (v[:, :T1] if k in ("x", "dt", "B", "C") else v) for k, v in inp.items()}
    y1, s1, _ = oracle.recurrence(**first)
    second = {k: (v[:, T1:] if k in ("x", "dt", "B", "C") else v) for k, v in inp.items()}
    second["initial_states"] = s1
    y2, s2, _ = oracle.recurrence(**second)
    assert oracle.rel_err(np.concatenate([y1, y2], axis=1), y) < 1e-13
    assert oracle.rel_err(s2, final) < 1e-13


def test_linearity_in_x_and_initial_state():
    inp = rnd(T=30, seed=11, init=True)
    inp2 = rnd(T=30, seed=12, init=True)
    al, be = 0.75, -1.5
    mix = dict(inp)
    mix["x"] = al * f64(inp["x"]) + be * f64(inp2["x"])
    mix["initial_states"] = al * f64(inp["initial_states"]) + be * f64(inp2["initial_states"])
    y_mix, f_mix, _ = oracle.recurrence(**mix)
    y1, f1, _ = oracle.recurrence(**inp)
    other = dict(inp)
    other["x"], other["initial_states"] = inp2["x"], inp2["initial_states"]
    y2, f2, _ = oracle.recurrence(**other)
    assert oracle.rel_err(y_mix, al * y1 + be * y2) < 1e-12
    assert oracle.rel_err(f_mix, al * f1 + be * f2) < 1e-12


def test_reset_forgets_the_past():
    # Knowl 8 (variable length): a_t = 0 at a boundary resets the state, so outputs from
    # the boundary on do not depend on earlier inputs or on the initial state.
    inp = rnd(T=40, seed=13, init=True)
    dt = f64(inp["dt"]).copy()
    tr = 23
    dt[:, tr, :] = 1000.0          # exp(1000 * A) underflows to exactly 0 for A <= -1
    base = dict(inp, dt=dt)
    y, _, _ = oracle.recurrence(**base)
    pert = dict(base)
    x = f64(inp["x"]).copy()
    x[:, :tr] += np.random.default_rng(0).standard_normal(x[:, :tr].shape)
    pert["x"] = x
    pert["initial_states"] = f64(inp["initial_states"]) * 3.0
    y2, _, _ = oracle.recurrence(**pert)
    assert np.array_equal(y[:, tr:], y2[:, tr:])
    assert not np.array_equal(y[:, :tr], y2[:, :tr])


def test_semiseparable_rank():
    # Knowl 3: the SSM matrix M (y = M x for one channel) is N-semiseparable: every block
    # strictly below the diagonal has rank <= N.
    rng = np.random.default_rng(14)
    T, N = 24, 3
    dt = np.exp(rng.uniform(math.log(1e-2), math.log(0.5), size=(1, T, 1)))
    A = np.array([-1.7])
    B = rng.standard_normal((1, T, 1, N))
    C = rng.standard_normal((1, T, 1, N))
    M = np.zeros((T, T))
    for i in range(T):
        e = np.zeros((1, T, 1, 1))
        e[0, i, 0, 0] = 1.0
        y, _, _ = oracle.recurrence(e, dt, A, B, C)
        M[:, i] = y[0, :, 0, 0]
    assert np.allclose(np.triu(M, 1), 0.0)
    for split in (6, 12, 18):
        s = np.linalg.svd(M[split:, :split], compute_uv=False)
        assert s[N] <= 1e-10 * s[0]
        assert s[N - 1] > 1e-8 * s[0]
    # a block reaching the diagonal is generically of full rank min(rows, cols) > N
    s = np.linalg.svd(M[8:16, 8:16], compute_uv=False)
    assert s[N] > 1e-8 * s[0]


@pytest.mark.parametrize("which", ["B", "C"])
def test_zero_projection_leaves_skip_term(which):
    inp = rnd(T=20, seed=15)
    inp[which] = inp[which] * 0
    y, _, _ = oracle.recurrence(**inp)
    want = f64(inp["D"])[None, None, :, None] * f64(inp["x"])
    assert np.array_equal(y, want)


def test_bh_subset_matches_full_run():
    inp = rnd(T=33, seed=16, init=True)
    y, f, _ = oracle.recurrence(**inp)
    sel = [(1, 3), (0, 0)]
    ys, fs, _ = oracle.recurrence(**inp, bh_list=sel)
    for b, h in sel:
        assert np.array_equal(ys[b, :, h], y[b, :, h])
        assert np.array_equal(fs[b, h], f[b, h])
    assert np.isnan(ys[0, :, 1]).all()


def test_golden_fixture():
    # Regression fixture written by tests/golden/make_golden.py (which calls only oracle/).
    with open(os.path.join(HERE, "golden", "tiny_recurrence.json")) as fh:
        g = json.load(fh)
    arr = {k: np.array(v, dtype=np.float64) for k, v in g["inputs"].items()}
    y, final, _ = oracle.recurrence(arr["x"], arr["dt"], arr["A"], arr["B"], arr["C"], arr["D"],
                                    arr["initial_states"])
    np.testing.assert_allclose(y, np.array(g["y"]), rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(final, np.array(g["final_states"]), rtol=1e-13, atol=1e-15)


# ---------------------------------------------------------------- gate + norm (Knowl 6)
def _gate_inputs(seed, rows=6, H=4, P=8):
    rng = np.random.Generator(np.random.PCG64(seed))
    y = rng.standard_normal((rows, H, P))
    z = rng.standard_normal((rows, H, P)) * 2.0
    w = rng.uniform(0.5, 1.5, size=(H * P,))
    return y, z, w


@pytest.mark.parametrize("group_size", [32, 16, 8, 1])
def test_gated_rmsnorm_matches_library_rmsnorm(group_size):
    """Against torch's own SiLU and RMSNorm routines (fp64), groups as reshapes."""
    import torch
    y, z, w = _gate_inputs(1)
    eps = 1e-5
    got = oracle.gated_rmsnorm(y, z, w, group_size, eps)
    ty, tz = torch.from_numpy(y), torch.from_numpy(z)
    g = (ty * torch.nn.functional.silu(tz)).reshape(y.shape[0], -1, group_size)
    ref = torch.nn.functional.rms_norm(g, (group_size,), eps=eps)
    ref = (ref * torch.from_numpy(w).reshape(-1, group_size)).reshape(y.shape).numpy()
    assert np.max(np.abs(got - ref)) <= 1e-12 * np.max(np.abs(ref))


def test_gated_rmsnorm_identities():
    y, z, w = _gate_inputs(2)
    ones = np.ones_like(w)
    # eps = 0: scale invariant, odd in y, and every group comes out with unit RMS
    a = oracle.gated_rmsnorm(y, z, w, 16, 0.0)
    assert np.allclose(oracle.gated_rmsnorm(3.7 * y, z, w, 16, 0.0), a, rtol=1e-13, atol=0)
    assert np.allclose(oracle.gated_rmsnorm(-y, z, w, 16, 0.0), -a, rtol=1e-13, atol=0)
    u = oracle.gated_rmsnorm(y, z, ones, 16, 0.0).reshape(y.shape[0], -1, 16)
    assert np.allclose(np.mean(u * u, axis=-1), 1.0, rtol=1e-13)
    # a closed gate (z = 0) gives 0; SiLU(z) -> z for large z and -> 0 for very negative z
    assert np.all(oracle.gated_rmsnorm(y, np.zeros_like(z), w, 16, 1e-5) == 0)
    big = np.full_like(z, 40.0)
    ref = oracle.gated_rmsnorm(y * 40.0, np.full_like(z, 1e9), w, 16, 0.0)
    assert np.allclose(oracle.gated_rmsnorm(y, big, w, 16, 0.0), ref, rtol=1e-12)


def test_gated_rmsnorm_hand_example():
    """One group of two channels, gate open (SiLU(z) = z for z -> inf, here z = 60
    where 1/(1+e^-60) = 1 in fp64): values 3*60 and 4*60; RMS = 60*sqrt((9+16)/2),
    so the outputs are 3/sqrt(12.5) and 4/sqrt(12.5) times the weights 2 and 1."""
    y = np.array([[[3.0, 4.0]]])
    z = np.full_like(y, 60.0)
    out = oracle.gated_rmsnorm(y, z, np.array([2.0, 1.0]), 2, 0.0)
    assert np.allclose(out.ravel(), [2 * 3 / math.sqrt(12.5), 4 / math.sqrt(12.5)], rtol=1e-15)


# ---------------------------------------------------------------- packed documents (Knowl 8)
def _packed(cu, seed, H=2, P=3, G=1, N=4):
    T = cu[-1]
    inp = make_inputs(1, T, H, P, G, N, dtype="f32", dt_dist="softplus", seed=seed)
    inp.pop("initial_states")
    rng = np.random.Generator(np.random.PCG64(seed + 1))
    init = rng.standard_normal((len(cu) - 1, H, P, N)) * 0.1
    return inp, init


@pytest.mark.parametrize("cu", [[0, 7, 8, 20, 33], [0, 33], [0, 1, 2, 3, 33], [0, 12, 12, 33]])
def test_packed_documents_equal_resets_in_dual_form(cu):
    """Knowl 8 literally: a_t = 0 at each document start in one flat sequence. The dual
    form with those resets (brute force, products of a) must equal running every
    document as its own sequence; documents of length 0 and 1 included."""
    inp, _ = _packed(cu, seed=31)
    y, _ = oracle.recurrence_varlen(**inp, cu_seqlens=cu)
    resets = np.zeros((1, cu[-1]), dtype=bool)
    for s in cu[1:-1]:
        if s < cu[-1]:
            resets[0, s] = True
    y_ref = oracle.dual_form(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], inp["D"],
                             resets=resets)
    assert oracle.rel_err(y, y_ref) < 1e-12


def test_packed_documents_are_independent():
    cu = [0, 9, 21, 33]
    inp, init = _packed(cu, seed=32)
    y, fin = oracle.recurrence_varlen(**inp, cu_seqlens=cu, initial_states=init)
    pert = dict(inp)
    x = f64(inp["x"]).copy()
    x[:, 9:21] += 1.0                       # change document 1 only
    pert["x"] = x
    init2 = init.copy()
    init2[1] *= -2.0
    y2, fin2 = oracle.recurrence_varlen(**pert, cu_seqlens=cu, initial_states=init2)
    assert np.array_equal(y[:, :9], y2[:, :9]) and np.array_equal(y[:, 21:], y2[:, 21:])
    assert np.array_equal(fin[[0, 2]], fin2[[0, 2]])
    assert not np.array_equal(y[:, 9:21], y2[:, 9:21])
    # one document is the plain recurrence
    y1, f1 = oracle.recurrence_varlen(**inp, cu_seqlens=[0, 33], initial_states=init[:1])
    y_ref, f_ref, _ = oracle.recurrence(**inp, initial_states=init[:1])
    assert np.array_equal(y1, y_ref) and np.array_equal(f1, f_ref)


@pytest.mark.parametrize("cu,Q", [([0, 7, 8, 20, 33], 8), ([0, 16, 32, 33], 16), ([0, 1, 2, 3, 33], 4),
                                  ([0, 12, 12, 33], 5), ([0, 5, 9, 30, 31, 33], 7), ([0, 0, 33], 33)])
@pytest.mark.parametrize("with_init", [False, True])
def test_chunked_algorithm_on_packed_documents(cu, Q, with_init):
    """Knowl 2's chunked algorithm with segment-aware decays (the blueprint for the
    kernels) equals every document run as its own sequence: documents starting on
    and off chunk boundaries, several in one chunk, empty and one-token ones."""
    inp, init = _packed(cu, seed=40 + Q, H=4, P=3, G=2, N=5)
    ini = init if with_init else None
    y, f = oracle.recurrence_varlen(**inp, cu_seqlens=cu, initial_states=ini)
    y2, f2 = oracle.chunked_varlen(**inp, cu_seqlens=cu, chunk_size=Q, initial_states=ini)
    assert oracle.rel_err(y2, y) < 1e-12
    assert oracle.rel_err(f2, f) < 1e-12
