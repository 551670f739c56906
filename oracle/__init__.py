"""Oracle for the SSD layer forward: plain, slow, fp64, CPU only.

Test infrastructure. Only ``tests/``, ``__graft_entry__.smoke()`` and the
benchmark's ``cpu_baseline`` / ``--impl reference`` legs use it. It shares no
code with the CUDA path and never imports it.

Source of every definition: "Transformers are SSMs: Generalized Models and
Efficient Algorithms Through Structured State Space Duality" (summary page),
Knowl 1 (linear and dual forms), Knowl 2 (block-decomposition algorithm) and
Knowl 6 (Mamba-2 block: gate and norm), Knowl 7 (head patterns); "Mamba-2 and
State Space Duality (SSD)", section
"The Concept of State Space Duality" (dual form Y = (L o C B^T) X).

Functions
  recurrence()    the definition: the linear (recurrent) form in C, fp64.
  chunk_cumsum()  intra-chunk inclusive cumulative sums of dt*A (log of the
                  cumulative products of a_t, Knowl 2 step 2).
  chunk_states()  per-chunk states S_c: the recurrence run over chunk c alone
                  from a zero state (Knowl 2, "right factor chunk state").
  dual_form()     the quadratic (masked attention) form, tiny T only; optional
                  resets (a_t = 0) for packed documents.
  recurrence_varlen()  packed variable-length documents (Knowl 8), each its own
                  sequence.
  chunked_varlen() the block-decomposition algorithm on packed documents, with
                  segment-aware decays, step by step (the kernels' blueprint).
  chunked()       the block-decomposition algorithm, step by step, fp64.
  gated_rmsnorm() the gate and RMSNorm after the layer (Knowl 6), fp64.
Every function is pinned by ``tests/test_oracle.py`` against closed forms,
library routines and the identities the pages state.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ssd_oracle.c")
_BUILD_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD_DIR, "libssd_oracle.so")
_lib = None
_lock = threading.Lock()


def build(force: bool = False) -> str:
    """Compile the C oracle with gcc (no fast-math) into oracle/_build/."""
    os.makedirs(_BUILD_DIR, exist_ok=True)
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            d = ctypes.POINTER(ctypes.c_double)
            i64 = ctypes.c_int64
            lib.ssd_oracle_recurrence.argtypes = [i64] * 6 + [d] * 9 + [i64, d,
                                                  ctypes.POINTER(ctypes.c_int64), i64]
            lib.ssd_oracle_recurrence.restype = ctypes.c_int
            lib.ssd_oracle_max_threads.restype = ctypes.c_int
            _lib = lib
    return _lib


def max_threads() -> int:
    return int(_load().ssd_oracle_max_threads())


def _f64(a):
    """Exact upcast of a numpy array or a torch tensor (any float dtype) to fp64."""
    if a is None:
        return None
    if hasattr(a, "detach"):
        a = a.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(a, dtype=np.float64)


def _ptr(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def recurrence(x, dt, A, B, C, D=None, initial_states=None, chunk_size=None,
               bh_list=None):
    """Linear (recurrent) form, fp64 (Knowl 1 with dt and D).

    Returns (y [b,T,H,P], final_states [b,H,P,N], entry) where ``entry`` is
    None, or, when ``chunk_size`` is given, the states entering each chunk
    [b, nc, H, P, N]. With ``bh_list`` (pairs (b, h)) only those sequences are
    run; the other outputs are NaN.
    """
    x, dt, A, B, C, D, init = map(_f64, (x, dt, A, B, C, D, initial_states))
    b, T, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    y = np.full((b, T, H, P), np.nan)
    final = np.full((b, H, P, N), np.nan)
    entry = None
    if chunk_size is not None:
        nc = -(-T // chunk_size)
        entry = np.full((b, nc, H, P, N), np.nan)
    bl = None
    nbh = 0
    if bh_list is not None:
        bl = np.ascontiguousarray(np.asarray(bh_list, dtype=np.int64).reshape(-1, 2))
        nbh = bl.shape[0]
    rc = _load().ssd_oracle_recurrence(
        b, T, H, P, G, N, _ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(init),
        _ptr(y), _ptr(final), int(chunk_size or 0), _ptr(entry),
        bl.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)) if bl is not None else None, nbh)
    if rc != 0:
        raise ValueError("oracle recurrence rejected its arguments")
    return y, final, entry


def chunk_cumsum(dt, A, chunk_size):
    """cs[b,h,c,k] = sum_{k' <= k} dt[b, cQ+k', h] * A[h] (inclusive, within chunk c).

    Positions past the end of a partial last chunk repeat the chunk's last value
    (they stand for padding tokens with dt = 0, which leave the state unchanged).
    """
    dt, A = _f64(dt), _f64(A)
    b, T, H = dt.shape
    Q = chunk_size
    nc = -(-T // Q)
    dA = np.zeros((b, nc * Q, H))
    dA[:, :T, :] = dt * A[None, None, :]
    dA = dA.reshape(b, nc, Q, H).transpose(0, 3, 1, 2)   # [b, H, nc, Q]
    return np.cumsum(dA, axis=-1)


def chunk_states(x, dt, A, B, chunk_size):
    """S_c = state reached from zero by running chunk c alone: [b, nc, H, P, N].

    A partial last chunk is padded with dt = 0, x = 0 tokens, which leave the
    state unchanged, so the padding does not alter S.
    """
    x, dt, A, B = map(_f64, (x, dt, A, B))
    b, T, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    Q = chunk_size
    nc = -(-T // Q)
    pad = nc * Q - T

    def padT(a):
        if pad == 0:
            return a
        z = np.zeros((a.shape[0], pad) + a.shape[2:])
        return np.concatenate([a, z], axis=1)

    xs = padT(x).reshape(b * nc, Q, H, P)
    dts = padT(dt).reshape(b * nc, Q, H)
    Bs = padT(B).reshape(b * nc, Q, G, N)
    zeroC = np.zeros_like(Bs)
    _, final, _ = recurrence(xs, dts, A, Bs, zeroC)
    return final.reshape(b, nc, H, P, N)


def dual_form(x, dt, A, B, C, D=None, resets=None):
    """Quadratic (masked attention) form, fp64, one dense T x T matrix per (b, h).

    y = (L o (C B^T)) diag(dt) x + D x with the 1-semiseparable mask
    L_ji = prod_{s=i+1}^{j} a_s for j >= i and 0 above the diagonal
    (Knowl 1, dual form; "Mamba-2 and State Space Duality", Y = (L o C B^T) X).
    The products are taken directly, not through exponentials of sums.
    ``resets`` (bool [b, T], optional) sets a_t = 0 where true, the document
    boundaries of packed variable-length input (Knowl 8).
    """
    x, dt, A, B, C, D = map(_f64, (x, dt, A, B, C, D))
    rs = None if resets is None else np.asarray(resets, dtype=bool)
    b, T, H, P = x.shape
    G = B.shape[2]
    hpg = H // G
    y = np.zeros_like(x)
    for bi in range(b):
        for h in range(H):
            g = h // hpg
            a = np.exp(dt[bi, :, h] * A[h])
            if rs is not None:
                a = np.where(rs[bi], 0.0, a)
            L = np.zeros((T, T))
            for j in range(T):
                L[j, j] = 1.0
                for i in range(j - 1, -1, -1):
                    L[j, i] = L[j, i + 1] * a[i + 1]
            G_ = C[bi, :, g, :] @ B[bi, :, g, :].T
            M = L * G_ * dt[bi, :, h][None, :]
            y[bi, :, h, :] = M @ x[bi, :, h, :]
            if D is not None:
                y[bi, :, h, :] += D[h] * x[bi, :, h, :]
    return y


def recurrence_varlen(x, dt, A, B, C, D=None, cu_seqlens=None, initial_states=None):
    """Packed variable-length input (Knowl 8): documents concatenated along the
    sequence of batch row 0, document k at tokens cu_seqlens[k] .. cu_seqlens[k+1]-1,
    each run as its own sequence (the state does not cross a boundary).

    x [1, T, H, P], dt [1, T, H], B/C [1, T, G, N]; cu_seqlens [n_docs + 1] with
    cu_seqlens[0] = 0, non-decreasing, cu_seqlens[-1] = T; initial_states
    [n_docs, H, P, N] or None. Returns (y [1, T, H, P], final_states [n_docs, H, P, N]).
    """
    x, dt, A, B, C, D, init = map(_f64, (x, dt, A, B, C, D, initial_states))
    cu = [int(v) for v in np.asarray(cu_seqlens).ravel()]
    if x.shape[0] != 1 or cu[0] != 0 or cu[-1] != x.shape[1] or any(b < a for a, b in zip(cu, cu[1:])):
        raise ValueError("packed input needs batch 1 and cu_seqlens from 0 to T, non-decreasing")
    ndoc = len(cu) - 1
    H, P, N = x.shape[2], x.shape[3], B.shape[3]
    y = np.zeros_like(x)
    final = np.zeros((ndoc, H, P, N))
    for k in range(ndoc):
        sl = slice(cu[k], cu[k + 1])
        yk, fk, _ = recurrence(x[:, sl], dt[:, sl], A, B[:, sl], C[:, sl], D,
                               init[k:k + 1] if init is not None else None)
        y[:, sl] = yk
        final[k] = fk[0]
    return y, final


def chunked(x, dt, A, B, C, D=None, chunk_size=64, initial_states=None):
    """Block-decomposition SSD algorithm (Knowl 2), fp64, taken step by step.

    Readings where the page leaves a step open:
      * "decayed X" in the chunk state: token k of chunk c is weighted by
        exp(cs_last - cs_k) * dt_k (the decay from after token k to the chunk end).
      * chunk decay in state passing: prod_{t=0}^{Q-1} a_t = exp(cs_last).
      * "decayed h_c" in the off-diagonal output: row j is scaled by exp(cs_j),
        the decay from the chunk start through token j inclusive.
      * the initial state h_0 is ``initial_states`` when given, else 0.
      * a partial last chunk has fewer rows; nothing else changes.
    Returns (y, final_states, cs, S, entry).
    """
    x, dt, A, B, C, D, init = map(_f64, (x, dt, A, B, C, D, initial_states))
    b, T, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    hpg = H // G
    Q = chunk_size
    nc = -(-T // Q)
    y = np.zeros_like(x)
    final = np.zeros((b, H, P, N))
    cs_all = chunk_cumsum(dt, A, Q)
    S_all = np.zeros((b, nc, H, P, N))
    entry = np.zeros((b, nc, H, P, N))
    for bi in range(b):
        for h in range(H):
            g = h // hpg
            # step 1: partition into chunks
            parts = [slice(c * Q, min(T, (c + 1) * Q)) for c in range(nc)]
            Ydiag, S = [], []
            for c, sl in enumerate(parts):
                n_c = sl.stop - sl.start
                Xc, Bc, Cc = x[bi, sl, h, :], B[bi, sl, g, :], C[bi, sl, g, :]
                dtc = dt[bi, sl, h]
                # step 2: intra-chunk cumulative products of a, kept as log sums
                cs = cs_all[bi, h, c, :n_c]
                # step 3: 1-SS chunk mask L_ji = prod_{s=i+1}^{j} a_s (j >= i)
                Lc = np.zeros((n_c, n_c))
                for j in range(n_c):
                    for i in range(j + 1):
                        Lc[j, i] = np.exp(cs[j] - cs[i])
                # step 4: diagonal block output (L o C B^T) (dt x)
                Ydiag.append((Lc * (Cc @ Bc.T)) @ (dtc[:, None] * Xc))
                # step 5: right-factor chunk state B^T (decayed X), stored as [P, N]
                w = np.exp(cs[-1] - cs) * dtc
                Sc = (w[:, None] * Xc).T @ Bc
                S.append(Sc)
                S_all[bi, c, h] = Sc
            # steps 6-7: state passing across chunks
            hc = init[bi, h].copy() if init is not None else np.zeros((P, N))
            hs = []
            for c, sl in enumerate(parts):
                hs.append(hc)
                entry[bi, c, h] = hc
                n_c = sl.stop - sl.start
                hc = np.exp(cs_all[bi, h, c, n_c - 1]) * hc + S[c]
            final[bi, h] = hc
            # steps 8-9: off-diagonal output from the incoming state, combine, assemble
            for c, sl in enumerate(parts):
                n_c = sl.stop - sl.start
                cs = cs_all[bi, h, c, :n_c]
                Cc = C[bi, sl, g, :]
                Yoff = np.exp(cs)[:, None] * (Cc @ hs[c].T)
                y[bi, sl, h, :] = Ydiag[c] + Yoff
            if D is not None:
                y[bi, :, h, :] += D[h] * x[bi, :, h, :]
    return y, final, cs_all, S_all, entry


def gated_rmsnorm(y, z, weight, group_size, eps):
    """Gate and normalisation after the SSD layer, fp64.

    "Transformers are SSMs" (summary page), Knowl 6, step 4 of the Mamba-2
    block: the layer output is gated elementwise by the SiLU of the gate branch
    z, Y_g = Y * SiLU(z) with SiLU(v) = v / (1 + exp(-v)), then normalised
    (RMSNorm) before the output projection. Reading where the page is silent:
    the channels of a token (H * P, head-major as in y) are split into
    contiguous groups of ``group_size``; each group is divided by
    sqrt(mean over the group of Y_g^2 + eps) and scaled by the per-channel
    ``weight`` [H * P].
    y, z: [..., H, P] (same shape); returns an array of that shape.
    """
    y, z, w = _f64(y), _f64(z), _f64(weight)
    shape = y.shape
    C = shape[-2] * shape[-1]
    if C % group_size != 0:
        raise ValueError("group_size must divide the channel count")
    yg = (y * (z / (1.0 + np.exp(-z)))).reshape(-1, C // group_size, group_size)
    ms = np.mean(yg * yg, axis=-1, keepdims=True)
    out = yg / np.sqrt(ms + eps) * w.reshape(C // group_size, group_size)
    return out.reshape(shape)


def chunked_varlen(x, dt, A, B, C, D=None, cu_seqlens=None, chunk_size=64, initial_states=None):
    """Block-decomposition algorithm (Knowl 2) on packed documents (Knowl 8), fp64.

    Same inputs and outputs as ``recurrence_varlen``. The chunk grid ignores the
    documents; each token carries its document index seg_t, and with cs the plain
    intra-chunk cumulative sum of dt*A (a_t = 0 at a document start is applied
    by the segment tests, so no log-decay is ever -inf):
      * mask: L_ji = exp(cs_j - cs_i) if seg_j == seg_i (j >= i), else 0;
      * chunk state: only tokens of the chunk's last document count,
        S_c = sum_{k: seg_k = seg_last} exp(cs_last - cs_k) dt_k x_k B_k^T;
      * the state entering chunk c belongs to the document of token cQ - 1 and
        survives to token j only if seg_j is that document: the off-diagonal term
        exp(cs_j) C_j h_c and the chunk decay exp(cs_last) h_c are kept only then;
      * a document starting at token s inside chunk c enters its initial state
        there: tokens j >= s of that document add exp(cs_j - cs_{s-1}) C_j h0
        (cs_{s-1} = 0 when s is the chunk's first token), and so does the chunk
        state when that document is the chunk's last;
      * the state at a document's last token e is the same sum stopped at e.
    Returns (y, final_states).
    """
    x, dt, A, B, C, D, init = map(_f64, (x, dt, A, B, C, D, initial_states))
    cu = [int(v) for v in np.asarray(cu_seqlens).ravel()]
    _, T, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    hpg = H // G
    Q = chunk_size
    ndoc = len(cu) - 1
    seg = np.zeros(T, dtype=np.int64)
    start = np.zeros(T, dtype=bool)
    for k in range(ndoc):
        seg[cu[k]:cu[k + 1]] = k
        if cu[k] < cu[k + 1]:
            start[cu[k]] = True
    y = np.zeros_like(x)
    final = np.zeros((ndoc, H, P, N))
    for k in range(ndoc):                       # empty documents keep their initial state
        if cu[k] == cu[k + 1] and init is not None:
            final[k] = init[k]
    nc = -(-T // Q)
    for h in range(H):
        g = h // hpg
        hc = np.zeros((P, N))                   # state entering the chunk
        for c in range(nc):
            t0, t1 = c * Q, min(T, (c + 1) * Q)
            n_c = t1 - t0
            sg = seg[t0:t1]
            Xc, Bc, Cc = x[0, t0:t1, h], B[0, t0:t1, g], C[0, t0:t1, g]
            dtc = dt[0, t0:t1, h]
            cs = np.cumsum(dtc * A[h])
            prev = seg[t0 - 1] if t0 > 0 else -1   # document of the entering state
            # the state entering this chunk counts only for the document of token t0-1,
            # and only until that document ends (a start at t0 ends it at once)
            keep = (sg == prev) & ~np.logical_or.accumulate(start[t0:t1])
            # diagonal block, segment-masked
            L = np.zeros((n_c, n_c))
            for j in range(n_c):
                for i in range(j + 1):
                    if sg[i] == sg[j]:
                        L[j, i] = np.exp(cs[j] - cs[i])
            Yc = (L * (Cc @ Bc.T)) @ (dtc[:, None] * Xc)
            Yc += keep[:, None] * np.exp(cs)[:, None] * (Cc @ hc.T)
            # initial states of documents starting inside this chunk
            h0 = {}
            for s in range(t0, t1):
                if start[s]:
                    k = seg[s]
                    h0[k] = (s - t0, init[k, h] if init is not None else np.zeros((P, N)))
            for k, (s, hk) in h0.items():
                base = cs[s - 1] if s > 0 else 0.0
                for j in range(s, n_c):
                    if sg[j] == k:
                        Yc[j] += np.exp(cs[j] - base) * (Cc[j] @ hk.T)
            y[0, t0:t1, h] = Yc
            # the state after token j of document k (for document ends and the chunk end)
            def state_at(j):
                k = sg[j]
                st = np.zeros((P, N))
                if keep[j]:
                    st += np.exp(cs[j]) * hc
                if k in h0:
                    s, hk = h0[k]
                    st += np.exp(cs[j] - (cs[s - 1] if s > 0 else 0.0)) * hk
                for i in range(j + 1):
                    if sg[i] == k:
                        st += np.exp(cs[j] - cs[i]) * dtc[i] * np.outer(Xc[i], Bc[i])
                return st
            for k in set(sg.tolist()):
                e = cu[k + 1] - 1
                if t0 <= e < t1:
                    final[k, h] = state_at(e - t0)
            hc = state_at(n_c - 1)
        if D is not None:
            y[0, :, h] += D[h] * x[0, :, h]
    return y, final


def rel_err(a, ref) -> float:
    """max|a - ref| / max|ref| over the whole tensor (the parity metric)."""
    a = _f64(a)
    ref = _f64(ref)
    m = np.max(np.abs(ref))
    if m == 0:
        return float(np.max(np.abs(a)))
    return float(np.max(np.abs(a - ref)) / m)
