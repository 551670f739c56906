"""Thin Python binding of libssd, the B200 SSD layer forward.

Argument marshalling only: every step of the computation runs in the CUDA
kernels of libssd.so. PyTorch supplies device memory and the current stream.
If the shared library is missing or fails to load, every call raises; there
is no fallback implementation.

    y, final = ssd_fwd(x, dt, A, B, C, D, chunk_size=256,
                       initial_states=None, return_final_states=True)

Shapes: x[b,T,H,P], dt[b,T,H], A[H], B/C[b,T,G,N], D[H], states[b,H,P,N]
("Transformers are SSMs: Generalized Models and Efficient Algorithms Through
Structured State Space Duality", Knowl 1, 2 and 7).
"""
from __future__ import annotations

import ctypes
import os

import torch

from ._lib import (SSD_BF16, SSD_F32, SSDError, ShapeT, check, lib, lib_path,  # noqa: F401
                   status_string)

__all__ = ["ssd_fwd", "ssd_fwd_host", "ssd_fwd_workspace_size", "ssd_fwd_plan", "ssd_fwd_check",
           "ssd_step", "ssd_fwd_cp", "ssd_cp_begin", "ssd_cp_end", "ssd_cp_record_floats",
           "ssd_gated_rmsnorm", "ssd_fwd_gated", "ssd_fwd_gated_workspace_size", "ssd_fwd_varlen", "ssd_fwd_varlen_workspace_size",
           "ssd_fwd_varlen_check", "ssd_chunk_cumsum",
           "ssd_chunk_state", "ssd_state_passing", "ssd_chunk_scan", "SSDError", "make_shape",
           "lib_path"]

_DT = {torch.float32: SSD_F32, torch.bfloat16: SSD_BF16}


def make_shape(x: torch.Tensor, B: torch.Tensor, chunk_size: int) -> ShapeT:
    b, T, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    if x.dtype not in _DT:
        raise TypeError(f"x must be float32 or bfloat16, got {x.dtype}")
    return ShapeT(b, T, H, P, G, N, int(chunk_size), _DT[x.dtype], 0)


def _p(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _need(t, name, dtype=None, device=True):
    if t is None:
        raise ValueError(f"{name} is required")
    if device and not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    return t


def ssd_fwd_plan(shape: ShapeT) -> tuple[str, int]:
    """(path name, kernel launches per ssd_fwd call) for this shape."""
    name = ctypes.c_char_p()
    n = ctypes.c_int(0)
    check(lib().ssd_fwd_plan(ctypes.byref(shape), ctypes.byref(name), ctypes.byref(n)), "ssd_fwd_plan")
    return name.value.decode(), int(n.value)


def ssd_fwd_workspace_size(shape: ShapeT) -> int:
    n = ctypes.c_size_t(0)
    check(lib().ssd_fwd_workspace_size(ctypes.byref(shape), ctypes.byref(n)), "ssd_fwd_workspace_size")
    return int(n.value)


def ssd_fwd(x, dt, A, B, C, D=None, chunk_size: int = 256, initial_states=None,
            return_final_states: bool = False, y=None, final_states=None, workspace=None,
            stream=None):
    """SSD layer forward on the GPU; returns y, or (y, final_states)."""
    _need(x, "x")
    _need(dt, "dt", torch.float32)
    _need(A, "A", torch.float32)
    _need(B, "B", x.dtype)
    _need(C, "C", x.dtype)
    if D is not None:
        _need(D, "D", torch.float32)
    if initial_states is not None:
        _need(initial_states, "initial_states", torch.float32)
    shape = make_shape(x, B, chunk_size)
    if y is None:
        y = torch.empty_like(x)
    if return_final_states and final_states is None:
        final_states = torch.empty((x.shape[0], x.shape[2], x.shape[3], B.shape[3]),
                                   dtype=torch.float32, device=x.device)
    nbytes = ssd_fwd_workspace_size(shape)
    if workspace is None or workspace.numel() < nbytes:
        workspace = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=x.device)
    check(lib().ssd_fwd(ctypes.byref(shape), _p(x), _p(dt), _p(A), _p(B), _p(C), _p(D),
                        _p(initial_states), _p(y), _p(final_states), _p(workspace),
                        ctypes.c_size_t(nbytes), _stream(stream)), "ssd_fwd")
    return (y, final_states) if return_final_states else y


def check_cu_seqlens(cu_seqlens, T: int) -> list[int]:
    """A host-side offset list as ints, or ValueError unless it runs from 0 to T, non-decreasing."""
    cu = [int(v) for v in (cu_seqlens.tolist() if hasattr(cu_seqlens, "tolist") else cu_seqlens)]
    if len(cu) < 2 or cu[0] != 0 or cu[-1] != T or any(b < a for a, b in zip(cu, cu[1:])):
        raise ValueError("cu_seqlens must run from 0 to T, non-decreasing")
    return cu


def ssd_fwd_gated_workspace_size(shape: ShapeT, group_size: int, fuse: bool = True) -> int:
    n = ctypes.c_size_t(0)
    check(lib().ssd_fwd_gated_workspace_size(ctypes.byref(shape), ctypes.c_int64(group_size), ctypes.c_int(int(fuse)),
                                             ctypes.byref(n)), "ssd_fwd_gated_workspace_size")
    return int(n.value)


def ssd_fwd_gated(x, dt, A, B, C, D=None, z=None, norm_weight=None, group_size: int = 64,
                  eps: float = 1e-5, fuse: bool = True, chunk_size: int = 256, initial_states=None,
                  return_final_states: bool = False, out=None, final_states=None, workspace=None,
                  stream=None):
    """The forward, then y * SiLU(z) RMS-normalised over channel groups times norm_weight
    (Knowl 6). With fuse, y is never stored when the single-pass kernel can apply the gate
    (groups of 8, 16, 32 or 64 channels); otherwise y passes through the workspace.
    Returns out, or (out, final_states)."""
    _need(x, "x")
    _need(z, "z", x.dtype)
    _need(norm_weight, "norm_weight", torch.float32)
    shape = make_shape(x, B, chunk_size)
    if out is None:
        out = torch.empty_like(x)
    if final_states is None and return_final_states:
        final_states = torch.empty((x.shape[0], x.shape[2], x.shape[3], B.shape[3]),
                                   dtype=torch.float32, device=x.device)
    nbytes = ssd_fwd_gated_workspace_size(shape, group_size, fuse)
    if workspace is None or workspace.numel() < nbytes:
        workspace = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=x.device)
    check(lib().ssd_fwd_gated(ctypes.byref(shape), _p(x), _p(dt), _p(A), _p(B), _p(C), _p(D),
                              _p(initial_states), _p(z), _p(norm_weight), ctypes.c_int64(group_size),
                              ctypes.c_float(eps), ctypes.c_int(int(fuse)), _p(out), _p(final_states),
                              _p(workspace),
                              ctypes.c_size_t(nbytes), _stream(stream)), "ssd_fwd_gated")
    return (out, final_states) if return_final_states else out


def ssd_fwd_varlen_workspace_size(shape: ShapeT, n_docs: int) -> int:
    n = ctypes.c_size_t(0)
    check(lib().ssd_fwd_varlen_workspace_size(ctypes.byref(shape), ctypes.c_int64(n_docs), ctypes.byref(n)),
          "ssd_fwd_varlen_workspace_size")
    return int(n.value)


def ssd_fwd_varlen(x, dt, A, B, C, D=None, cu_seqlens=None, chunk_size: int = 256,
                   initial_states=None, return_final_states: bool = False, y=None,
                   final_states=None, workspace=None, stream=None):
    """Packed variable-length documents (Knowl 8): batch row 0 of x [1, T, H, P]
    holds documents at tokens cu_seqlens[k] .. cu_seqlens[k+1]-1, each an
    independent sequence (a_t = 0 at its first token). Returns y, or
    (y, final_states [n_docs, H, P, N]); initial_states [n_docs, H, P, N] or None.

    cu_seqlens: a device int32 tensor [n_docs + 1] (passed as is), or a host list /
    tensor (copied to the device). One ssd_fwd_varlen call: every document runs in
    the single-pass kernel's one launch.
    """
    _need(x, "x")
    if x.shape[0] != 1:
        raise ValueError("packed documents need batch 1 (x [1, T, H, P])")
    if isinstance(cu_seqlens, torch.Tensor) and cu_seqlens.is_cuda:
        if cu_seqlens.dtype != torch.int32 or not cu_seqlens.is_contiguous() or cu_seqlens.dim() != 1:
            raise ValueError("device cu_seqlens must be a contiguous 1-D int32 tensor")
        if cu_seqlens.numel() < 1:
            raise ValueError("cu_seqlens needs at least one entry")
        cu_dev = cu_seqlens   # checked on the device; see ssd_fwd_varlen_check
    else:
        cu_dev = torch.tensor(check_cu_seqlens(cu_seqlens, x.shape[1]), dtype=torch.int32).to(x.device)
    ndoc = cu_dev.numel() - 1
    H, P, N = x.shape[2], x.shape[3], B.shape[3]
    shape = make_shape(x, B, chunk_size)
    if initial_states is not None:
        _need(initial_states, "initial_states", torch.float32)
        if tuple(initial_states.shape) != (ndoc, H, P, N):
            raise ValueError("initial_states must be [n_docs, H, P, N]")
    if y is None:
        y = torch.empty_like(x)
    if final_states is None and return_final_states:
        final_states = torch.empty((ndoc, H, P, N), dtype=torch.float32, device=x.device)
    nbytes = ssd_fwd_varlen_workspace_size(shape, ndoc)
    if workspace is None or workspace.numel() < nbytes:
        workspace = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=x.device)
    check(lib().ssd_fwd_varlen(ctypes.byref(shape), _p(x), _p(dt), _p(A), _p(B), _p(C), _p(D),
                               _p(cu_dev), ctypes.c_int64(ndoc), _p(initial_states), _p(y),
                               _p(final_states), _p(workspace), ctypes.c_size_t(nbytes),
                               _stream(stream)), "ssd_fwd_varlen")
    return (y, final_states) if return_final_states else y


def ssd_fwd_varlen_check(shape: ShapeT, n_docs: int, workspace, stream=None):
    """Status of the last ssd_fwd_varlen on `workspace` (waits for the stream): raises
    SSDError with SSD_ERR_INVALID_ARG for malformed cu_seqlens, SSD_ERR_TIMEOUT when a
    bounded wait gave up."""
    nbytes = ssd_fwd_varlen_workspace_size(shape, n_docs)
    check(lib().ssd_fwd_varlen_check(ctypes.byref(shape), ctypes.c_int64(n_docs), _p(workspace),
                                     ctypes.c_size_t(nbytes), _stream(stream)), "ssd_fwd_varlen_check")


def ssd_fwd_check(shape: ShapeT, workspace, stream=None):
    """Device-side status of the last ssd_fwd on `workspace` (waits for the stream);
    raises SSDError with SSD_ERR_TIMEOUT when the fused kernel's bounded waits gave up."""
    nbytes = ssd_fwd_workspace_size(shape)
    check(lib().ssd_fwd_check(ctypes.byref(shape), _p(workspace), ctypes.c_size_t(nbytes),
                              _stream(stream)), "ssd_fwd_check")


def ssd_fwd_host(x, dt, A, B, C, D=None, chunk_size: int = 256, initial_states=None,
                 y=None, final_states=None, device_workspace=None, stream=None):
    """ssd_fwd on host (CPU, ideally pinned) tensors; synchronous. Returns (y, final_states)."""
    for t, n in ((x, "x"), (dt, "dt"), (A, "A"), (B, "B"), (C, "C")):
        _need(t, n, device=False)
    shape = make_shape(x, B, chunk_size)
    if y is None:
        y = torch.empty_like(x)
    n = ctypes.c_size_t(0)
    check(lib().ssd_fwd_host_workspace_size(ctypes.byref(shape), ctypes.byref(n)),
          "ssd_fwd_host_workspace_size")
    if device_workspace is None or device_workspace.numel() < n.value:
        device_workspace = torch.empty(max(int(n.value), 1), dtype=torch.uint8, device="cuda")
    check(lib().ssd_fwd_host(ctypes.byref(shape), _p(x), _p(dt), _p(A), _p(B), _p(C), _p(D),
                             _p(initial_states), _p(y), _p(final_states), _p(device_workspace),
                             ctypes.c_size_t(n.value), _stream(stream)), "ssd_fwd_host")
    return y, final_states


def ssd_step(x, dt, A, B, C, D, state, y=None, stream=None):
    """Recurrent form from `state` (updated in place) for the tokens in x; returns y.

    x [b,T,H,P] (or [b,H,P] for one token), dt [b,T,H] (or [b,H]), B/C [b,T,G,N]
    (or [b,G,N]), state [b,H,P,N] fp32. y has x's shape and dtype.
    """
    one = x.dim() == 3
    if one:
        x, dt, B, C = x.unsqueeze(1), dt.unsqueeze(1), B.unsqueeze(1), C.unsqueeze(1)
    _need(x, "x")
    _need(dt, "dt", torch.float32)
    _need(A, "A", torch.float32)
    _need(B, "B", x.dtype)
    _need(C, "C", x.dtype)
    _need(state, "state", torch.float32)
    if D is not None:
        _need(D, "D", torch.float32)
    shape = make_shape(x, B, 0)
    if y is None:
        y = torch.empty_like(x)
    elif one:
        y = y.unsqueeze(1)
    check(lib().ssd_step(ctypes.byref(shape), _p(x), _p(dt), _p(A), _p(B), _p(C), _p(D),
                         _p(state), _p(y), _stream(stream)), "ssd_step")
    return y.squeeze(1) if one else y


def ssd_gated_rmsnorm(y, z, weight, group_size: int | None = None, eps: float = 1e-5, out=None,
                      stream=None):
    """out = RMSNorm over channel groups of (y * SiLU(z)), times weight (Knowl 6).

    y, z [b, T, H, P] (same dtype), weight [H * P] fp32; group_size defaults to H * P.
    """
    _need(y, "y")
    _need(z, "z", y.dtype)
    _need(weight, "weight", torch.float32)
    b, T, H, P = y.shape
    if y.dtype not in _DT:
        raise TypeError(f"y must be float32 or bfloat16, got {y.dtype}")
    shape = ShapeT(b, T, H, P, 1, 1, 64, _DT[y.dtype], 0)
    if out is None:
        out = torch.empty_like(y)
    gs = H * P if group_size is None else int(group_size)
    check(lib().ssd_gated_rmsnorm(ctypes.byref(shape), _p(y), _p(z), _p(weight), ctypes.c_int64(gs),
                                  ctypes.c_float(eps), _p(out), _stream(stream)), "ssd_gated_rmsnorm")
    return out


def ssd_cp_record_floats(shape: ShapeT) -> int:
    n = ctypes.c_size_t(0)
    check(lib().ssd_cp_record_floats(ctypes.byref(shape), ctypes.byref(n)), "ssd_cp_record_floats")
    return int(n.value)


def ssd_cp_workspace_size(shape: ShapeT) -> int:
    n = ctypes.c_size_t(0)
    check(lib().ssd_cp_workspace_size(ctypes.byref(shape), ctypes.byref(n)), "ssd_cp_workspace_size")
    return int(n.value)


def ssd_cp_begin(x, dt, A, B, chunk_size: int = 256, initial_states=None, record=None,
                 workspace=None, stream=None):
    """Sequence-parallel step 1 on this rank's slice; returns (record, workspace)."""
    _need(x, "x")
    _need(dt, "dt", torch.float32)
    _need(A, "A", torch.float32)
    _need(B, "B", x.dtype)
    if initial_states is not None:
        _need(initial_states, "initial_states", torch.float32)
    shape = make_shape(x, B, chunk_size)
    if record is None:
        record = torch.empty(max(ssd_cp_record_floats(shape), 4), dtype=torch.float32,
                             device=x.device)
    nbytes = ssd_cp_workspace_size(shape)
    if workspace is None or workspace.numel() < nbytes:
        workspace = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=x.device)
    check(lib().ssd_cp_begin(ctypes.byref(shape), _p(x), _p(dt), _p(A), _p(B), _p(initial_states),
                             _p(record), _p(workspace), ctypes.c_size_t(nbytes), _stream(stream)),
          "ssd_cp_begin")
    return record, workspace


def ssd_cp_end(x, dt, B, C, D, records, nranks: int, rank: int, workspace, chunk_size: int = 256,
               initial_states=None, y=None, final_states=None, stream=None):
    """Sequence-parallel step 3 on this rank's slice; returns (y, final_states)."""
    _need(x, "x")
    _need(dt, "dt", torch.float32)
    _need(B, "B", x.dtype)
    _need(C, "C", x.dtype)
    _need(records, "records", torch.float32)
    if D is not None:
        _need(D, "D", torch.float32)
    shape = make_shape(x, B, chunk_size)
    if y is None:
        y = torch.empty_like(x)
    if final_states is None:
        final_states = torch.empty((x.shape[0], x.shape[2], x.shape[3], B.shape[3]),
                                   dtype=torch.float32, device=x.device)
    nbytes = ssd_cp_workspace_size(shape)
    check(lib().ssd_cp_end(ctypes.byref(shape), int(nranks), int(rank), _p(records),
                           _p(initial_states), _p(x), _p(dt), _p(B), _p(C), _p(D), _p(y),
                           _p(final_states), _p(workspace), ctypes.c_size_t(nbytes),
                           _stream(stream)), "ssd_cp_end")
    return y, final_states


def _cp_exchange(record, world: int, group=None):
    """All ranks' records, gathered in rank order (one collective)."""
    import torch.distributed as dist
    out = torch.empty(world * record.numel(), dtype=record.dtype, device=record.device)
    dist.all_gather_into_tensor(out, record, group=group)
    return out


def ssd_fwd_cp(x, dt, A, B, C, D=None, chunk_size: int = 256, initial_states=None,
               return_final_states: bool = False, group=None):
    """Context-parallel SSD forward over the ranks of `group` (torch.distributed).

    Every rank passes its own contiguous slice of the sequence (x [b, T_r, H, P],
    dt, B, C likewise), rank order being sequence order; initial_states is read on
    rank 0 only. Returns this slice's y (and the state after the slice, which on
    the last rank is the sequence's final state).
    """
    import torch.distributed as dist
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    init = initial_states if rank == 0 else None
    record, ws = ssd_cp_begin(x, dt, A, B, chunk_size, initial_states=init)
    records = _cp_exchange(record, world, group)
    y, fin = ssd_cp_end(x, dt, B, C, D, records, world, rank, ws, chunk_size, initial_states=init)
    return (y, fin) if return_final_states else y


def ssd_chunk_cumsum(dt, A, chunk_size, shape: ShapeT, cs=None, stream=None):
    nc = -(-shape.seqlen // chunk_size)
    if cs is None:
        cs = torch.empty((shape.batch, shape.nheads, nc, chunk_size), dtype=torch.float32,
                         device=dt.device)
    check(lib().ssd_chunk_cumsum(ctypes.byref(shape), _p(dt), _p(A), _p(cs), _stream(stream)),
          "ssd_chunk_cumsum")
    return cs


def ssd_chunk_state(x, dt, B, cs, shape: ShapeT, states=None, stream=None):
    nc = cs.shape[2]
    if states is None:
        states = torch.empty((shape.batch, nc, shape.nheads, shape.headdim, shape.dstate),
                             dtype=torch.float32, device=x.device)
    check(lib().ssd_chunk_state(ctypes.byref(shape), _p(x), _p(dt), _p(B), _p(cs), _p(states),
                                _stream(stream)), "ssd_chunk_state")
    return states


def ssd_state_passing(states, cs, shape: ShapeT, initial_states=None, entry_states=None,
                      final_states=None, stream=None):
    if entry_states is None:
        entry_states = torch.empty_like(states)
    if final_states is None:
        final_states = torch.empty((shape.batch, shape.nheads, shape.headdim, shape.dstate),
                                   dtype=torch.float32, device=states.device)
    check(lib().ssd_state_passing(ctypes.byref(shape), _p(states), _p(cs), _p(initial_states),
                                  _p(entry_states), _p(final_states), _stream(stream)),
          "ssd_state_passing")
    return entry_states, final_states


def ssd_chunk_scan(x, dt, B, C, D, cs, entry_states, shape: ShapeT, y=None, stream=None):
    if y is None:
        y = torch.empty_like(x)
    check(lib().ssd_chunk_scan(ctypes.byref(shape), _p(x), _p(dt), _p(B), _p(C), _p(D), _p(cs),
                               _p(entry_states), _p(y), _stream(stream)), "ssd_chunk_scan")
    return y
