"""Host-only checks of the C ABI: the library loads, exports every declared
symbol, and rejects bad arguments before launching anything.

No test here computes on a GPU. On a machine without CUDA the calls use
placeholder addresses that the library never dereferences (every call is
expected to fail validation); on a machine with CUDA they use real device
buffers, so even a validation bug could not touch foreign memory.
"""
import ctypes
import os
import re

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    from structured_state_space_fwd_b200 import build
    build.build()
    from structured_state_space_fwd_b200 import _lib
    return _lib


def declared_functions():
    src = open(os.path.join(ROOT, "include", "ssd.h")).read()
    return sorted(set(re.findall(r"SSD_API\s+[\w\s\*]+?\b(ssd_\w+)\s*\(", src)))


def test_exports_every_declared_symbol(L):
    names = declared_functions()
    assert len(names) >= 11
    lib = L.lib()
    for n in names:
        assert hasattr(lib, n), n


def test_status_strings(L):
    for code, name in enumerate(["SSD_OK", "SSD_ERR_INVALID_ARG", "SSD_ERR_UNSUPPORTED",
                                 "SSD_ERR_CUDA", "SSD_ERR_TIMEOUT"]):
        assert L.status_string(code) == name
    assert L.lib().ssd_version() >= 100


def shape(**kw):
    from structured_state_space_fwd_b200._lib import ShapeT
    d = dict(batch=2, seqlen=300, nheads=4, headdim=64, ngroups=2, dstate=64, chunk_size=128,
             dtype=1, reserved=0)
    d.update(kw)
    return ShapeT(**d)


def ws_size(L, s):
    n = ctypes.c_size_t(0)
    st = L.lib().ssd_fwd_workspace_size(ctypes.byref(s), ctypes.byref(n))
    return st, n.value


@pytest.mark.parametrize("kw,code", [
    (dict(nheads=6, ngroups=4), 1),        # G does not divide H
    (dict(headdim=0), 1),
    (dict(dstate=-1), 1),
    (dict(batch=-1), 1),
    (dict(dtype=7), 1),
    (dict(reserved=3), 1),
    (dict(chunk_size=0), 1),
    (dict(chunk_size=96), 2),              # not a supported chunk size
    (dict(chunk_size=512), 2),
    (dict(headdim=512), 2),
    (dict(dstate=300), 2),
])
def test_shape_rejections(L, kw, code):
    st, _ = ws_size(L, shape(**kw))
    assert st == code


def test_workspace_size_monotone(L):
    st, a = ws_size(L, shape(seqlen=256))
    assert st == 0 and a > 0
    st, b = ws_size(L, shape(seqlen=512))
    assert st == 0 and b > a
    st, z = ws_size(L, shape(seqlen=0))
    assert st == 0 and z == 0


class Bufs:
    """Real device buffers on a CUDA machine, otherwise placeholder addresses."""

    def __init__(self, s):
        self.real = torch.cuda.is_available()
        b, T, H, P, G, N = s.batch, s.seqlen, s.nheads, s.headdim, s.ngroups, s.dstate
        es = 2 if s.dtype == 1 else 4
        sizes = dict(x=b * T * H * P * es, dt=b * T * H * 4, A=H * 4, B=b * T * G * N * es,
                     C=b * T * G * N * es, D=H * 4, init=b * H * P * N * 4, y=b * T * H * P * es,
                     final=b * H * P * N * 4)
        _, ws = ws_size(lib_mod(), s)
        sizes["ws"] = ws
        self.t = {}
        self.addr = {}
        base = 1 << 40
        for k, n in sizes.items():
            if self.real:
                self.t[k] = torch.empty(max(n, 16), dtype=torch.uint8, device="cuda")
                self.addr[k] = self.t[k].data_ptr()
            else:
                self.addr[k] = base
                base += ((n + 4095) // 4096 + 1) * 4096
        self.ws_bytes = ws

    def p(self, k):
        return ctypes.c_void_p(self.addr[k]) if k else None


def lib_mod():
    from structured_state_space_fwd_b200 import _lib
    return _lib


def call_fwd(L, s, bufs, **over):
    names = ["x", "dt", "A", "B", "C", "D", "init", "y", "final", "ws"]
    args = {k: bufs.p(k) for k in names}
    ws_bytes = over.pop("ws_bytes", bufs.ws_bytes)
    for k, v in over.items():
        args[k] = v
    return L.lib().ssd_fwd(ctypes.byref(s), args["x"], args["dt"], args["A"], args["B"],
                           args["C"], args["D"], args["init"], args["y"], args["final"],
                           args["ws"], ctypes.c_size_t(ws_bytes), None)


def off(bufs, k, delta):
    return ctypes.c_void_p(bufs.addr[k] + delta)


@pytest.mark.parametrize("case", ["null_x", "null_y", "null_dt", "misaligned_x", "misaligned_y",
                                  "y_is_x", "y_overlaps_B", "final_is_init", "final_overlaps_y",
                                  "small_ws", "null_ws", "ws_overlaps_x", "bad_shape"])
def test_fwd_argument_rejections(L, case):
    s = shape()
    bufs = Bufs(s)
    over = {
        "null_x": dict(x=None), "null_y": dict(y=None), "null_dt": dict(dt=None),
        "misaligned_x": dict(x=off(bufs, "x", 2)), "misaligned_y": dict(y=off(bufs, "y", 8)),
        "y_is_x": dict(y=bufs.p("x")), "y_overlaps_B": dict(y=off(bufs, "B", 16)),
        "final_is_init": dict(final=bufs.p("init")),
        "final_overlaps_y": dict(final=bufs.p("y")),
        "small_ws": dict(ws_bytes=bufs.ws_bytes - 1), "null_ws": dict(ws=None),
        "ws_overlaps_x": dict(ws=bufs.p("x")),
        "bad_shape": None,
    }[case]
    if over is None:
        st = call_fwd(L, shape(nheads=5, ngroups=2), bufs)
    else:
        st = call_fwd(L, s, bufs, **over)
    assert st == 1


def test_step_entry_rejections(L):
    s = shape()
    bufs = Bufs(s)
    lib = L.lib()
    assert lib.ssd_chunk_cumsum(ctypes.byref(s), None, bufs.p("A"), bufs.p("ws"), None) == 1
    assert lib.ssd_chunk_cumsum(ctypes.byref(s), bufs.p("dt"), bufs.p("A"), bufs.p("dt"), None) == 1
    assert lib.ssd_chunk_state(ctypes.byref(s), bufs.p("x"), bufs.p("dt"), bufs.p("B"),
                               bufs.p("ws"), bufs.p("x"), None) == 1
    assert lib.ssd_state_passing(ctypes.byref(s), bufs.p("ws"), bufs.p("ws"), None, None,
                                 None, None) == 1
    assert lib.ssd_chunk_scan(ctypes.byref(s), bufs.p("x"), bufs.p("dt"), bufs.p("B"),
                              bufs.p("C"), None, bufs.p("ws"), bufs.p("ws"), bufs.p("x"),
                              None) == 1
    bad = shape(chunk_size=100)
    assert lib.ssd_chunk_cumsum(ctypes.byref(bad), bufs.p("dt"), bufs.p("A"), bufs.p("ws"),
                                None) == 2


def test_binding_fails_loudly_without_library(tmp_path, monkeypatch):
    from structured_state_space_fwd_b200 import _lib
    monkeypatch.setattr(_lib, "_lib", None)
    monkeypatch.setattr(_lib, "lib_path", str(tmp_path / "missing.so"))
    with pytest.raises(ImportError):
        _lib.lib()


def test_recurrent_step_rejections(L):
    """ssd_step: state is in/out, so it may overlap neither an input nor y; the other
    rules are ssd_fwd's. chunk_size is not used by the recurrent form."""
    s = shape(seqlen=1)
    bufs = Bufs(s)
    lib = L.lib()

    def call(**over):
        names = ["x", "dt", "A", "B", "C", "D", "init", "y"]
        a = {k: bufs.p(k) for k in names}
        a.update(over)
        sh = over.pop("shape", s) if "shape" in over else s
        return lib.ssd_step(ctypes.byref(sh), a["x"], a["dt"], a["A"], a["B"], a["C"], a["D"],
                            a["init"], a["y"], None)
    assert call(init=None) == 1                       # state required
    assert call(x=None) == 1
    assert call(init=bufs.p("x")) == 1                # state overlaps x
    assert call(init=off(bufs, "B", 16)) == 1         # state overlaps B
    assert call(y=bufs.p("init")) == 1                # y overlaps state
    assert call(y=bufs.p("C")) == 1                   # y overlaps an input
    assert call(init=off(bufs, "init", 4)) == 1       # state misaligned
    assert call(shape=shape(seqlen=1, nheads=5, ngroups=2)) == 1
    assert call(shape=shape(seqlen=1, dstate=300)) == 2
    assert call(shape=shape(seqlen=1, dtype=5)) == 1


def test_context_parallel_sizes_and_rejections(L):
    """ssd_cp_*: record size is the documented layout; bad ranks, missing or
    overlapping buffers and a short workspace are rejected before any launch."""
    s = shape()
    lib = L.lib()
    n = ctypes.c_size_t(0)
    assert lib.ssd_cp_record_floats(ctypes.byref(s), ctypes.byref(n)) == 0
    bhpn, bh = s.batch * s.nheads * s.headdim * s.dstate, s.batch * s.nheads
    assert n.value == (bhpn + bh + 3) // 4 * 4
    rec_floats = n.value
    ws = ctypes.c_size_t(0)
    assert lib.ssd_cp_workspace_size(ctypes.byref(s), ctypes.byref(ws)) == 0 and ws.value > 0
    bufs = Bufs(s)
    # records of 4 ranks and one cp workspace, as placeholder or real device buffers
    if bufs.real:
        recs = torch.empty(4 * rec_floats, dtype=torch.float32, device="cuda")
        cpws = torch.empty(ws.value, dtype=torch.uint8, device="cuda")
        rp, wp = recs.data_ptr(), cpws.data_ptr()
    else:
        rp, wp = 1 << 44, 1 << 45
    R = ctypes.c_void_p(rp)
    WS = ctypes.c_void_p(wp)
    p = bufs.p

    def begin(record=R, x=None, ws_bytes=ws.value, workspace=WS):
        return lib.ssd_cp_begin(ctypes.byref(s), x or p("x"), p("dt"), p("A"), p("B"), None,
                                record, workspace, ctypes.c_size_t(ws_bytes), None)

    def end(nranks=4, rank=1, records=R, y=None, final=None, ws_bytes=ws.value):
        return lib.ssd_cp_end(ctypes.byref(s), nranks, rank, records, None, p("x"), p("dt"),
                              p("B"), p("C"), p("D"), y or p("y"), final, WS,
                              ctypes.c_size_t(ws_bytes), None)
    assert begin(record=None) == 1
    assert begin(record=p("x")) == 1                      # record overlaps x
    assert begin(ws_bytes=ws.value - 1) == 1
    assert begin(workspace=R) == 1                        # workspace overlaps the record
    assert end(rank=4) == 1 and end(rank=-1) == 1 and end(nranks=0, rank=0) == 1
    assert end(records=None) == 1
    assert end(y=R) == 1                                  # y overlaps the records
    assert end(final=p("x")) == 1
    assert end(ws_bytes=0) == 1


def test_gated_rmsnorm_rejections(L):
    s = shape()
    bufs = Bufs(s)
    lib = L.lib()

    def call(y="x", z="C", w="A", gs=256, eps=1e-5, out="y", sh=None):
        return lib.ssd_gated_rmsnorm(ctypes.byref(sh or s), bufs.p(y) if y else None,
                                     bufs.p(z) if z else None, bufs.p(w) if w else None,
                                     ctypes.c_int64(gs), ctypes.c_float(eps),
                                     bufs.p(out) if out else None, None)
    # H * P = 256 channels in this shape
    assert call(gs=0) == 1 and call(gs=100) == 1 and call(gs=512) == 1
    assert call(eps=-1.0) == 1 and call(eps=float("nan")) == 1 and call(eps=float("inf")) == 1
    assert call(out=None) == 1 and call(w=None) == 1
    assert call(out="x") == 1                           # out overlaps y
    assert call(sh=shape(dtype=9)) == 1


def test_binding_declares_every_entry_point(L):
    """The Python binding gives every C entry point of include/ssd.h its signature."""
    missing = [n for n in declared_functions() if n not in L._SIGS]
    assert not missing, missing
