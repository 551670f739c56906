#!/usr/bin/env python
"""Benchmark of the SSD layer forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = one ssd_fwd call (every step of the block-decomposition algorithm)
on the Mamba-2 2.7B layer shape: batch 8, T 2048, 80 heads, head dim 64,
state 128, 1 group, chunk 256, bf16 x/B/C/y, fp32 dt/A/D, final states
returned. Inputs are seeded synthetic data resident in HBM; their working set
(x and y alone are 168 MB each) exceeds the 126 MB L2, so no flush is needed
between steps. Under torchrun every rank runs its own copy of the workload
(weak scaling, no collective on the data path) and rank 0 prints one JSON
line with the whole-job throughput, timed on the device as the max over ranks.

--impl reference times the fp64 CPU oracle on the host cores instead (a
bounded sample of the same workload per step); it is a deliberately slow
program, reported for context.
"""
from __future__ import annotations

import argparse
import json
import os
import shutil
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import ssd_inputs as W  # noqa: E402

WORKLOAD = W.MAMBA2_27B_LAYER
METRIC = "SSD fwd Mtokens/s & TFLOP/s at 2.7B layer shape; % of bf16/HBM roofline"
UNIT = "Mtokens/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# dram__bytes_read.sum + dram__bytes_write.sum per launch of the dominant kernel, from
# one ncu capture of this workload (profiles/); None until captured for the current kernel
TRAFFIC = {"fused": 359387648}
KERNEL_NAMES = {"fused": "ssd_fused_kernel",
                "segmented": "segment_state_kernel + segment_scan_kernel + ssd_fused_kernel",
                "steps": "chunk_cumsum + chunk_state_tc + state_passing + chunk_scan_tc",
                "simt": "chunk_cumsum + chunk_state + state_passing + chunk_scan"}


# ------------------------------------------------------------------ counts
def alg_counts(w: W.Workload, with_final=True, with_init=False):
    """Algorithmic FLOPs and bytes of one forward (tensor-core flops, causal half).

    F = b T [ G (Q+1) N + H ((Q+1) P + 4 N P + 2 P N / Q) ]
    Bytes = b T H P (s_x + s_y) + 4 b T H + 2 b T G N s_bc + 8 H + 4 b H P N per state tensor
    """
    b, T, H, P, G, N, Q = w.batch, w.seqlen, w.nheads, w.headdim, w.ngroups, w.dstate, w.chunk_size
    s = 2 if w.dtype == "bf16" else 4
    F = b * T * (G * (Q + 1) * N + H * ((Q + 1) * P + 4 * N * P + 2 * P * N / Q))
    by = b * T * H * P * 2 * s + 4 * b * T * H + 2 * b * T * G * N * s + 8 * H
    by += 4 * b * H * P * N * (int(with_final) + int(with_init))
    return float(F), float(by)


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as fh:
            d = json.load(fh)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ------------------------------------------------------------------ clocks
class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.proc = None
        self.path = None
        smi = shutil.which("nvidia-smi")
        if smi is None:
            return
        try:
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            ident = uuid if uuid.startswith("GPU-") else f"GPU-{uuid}"
        except Exception:
            ident = str(device_index)
        self.path = f"/tmp/ssd_bench_clocks_{os.getpid()}.csv"
        self.fh = open(self.path, "w")
        self.proc = subprocess.Popen([smi, "-i", ident, f"--query-gpu={self.FIELDS}",
                                      "--format=csv,noheader,nounits", "-lms", "100"],
                                     stdout=self.fh, stderr=subprocess.DEVNULL)
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.fh.close()
        rows = []
        with open(self.path) as fh:
            for line in fh:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 8:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        sm = [float(r[0]) for r in rows if r[0].replace(".", "").isdigit()]
        mx = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[4 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons, "samples": len(rows)}


# ------------------------------------------------------------------ helpers
def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def max_over_ranks(v: float, world: int, device) -> float:
    if world == 1:
        return v
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def oracle_sample(w: W.Workload, budget_s: float, inputs64=None):
    """Prepare a bounded sample of the workload for the fp64 oracle: the first
    n heads of batch row 0 (one group, so heads slice freely), n chosen so one
    run takes about budget_s on the host cores. Returns (run, tokens_equiv, desc)."""
    import oracle
    inp = inputs64 if inputs64 is not None else W.workload_inputs(w)
    x = inp["x"][:1].double().numpy()
    dt = inp["dt"][:1].double().numpy()
    A = inp["A"].double().numpy()
    B = inp["B"][:1].double().numpy()
    C = inp["C"][:1].double().numpy()
    D = inp["D"].double().numpy() if inp["D"] is not None else None
    assert w.ngroups == 1

    def make(nh):
        xs = np.ascontiguousarray(x[:, :, :nh])
        dts = np.ascontiguousarray(dt[:, :, :nh])
        As = np.ascontiguousarray(A[:nh])
        Ds = np.ascontiguousarray(D[:nh]) if D is not None else None
        return lambda: oracle.recurrence(xs, dts, As, B, C, Ds)

    threads = oracle.max_threads()
    nh = min(w.nheads, max(1, threads))
    t0 = time.perf_counter()
    make(nh)()
    t1 = time.perf_counter() - t0
    scale = budget_s / max(t1, 1e-6)
    nh2 = int(min(w.nheads, max(1, nh * scale)))
    run = make(nh2)
    tokens_equiv = w.seqlen * nh2 / w.nheads   # token-heads of one batch row / heads per token
    desc = (f"batch row 0, heads 0..{nh2 - 1} of {w.nheads} (T={w.seqlen}); "
            f"{nh2 * w.seqlen} token-heads = {tokens_equiv:.0f} token-equivalents per run")
    return run, tokens_equiv, desc, threads


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as fh:
            for line in fh:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def oracle_single_thread(w: W.Workload, inp, budget_s: float = 3.0):
    """The oracle's recurrence on one thread (one head of batch row 0, repeated for
    about budget_s), in the bench unit: what one host core sustains."""
    import oracle
    x = np.ascontiguousarray(inp["x"][:1, :, :1].double().numpy())
    dt = np.ascontiguousarray(inp["dt"][:1, :, :1].double().numpy())
    A = np.ascontiguousarray(inp["A"][:1].double().numpy())
    B = inp["B"][:1].double().numpy()
    C = inp["C"][:1].double().numpy()
    D = np.ascontiguousarray(inp["D"][:1].double().numpy()) if inp["D"] is not None else None
    reps, t0 = 0, time.perf_counter()
    while time.perf_counter() - t0 < budget_s:
        oracle.recurrence(x, dt, A, B, C, D)
        reps += 1
    el = time.perf_counter() - t0
    tok = w.seqlen / w.nheads * reps     # one head of T tokens = T / H token-equivalents
    return {"value": tok / el / 1e6, "unit": UNIT, "threads": 1,
            "sample": f"batch row 0, head 0 (T={w.seqlen}), {reps} runs in {el:.1f} s"}


# ------------------------------------------------------------------ sweeps
def measure_workload(ssd, dev, stream, w: W.Workload, steps, warmup, seed=0):
    """One ssd_fwd step of workload w (final states returned), timed with CUDA events:
    throughput, path, and the fraction of the HBM roofline the whole step reaches
    (algorithmic bytes of the step / step time)."""
    inp = W.workload_inputs(w, seed=seed)
    d = {k: (v.to(dev) if v is not None else None) for k, v in inp.items()}
    shp = ssd.make_shape(d["x"], d["B"], w.chunk_size)
    ws = torch.empty(max(ssd.ssd_fwd_workspace_size(shp), 1), dtype=torch.uint8, device=dev)
    y = torch.empty_like(d["x"])
    fin = torch.empty((w.batch, w.nheads, w.headdim, w.dstate), dtype=torch.float32, device=dev)

    def step():
        ssd.ssd_fwd(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], chunk_size=w.chunk_size,
                    initial_states=d["initial_states"], y=y, final_states=fin,
                    return_final_states=True, workspace=ws, stream=stream)
    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    ssd.ssd_fwd_check(shp, ws, stream=stream)
    ms = e0.elapsed_time(e1) / steps
    path, nk = ssd.ssd_fwd_plan(shp)
    _, by = alg_counts(w, with_final=True, with_init=w.initial_states)
    pk, pk_kind = peaks()
    ach = by / (ms / 1e3) / 1e9
    return {"workload": w.name, "value": w.tokens / (ms / 1e3) / 1e6, "unit": UNIT, "ms_per_step": ms,
            "steps": steps, "warmup": warmup, "path": path, "gpu_launches_per_step": nk,
            "roofline": {"kernel": KERNEL_NAMES[path] + " (whole step)", "bound": "hbm",
                         "achieved": ach, "peak": pk["hbm_gbs"], "unit": "GB/s",
                         "frac": ach / pk["hbm_gbs"], "alg_bytes_per_step": by, "traffic": None,
                         "peak_source": pk_kind}}


def measure_sweeps(ssd, dev, stream, seed=0):
    """The sequence-length sweep (32768 tokens at every T), the state-size sweep and the
    long-context workload, each as its own row."""
    rows = {}
    for w in W.seqlen_sweep():
        rows[f"seqlen_T{w.seqlen}"] = measure_workload(ssd, dev, stream, w, 20, 3, seed=seed)
    for w in W.dstate_sweep():
        rows[f"dstate_N{w.dstate}"] = measure_workload(ssd, dev, stream, w, 20, 3, seed=seed)
    rows["long_context"] = measure_workload(ssd, dev, stream, W.LONG_CONTEXT, 20, 3, seed=seed)
    return rows


# ------------------------------------------------------------------ reference arm
def run_reference(args):
    world, rank, local = dist_env()
    if rank != 0:
        return 0
    w = WORKLOAD
    per_step_budget = max(0.05, min(10.0, 150.0 / max(1, args.steps + args.warmup)))
    run, tok, desc, threads = oracle_sample(w, per_step_budget)
    for _ in range(args.warmup):
        run()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        run()
    el = time.perf_counter() - t0
    value = tok * args.steps / el / 1e6
    cpu = {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
           "sample": f"fp64 sequential recurrence (C, OpenMP over heads) per step: {desc}"}
    line = {"metric": METRIC, "value": value, "unit": UNIT, "impl": "reference",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": el / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w.name, **w.shape_dict(), "input_dtype": w.dtype},
            "cpu_baseline": cpu,
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ decoding step
DECODE = W.DECODE_STEP_27B
DECODE_METRIC = "SSD decode step (recurrent form) Mtokens/s at 2.7B layer shape, 128 sequences"
# dram__bytes_read.sum + dram__bytes_write.sum of one ssd_step_kernel launch on this
# workload, from one ncu capture (profiles/); None once the kernel changes
DECODE_TRAFFIC = 614955264
# ncu DRAM bytes (read + write) of one gate launch, one group of 5120 channels
# (profiles/gated_rmsnorm_kernel_2.7b_layer.md); the rest of out is still in L2
GATE_TRAFFIC = 446482176


def decode_bytes(w: W.Workload) -> float:
    """Algorithmic bytes of one decoding step: the fp32 state read and written
    (8 b H P N) plus the token's x, y, dt, B, C and A, D."""
    b, T, H, P, G, N = w.batch, w.seqlen, w.nheads, w.headdim, w.ngroups, w.dstate
    s = 2 if w.dtype == "bf16" else 4
    return 8.0 * b * H * P * N + b * T * (H * P * 2 * s + 4 * H + 2 * G * N * s) + 8.0 * H


def measure_decode(ssd, dev, stream, steps, warmup, rank, with_cpu):
    """Decoding steps on the 2.7B layer shape for 128 sequences: each step runs
    ssd_step once, updating a carried fp32 state (335 MB) in place. Two state sets
    are alternated so that a step never finds its state in L2 from the step before."""
    w = DECODE
    inp = W.workload_inputs(w, seed=rank)
    d = {k: (v.to(dev) if v is not None else None) for k, v in inp.items()}
    states = [d["initial_states"].clone(), d["initial_states"].clone()]
    y = torch.empty_like(d["x"])

    def step(i):
        ssd.ssd_step(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], states[i & 1], y=y,
                     stream=stream)
    for i in range(warmup):
        step(i)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(steps):
        step(i)
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    by = decode_bytes(w)
    pk, pk_kind = peaks()
    achieved = by / (ms / 1e3) / 1e9
    out = {"metric": DECODE_METRIC, "value": w.tokens / (ms / 1e3) / 1e6, "unit": UNIT,
           "ms_per_step": ms, "steps": steps, "warmup": warmup, "dtype": "bf16",
           "config": {"workload": w.name, **w.shape_dict(), "input_dtype": w.dtype,
                      "state_mb": 4.0 * w.batch * w.nheads * w.headdim * w.dstate / 1e6,
                      "l2": "two 335 MB state sets alternated, no flush"},
           "roofline": {"kernel": "ssd_step_kernel", "bound": "hbm", "achieved": achieved,
                        "peak": pk["hbm_gbs"], "unit": "GB/s", "frac": achieved / pk["hbm_gbs"],
                        "traffic": DECODE_TRAFFIC, "alg_bytes_per_launch": by,
                        "peak_source": pk_kind + " (burst copy, MEASURED_PEAKS hbm_gbs)"},
           "gpu_launches": steps}
    if with_cpu:
        import oracle
        f64 = {k: (v.double().numpy() if v is not None else None) for k, v in inp.items()}
        t0 = time.perf_counter()
        reps = 0
        while time.perf_counter() - t0 < 3.0 or reps == 0:
            oracle.recurrence(**f64)
            reps += 1
        el = time.perf_counter() - t0
        out["cpu_baseline"] = {"value": w.tokens * reps / el / 1e6, "unit": UNIT,
                               "cores": oracle.max_threads(), "kind": "oracle",
                               "sample": f"fp64 recurrence, the whole step (128 sequences x 80 "
                                         f"heads, one token); {reps} runs in {el:.1f} s"}
    return out


# ------------------------------------------------------------------ gate + norm
GATE_METRIC = "SSD gate + RMSNorm (y * SiLU(z), one group of 5120 channels) at 2.7B layer shape"


def measure_gate(ssd, dev, stream, steps, warmup, seed=0):
    """ssd_gated_rmsnorm on the layer output of the 2.7B shape: y, z bf16
    [8, 2048, 80, 64] (168 MB each, larger than L2), weight [5120], one norm group
    per token. Algorithmic bytes: y and z read, out written, weight read."""
    w = WORKLOAD
    g = torch.Generator(device="cpu").manual_seed(seed)
    shp = (w.batch, w.seqlen, w.nheads, w.headdim)
    y = torch.randn(shp, generator=g).to(torch.bfloat16).to(dev)
    z = (torch.randn(shp, generator=g) * 2.0).to(torch.bfloat16).to(dev)
    wt = (torch.rand(w.nheads * w.headdim, generator=g) + 0.5).to(dev)
    out = torch.empty_like(y)

    def step():
        ssd.ssd_gated_rmsnorm(y, z, wt, group_size=w.nheads * w.headdim, out=out, stream=stream)
    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    by = 3.0 * y.numel() * 2 + 4.0 * wt.numel()
    pk, pk_kind = peaks()
    return {"metric": GATE_METRIC, "value": w.tokens / (ms / 1e3) / 1e6, "unit": UNIT,
            "ms_per_step": ms, "steps": steps, "warmup": warmup, "dtype": "bf16",
            "config": {"workload": "gate_rmsnorm_b8_T2048_C5120_group5120", "batch": w.batch,
                       "seqlen": w.seqlen, "channels": w.nheads * w.headdim,
                       "group_size": w.nheads * w.headdim,
                       "l2": "y and z 168 MB each, larger than L2, no flush"},
            "roofline": {"kernel": "gated_rmsnorm_pipelined_kernel", "bound": "hbm",
                         "achieved": by / (ms / 1e3) / 1e9, "peak": pk["hbm_gbs"], "unit": "GB/s",
                         "frac": by / (ms / 1e3) / 1e9 / pk["hbm_gbs"], "traffic": GATE_TRAFFIC,
                         "alg_bytes_per_launch": by,
                         "peak_source": pk_kind + " (burst copy, MEASURED_PEAKS hbm_gbs)"},
            "gpu_launches": steps}


# ------------------------------------------------------------------ packed documents
VARLEN_METRIC = ("SSD fwd Mtokens/s on packed variable-length documents (16 docs, 16384 tokens, "
                 "2.7B head shape)")


def measure_varlen(ssd, dev, stream, steps, warmup, seed=0):
    """ssd_fwd_varlen on 16 packed documents of mixed lengths (16384 tokens, H80 P64
    N128 G1 bf16), per-document final states returned. Algorithmic bytes: x, y, dt,
    B, C of the pack and one final state per document."""
    w = W.PACKED_DOCS_27B
    cu = W.packed_cu_seqlens()
    inp = W.workload_inputs(w, seed=seed)
    d = {k: (v.to(dev) if v is not None else None) for k, v in inp.items()}
    ndoc = len(cu) - 1
    y = torch.empty_like(d["x"])
    fin = torch.empty((ndoc, w.nheads, w.headdim, w.dstate), dtype=torch.float32, device=dev)
    cu_dev = torch.tensor(cu, dtype=torch.int32, device=dev)
    shp = ssd.make_shape(d["x"], d["B"], w.chunk_size)
    ws = torch.empty(ssd.ssd_fwd_varlen_workspace_size(shp, ndoc), dtype=torch.uint8, device=dev)

    def step():
        ssd.ssd_fwd_varlen(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], cu_seqlens=cu_dev,
                           chunk_size=w.chunk_size, return_final_states=True, y=y,
                           final_states=fin, workspace=ws, stream=stream)
    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    _, by = alg_counts(w, with_final=False)
    by += 4.0 * ndoc * w.nheads * w.headdim * w.dstate
    pk, pk_kind = peaks()
    return {"metric": VARLEN_METRIC, "value": w.tokens / (ms / 1e3) / 1e6, "unit": UNIT,
            "ms_per_step": ms, "steps": steps, "warmup": warmup, "dtype": "bf16",
            "config": {"workload": w.name, "documents": ndoc, "doc_lengths": list(W.PACKED_DOC_LENGTHS),
                       **w.shape_dict(), "input_dtype": w.dtype,
                       "dispatch": "one single-pass launch over the pack, a unit per (document, "
                                   "head pair), longest documents first"},
            "roofline": {"kernel": "ssd_fused_kernel (packed documents) + document ordering", "bound": "hbm",
                         "achieved": by / (ms / 1e3) / 1e9, "peak": pk["hbm_gbs"], "unit": "GB/s",
                         "frac": by / (ms / 1e3) / 1e9 / pk["hbm_gbs"], "traffic": None,
                         "alg_bytes_per_step": by,
                         "peak_source": pk_kind + " (burst copy, MEASURED_PEAKS hbm_gbs)"},
            "gpu_launches": steps * 2}   # document ordering + the single-pass kernel


# ------------------------------------------------------------------ forward + gate, fused
GATED_METRIC = ("SSD fwd + gate + RMSNorm (per-head groups of 64) Mtokens/s at 2.7B layer shape, "
                "gate in the forward's stores (fuse)")


def measure_fwd_gated(ssd, dev, stream, steps, warmup, seed=0):
    """ssd_fwd_gated at the 2.7B layer shape with norm groups of 64 channels (one head),
    both ways: fuse (the single-pass kernel gates and normalises each row before storing
    it, so y never reaches HBM and needs no buffer) and separate (y through the
    workspace, then the gate kernel)."""
    w = WORKLOAD
    inp = W.workload_inputs(w, seed=seed)
    d = {k: (v.to(dev) if v is not None else None) for k, v in inp.items()}
    g = torch.Generator().manual_seed(seed + 11)
    z = (torch.randn(w.batch, w.seqlen, w.nheads, w.headdim, generator=g) * 2.0).to(torch.bfloat16).to(dev)
    nw = (torch.rand(w.nheads * w.headdim, generator=g) + 0.5).float().to(dev)
    gs = 64
    shp = ssd.make_shape(d["x"], d["B"], w.chunk_size)
    out = torch.empty_like(d["x"])
    fin = torch.empty((w.batch, w.nheads, w.headdim, w.dstate), dtype=torch.float32, device=dev)
    wss = {f: torch.empty(max(ssd.ssd_fwd_gated_workspace_size(shp, gs, f), 1), dtype=torch.uint8, device=dev)
           for f in (True, False)}

    def run(f):
        ssd.ssd_fwd_gated(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], z=z, norm_weight=nw, group_size=gs,
                          eps=1e-5, fuse=f, chunk_size=w.chunk_size, out=out, final_states=fin,
                          return_final_states=True, workspace=wss[f], stream=stream)

    def timed(f):
        for _ in range(warmup):
            run(f)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(steps):
            run(f)
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / steps
    ms_f = timed(True)
    ms_s = timed(False)
    _, by = alg_counts(w, with_final=True)
    by += 2.0 * w.batch * w.seqlen * w.nheads * w.headdim + 4.0 * w.nheads * w.headdim   # z, weight
    pk, pk_kind = peaks()
    ach = by / (ms_f / 1e3) / 1e9
    ybytes = 2.0 * w.batch * w.seqlen * w.nheads * w.headdim
    return {"metric": GATED_METRIC, "value": w.tokens / (ms_f / 1e3) / 1e6, "unit": UNIT,
            "ms_per_step": ms_f, "steps": steps, "warmup": warmup, "dtype": "bf16",
            "config": {"workload": w.name, **w.shape_dict(), "group_size": gs, "eps": 1e-5,
                       "plan": ssd.ssd_fwd_plan(shp)[0]},
            "separate_ms_per_step": ms_s, "fused_minus_separate_ms": ms_f - ms_s,
            "y_round_trip_bytes_saved": 2.0 * ybytes, "y_buffer_bytes_saved": ybytes,
            "roofline": {"kernel": "ssd_fused_kernel (gated stores)", "bound": "hbm", "achieved": ach,
                         "peak": pk["hbm_gbs"], "unit": "GB/s", "frac": ach / pk["hbm_gbs"],
                         "alg_bytes_per_step": by, "traffic": None, "peak_source": pk_kind},
            "gpu_launches": steps}


# ------------------------------------------------------------------ context parallelism
CP = W.LONG_CONTEXT
CP_METRIC = ("SSD fwd Mtokens/s, long context (b1 T65536 H32 P64 N128 G8) split over the "
             "ranks along the sequence")


def cp_slice_bytes(w: W.Workload, T_slice: int, nranks: int) -> float:
    """Algorithmic bytes of one rank's slice: its x, y, dt, B, C (and A, D), the
    initial and final states, and the gathered records it reads."""
    ws = W.Workload(w.name, w.batch, T_slice, w.nheads, w.headdim, w.ngroups, w.dstate,
                    w.chunk_size, w.dtype, w.dt_dist, w.initial_states)
    _, by = alg_counts(ws, with_final=True, with_init=True)
    return by + 4.0 * nranks * w.batch * w.nheads * (w.headdim * w.dstate + 1)


def cp_setup(ssd, dev, w, nranks, rank, seed=0):
    """Inputs of rank `rank`'s slice of the long-context sequence (the whole
    sequence is drawn once with `seed`, then sliced)."""
    inp = W.workload_inputs(w, seed=seed)
    Ts = w.seqlen // nranks
    sl = slice(rank * Ts, (rank + 1) * Ts)
    d = {k: (inp[k][:, sl].contiguous().to(dev)) for k in ("x", "dt", "B", "C")}
    d.update({k: (inp[k].to(dev) if inp[k] is not None else None) for k in ("A", "D", "initial_states")})
    return d, Ts


def cp_kernels_per_step(ssd, d, w, rank):
    """Launches of one rank's ssd_cp_begin + ssd_cp_end: on the single-pass plan the
    segment-state pass and its scan, then the fold (ranks > 0), the scan from the
    entering state and the single-pass kernel over the slice's segments; otherwise
    chunk cumsum, chunk states, state passing and the slice decay, then the fold,
    state passing and the chunk scan (slices of several segments assumed)."""
    path, _ = ssd.ssd_fwd_plan(ssd.make_shape(d["x"], d["B"], w.chunk_size))
    fold = 1 if rank > 0 else 0
    return 2 + fold + 2 if path in ("fused", "segmented") else 4 + fold + 2


def measure_cp_slice(ssd, dev, stream, steps, warmup, nranks=8):
    """One rank's work in an nranks-way split of the long-context sequence, timed on
    one GPU: ssd_cp_begin, then ssd_cp_end of the last rank (which folds the most
    records) with a records buffer standing in for the all-gather's result. The
    collective itself needs several GPUs and is not in this number."""
    w = CP
    rank = nranks - 1
    d, Ts = cp_setup(ssd, dev, w, nranks, rank)
    rec, ws = ssd.ssd_cp_begin(d["x"], d["dt"], d["A"], d["B"], w.chunk_size)
    records = rec.repeat(nranks)
    y = torch.empty_like(d["x"])
    fin = torch.empty_like(d["initial_states"])

    def step():
        ssd.ssd_cp_begin(d["x"], d["dt"], d["A"], d["B"], w.chunk_size, record=rec, workspace=ws,
                         stream=stream)
        ssd.ssd_cp_end(d["x"], d["dt"], d["B"], d["C"], d["D"], records, nranks, rank, ws,
                       w.chunk_size, y=y, final_states=fin, stream=stream)
    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    by = cp_slice_bytes(w, Ts, nranks)
    pk, pk_kind = peaks()
    return {"what": f"one rank of {nranks}: ssd_cp_begin + ssd_cp_end on a {Ts}-token slice "
                    f"(rank {rank}); the all-gather of {nranks} records of "
                    f"{4 * w.batch * w.nheads * (w.headdim * w.dstate + 1) / 2**20:.2f} MiB is not timed",
            "ms_per_rank_step": ms, "slice_tokens": Ts, "workload": w.name,
            "kernels_per_rank_step": cp_kernels_per_step(ssd, d, w, rank),
            "roofline": {"bound": "hbm", "achieved": by / (ms / 1e3) / 1e9, "peak": pk["hbm_gbs"],
                         "unit": "GB/s", "frac": by / (ms / 1e3) / 1e9 / pk["hbm_gbs"],
                         "alg_bytes_per_rank_step": by, "traffic": None,
                         "peak_source": pk_kind + " (burst copy, MEASURED_PEAKS hbm_gbs)"}}


def run_cp(args):
    """--workload long_context_cp: the long-context sequence split along its length
    over the torchrun ranks (strong scaling: the sequence is fixed), one all-gather of
    the per-rank records per step (NCCL), timed on the device, max over ranks."""
    import datetime
    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    import torch.distributed as dist
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    from structured_state_space_fwd_b200 import build as _b
    _b.build()
    import structured_state_space_fwd_b200 as ssd
    w = CP
    if w.seqlen % world:
        raise SystemExit(f"seqlen {w.seqlen} does not split over {world} ranks")
    d, Ts = cp_setup(ssd, dev, w, world, rank)
    stream = torch.cuda.current_stream(dev)
    init = d["initial_states"] if rank == 0 else None
    rec, ws = ssd.ssd_cp_begin(d["x"], d["dt"], d["A"], d["B"], w.chunk_size, initial_states=init)
    records = torch.empty(world * rec.numel(), dtype=torch.float32, device=dev)
    y = torch.empty_like(d["x"])
    fin = torch.empty_like(d["initial_states"])

    def step():
        ssd.ssd_cp_begin(d["x"], d["dt"], d["A"], d["B"], w.chunk_size, initial_states=init,
                         record=rec, workspace=ws, stream=stream)
        if world > 1:
            dist.all_gather_into_tensor(records, rec)
        else:
            records.copy_(rec)
        ssd.ssd_cp_end(d["x"], d["dt"], d["B"], d["C"], d["D"], records, world, rank, ws,
                       w.chunk_size, initial_states=init, y=y, final_states=fin, stream=stream)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    barrier(world)
    clocks = ClockSampler(local)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop()
    ms = max_over_ranks(e0.elapsed_time(e1), world, dev) / args.steps
    by = cp_slice_bytes(w, Ts, world)
    pk, pk_kind = peaks()
    if rank == 0:
        line = {"metric": CP_METRIC, "value": w.tokens / (ms / 1e3) / 1e6, "unit": UNIT,
                "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
                "higher_is_better": True, "scaling": "strong", "vs_baseline": None,
                "dtype": "bf16", "data": "synthetic",
                "config": {"workload": w.name, **w.shape_dict(), "input_dtype": w.dtype,
                           "slice_tokens": Ts, "exchange": "NCCL all-gather of per-rank records"
                           if world > 1 else "none (one rank)",
                           "l2": "per-rank slice inputs 34 MB + outputs; timed back to back"},
                "roofline": {"kernel": f"rank step ({cp_kernels_per_step(ssd, d, w, rank)} kernels + all-gather)",
                             "bound": "hbm",
                             "achieved": by / (ms / 1e3) / 1e9, "peak": pk["hbm_gbs"],
                             "unit": "GB/s", "frac": by / (ms / 1e3) / 1e9 / pk["hbm_gbs"],
                             "traffic": None, "alg_bytes_per_rank_step": by,
                             "peak_source": pk_kind + " (burst copy, MEASURED_PEAKS hbm_gbs)"},
                "gpu_launches": cp_kernels_per_step(ssd, d, w, rank) * args.steps, "clocks": clk}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


# ------------------------------------------------------------------ our arm
def kernel_plan(ssd, w, d, bufs, stream):
    """The kernels of the unfused path as individually timed launches, with the
    algorithmic bytes each must move per launch."""
    b, T, H, P, G, N, Q = w.batch, w.seqlen, w.nheads, w.headdim, w.ngroups, w.dstate, w.chunk_size
    nc = -(-T // Q)
    s = 2 if w.dtype == "bf16" else 4
    shp = ssd.make_shape(d["x"], d["B"], Q)
    cs, S, entry, y, fin = bufs["cs"], bufs["S"], bufs["entry"], bufs["y"], bufs["final"]
    st_bytes = 4.0 * b * nc * H * P * N
    plan = [
        ("chunk_cumsum", lambda: ssd.ssd_chunk_cumsum(d["dt"], d["A"], Q, shp, cs=cs, stream=stream),
         4.0 * b * T * H + 4.0 * b * H * nc * Q),
        ("chunk_state", lambda: ssd.ssd_chunk_state(d["x"], d["dt"], d["B"], cs, shp, states=S,
                                                    stream=stream),
         s * b * T * H * P + s * b * T * G * N + 4.0 * b * T * H + 4.0 * b * H * nc * Q + st_bytes),
        ("state_passing", lambda: ssd.ssd_state_passing(S, cs, shp, entry_states=entry,
                                                        final_states=fin, stream=stream),
         2 * st_bytes + 4.0 * b * H * P * N + 4.0 * b * H * nc),
        ("chunk_scan", lambda: ssd.ssd_chunk_scan(d["x"], d["dt"], d["B"], d["C"], d["D"], cs, entry,
                                                  shp, y=y, stream=stream),
         2.0 * s * b * T * H * P + 2.0 * s * b * T * G * N + 4.0 * b * T * H + 4.0 * b * H * nc * Q
         + st_bytes),
    ]
    return plan


def run_ours(args):
    world, rank, local = dist_env()
    if world > 1:
        import datetime

        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    from structured_state_space_fwd_b200 import build as _b
    _b.build()
    import structured_state_space_fwd_b200 as ssd

    w = WORKLOAD
    # each rank's shard: its own batch of the workload (seeded by rank)
    inp = W.workload_inputs(w, seed=rank)
    d = {k: (v.to(dev) if v is not None else None) for k, v in inp.items()}
    b, T, H, P, G, N, Q = w.batch, w.seqlen, w.nheads, w.headdim, w.ngroups, w.dstate, w.chunk_size
    nc = -(-T // Q)
    stream = torch.cuda.current_stream(dev)
    shp = ssd.make_shape(d["x"], d["B"], Q)
    bufs = dict(y=torch.empty_like(d["x"]),
                final=torch.empty((b, H, P, N), dtype=torch.float32, device=dev),
                cs=torch.empty((b, H, nc, Q), dtype=torch.float32, device=dev),
                S=torch.empty((b, nc, H, P, N), dtype=torch.float32, device=dev),
                entry=torch.empty((b, nc, H, P, N), dtype=torch.float32, device=dev))
    ws_bytes = ssd.ssd_fwd_workspace_size(shp)
    ws = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=dev)

    def step():
        ssd.ssd_fwd(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], chunk_size=Q,
                    y=bufs["y"], final_states=bufs["final"], return_final_states=True,
                    workspace=ws, stream=stream)

    path_name, kernels_per_step = ssd.ssd_fwd_plan(shp)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()

    clocks = ClockSampler(local)
    # keep the GPU busy for ~0.5 s before the timed region so that the clock
    # samples taken around it reflect clocks under this load (untimed)
    t_soak = time.perf_counter()
    while time.perf_counter() - t_soak < args.soak_s:
        for _ in range(20):
            step()
        torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop()
    ms_total = max_over_ranks(e0.elapsed_time(e1), world, dev)
    ms_step = ms_total / args.steps
    tokens_total = w.tokens * world
    value = tokens_total * args.steps / (ms_total / 1e3) / 1e6

    F, by = alg_counts(w, with_final=True, with_init=w.initial_states)
    pk, pk_kind = peaks()
    t_roof = max(F / (pk["bf16_tflops"] * 1e12), by / (pk["hbm_gbs"] * 1e9))
    step_s = ms_step / 1e3

    # dominant kernel and its average launch duration (CUDA events on its stream)
    if path_name == "fused":
        # one kernel per step: the single-pass forward; its launch duration is the
        # timed step (which also holds the small counter memset before it)
        ktimes = {"ssd_fused_kernel": ms_step}
        dom = ("ssd_fused_kernel", None, by)
    else:
        plan = kernel_plan(ssd, w, d, bufs, stream)
        ktimes = {}
        reps = max(3, min(50, args.steps))
        for name, fn, _ in plan:
            for _ in range(2):
                fn()
            k0, k1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            k0.record(stream)
            for _ in range(reps):
                fn()
            k1.record(stream)
            torch.cuda.synchronize()
            ktimes[name] = k0.elapsed_time(k1) / reps
        dom = max(plan, key=lambda p: ktimes[p[0]])
    dom_s = ktimes[dom[0]] / 1e3
    achieved = dom[2] / dom_s / 1e9
    roofline = {"kernel": dom[0], "bound": "hbm", "achieved": achieved, "peak": pk["hbm_gbs"],
                "unit": "GB/s", "frac": achieved / pk["hbm_gbs"], "traffic": TRAFFIC.get(path_name),
                "peak_source": pk_kind + " (burst copy, MEASURED_PEAKS hbm_gbs)",
                "alg_bytes_per_launch": dom[2], "path": path_name,
                "kernel_ms": {k: round(v, 5) for k, v in ktimes.items()}}

    # end to end through the host-buffer entry point (pinned host memory)
    e2e = None
    if not args.no_e2e and not args.profile:
        hp = {k: (v.pin_memory() if v is not None else None) for k, v in inp.items()}
        hy = torch.empty_like(hp["x"]).pin_memory()
        hf = torch.empty((b, H, P, N), dtype=torch.float32).pin_memory()
        n = 0
        import ctypes
        nb = ctypes.c_size_t(0)
        ssd.lib().ssd_fwd_host_workspace_size(ctypes.byref(shp), ctypes.byref(nb))
        dws = torch.empty(int(nb.value), dtype=torch.uint8, device=dev)

        def e2e_step():
            ssd.ssd_fwd_host(hp["x"], hp["dt"], hp["A"], hp["B"], hp["C"], hp["D"], chunk_size=Q,
                             y=hy, final_states=hf, device_workspace=dws, stream=stream)
        for _ in range(2):
            e2e_step()
        ke = max(3, min(20, args.steps))
        barrier(world)
        torch.cuda.synchronize()
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        for _ in range(ke):
            e2e_step()
        a1.record(stream)
        torch.cuda.synchronize()
        barrier(world)
        ms_e2e = max_over_ranks(a0.elapsed_time(a1), world, dev) / ke
        h2d = sum(v.numel() * v.element_size() for v in hp.values() if v is not None)
        d2h = hy.numel() * hy.element_size() + hf.numel() * hf.element_size()
        # the same bytes copied alone (one pinned copy each way), for the copy engines' rate
        hx = torch.empty(int(h2d), dtype=torch.uint8).pin_memory()
        dx = torch.empty(int(h2d), dtype=torch.uint8, device=dev)
        hyb = torch.empty(int(d2h), dtype=torch.uint8).pin_memory()
        dyb = torch.empty(int(d2h), dtype=torch.uint8, device=dev)
        for _ in range(2):
            dx.copy_(hx, non_blocking=True)
            hyb.copy_(dyb, non_blocking=True)
        torch.cuda.synchronize()
        c0, c1, c2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
        c0.record(stream)
        dx.copy_(hx, non_blocking=True)
        c1.record(stream)
        hyb.copy_(dyb, non_blocking=True)
        c2.record(stream)
        torch.cuda.synchronize()
        h2d_gbs = h2d / (c0.elapsed_time(c1) / 1e3) / 1e9
        d2h_gbs = d2h / (c1.elapsed_time(c2) / 1e3) / 1e9
        del hx, dx, hyb, dyb
        e2e = {"value": w.tokens * world / (ms_e2e / 1e3) / 1e6, "unit": UNIT,
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "ms_per_step": ms_e2e, "api": "ssd_fwd_host (pinned host buffers)",
               "copy_gbs": {"h2d_alone": h2d_gbs, "d2h_alone": d2h_gbs,
                            "h2d_plus_d2h_over_step": (h2d + d2h) / (ms_e2e / 1e3) / 1e9},
               "copy_bound_ms": (h2d / h2d_gbs + d2h / d2h_gbs) / 1e6}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and not args.profile:
        run, tok, desc, threads = oracle_sample(w, 15.0, inputs64=inp)
        t0 = time.perf_counter()
        run()
        t1 = time.perf_counter() - t0
        # the sample is capped at one batch row; repeat it for about 12 s of CPU work
        reps = max(1, int(12.0 / max(t1, 1e-3)))
        t0 = time.perf_counter()
        for _ in range(reps):
            run()
        el = time.perf_counter() - t0
        cpu = {"value": tok * reps / el / 1e6, "unit": UNIT, "cores": threads, "kind": "oracle",
               "sample": f"fp64 sequential recurrence, {desc}; {reps} runs in {el:.1f} s",
               "cpu_model": cpu_model(), "single_thread": oracle_single_thread(w, inp)}

    decode = None
    cp = None
    gate = None
    varlen = None
    sweeps = None
    gated = None
    if not args.profile:
        # secondary rows, measured after the headline: a failure here is reported in
        # its own entry and does not take the headline line down with it
        def guarded(fn, *a, **k):
            try:
                return fn(*a, **k)
            except Exception as e:  # noqa: BLE001
                try:
                    torch.cuda.synchronize()
                except Exception:  # noqa: BLE001
                    pass
                return {"error": f"{type(e).__name__}: {e}"[:300]}
        decode = guarded(measure_decode, ssd, dev, stream, 200, 10, rank,
                         rank == 0 and world == 1 and not args.no_cpu_baseline)
        cp = guarded(measure_cp_slice, ssd, dev, stream, 50, 5)
        gate = guarded(measure_gate, ssd, dev, stream, 100, 5, seed=rank)
        varlen = guarded(measure_varlen, ssd, dev, stream, 20, 3, seed=rank)
        sweeps = guarded(measure_sweeps, ssd, dev, stream, seed=rank)
        gated = guarded(measure_fwd_gated, ssd, dev, stream, 50, 5, seed=rank)

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": w.name, **w.shape_dict(), "input_dtype": w.dtype,
                       "final_states": True, "per_rank_batch": b,
                       "l2": "inputs larger than L2 (x and y 168 MB each), no flush"},
            "tflops": F * world / step_s / 1e12,
            "step_roofline": {"t_roof_us": t_roof * 1e6, "t_step_us": step_s * 1e6,
                              "frac": t_roof / step_s, "alg_gflop": F / 1e9, "alg_mb": by / 1e6,
                              "peaks": pk_kind},
            "roofline": roofline,
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": kernels_per_step * args.steps,
            "clocks": clk,
            "workload_rows": sweeps,
            "next_rows": {"decode_step": decode, "context_parallel": cp, "gate_norm": gate,
                          "fwd_gate_fused": gated, "packed_docs": varlen},
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def run_decode_only(args):
    """--workload decode_step / gate_norm / long_context: that step alone, as the printed
    line (long_context: ssd_fwd on the long-context workload, the segmented path)."""
    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    from structured_state_space_fwd_b200 import build as _b
    _b.build()
    import structured_state_space_fwd_b200 as ssd
    stream = torch.cuda.current_stream(dev)
    if args.workload == "gate_norm":
        out = measure_gate(ssd, dev, stream, args.steps, args.warmup, seed=rank)
    elif args.workload == "long_context":
        out = measure_workload(ssd, dev, stream, W.LONG_CONTEXT, args.steps, args.warmup, seed=rank)
        out["metric"] = "SSD fwd Mtokens/s, long context (b1 T65536 H32 P64 N128 G8, state carry)"
    else:
        out = measure_decode(ssd, dev, stream, args.steps, args.warmup, rank,
                             world == 1 and not args.no_cpu_baseline and not args.profile)
    if rank == 0:
        out.update({"n_gpus": 1, "higher_is_better": True, "scaling": "weak",
                    "vs_baseline": None, "data": "synthetic"})
        print(json.dumps(out), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--soak-s", type=float, default=0.5,
                    help="untimed load before the timed region, for the clock samples")
    ap.add_argument("--profile", action="store_true",
                    help="warmup and timed steps only (for ncu): no e2e, no CPU baseline")
    ap.add_argument("--workload", choices=["layer", "decode_step", "gate_norm", "long_context", "long_context_cp"],
                    default="layer",
                    help="decode_step: time only the recurrent decoding step; long_context: one ssd_fwd "
                         "on the long-context workload; long_context_cp: the long-context sequence split "
                         "over the ranks (context parallel)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        return run_reference(args)
    if args.workload in ("decode_step", "gate_norm", "long_context"):
        return run_decode_only(args)
    if args.workload == "long_context_cp":
        return run_cp(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
