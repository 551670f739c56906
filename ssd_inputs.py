"""Seeded synthetic inputs and workload shapes for the SSD layer forward.

This module is shared by the tests, the smoke check and the benchmark. It holds
no arithmetic of the method itself: it only draws random numbers and casts them
to the stored dtypes, so that the oracle and the CUDA path see the same values.

Shapes follow the Mamba-2 layer: x[b,T,H,P], dt[b,T,H], A[H], B/C[b,T,G,N],
D[H], states[b,H,P,N] (state expansion N, head dim P, G groups of heads sharing
B and C; "Transformers are SSMs", Knowl 7, multi-input / grouped-input patterns).

Value distributions (one recipe for every workload):
  x ~ N(0,1); B, C ~ N(0,1)/sqrt(N); A_h = -exp(U(0, ln 16)); D ~ N(0,1);
  dt = clamp(softplus(N(0,1) - 3), 1e-3, 0.1) for the tiny fp32 case and
  dt = exp(U(ln 1e-3, ln 0.1)) (log-uniform) for the bf16 workloads;
  initial_states ~ N(0, 0.1^2) where a workload carries state in.
Draws are float64 from numpy's PCG64 in the fixed order A, D, dt, x, B, C,
initial_states, then cast (bf16 by round-to-nearest-even through torch).
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np
import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    seqlen: int
    nheads: int
    headdim: int
    ngroups: int
    dstate: int
    chunk_size: int
    dtype: str            # "f32" or "bf16": storage type of x, B, C and y
    dt_dist: str          # "softplus" or "loguniform"
    initial_states: bool = False

    @property
    def tokens(self) -> int:
        return self.batch * self.seqlen

    def shape_dict(self) -> dict:
        return dict(batch=self.batch, seqlen=self.seqlen, nheads=self.nheads,
                    headdim=self.headdim, ngroups=self.ngroups, dstate=self.dstate,
                    chunk_size=self.chunk_size)


TINY_FP32 = Workload("tiny_fp32_b1_T256_H2_P16_N16_Q64", 1, 256, 2, 16, 1, 16, 64,
                     "f32", "softplus")
MAMBA2_27B_LAYER = Workload("mamba2_2.7b_layer_b8_T2048_H80_P64_N128_G1_Q256", 8, 2048,
                            80, 64, 1, 128, 256, "bf16", "loguniform")


def seqlen_sweep() -> list[Workload]:
    out = []
    for T in (512, 1024, 2048, 4096, 8192, 16384):
        out.append(Workload(f"seqlen_sweep_T{T}_b{32768 // T}_H32_P64_N128", 32768 // T, T,
                            32, 64, 1, 128, 256, "bf16", "loguniform"))
    return out


def dstate_sweep() -> list[Workload]:
    out = []
    for N in (16, 32, 64, 128, 256):
        out.append(Workload(f"dstate_sweep_N{N}_b4_T4096_H64_P64", 4, 4096, 64, 64, 1, N,
                            256, "bf16", "loguniform"))
    return out


LONG_CONTEXT = Workload("long_context_b1_T65536_H32_P64_N128_G8_state_carry", 1, 65536, 32,
                        64, 8, 128, 256, "bf16", "loguniform", initial_states=True)


# one decoding step of the same layer for 128 sequences: the recurrent form on the
# carried state [128, 80, 64, 128] fp32 (335 MB, larger than L2)
DECODE_STEP_27B = Workload("decode_step_mamba2_2.7b_b128_H80_P64_N128_G1", 128, 1, 80, 64, 1,
                           128, 256, "bf16", "loguniform", initial_states=True)


# packed documents (variable length): 16 documents of mixed lengths, 16384 tokens in
# all (the 2.7B layer's b*T), at the 2.7B head shape, in batch row 0
PACKED_DOC_LENGTHS = (2048, 512, 1024, 256, 3072, 768, 1536, 128, 2048, 640, 1408, 896, 1152,
                      384, 320, 192)
PACKED_DOCS_27B = Workload("packed_docs_mamba2_2.7b_16docs_T16384_H80_P64_N128_G1", 1,
                           sum(PACKED_DOC_LENGTHS), 80, 64, 1, 128, 256, "bf16", "loguniform")


def packed_cu_seqlens(lengths=PACKED_DOC_LENGTHS) -> list[int]:
    cu = [0]
    for n in lengths:
        cu.append(cu[-1] + n)
    return cu


def all_workloads() -> list[Workload]:
    return [TINY_FP32, MAMBA2_27B_LAYER, *seqlen_sweep(), *dstate_sweep(), LONG_CONTEXT]


def _softplus(v: np.ndarray) -> np.ndarray:
    return np.logaddexp(0.0, v)


def make_inputs(batch: int, seqlen: int, nheads: int, headdim: int, ngroups: int,
                dstate: int, dtype: str = "bf16", dt_dist: str = "loguniform",
                initial_states: bool = False, with_D: bool = True, seed: int = 0,
                **_ignored) -> dict:
    """Draw one seeded input set; returns CPU torch tensors in their stored dtype.

    x, B, C are float32 or bfloat16 (``dtype``); dt, A, D, initial_states are
    float32. ``D`` is None when ``with_D`` is false, ``initial_states`` is None
    unless requested.
    """
    rng = np.random.Generator(np.random.PCG64(seed))
    H, P, N, G = nheads, headdim, dstate, ngroups
    A = -np.exp(rng.uniform(0.0, math.log(16.0), size=(H,)))
    D = rng.standard_normal(size=(H,))
    if dt_dist == "softplus":
        dt = np.clip(_softplus(rng.standard_normal(size=(batch, seqlen, H)) - 3.0), 1e-3, 0.1)
    elif dt_dist == "loguniform":
        dt = np.exp(rng.uniform(math.log(1e-3), math.log(0.1), size=(batch, seqlen, H)))
    else:
        raise ValueError(f"unknown dt distribution {dt_dist!r}")
    x = rng.standard_normal(size=(batch, seqlen, H, P))
    B = rng.standard_normal(size=(batch, seqlen, G, N)) / math.sqrt(N)
    C = rng.standard_normal(size=(batch, seqlen, G, N)) / math.sqrt(N)
    init = rng.standard_normal(size=(batch, H, P, N)) * 0.1 if initial_states else None

    tdt = {"f32": torch.float32, "bf16": torch.bfloat16}[dtype]

    def cast(a, t):
        return torch.from_numpy(np.ascontiguousarray(a)).to(t).contiguous()

    return dict(
        x=cast(x, tdt), dt=cast(dt, torch.float32), A=cast(A, torch.float32),
        B=cast(B, tdt), C=cast(C, tdt),
        D=cast(D, torch.float32) if with_D else None,
        initial_states=cast(init, torch.float32) if init is not None else None,
    )


def workload_inputs(w: Workload, seed: int = 0, **overrides) -> dict:
    kw = dict(w.shape_dict(), dtype=w.dtype, dt_dist=w.dt_dist,
              initial_states=w.initial_states, seed=seed)
    kw.update(overrides)
    return make_inputs(**kw)
