"""Seeded synthetic inputs for the SSD layer core, shared by tests and benchmark.

This module holds no arithmetic of the method: it only draws random numbers
and rounds them to the storage dtype.  Both the CUDA path and the float64
oracle consume the arrays it returns (the oracle reads the exact float64 value
of every stored bf16/fp32 element).

Recipe (value distributions of the workloads the method is benchmarked on):

- x, B, C, dt_raw ~ N(0, 1)
- dt_bias = log(expm1(U[1e-3, 1e-1]))   (so softplus(dt_bias) ~ U[1e-3, 1e-1])
- A = -U[1, 16]
- D ~ N(0, 1)
- decode state ~ N(0, 0.1^2)

Streams: numpy ``default_rng`` seeded with a tuple so that any batch slice can
be regenerated on its own (needed to check a few sequences of a very large
batch against the oracle):

- per-head parameters: ``default_rng([seed, 0])`` draws dt_bias, A, D;
- batch element b of a prefill: ``default_rng([seed, 1, b])`` draws x, dt_raw,
  B, C in that order;
- batch element b of a decode state: ``default_rng([seed, 2, b])``;
- decode step t: ``default_rng([seed, 3, t])`` draws x, dt_raw, B, C for the
  whole batch.

Everything is drawn in float64, then rounded to the storage dtype (fp32: IEEE
round-to-nearest-even; bf16: via fp32, then round-to-nearest-even on the top
16 bits).  bf16 arrays are returned as ``uint16`` bit patterns.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

F32 = "f32"
BF16 = "bf16"


# --------------------------------------------------------------------------
# dtype helpers
# --------------------------------------------------------------------------
def to_storage(a64: np.ndarray, dtype: str) -> np.ndarray:
    """Round float64 values to the storage dtype (float32 array or bf16 bits)."""
    f32 = np.asarray(a64, dtype=np.float64).astype(np.float32)
    if dtype == F32:
        return f32
    if dtype == BF16:
        u = f32.view(np.uint32)
        bias = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
        return ((u + bias) >> np.uint32(16)).astype(np.uint16)
    raise ValueError(f"unknown dtype {dtype!r}")


def to_f64(a: np.ndarray) -> np.ndarray:
    """Exact float64 value of a storage array (float32, float64 or bf16 bits)."""
    if a.dtype == np.uint16:
        return (a.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)
    return a.astype(np.float64)


def storage_dtype_of(a: np.ndarray) -> str:
    if a.dtype == np.uint16:
        return BF16
    if a.dtype == np.float32:
        return F32
    raise ValueError(f"not a storage array: {a.dtype}")


# --------------------------------------------------------------------------
# draws
# --------------------------------------------------------------------------
def draw_head_params(nheads: int, seed: int) -> dict:
    """dt_bias, A, D per head, rounded to fp32 (the API takes them in fp32)."""
    rng = np.random.default_rng([seed, 0])
    dt_bias = np.log(np.expm1(rng.uniform(1e-3, 1e-1, nheads)))
    A = -rng.uniform(1.0, 16.0, nheads)
    D = rng.standard_normal(nheads)
    return {"dt_bias": to_storage(dt_bias, F32), "A": to_storage(A, F32), "D": to_storage(D, F32)}


def draw_prefill_batch(b: int, seqlen: int, nheads: int, headdim: int, dstate: int,
                       ngroups: int, seed: int, dtype: str) -> dict:
    """x [L,H,P], dt_raw [L,H], B [L,G,N], C [L,G,N] of batch element b."""
    rng = np.random.default_rng([seed, 1, b])
    x = rng.standard_normal((seqlen, nheads, headdim))
    dt_raw = rng.standard_normal((seqlen, nheads))
    Bm = rng.standard_normal((seqlen, ngroups, dstate))
    Cm = rng.standard_normal((seqlen, ngroups, dstate))
    return {k: to_storage(v, dtype) for k, v in (("x", x), ("dt_raw", dt_raw), ("B", Bm), ("C", Cm))}


def draw_decode_state(b: int, nheads: int, headdim: int, dstate: int, seed: int,
                      dtype: str, std: float = 0.1) -> np.ndarray:
    rng = np.random.default_rng([seed, 2, b])
    return to_storage(rng.normal(0.0, std, (nheads, dstate, headdim)), dtype)


def draw_decode_step(t: int, batch: int, nheads: int, headdim: int, dstate: int,
                     ngroups: int, seed: int, dtype: str) -> dict:
    """x [b,H,P], dt_raw [b,H], B [b,G,N], C [b,G,N] of decode step t."""
    rng = np.random.default_rng([seed, 3, t])
    x = rng.standard_normal((batch, nheads, headdim))
    dt_raw = rng.standard_normal((batch, nheads))
    Bm = rng.standard_normal((batch, ngroups, dstate))
    Cm = rng.standard_normal((batch, ngroups, dstate))
    return {k: to_storage(v, dtype) for k, v in (("x", x), ("dt_raw", dt_raw), ("B", Bm), ("C", Cm))}


def draw_mimo_step(t: int, batch: int, nheads: int, headdim: int, dstate: int,
                   ngroups: int, rank: int, seed: int, dtype: str) -> dict:
    """x [b,H,R,P], dt_raw [b,H], B [b,G,R,N], C [b,G,R,N] of a rank-R decode step t."""
    rng = np.random.default_rng([seed, 4, t])
    x = rng.standard_normal((batch, nheads, rank, headdim))
    dt_raw = rng.standard_normal((batch, nheads))
    Bm = rng.standard_normal((batch, ngroups, rank, dstate))
    Cm = rng.standard_normal((batch, ngroups, rank, dstate))
    return {k: to_storage(v, dtype) for k, v in (("x", x), ("dt_raw", dt_raw), ("B", Bm), ("C", Cm))}


def draw_output_grads(batch: int, seqlen: int, nheads: int, headdim: int, dstate: int, seed: int,
                      dtype: str, state_dtype: str) -> dict:
    """Seeds of a backward pass: dy [b,L,H,P] (unit normal) and dfinal [b,H,N,P]
    (normal, std 0.1, like the states)."""
    rng = np.random.default_rng([seed, 5])
    dy = rng.standard_normal((batch, seqlen, nheads, headdim))
    dfinal = 0.1 * rng.standard_normal((batch, nheads, dstate, headdim))
    return {"dy": to_storage(dy, dtype), "dfinal": to_storage(dfinal, state_dtype)}


def draw_mamba3_extras(batch: int, seqlen: int, nheads: int, ngroups: int, dstate: int, seed: int) -> dict:
    """Mamba-3 prefill inputs beyond Mamba-2's: the trapezoid's mix lam [b,L,H]
    ~ U[0, 1] and the rotation angle per step and state pair theta [b,L,G,N/2]
    ~ U[-0.5, 0.5] rad, both fp32."""
    rng = np.random.default_rng([seed, 6])
    lam = rng.uniform(0.0, 1.0, (batch, seqlen, nheads))
    theta = rng.uniform(-0.5, 0.5, (batch, seqlen, ngroups, dstate // 2))
    return {"lam": to_storage(lam, F32), "theta": to_storage(theta, F32)}


def prefill_inputs(batch: int, seqlen: int, nheads: int, headdim: int, dstate: int,
                   ngroups: int, seed: int, dtype: str, batches=None) -> dict:
    """Whole prefill input set (or the listed batch elements, in that order)."""
    idx = list(range(batch)) if batches is None else list(batches)
    parts = [draw_prefill_batch(b, seqlen, nheads, headdim, dstate, ngroups, seed, dtype) for b in idx]
    out = {k: np.stack([p[k] for p in parts]) for k in ("x", "dt_raw", "B", "C")}
    out.update(draw_head_params(nheads, seed))
    return out


# --------------------------------------------------------------------------
# the workloads
# --------------------------------------------------------------------------
@dataclass(frozen=True)
class PrefillShape:
    batch: int
    seqlen: int
    nheads: int
    headdim: int
    dstate: int
    ngroups: int
    chunk: int
    dtype: str
    seed: int
    name: str = ""

    @property
    def tokens(self) -> int:
        return self.batch * self.seqlen

    def inputs(self, batches=None) -> dict:
        return prefill_inputs(self.batch, self.seqlen, self.nheads, self.headdim, self.dstate,
                              self.ngroups, self.seed, self.dtype, batches)


@dataclass(frozen=True)
class DecodeShape:
    batch: int
    nheads: int
    headdim: int
    dstate: int
    ngroups: int
    steps: int
    io_dtype: str
    state_dtype: str
    seed: int
    name: str = ""


# tiny fp32 prefill: batch 1, seqlen 256, 4 heads, P=64, N=16, 1 group, chunk 64
TINY_FP32 = PrefillShape(1, 256, 4, 64, 16, 1, 64, F32, 0, "tiny_fp32_b1_L256_H4_P64_N16_G1_Q64")
# Mamba-2 1.3B-shaped layer: d_inner 4096 = 64 heads x 64, N=128, 1 group, chunk 256
MAMBA2_1P3B = PrefillShape(4, 2048, 64, 64, 128, 1, 256, BF16, 1,
                           "mamba2_1.3b_layer_b4_L2048_H64_P64_N128_G1_Q256")


def long_sequence_sweep() -> list:
    """Long sequences x state sizes, batch 1, 64 heads, P=64, 8 groups, chunk 256."""
    return [PrefillShape(1, L, 64, 64, N, 8, 256, BF16, 2, f"long_b1_L{L}_H64_P64_N{N}_G8_Q256")
            for L in (4096, 16384, 65536) for N in (64, 128, 256)]


# decode: batch 256, 128 heads, P=64, N=128, 8 groups, fp32 state, 64 steps
DECODE_B256 = DecodeShape(256, 128, 64, 128, 8, 64, BF16, F32, 3, "decode_b256_H128_P64_N128_G8_f32state")
# prefill batch 512 x 1024 tokens, then 32 decode steps on a bf16 state
HANDOFF_PREFILL = PrefillShape(512, 1024, 128, 64, 128, 8, 256, BF16, 4,
                               "handoff_prefill_b512_L1024_H128_P64_N128_G8_Q256")
HANDOFF_DECODE = DecodeShape(512, 128, 64, 128, 8, 32, BF16, BF16, 4,
                             "handoff_decode_b512_H128_P64_N128_G8_bf16state")
