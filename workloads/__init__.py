"""Seeded synthetic inputs for single-token GQA decode over a packed ragged KV cache.

This module holds the input recipe only: shapes, value distributions, draw order and
the bf16 cast.  It contains none of the method's arithmetic (no attention, no scores,
no quantisation), so both the CUDA path and the fp64 oracle can be fed from it
without sharing any of the computation they are compared on.

Layout produced (what the library consumes):
  q           [B, Hq, D]      Hq = Hkv * G, query head h = kvh * G + g
  k, v        [Hkv, T, D]     T = sum_b L_b, sequence b occupies tokens cu_seqlens[b] .. cu_seqlens[b+1]
  cu_seqlens  [B + 1] int32   prefix sum of the sequence lengths

Draw order for a given seed.  ``SeedSequence(seed).spawn(1 + 2*Hkv)`` gives independent
numpy PCG64 streams: stream 0 draws, in this order,
  1. ragged lengths (only for workloads with a length range),
  2. the outlier channels of K (only for the "outlier" distribution): ``n_outlier`` distinct
     channels, the same for every head and sequence,
  3. q, as one [B, Hq, D] float32 standard-normal draw ([B, M, Hq, D] with M > 1 query tokens);
stream 1 + kvh draws k[kvh] as one [T, D] float32 standard-normal draw; stream 1 + Hkv + kvh
draws v[kvh] as one [T, D] float32 standard-normal draw followed (outlier distribution only)
by one [T] LogNormal(0, 1) draw of per-token magnitudes s_t, V[t] = N(0,1)^D * s_t.
The "outlier" distribution multiplies the chosen K channels by ``outlier_gain`` (x20).
bf16 tensors are the round-to-nearest-even cast of the float32 draws (torch ``.to``).
"""
from __future__ import annotations

import concurrent.futures
import dataclasses
import math
import os
from typing import Optional, Sequence

import numpy as np
import torch

__all__ = ["Workload", "Batch", "CONFIGS", "config", "generate"]


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic decode workload.

    ``lengths`` fixes every sequence length; otherwise ``length_range`` = (lo, hi) draws
    B lengths log-uniformly, L_b = round(exp(U[ln lo, ln hi])).
    """

    name: str
    B: int
    Hkv: int
    G: int
    D: int
    kv_dtype: str  # "f32" or "bf16" (the cache as the caller holds it before any quantisation)
    dist: str  # "normal" or "outlier"
    lengths: Optional[Sequence[int]] = None
    length_range: Optional[tuple] = None
    n_outlier: int = 4
    outlier_gain: float = 20.0
    # what the method does on this workload
    scheme: Optional[str] = None  # None (no INT8), "A" or "B"
    oam: bool = False
    beta: float = 1.0
    eps: float = 1e-6
    keep_num: int = 1  # keep ceil(L_b * keep_num / keep_den) tokens per (sequence, KV head)
    keep_den: int = 8
    n_splits: int = 0  # 0 = equal-work split over all SMs; >0 forces that many CTAs
    select_on_codes: bool = False  # the cache is quantised beforehand; OAM scores its INT8 K codes
    q_quant: Optional[str] = None  # None, "token" or "tensor": the attention's q.k runs on INT8 query codes
    seed: Optional[int] = None  # the draw's seed when it is not the workload's number
    M: int = 1  # query tokens per sequence and step (speculative decode: 1 + draft tokens)
    blocks: bool = False  # OAM keeps whole 64-token blocks (ranked by their best token)
    calibrated: bool = False  # the per-tensor scales are given (calibrated once) instead of computed

    @property
    def Hq(self) -> int:
        return self.Hkv * self.G

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The seeded workloads.  Seed = workload number.
CONFIGS = {
    1: Workload("tiny_dense_f32_L256", B=1, Hkv=1, G=4, D=64, kv_dtype="f32", dist="normal",
                lengths=(256,), n_splits=4),
    2: Workload("bf16_gqa_B8_L32K", B=8, Hkv=8, G=8, D=128, kv_dtype="bf16", dist="normal",
                lengths=(32768,) * 8),
    3: Workload("ragged_bf16_B16_L512-128K", B=16, Hkv=8, G=8, D=128, kv_dtype="bf16",
                dist="normal", length_range=(512, 131072)),
    4: Workload("int8_B8_L128K", B=8, Hkv=8, G=8, D=128, kv_dtype="bf16", dist="outlier",
                lengths=(131072,) * 8, scheme="A"),
    5: Workload("oam_int8A_B4_L32K-128K", B=4, Hkv=8, G=8, D=128, kv_dtype="bf16",
                dist="outlier", length_range=(32768, 131072), scheme="A", oam=True),
    6: Workload("oam_on_int8cache_A_B4_L32K-128K", B=4, Hkv=8, G=8, D=128, kv_dtype="bf16",
                dist="outlier", length_range=(32768, 131072), scheme="A", oam=True, select_on_codes=True),
    # workload 5 with INT8 query codes, drawn from workload 5's seed: the same batch, so the
    # two decode stages compare directly
    7: Workload("oam_int8A_qcodes_B4_L32K-128K", B=4, Hkv=8, G=8, D=128, kv_dtype="bf16",
                dist="outlier", length_range=(32768, 131072), scheme="A", oam=True, q_quant="token", seed=5),
    # workload 4 with two query tokens per sequence (one draft token): 16 columns per KV head
    8: Workload("spec_M2_int8_B8_L128K", B=8, Hkv=8, G=8, D=128, kv_dtype="bf16", dist="outlier",
                lengths=(131072,) * 8, scheme="A", M=2, seed=4),
    # workload 6 with block-granular selection: whole 64-token blocks kept, read as contiguous tiles
    9: Workload("oam_blocks_on_int8cache_A_B4_L32K-128K", B=4, Hkv=8, G=8, D=128, kv_dtype="bf16",
                dist="outlier", length_range=(32768, 131072), scheme="A", oam=True, select_on_codes=True,
                blocks=True, seed=6),
    # workload 4's cache with four query tokens (three draft tokens): 32 columns per KV head, two
    # CTAs per split range
    10: Workload("spec_M4_int8_B8_L128K", B=8, Hkv=8, G=8, D=128, kv_dtype="bf16", dist="outlier",
                 lengths=(131072,) * 8, scheme="A", M=4, seed=4),
    # the INT8 scheme table on workload 4's batch: scheme B (per-tensor K), the per-tensor Q/K/V
    # baseline (scheme B with one query scale) and scheme A with query codes per (sequence, head)
    11: Workload("int8B_B8_L128K", B=8, Hkv=8, G=8, D=128, kv_dtype="bf16", dist="outlier",
                 lengths=(131072,) * 8, scheme="B", seed=4),
    12: Workload("int8_qkv_per_tensor_B8_L128K", B=8, Hkv=8, G=8, D=128, kv_dtype="bf16", dist="outlier",
                 lengths=(131072,) * 8, scheme="B", q_quant="tensor", seed=4),
    13: Workload("int8A_qcodes_B8_L128K", B=8, Hkv=8, G=8, D=128, kv_dtype="bf16", dist="outlier",
                 lengths=(131072,) * 8, scheme="A", q_quant="token", seed=4),
    # the ragged batch of workload 3 (its seed, so the same 16 log-uniform lengths in [512, 128K]:
    # the lengths are the first draw) over workload 4's INT8 scheme-A cache distribution
    14: Workload("ragged_int8A_B16_L512-128K", B=16, Hkv=8, G=8, D=128, kv_dtype="bf16", dist="outlier",
                 length_range=(512, 131072), scheme="A", seed=3),
    # workload 5 (its seed: the same batch) with the V scale calibrated: one pass writes every code
    15: Workload("oam_int8A_calibrated_B4_L32K-128K", B=4, Hkv=8, G=8, D=128, kv_dtype="bf16",
                 dist="outlier", length_range=(32768, 131072), scheme="A", oam=True, calibrated=True, seed=5),
}


def config(n: int, **overrides) -> Workload:
    """Workload ``n`` (1..15), optionally with fields replaced (e.g. shorter lengths for tests)."""
    return CONFIGS[n].with_(**overrides) if overrides else CONFIGS[n]


@dataclasses.dataclass
class Batch:
    """Host tensors of one workload instance (CPU, contiguous)."""

    wl: Workload
    seed: int
    lengths: np.ndarray  # int64 [B]
    cu_seqlens: torch.Tensor  # int32 [B+1]
    q: torch.Tensor  # [B, Hq, D] (M = 1) or [B, M, Hq, D], float32 or bfloat16
    k: torch.Tensor  # [Hkv, T, D] float32 or bfloat16
    v: torch.Tensor  # [Hkv, T, D]
    outlier_channels: Optional[np.ndarray]

    @property
    def T(self) -> int:
        return int(self.cu_seqlens[-1])

    def row(self, b: int, kvh: int):
        """(q [G, D], k [L_b, D], v [L_b, D]) of sequence b, KV head kvh as float32 numpy arrays."""
        G = self.wl.G
        s, e = int(self.cu_seqlens[b]), int(self.cu_seqlens[b + 1])
        q = self.q[b, kvh * G:(kvh + 1) * G].float().numpy()
        return q, self.k[kvh, s:e].float().numpy(), self.v[kvh, s:e].float().numpy()


def draw_lengths(wl: Workload, rng: np.random.Generator) -> np.ndarray:
    if wl.lengths is not None:
        if len(wl.lengths) != wl.B:
            raise ValueError("lengths must have B entries")
        return np.asarray(wl.lengths, dtype=np.int64)
    lo, hi = wl.length_range
    u = rng.uniform(math.log(lo), math.log(hi), size=wl.B)
    return np.rint(np.exp(u)).astype(np.int64)


def _cast(x: np.ndarray, dtype: str) -> torch.Tensor:
    t = torch.from_numpy(x)
    return t if dtype == "f32" else t.to(torch.bfloat16)  # round-to-nearest-even


def generate(wl: Workload, seed: Optional[int] = None) -> Batch:
    """Draw one instance of ``wl`` (see the module docstring for the exact recipe)."""
    if seed is None:
        seed = wl.seed if wl.seed is not None else next((n for n, c in CONFIGS.items() if c.name == wl.name), 0)
    streams = np.random.SeedSequence(seed).spawn(1 + 2 * wl.Hkv)
    rng = np.random.default_rng(streams[0])
    lengths = draw_lengths(wl, rng)
    if (lengths < 1).any():
        raise ValueError("every sequence needs at least one token")
    cu = np.zeros(wl.B + 1, dtype=np.int64)
    np.cumsum(lengths, out=cu[1:])
    T = int(cu[-1])
    outl = None
    if wl.dist == "outlier":
        outl = np.sort(rng.choice(wl.D, size=wl.n_outlier, replace=False))
    elif wl.dist != "normal":
        raise ValueError(f"unknown distribution {wl.dist}")
    qshape = (wl.B, wl.Hq, wl.D) if wl.M == 1 else (wl.B, wl.M, wl.Hq, wl.D)
    q = _cast(rng.standard_normal(qshape, dtype=np.float32),
              "f32" if wl.kv_dtype == "f32" else "bf16")
    tdt = torch.float32 if wl.kv_dtype == "f32" else torch.bfloat16
    k = torch.empty((wl.Hkv, T, wl.D), dtype=tdt)
    v = torch.empty((wl.Hkv, T, wl.D), dtype=tdt)

    def draw(job):
        which, h = job
        r = np.random.default_rng(streams[1 + h + (wl.Hkv if which == "v" else 0)])
        buf = np.empty((T, wl.D), dtype=np.float32)
        r.standard_normal(dtype=np.float32, out=buf)
        if which == "k" and outl is not None:
            buf[:, outl] *= np.float32(wl.outlier_gain)
        if which == "v" and wl.dist == "outlier":
            buf *= r.lognormal(0.0, 1.0, size=T).astype(np.float32)[:, None]
        (k if which == "k" else v)[h].copy_(torch.from_numpy(buf))

    jobs = [("k", h) for h in range(wl.Hkv)] + [("v", h) for h in range(wl.Hkv)]
    workers = max(1, min(len(jobs), os.cpu_count() or 1, 8))
    with concurrent.futures.ThreadPoolExecutor(workers) as ex:
        list(ex.map(draw, jobs))
    return Batch(wl=wl, seed=seed, lengths=lengths,
                 cu_seqlens=torch.from_numpy(cu.astype(np.int32)), q=q, k=k, v=v,
                 outlier_channels=outl)
