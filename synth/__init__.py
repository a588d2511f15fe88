"""Seeded synthetic inputs for the attention workloads.

This module is shared by the CUDA path's tests and bench and by the float64
oracle's callers. It draws random tensors and rounds them to the storage dtype.
It holds none of the attention arithmetic.

Recipe. Every (tensor, batch, head) slice has its own NumPy PCG64 stream seeded
with SeedSequence([seed, tensor_id, b, h]). A slice can therefore be
regenerated on its own, which lets the oracle rebuild only the heads it
samples. Values are iid N(0, 1) float32, multiplied by `std`. For bf16
workloads they are then rounded to the nearest bf16, ties to even, so the
GPU and the oracle receive bit-identical numbers. The oracle upcasts them
exactly to float64. For E4M3 workloads the values are divided by a static
per-tensor descale (8 std / 448, so that 8 standard deviations map to the
largest finite E4M3 value) and rounded to the nearest E4M3 value, ties to even,
saturating at +-448; the slice then holds those codes, and the real input is
code * descale (exact in float64).

Workloads (shapes from the pages' long-context regime; all synthetic, no dataset):
  c1  fp32 fwd,  B=1 H=1 N=128 d=64, non-causal
  c2  bf16 fwd+bwd, B=4 H=16 N=2048 d=64, causal, 1% of query rows x20
  c3  bf16 fwd+bwd, B=2 H=32 N=8192 d=128, causal, std 1/sqrt(2)
  c4  bf16 fwd,  B=1 H=16 N=65536 d=128, causal
  c5  bf16 fwd+bwd GQA, B=1 Hq=32 Hkv=8 N=32768 d=128, causal
  c3n bf16 fwd+bwd, c3's shape without the causal mask
  c6  bf16 fwd,  B=2 H=16 N=8192 d=256, causal
  c6b bf16 fwd+bwd, c6's shape
  f3  E4M3 fwd,  B=2 H=32 N=8192 d=128, causal, std 1/sqrt(2) (c3's shape)
  f4  E4M3 fwd,  B=1 H=16 N=65536 d=128, causal (c4's shape)
  f5  E5M2 fwd,  c3's shape
  dec decode,    B=16 Hq=32 Hkv=8, Nq=1 new query against Nk=32768 cached keys, d=128
  dec4 decode,   B=16 Hq=32 Hkv=4, Nq=4 (32 query rows a group)
  dec8 decode,   B=16 Hq=64 Hkv=8, Nq=8 (64 query rows a group)
"""
from __future__ import annotations

import concurrent.futures as _cf
import math
import os
from dataclasses import dataclass, field

import numpy as np

# tensor ids used in the per-slice seed
TID_Q, TID_K, TID_V, TID_DO, TID_SPIKE = 0, 1, 2, 3, 4


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    N: int
    d: int
    causal: bool
    dtype: str  # "f32", "bf16", "e4m3" or "e5m2"
    backward: bool
    seed: int
    std: float = 1.0
    spike_frac: float = 0.0  # fraction of query rows per (b, h) multiplied by spike_mul
    spike_mul: float = 1.0
    # oracle sampling for the large shapes: (b, hq) heads and number of query rows
    sample_heads: tuple = field(default=())
    sample_rows: int = 0

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    @property
    def group(self) -> int:
        return self.Hq // self.Hkv

    @property
    def descale(self) -> float:
        """FP8 workloads: the float32 value that multiplies every stored code
        (8 standard deviations map to the format's largest finite value)."""
        top = E5M2_MAX if self.dtype == "e5m2" else E4M3_MAX
        return float(np.float32(8.0 * self.std / top))

    def fwd_flops(self) -> float:
        f = 4.0 * self.B * self.Hq * self.N * self.N * self.d
        return f / 2 if self.causal else f

    def bwd_flops(self) -> float:
        return 2.5 * self.fwd_flops()


WORKLOADS = {
    "c1": Workload("c1", 1, 1, 1, 128, 64, False, "f32", False, 1001),
    "c2": Workload("c2", 4, 16, 16, 2048, 64, True, "bf16", True, 1002,
                   spike_frac=0.01, spike_mul=20.0),
    "c3": Workload("c3", 2, 32, 32, 8192, 128, True, "bf16", True, 1003,
                   std=1.0 / math.sqrt(2.0),
                   sample_heads=((0, 0), (0, 17), (1, 6), (1, 31)), sample_rows=256),
    "c4": Workload("c4", 1, 16, 16, 65536, 128, True, "bf16", False, 1004,
                   sample_heads=((0, 0), (0, 5), (0, 10), (0, 15)), sample_rows=256),
    "c5": Workload("c5", 1, 32, 8, 32768, 128, True, "bf16", True, 1005,
                   sample_heads=((0, 0), (0, 1), (0, 2), (0, 3),
                                 (0, 28), (0, 29), (0, 30), (0, 31)), sample_rows=256),
    "c3n": Workload("c3n", 2, 32, 32, 8192, 128, False, "bf16", True, 1008,
                    std=1.0 / math.sqrt(2.0),
                    sample_heads=((0, 0), (0, 17), (1, 6), (1, 31)), sample_rows=256),
    "c6": Workload("c6", 2, 16, 16, 8192, 256, True, "bf16", False, 1009,
                   std=1.0 / math.sqrt(2.0),
                   sample_heads=((0, 0), (0, 9), (1, 4), (1, 15)), sample_rows=256),
    "c6b": Workload("c6b", 2, 16, 16, 8192, 256, True, "bf16", True, 1012,
                    std=1.0 / math.sqrt(2.0),
                    sample_heads=((0, 0), (0, 9), (1, 4), (1, 15)), sample_rows=256),
    "f3": Workload("f3", 2, 32, 32, 8192, 128, True, "e4m3", False, 1006,
                   std=1.0 / math.sqrt(2.0),
                   sample_heads=((0, 0), (0, 17), (1, 6), (1, 31)), sample_rows=256),
    "f5": Workload("f5", 2, 32, 32, 8192, 128, True, "e5m2", False, 1011,
                   std=1.0 / math.sqrt(2.0),
                   sample_heads=((0, 0), (0, 17), (1, 6), (1, 31)), sample_rows=256),
    "f4": Workload("f4", 1, 16, 16, 65536, 128, True, "e4m3", False, 1007,
                   sample_heads=((0, 0), (0, 5), (0, 10), (0, 15)), sample_rows=256),
}

E4M3_MAX = 448.0
E5M2_MAX = 57344.0


def _round_to_fp8(x: np.ndarray, mant_bits: int, min_exp: int, top: float) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32).astype(np.float64)
    a = np.minimum(np.abs(x), top)
    with np.errstate(divide="ignore"):
        e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.maximum(e, float(min_exp))    # below the smallest normal the step stays (subnormals)
    step = np.exp2(e - mant_bits)
    r = np.minimum(np.round(a / step) * step, top)   # numpy rounds halves to even
    return (np.sign(x) * r).astype(np.float32)


def round_to_e5m2(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest E5M2 value (OCP FP8: 2 mantissa bits,
    exponent bias 15, subnormal step 2^-16), ties to even, saturating at +-57344.
    Returns float32."""
    return _round_to_fp8(x, 2, -14, E5M2_MAX)


def round_to_e4m3(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest E4M3 value (OCP FP8: 3 mantissa bits,
    exponent bias 7, subnormal step 2^-9, no infinities), ties to even,
    saturating at +-448. Returns float32."""
    x = np.ascontiguousarray(x, dtype=np.float32).astype(np.float64)
    a = np.minimum(np.abs(x), E4M3_MAX)
    with np.errstate(divide="ignore"):
        e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.maximum(e, -6.0)           # below 2^-6 the step stays 2^-9 (subnormals)
    step = np.exp2(e - 3.0)
    r = np.round(a / step) * step     # numpy rounds halves to even
    r = np.minimum(r, E4M3_MAX)
    return (np.sign(x) * r).astype(np.float32)


def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16 (ties to even); returns float32."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32)
    bias = ((u >> 16) & np.uint32(1)) + np.uint32(0x7FFF)
    r = ((u + bias) & np.uint32(0xFFFF0000)).astype(np.uint32)
    return r.view(np.float32)


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """Upper 16 bits of float32 values that are already bf16-representable."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    return (x.view(np.uint32) >> 16).astype(np.uint16)


def _rng(seed: int, tid: int, b: int, h: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, tid, b, h])))


def head_slice(w: Workload, tid: int, b: int, h: int, n: int | None = None) -> np.ndarray:
    """One [N, d] float32 slice of tensor `tid` for (b, h), already in storage precision."""
    n = w.N if n is None else n
    x = _rng(w.seed, tid, b, h).standard_normal((n, w.d), dtype=np.float32)
    if w.std != 1.0:
        x *= np.float32(w.std)
    if tid == TID_Q and w.spike_frac > 0.0:
        k = int(round(w.spike_frac * n))
        rows = _rng(w.seed, TID_SPIKE, b, h).permutation(n)[:k]
        x[rows] *= np.float32(w.spike_mul)
    if w.dtype == "bf16":
        x = round_to_bf16(x)
    elif w.dtype == "e4m3":
        x = round_to_e4m3(x / np.float32(w.descale))
    elif w.dtype == "e5m2":
        x = round_to_e5m2(x / np.float32(w.descale))
    return x


def spiked_rows(w: Workload, b: int, h: int) -> np.ndarray:
    """The query rows of (b, h) that `head_slice` scaled by spike_mul."""
    if w.spike_frac <= 0.0:
        return np.zeros(0, dtype=np.int64)
    k = int(round(w.spike_frac * w.N))
    return np.sort(_rng(w.seed, TID_SPIKE, b, h).permutation(w.N)[:k])


def _fill(args):
    w, tid, b, h, out = args
    out[b, h] = head_slice(w, tid, b, h)


def tensor(w: Workload, tid: int, workers: int | None = None) -> np.ndarray:
    """Full [B, H, N, d] float32 tensor (H = Hq for Q/dO, Hkv for K/V)."""
    H = w.Hq if tid in (TID_Q, TID_DO) else w.Hkv
    out = np.empty((w.B, H, w.N, w.d), dtype=np.float32)
    jobs = [(w, tid, b, h, out) for b in range(w.B) for h in range(H)]
    workers = workers or min(len(jobs), os.cpu_count() or 1)
    if workers <= 1 or len(jobs) == 1:
        for j in jobs:
            _fill(j)
    else:
        with _cf.ThreadPoolExecutor(workers) as ex:
            list(ex.map(_fill, jobs))
    return out


def small(B, Hq, Hkv, N, d, causal, seed, dtype="bf16", std=1.0, backward=True,
          spike_frac=0.0, spike_mul=1.0) -> Workload:
    """An ad-hoc workload for parity tests at small sizes."""
    return Workload(f"t{B}x{Hq}x{Hkv}x{N}x{d}{'c' if causal else ''}", B, Hq, Hkv, N, d,
                    causal, dtype, backward, seed, std=std, spike_frac=spike_frac,
                    spike_mul=spike_mul)


@dataclass(frozen=True)
class DecodeWorkload:
    """Nq new queries against a cache of Nk keys/values (bf16)."""
    name: str
    B: int
    Hq: int
    Hkv: int
    Nq: int
    Nk: int
    d: int
    causal: bool
    seed: int
    std: float = 1.0

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    @property
    def group(self) -> int:
        return self.Hq // self.Hkv

    def flops(self) -> float:
        return 4.0 * self.B * self.Hq * self.Nq * self.Nk * self.d

    def kv_bytes(self) -> int:
        return 2 * self.B * self.Hkv * self.Nk * self.d * 2


DECODE_WORKLOADS = {
    # one decode step of a GQA model (32 query heads, 8 kv heads) over a 32K-token cache
    "dec": DecodeWorkload("dec", 16, 32, 8, 1, 32768, 128, True, 1010),
    # speculative / multi-token decode: 4 new tokens per sequence, GQA group 8 (32 query rows a CTA)
    "dec4": DecodeWorkload("dec4", 16, 32, 4, 4, 32768, 128, True, 1011),
    # 8 new tokens per sequence, 64 query heads over 8 kv heads: 64 query rows a group,
    # the 128-row-block kernel
    "dec8": DecodeWorkload("dec8", 16, 64, 8, 8, 32768, 128, True, 1013),
    # the step of "dec" with a head dim of 64 (4 query rows a group: the 128-row-block kernel
    # with the rows duplicated over both lane halves)
    "dec64": DecodeWorkload("dec64", 16, 32, 8, 1, 32768, 64, True, 1014),
}


def decode_inputs(w: DecodeWorkload, workers: int | None = None):
    """(q [B,Hq,Nq,d], k, v [B,Hkv,Nk,d]) float32, bf16-representable, one seeded
    stream per (tensor, batch, head) as for the other workloads."""
    def fill(args):
        out, tid, b, h = args
        x = _rng(w.seed, tid, b, h).standard_normal(out.shape[2:], dtype=np.float32)
        if w.std != 1.0:
            x *= np.float32(w.std)
        out[b, h] = round_to_bf16(x)

    q = np.empty((w.B, w.Hq, w.Nq, w.d), dtype=np.float32)
    k = np.empty((w.B, w.Hkv, w.Nk, w.d), dtype=np.float32)
    v = np.empty_like(k)
    jobs = [(q, TID_Q, b, h) for b in range(w.B) for h in range(w.Hq)]
    jobs += [(t, tid, b, h) for t, tid in ((k, TID_K), (v, TID_V)) for b in range(w.B) for h in range(w.Hkv)]
    workers = workers or min(len(jobs), os.cpu_count() or 1)
    with _cf.ThreadPoolExecutor(workers) as ex:
        list(ex.map(fill, jobs))
    return q, k, v


def sample_rows(w: Workload, b: int, h: int, count: int | None = None) -> np.ndarray:
    """Sorted query (or key) row indices checked for a large workload.

    Always includes the first rows, the tile edges at 127/128, the middle and the
    last row, then seeded random rows up to `count`.
    """
    count = count or w.sample_rows or w.N
    fixed = {0, 1, 127, 128, w.N // 2, w.N - 1}
    fixed = {r for r in fixed if 0 <= r < w.N}
    rng = _rng(w.seed, 99, b, h)
    extra = rng.choice(w.N, size=min(w.N, count + len(fixed)), replace=False)
    rows = list(sorted(fixed))
    for r in extra:
        if len(rows) >= count:
            break
        if r not in fixed:
            rows.append(int(r))
    return np.array(sorted(set(rows)), dtype=np.int64)
