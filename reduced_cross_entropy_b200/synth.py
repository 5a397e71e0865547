"""Seeded synthetic inputs for the reduced cross-entropy loss.

This module only draws numbers: it holds none of the loss's arithmetic, so both the
CUDA path and the CPU oracle can be fed from it.  Everything is drawn with numpy's
PCG64 from an explicit seed, in a fixed order (X, then Y, then the targets), in fp32,
then rounded to bf16 (round to nearest even) where a workload is bf16.  A matrix of more
than 2^24 elements is drawn instead in blocks of 2^22 elements, block b from its own
PCG64 stream (the b-th child of SeedSequence([seed, 0 for X / 1 for Y])), filled by a
thread pool: the values depend on the seed only, never on the thread count.

Workloads follow the shapes of the RECE paper's experiments (section 4, Table 1:
catalogues of 22k to 174k items, SASRec outputs of batch x sequence rows) and extend
them to larger catalogues and an LM-sized vocabulary:

* targets are uniform or truncated Zipf over the catalogue, P(j) ~ (j+1)^-alpha,
  drawn by inverse CDF (item 0 is the most popular);
* X, Y rows are Gaussian; the large-catalogue workload scales item j's row by a
  Zipf-like factor (j+1)^-alpha normalised to unit mean square, so that popular
  items have long embeddings.

The random projection vectors B of the method are drawn here too, from their own
stream keyed by (seed, step), and are passed to both sides as an input.
"""
from __future__ import annotations

import dataclasses
import os
from concurrent.futures import ThreadPoolExecutor
from typing import Optional

import numpy as np


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    N: int          # rows = batch x sequence length
    d: int          # embedding width
    C: int          # catalogue size
    dtype: str      # "fp32" or "bf16"
    n_b: int        # random vectors (buckets) per round
    n_c: int        # chunks
    n_ec: int       # neighbouring chunks on each side
    n_r: int        # rounds
    k: int          # negatives kept per row
    target_alpha: float = 0.0   # 0 -> uniform targets, else truncated Zipf exponent
    x_std: Optional[float] = None  # None -> 1/sqrt(d)
    y_std: Optional[float] = None  # None -> 1/sqrt(d)
    y_norm_alpha: float = 0.0      # >0 -> Zipf-scaled item norms

    def scaled(self, N: int, C: int, **over) -> "Workload":
        """Same recipe at other sizes (for tests that the oracle finishes quickly)."""
        return dataclasses.replace(self, name=f"{self.name}@N{N}C{C}", N=N, C=C, **over)


WORKLOADS = {
    "tiny": Workload("tiny", N=256, d=64, C=4096, dtype="fp32", n_b=16, n_c=8, n_ec=1,
                     n_r=1, k=32),
    "sasrec": Workload("sasrec", N=25_600, d=64, C=100_000, dtype="bf16", n_b=256, n_c=64,
                       n_ec=1, n_r=2, k=256, target_alpha=1.0),
    "large": Workload("large", N=51_200, d=128, C=1_000_000, dtype="bf16", n_b=1024,
                      n_c=256, n_ec=1, n_r=2, k=512, target_alpha=1.1, y_norm_alpha=1.1),
    "very_large": Workload("very_large", N=65_536, d=256, C=4_000_000, dtype="bf16",
                           n_b=4096, n_c=1024, n_ec=2, n_r=1, k=1024, target_alpha=1.2),
    "lm": Workload("lm", N=16_384, d=4096, C=128_000, dtype="bf16", n_b=512, n_c=128,
                   n_ec=1, n_r=2, k=512, target_alpha=1.0, x_std=1.0, y_std=0.02),
}


def _bf16_rounded_u32(a: np.ndarray) -> np.ndarray:
    """fp32 bit patterns rounded to nearest even at bit 16 (low 16 bits left as they are
    after the add; finite inputs: the largest sum, 0xFF7FFFFF + 0x8000, stays in 32 bits)."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    r = (u >> np.uint32(16)) & np.uint32(1)
    r += u
    r += np.uint32(0x7FFF)
    return r


def bf16_bits(a: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns (uint16), round to nearest even (finite inputs)."""
    return (_bf16_rounded_u32(a) >> np.uint32(16)).astype(np.uint16)


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> their exact fp32 values."""
    return (np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(
        np.float32)


def round_bf16(a: np.ndarray) -> np.ndarray:
    r = _bf16_rounded_u32(a)
    r &= np.uint32(0xFFFF0000)
    return r.view(np.float32).reshape(np.shape(a))


def zipf_targets(rng: np.random.Generator, n: int, C: int, alpha: float) -> np.ndarray:
    """n draws from P(j) ~ (j+1)^-alpha on [0, C) by inverse CDF (alpha 0 = uniform)."""
    if alpha == 0.0:
        return rng.integers(0, C, size=n, dtype=np.int64).astype(np.int32)
    w = np.arange(1, C + 1, dtype=np.float64) ** (-alpha)
    cdf = np.cumsum(w)
    cdf /= cdf[-1]
    u = rng.random(n)
    return np.minimum(np.searchsorted(cdf, u, side="right"), C - 1).astype(np.int32)


_BLOCK = 1 << 22
_SINGLE_STREAM_MAX = 1 << 24


def _standard_normal(rng: np.random.Generator, seed: int, tag: int, shape) -> np.ndarray:
    """fp32 N(0, 1) draws: from `rng` for up to 2^24 elements, else block by block."""
    n = int(np.prod(shape))
    if n <= _SINGLE_STREAM_MAX:
        return rng.standard_normal(shape, dtype=np.float32)
    out = np.empty(n, np.float32)
    nb = (n + _BLOCK - 1) // _BLOCK
    kids = np.random.SeedSequence([seed, tag]).spawn(nb)

    def fill(b):
        np.random.Generator(np.random.PCG64(kids[b])).standard_normal(
            out=out[b * _BLOCK:(b + 1) * _BLOCK], dtype=np.float32)

    with ThreadPoolExecutor(max_workers=os.cpu_count() or 1) as ex:
        list(ex.map(fill, range(nb)))
    return out.reshape(shape)


def make_inputs(w: Workload, seed: int = 0):
    """(X, Y, targets) as fp32 numpy arrays (bf16 workloads already rounded to bf16)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    xs = w.x_std if w.x_std is not None else w.d ** -0.5
    ys = w.y_std if w.y_std is not None else w.d ** -0.5
    X = _standard_normal(rng, seed, 0, (w.N, w.d))
    X *= np.float32(xs)
    Y = _standard_normal(rng, seed, 1, (w.C, w.d))
    Y *= np.float32(ys)
    if w.y_norm_alpha > 0.0:
        s = np.arange(1, w.C + 1, dtype=np.float64) ** (-w.y_norm_alpha)
        s /= np.sqrt(np.mean(s * s))
        Y = (Y * s[:, None].astype(np.float32)).astype(np.float32)
    t = zipf_targets(rng, w.N, w.C, w.target_alpha)
    if w.dtype == "bf16":
        X, Y = round_bf16(X), round_bf16(Y)
    return X, Y, t


def projections(seed: int, step: int, n_r: int, n_b: int, d: int, dtype: str = "fp32"):
    """Random vectors B [n_r, n_b, d] ~ N(0,1) for one call of the loss.

    The RECE paper draws B afresh inside the loss (Algorithm 1, the randn step); here
    it is keyed by (seed, step) so every call is reproducible."""
    ss = np.random.SeedSequence([seed, step, 0x5EED])
    B = np.random.Generator(np.random.PCG64(ss)).standard_normal((n_r, n_b, d),
                                                                  dtype=np.float32)
    return round_bf16(B) if dtype == "bf16" else B


def uniform_negatives(seed: int, N: int, C: int, n: int) -> np.ndarray:
    """n negatives per row drawn uniformly from the catalogue [0, C), with replacement
    (the uniform sampling of the sampled baselines, RECE section 2), int32 [N, n].  The
    draw may hit the row's positive or repeat an item; the losses take the ids as given."""
    ss = np.random.SeedSequence([seed, 0x5A4D])
    rng = np.random.Generator(np.random.PCG64(ss))
    return rng.integers(0, C, size=(N, n), dtype=np.int64).astype(np.int32)


def integer_inputs(N: int, C: int, d: int, lo: int = -3, hi: int = 3, seed: int = 0,
                   scale: float = 0.25):
    """Small-integer multiples of `scale` (a power of two): every product and partial
    sum is exact in fp32, so any summation order gives the same score, and ties are
    frequent.  Used to pin the oracle against brute force."""
    rng = np.random.Generator(np.random.PCG64(seed))
    X = rng.integers(lo, hi + 1, size=(N, d)).astype(np.float32) * np.float32(scale)
    Y = rng.integers(lo, hi + 1, size=(C, d)).astype(np.float32) * np.float32(scale)
    t = rng.integers(0, C, size=N).astype(np.int32)
    return X, Y, t
