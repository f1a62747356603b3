"""Seeded synthetic workloads for the LLM.int8() mixed-precision matmul.

This module only draws random inputs. It holds none of the method's
arithmetic (no detection, no quantisation, no products), so both the CPU
oracle's tests and the CUDA path's tests and benchmark can use it without
sharing any of the computation under test.

Random numbers come from numpy's Philox4x32-10 bit generator, a
counter-based generator (Salmon et al., "Parallel random numbers: as easy
as 1, 2, 3", SC'11), seeded per workload.

Shapes and value statistics follow the pages' description of activation
outliers (AIInfra "05Quantization01", LLM.int8() section: outliers are
about 0.1% of values, live in ~6-7 fixed feature dimensions, are more than
20x the normal magnitude, appear on ~75% of sequence positions and are
almost always one-sided). Those pages evaluate on C4/WikiText-2 with
trained OPT/BLOOM/LLaMA models; these synthetic tensors stand in for the
activation statistics of such models.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

# Background activations are N(0,1) resampled while |x| > BACKGROUND_CLIP,
# so that at the default threshold (6.0) the detected outlier columns are
# exactly the planted ones.
BACKGROUND_CLIP = 6.0
# Fraction of rows (tokens) of an outlier column that hold an outlier value.
OUTLIER_ROW_FRACTION = 0.75


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    M: int            # tokens (rows of X)
    K: int            # input features
    N: int            # output features (rows of W)
    n_outliers: int   # planted outlier columns
    lo: float         # outlier magnitude ~ U(lo, hi)
    hi: float
    w_std: float      # W ~ N(0, w_std)
    seed: int
    threshold: float = 6.0
    description: str = ""

    @property
    def ops(self) -> int:
        """Algorithmic integer+float operations of one Y = X.W^T (2MNK)."""
        return 2 * self.M * self.N * self.K


WORKLOADS: dict[str, Workload] = {
    w.name: w
    for w in [
        Workload("tiny", 16, 256, 256, 2, 8.0, 40.0, 0.02, 1,
                 description="tiny correctness case, 16x256 . 256x256"),
        Workload("opt-6.7b-ffn-up-prefill", 2048, 4096, 16384, 6, 6.0, 60.0, 0.02, 2,
                 description="OPT-6.7B-like FFN up-projection prefill, 2048x4096 . 16384x4096"),
        Workload("decode", 16, 4096, 4096, 6, 6.0, 60.0, 0.02, 3,
                 description="decode shape, 16x4096 . 4096x4096, weight-read bound"),
        Workload("llama-70b-ffn-prefill", 4096, 8192, 28672, 7, 6.0, 100.0, 0.015, 4,
                 description="Llama-70B-like FFN prefill, 4096x8192 . 28672x8192"),
        Workload("stress-o0", 4096, 4096, 4096, 0, 6.0, 60.0, 0.02, 5,
                 description="outlier-density stress, 0 outlier columns"),
        Workload("stress-o7", 4096, 4096, 4096, 7, 6.0, 60.0, 0.02, 6,
                 description="outlier-density stress, 7 outlier columns"),
        Workload("stress-o64", 4096, 4096, 4096, 64, 6.0, 60.0, 0.02, 7,
                 description="outlier-density stress, 64 outlier columns"),
        Workload("stress-o256", 4096, 4096, 4096, 256, 6.0, 60.0, 0.02, 8,
                 description="outlier-density stress, 256 outlier columns"),
        Workload("stress-thr-inf", 4096, 4096, 4096, 7, 6.0, 60.0, 0.02, 9, math.inf,
                 description="stress endpoint: threshold=inf (pure vector-wise INT8)"),
        Workload("stress-thr-0", 4096, 4096, 4096, 7, 6.0, 60.0, 0.02, 10, 0.0,
                 description="stress endpoint: threshold=0 (pure FP16)"),
    ]
}


def rng(seed: int, stream: int = 0) -> np.random.Generator:
    """Counter-based generator for (seed, stream)."""
    return np.random.Generator(np.random.Philox(key=[seed, stream]))


def truncated_normal(g: np.random.Generator, shape, clip: float) -> np.ndarray:
    """N(0,1) samples in float64, each redrawn while |x| > clip."""
    x = g.standard_normal(size=shape)
    bad = np.abs(x) > clip
    while bad.any():
        x[bad] = g.standard_normal(size=int(bad.sum()))
        bad = np.abs(x) > clip
    return x


def make_activations(M: int, K: int, n_outliers: int, lo: float, hi: float, seed: int,
                     row_fraction: float = OUTLIER_ROW_FRACTION):
    """X fp16 [M, K] and the planted outlier column indices (sorted).

    Background entries are truncated N(0,1); each planted column gets a
    fixed random sign, and each of its rows independently (probability
    `row_fraction`) holds sign*U(lo, hi) instead of its background value.
    """
    g = rng(seed, 0)
    x = truncated_normal(g, (M, K), BACKGROUND_CLIP)
    cols = np.sort(g.choice(K, size=n_outliers, replace=False)) if n_outliers else np.zeros(0, np.int64)
    if n_outliers:
        signs = np.where(g.random(n_outliers) < 0.5, -1.0, 1.0)
        hit = g.random((M, n_outliers)) < row_fraction
        mag = g.uniform(lo, hi, size=(M, n_outliers))
        block = x[:, cols]
        block = np.where(hit, signs[None, :] * mag, block)
        x[:, cols] = block
    return x.astype(np.float16), cols.astype(np.int64)


def make_weight(N: int, K: int, std: float, seed: int) -> np.ndarray:
    """W fp16 [N, K] ~ N(0, std), out-features by in-features."""
    g = rng(seed, 1)
    w = g.standard_normal(size=(N, K), dtype=np.float32)
    w *= np.float32(std)
    return w.astype(np.float16)


def make_workload(w: Workload | str):
    """(X fp16 [M,K], W fp16 [N,K], planted outlier columns) for a workload."""
    if isinstance(w, str):
        w = WORKLOADS[w]
    X, cols = make_activations(w.M, w.K, w.n_outliers, w.lo, w.hi, w.seed)
    W = make_weight(w.N, w.K, w.w_std, w.seed)
    return X, W, cols


def make_workload_shard(w: Workload | str, part: int, parts: int):
    """Rows [part*M, (part+1)*M) of a batch of parts*M tokens drawn like the
    workload (same weight, same planted columns and signs); with parts = 1 it is
    make_workload(w). Returns (X shard fp16 [M,K], W fp16 [N,K], planted columns)."""
    if isinstance(w, str):
        w = WORKLOADS[w]
    X, cols = make_activations(parts * w.M, w.K, w.n_outliers, w.lo, w.hi, w.seed)
    W = make_weight(w.N, w.K, w.w_std, w.seed)
    return np.ascontiguousarray(X[part * w.M:(part + 1) * w.M]), W, cols


def random_case(M: int, K: int, N: int, n_outliers: int, seed: int, lo: float = 6.0,
                hi: float = 60.0, w_std: float = 0.02, row_fraction: float = OUTLIER_ROW_FRACTION):
    """An arbitrary-shape case with the same statistics (for ragged-shape tests)."""
    X, cols = make_activations(M, K, n_outliers, lo, hi, seed, row_fraction)
    W = make_weight(N, K, w_std, seed)
    return X, W, cols
