"""Seeded synthetic inputs for the LLM.int8() decomposed matmul.

This module only draws random numbers.  It holds none of the method's
arithmetic (no outlier test, no scale, no rounding to int8): both the CPU
oracle and the CUDA path receive exactly the arrays made here.

Every array is drawn with numpy's PCG64 generator from an explicit seed.  The
convention for the named workloads is ``seed = 1000 * workload_id + repeat``.

The value distributions follow what the pages report about the input of an
FFN expansion layer in a >6.7B-parameter transformer:

* "LLM.int8() — 大模型激活值里藏着几个超大异常通道", 案例1: in OPT-13B, 4095
  ordinary channels with mean |x| 0.5 and max 5, and 7 outlier channels with
  mean |x| 65 and max 130.
* "AI 十大核心论文解读" §2.1: the outlier dimensions are few (at most 7) and
  cover about 75% of the sequence positions.

Ordinary activation columns are Gaussian and clipped below the threshold
(|x| <= 5.5 < 6.0), so only the planted columns can be outliers.  Weights are
N(0, 0.02^2).  All values are rounded once to IEEE binary16 by numpy.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

# The sigma of N(0, s^2) whose mean absolute value is 0.5: E|z| = s*sqrt(2/pi).
SIGMA_MEAN_ABS_HALF = 0.5 * math.sqrt(math.pi / 2.0)
NORMAL_CLIP = 5.5
W_SIGMA = 0.02
DEFAULT_ALPHA = 6.0


@dataclasses.dataclass
class Problem:
    """One decomposed-matmul input: X [M,K] fp16, W [K,N] fp16, threshold alpha."""

    name: str
    X: np.ndarray  # float16 [M, K], C order
    W: np.ndarray  # float16 [K, N], C order
    alpha: float
    planted: np.ndarray  # int64 column indices that carry planted outliers (sorted)
    seed: int

    @property
    def shape(self):
        return self.X.shape[0], self.X.shape[1], self.W.shape[1]


def _rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def _normal_f16(rng, shape, sigma, clip=None) -> np.ndarray:
    a = rng.standard_normal(size=shape, dtype=np.float32)
    a *= np.float32(sigma)
    if clip is not None:
        np.clip(a, -clip, clip, out=a)
    return a.astype(np.float16)


def weight(K: int, N: int, seed: int) -> np.ndarray:
    """W ~ N(0, 0.02^2) in fp16, [K, N] row-major."""
    return _normal_f16(_rng(seed), (K, N), W_SIGMA)


def activations(M: int, K: int, n_outliers: int, seed: int, *,
                normal_sigma: float = 1.0, normal_clip: float = NORMAL_CLIP,
                outlier_lo: float = 20.0, outlier_hi: float = 130.0,
                row_fraction: float = 0.75, force_max: float | None = None):
    """X [M,K] fp16 with ``n_outliers`` planted outlier columns.

    Ordinary entries are N(0, normal_sigma^2) clipped to +-normal_clip.  In each
    planted column, a seeded subset of ceil(row_fraction*M) rows holds
    |x| ~ U[outlier_lo, outlier_hi] with a random sign; the other rows stay
    ordinary.  With ``force_max`` set, one of those rows (seeded) is set to
    exactly +-force_max so the column maximum is pinned.
    Returns (X, planted_columns_sorted).
    """
    rng = _rng(seed)
    X = rng.standard_normal(size=(M, K), dtype=np.float32)
    X *= np.float32(normal_sigma)
    np.clip(X, -normal_clip, normal_clip, out=X)
    cols = np.sort(rng.permutation(K)[:n_outliers]).astype(np.int64)
    n_rows = int(math.ceil(row_fraction * M))
    for j in cols:
        rows = rng.permutation(M)[:n_rows]
        mag = rng.uniform(outlier_lo, outlier_hi, size=n_rows).astype(np.float32)
        sign = np.where(rng.integers(0, 2, size=n_rows) == 0, -1.0, 1.0).astype(np.float32)
        if force_max is not None and n_rows > 0:
            mag[int(rng.integers(0, n_rows))] = np.float32(force_max)
        X[rows, j] = sign * mag
    return X.astype(np.float16), cols


# ---------------------------------------------------------------------------
# Named workloads.  ids: 0 tiny, 1 OPT-13B prefill, 2 175B prefill,
# 3 decode, 4 sweep.  seed = 1000*id + repeat.

def tiny(repeat: int = 0) -> Problem:
    """M=16, K=256, N=128; 2 outlier columns, |x|~U[20,130] in 75% of rows."""
    seed = 0 * 1000 + repeat
    X, cols = activations(16, 256, 2, seed)
    W = weight(256, 128, seed + 500_000)
    return Problem("tiny_m16_k256_n128", X, W, DEFAULT_ALPHA, cols, seed)


def _ffn_prefill(name, wid, M, K, N, repeat, w=True):
    seed = wid * 1000 + repeat
    X, cols = activations(M, K, 7, seed, normal_sigma=SIGMA_MEAN_ABS_HALF,
                          outlier_lo=0.0, outlier_hi=130.0, force_max=130.0)
    W = weight(K, N, seed + 500_000) if w else None
    return Problem(name, X, W, DEFAULT_ALPHA, cols, seed)


def opt13b_prefill(repeat: int = 0, M: int = 2048, with_weight: bool = True) -> Problem:
    """OPT-13B FFN expansion: M=2048 tokens, K=5120, N=20480, 7 outlier columns
    with mean |x| 65 and max 130 in 75% of rows; ordinary mean |x| 0.5."""
    return _ffn_prefill(f"opt13b_ffn1_m{M}_k5120_n20480", 1, M, 5120, 20480, repeat, with_weight)


def gpt175b_prefill(repeat: int = 0, M: int = 2048, with_weight: bool = True) -> Problem:
    """175B-scale FFN expansion: M=2048, K=12288, N=49152, same distributions."""
    return _ffn_prefill(f"175b_ffn1_m{M}_k12288_n49152", 2, M, 12288, 49152, repeat, with_weight)


def opt13b_contraction(repeat: int = 0, M: int = 2048, with_weight: bool = True) -> Problem:
    """OPT-13B FFN contraction, the layer after the expansion: M=2048 tokens,
    K=20480, N=5120 (K > N), the same activation statistics (7 outlier
    columns, mean |x| 65, max 130, in 75% of rows; ordinary mean |x| 0.5)."""
    return _ffn_prefill(f"opt13b_ffn2_m{M}_k20480_n5120", 6, M, 20480, 5120, repeat, with_weight)


def decode(M: int, repeat: int = 0, K: int = 12288, N: int = 49152,
           with_weight: bool = True) -> Problem:
    """Decode step: M in {1, 8, 32} tokens, K=12288, N=49152.  The 7 outlier
    columns hold an outlier magnitude (U[20,130], random sign) in every row."""
    seed = 3 * 1000 + repeat
    X, cols = activations(M, K, 7, seed, normal_sigma=SIGMA_MEAN_ABS_HALF,
                          row_fraction=1.0)
    W = weight(K, N, seed + 500_000) if with_weight else None
    return Problem(f"decode_m{M}_k{K}_n{N}", X, W, DEFAULT_ALPHA, cols, seed)


def sweep(M: int, n_outliers: int, repeat: int = 0, K: int = 8192, N: int = 8192,
          alpha: float = DEFAULT_ALPHA, with_weight: bool = True) -> Problem:
    """K=N=8192 sweep point: ordinary N(0,1) clipped to +-5.5 and ``n_outliers``
    columns with |x|~U[20,130] in 75% of rows."""
    seed = 4 * 1000 + repeat + 10 * n_outliers + 100_000 * (M % 97)
    X, cols = activations(M, K, n_outliers, seed)
    W = weight(K, N, seed + 500_000) if with_weight else None
    a = "inf" if math.isinf(alpha) else f"{alpha:g}"
    return Problem(f"sweep_m{M}_k{K}_n{N}_o{n_outliers}_a{a}", X, W, alpha, cols, seed)


def worked_example(K: int = 4102, M: int = 2048, N: int = 256, repeat: int = 0) -> Problem:
    """The OPT-13B activation of the pages' first case study: 7 outlier channels
    (mean |x| 65, max 130) among K-7 ordinary channels (mean |x| 0.5, max 5)."""
    seed = 5 * 1000 + repeat
    X, cols = activations(M, K, 7, seed, normal_sigma=SIGMA_MEAN_ABS_HALF,
                          normal_clip=5.0, outlier_lo=0.0, outlier_hi=130.0,
                          force_max=130.0)
    W = weight(K, N, seed + 500_000)
    return Problem(f"worked_example_m{M}_k{K}_n{N}", X, W, DEFAULT_ALPHA, cols, seed)


def small(M: int, K: int, N: int, n_outliers: int, seed: int,
          alpha: float = DEFAULT_ALPHA, row_fraction: float = 0.75) -> Problem:
    """A small problem of any shape for edge-case and parity tests."""
    X, cols = activations(M, K, n_outliers, seed, row_fraction=row_fraction)
    W = weight(K, N, seed + 500_000)
    return Problem(f"small_m{M}_k{K}_n{N}_o{n_outliers}", X, W, alpha, cols, seed)


WORKLOADS = {
    "tiny": tiny,
    "opt13b": opt13b_prefill,
    "175b": gpt175b_prefill,
    "opt13b_ffn2": opt13b_contraction,
}
