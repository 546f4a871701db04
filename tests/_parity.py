"""Comparison helpers for the GPU-vs-oracle parity tests."""
import numpy as np


def y_tolerance(y_oracle: np.ndarray, X: np.ndarray, W: np.ndarray, idx: np.ndarray, rows=None) -> np.ndarray:
    """Per-element bound max(2 fp16 ulp at the oracle value, 1e-3 * sum_{k in O} |x_ik w_kj|).

    The ulp is that of the binade holding the oracle's fp16 value (2^-24 at
    and below the subnormal range).  The second term covers the fp32 (GPU)
    versus double (oracle) accumulation of the fp16 outlier product.
    """
    yo = np.abs(y_oracle.astype(np.float64))
    e = np.floor(np.log2(np.maximum(yo, 2.0 ** -14)))
    ulp = np.exp2(e - 10)
    Xr = X if rows is None else X[np.asarray(rows)]
    if idx.size:
        s = np.abs(Xr[:, idx].astype(np.float64)) @ np.abs(W[idx, :].astype(np.float64))
    else:
        s = np.zeros_like(yo)
    return np.maximum(2 * ulp, 1e-3 * s)


def assert_y_close(y_gpu: np.ndarray, y_oracle: np.ndarray, X, W, idx, rows=None):
    yg = y_gpu.astype(np.float64)
    yo = y_oracle.astype(np.float64)
    assert np.isfinite(yg).all(), "non-finite GPU output"
    tol = y_tolerance(y_oracle, X, W, idx, rows)
    err = np.abs(yg - yo)
    bad = err > tol
    if bad.any():
        i, j = np.argwhere(bad)[0]
        raise AssertionError(
            f"{int(bad.sum())} of {bad.size} outputs out of tolerance; first at [{i},{j}]: "
            f"gpu={yg[i, j]!r} oracle={yo[i, j]!r} tol={tol[i, j]!r}")
    return float(err.max()) if err.size else 0.0


def sample_rows(M: int, n: int, seed: int) -> np.ndarray:
    """Seeded sample of about n distinct row indices that always includes
    the first and the last row (the ragged tail of the last 128-row tile)."""
    if M <= n:
        return np.arange(M)
    rng = np.random.default_rng(seed)
    inner = rng.choice(np.arange(1, M - 1), size=max(0, n - 2), replace=False)
    return np.unique(np.concatenate([[0, M - 1], inner]))
