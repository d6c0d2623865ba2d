"""Error and bias statistics used by the tests and the bench (NumPy, host).

These measure outputs; they hold none of the attention arithmetic.
"""
from __future__ import annotations

import numpy as np

__all__ = ["lse_rel_err", "normwise_rel_err", "max_rel_err", "bias_stats"]


def lse_rel_err(lse, ref) -> float:
    """max |LSE - LSE_ref| / max(|LSE_ref|, 1): relative, floored at 1 near zero."""
    lse, ref = np.asarray(lse, np.float64), np.asarray(ref, np.float64)
    return float(np.max(np.abs(lse - ref) / np.maximum(np.abs(ref), 1.0)))


def normwise_rel_err(x, ref, rms_floor: float = 1e-3) -> float:
    """||X - X_ref||_F / max(||X_ref||_F, rms_floor * sqrt(numel)).

    The floor only matters where the exact gradient vanishes (one visible key
    gives dQ = dK = 0 exactly); there the error is judged against an RMS of
    1e-3 instead of against zero.
    """
    x, ref = np.asarray(x, np.float64), np.asarray(ref, np.float64)
    denom = max(np.linalg.norm(ref.ravel()), rms_floor * np.sqrt(ref.size), 1e-300)
    return float(np.linalg.norm((x - ref).ravel()) / denom)


def max_rel_err(x, ref) -> float:
    """max |X - X_ref| / max |X_ref| over the tensor (the deviation measure used
    for the Llama 2 7B numbers in "Is Flash Attention Stable?")."""
    x, ref = np.asarray(x, np.float64), np.asarray(ref, np.float64)
    return float(np.max(np.abs(x - ref)) / max(np.max(np.abs(ref)), 1e-300))


def bias_stats(o, ref, rows) -> dict:
    """Mean signed error of O on the selected rows, with per-row standard errors.

    o, ref: [..., N, d]; rows: boolean [..., N].  Each selected row contributes
    e_r = mean_k (o - ref)[r, k] and a_r = mean_k sign(ref[r, k]) (o - ref)[r, k];
    rows are the independent samples.
    """
    o, ref = np.asarray(o, np.float64), np.asarray(ref, np.float64)
    rows = np.asarray(rows, bool)
    e = (o - ref)[rows]
    r = ref[rows]
    n = e.shape[0]
    er = e.mean(axis=-1)
    ar = (np.sign(r) * e).mean(axis=-1)
    se_e = er.std(ddof=1) / np.sqrt(n) if n > 1 else float("nan")
    se_a = ar.std(ddof=1) / np.sqrt(n) if n > 1 else float("nan")
    return {
        "rows": int(n),
        "mean": float(er.mean()),
        "se_mean": float(se_e),
        "z_mean": float(er.mean() / se_e) if se_e > 0 else 0.0,
        "aligned_mean": float(ar.mean()),
        "se_aligned": float(se_a),
        "z_aligned": float(ar.mean() / se_a) if se_a > 0 else 0.0,
        "mean_abs_ref": float(np.abs(r).mean()),
        "max_abs_err": float(np.abs(e).max()) if n else 0.0,
    }
