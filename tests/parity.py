"""Comparison helpers for the CUDA path against the oracle.

Rules (the tolerances of the comparison):
  * Index sets: bit-exact, except that an element may differ when the
    oracle's float64 score of every differing element lies within
    1e-6 * max|score| of the oracle's k-th score (a tie at the boundary within
    float32 rounding).  The number of accepted swaps is returned.
  * When the GPU's level-1 set differs inside that band, the oracle's later
    stages are re-run on the GPU's set (conditional oracle), so each stage is
    checked on the same inputs.
  * Attention outputs: per (batch, head) row, max|out - ref| / max|ref| <= 2e-3.
"""

from __future__ import annotations

import numpy as np

import oracle

BAND_REL = 1e-6
OUT_REL = 2e-3


def check_selection(gpu_sel, ref_scores, k, where=""):
    """gpu_sel: positions into ref_scores (any int array). Returns #swaps."""
    gpu_sel = np.asarray(gpu_sel, dtype=np.int64)
    assert gpu_sel.size == k, f"{where}: expected {k} indices, got {gpu_sel.size}"
    assert np.all(np.diff(gpu_sel) > 0), f"{where}: indices not strictly ascending"
    assert gpu_sel.min() >= 0 and gpu_sel.max() < ref_scores.size, f"{where}: index out of range"
    ref_sel = oracle.topk_ascending(ref_scores, k)
    if np.array_equal(ref_sel, gpu_sel):
        return 0
    s = np.asarray(ref_scores, dtype=np.float64)
    tau = np.sort(s)[::-1][k - 1]
    scale = np.max(np.abs(s))
    diff = np.setxor1d(ref_sel, gpu_sel)
    bad = diff[np.abs(s[diff] - tau) > BAND_REL * scale]
    assert bad.size == 0, (f"{where}: selection differs outside the tie band: {bad[:8]} "
                           f"scores {s[bad[:8]]} tau {tau} scale {scale}")
    return int(diff.size // 2)


def check_output(out, ref, where=""):
    out = np.asarray(out, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert out.shape == ref.shape, f"{where}: shape {out.shape} vs {ref.shape}"
    assert np.all(np.isfinite(out)), f"{where}: non-finite output"
    err = np.max(np.abs(out - ref), axis=-1) / np.maximum(np.max(np.abs(ref), axis=-1), 1e-30)
    worst = float(err.max())
    assert worst <= OUT_REL, f"{where}: max row relative error {worst:.3e} > {OUT_REL}"
    return worst
