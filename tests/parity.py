"""Comparison rules between a GPU result and the oracle.

Integer-valued inputs: scores bit-equal and index sets equal.
bf16 inputs (tolerance rule): for each row, with kth = the oracle's k-th
score (the smallest selected one) and tol = rel * max(|kth|, rms_row):
  - both sides hold the same number of valid (>= 0) indices;
  - GPU indices are eligible and unique;
  - every GPU index the oracle did not select has oracle score >= kth - tol;
  - every oracle index the GPU did not select has oracle score <= kth + tol.
rms_row is the root mean square of the row's oracle scores over the set the
row ranks (a floor for k-th scores near zero).  rel = 2e-3.
"""
from __future__ import annotations

import numpy as np

REL_TOL = 2e-3


def valid(row):
    return row[row >= 0]


def check_exact_sets(gpu_idx, ref_idx, what="idx"):
    gpu_idx, ref_idx = np.asarray(gpu_idx), np.asarray(ref_idx)
    assert gpu_idx.shape == ref_idx.shape, (gpu_idx.shape, ref_idx.shape)
    bad = []
    for r in range(gpu_idx.shape[0]):
        g, o = np.sort(valid(gpu_idx[r])), np.sort(valid(ref_idx[r]))
        if g.size != o.size or not np.array_equal(g, o):
            bad.append(r)
        elif valid(gpu_idx[r]).size != np.count_nonzero(gpu_idx[r] >= 0) or \
                np.any(gpu_idx[r][g.size:] != -1):
            bad.append(r)
    assert not bad, f"{what}: {len(bad)} rows differ, first {bad[:5]}"


def check_tolerance_row(gpu_row, ref_row, score_of, rms, rel=REL_TOL, eligible=None):
    """One row under the tolerance rule.  score_of(indices) -> oracle scores.

    Returns None when the row passes, else a message.
    """
    g, o = valid(np.asarray(gpu_row)), valid(np.asarray(ref_row))
    if g.size != o.size:
        return f"count {g.size} != {o.size}"
    if np.any(np.asarray(gpu_row)[g.size:] != -1):
        return "valid entries not packed before the -1 padding"
    if np.unique(g).size != g.size:
        return "duplicate indices"
    if g.size == 0:
        return None
    if eligible is not None and not np.all(eligible(g)):
        return "ineligible index"
    ref_scores = score_of(o)
    kth = float(np.min(ref_scores))
    tol = rel * max(abs(kth), rms)
    extra = np.setdiff1d(g, o)
    missing = np.setdiff1d(o, g)
    if extra.size:
        s = score_of(extra)
        if np.any(s < kth - tol):
            return f"selected index with score {float(np.min(s))} < kth {kth} - tol {tol}"
    if missing.size:
        s = score_of(missing)
        if np.any(s > kth + tol):
            return f"dropped index with score {float(np.max(s))} > kth {kth} + tol {tol}"
    return None


def check_tolerance_rows(gpu_idx, ref_idx, all_scores, rel=REL_TOL, what="idx"):
    """Rows whose oracle scores are all known: all_scores[r][s] (-inf = ineligible)."""
    bad = []
    for r in range(len(gpu_idx)):
        row = all_scores[r]
        fin = row[np.isfinite(row)]
        rms = float(np.sqrt(np.mean(fin ** 2))) if fin.size else 0.0
        msg = check_tolerance_row(gpu_idx[r], ref_idx[r], lambda ix: row[ix], rms, rel,
                                  eligible=lambda ix: np.isfinite(row[ix]))
        if msg:
            bad.append((r, msg))
    assert not bad, f"{what}: {len(bad)} rows fail the tolerance rule, first {bad[:3]}"


def check_scores_close(gpu, ref, rel=REL_TOL):
    """Element-wise score check: |g - r| <= rel * max(|r|, rms_row); -inf must match."""
    gpu, ref = np.asarray(gpu, np.float64), np.asarray(ref, np.float64)
    assert gpu.shape == ref.shape
    ninf_r, ninf_g = np.isneginf(ref), np.isneginf(gpu)
    assert np.array_equal(ninf_r, ninf_g), "masked (-inf) pattern differs"
    for r in range(ref.shape[0]):
        fin = np.isfinite(ref[r])
        if not fin.any():
            continue
        rms = np.sqrt(np.mean(ref[r][fin] ** 2))
        err = np.abs(gpu[r][fin] - ref[r][fin])
        lim = rel * np.maximum(np.abs(ref[r][fin]), rms)
        assert np.all(err <= lim), f"row {r}: max err {err.max()} vs limit {lim[np.argmax(err - lim)]}"
