"""Comparison rules between the CUDA path and the oracle (test helpers).

Rules (leaf ids and final ids identical to the oracle except swaps among items
whose oracle scores differ by less than the tolerance; fp32 scores within the
tolerance; uint8 mode bit-exact):

* tol(s) = 2e-5 * max(1, |s|): 2e-5 absolute on unit-norm data, relative for
  data whose scores are far above 1 (integer-valued points).
* A ranked GPU list matches the oracle's ranked list when it has the same
  length, its ids are distinct, and at every rank i the oracle's own score of
  the GPU's id is within tol of the oracle's i-th score.  Where the oracle's
  scores are separated by more than 2 tol, that forces the same id at the same
  rank; where several items are within tol of each other (or of the cut-off)
  it allows them to swap.
* Each GPU score is within tol of the oracle's score of the same id.
"""
from __future__ import annotations

import numpy as np

TOL = 2e-5


def tol(s):
    return TOL * np.maximum(1.0, np.abs(s))


def ranked_match(gpu_ids, gpu_scores, ora_ids, ora_scores, score_of, what=""):
    """Check one query's ranked list.  ``score_of(ids) -> oracle scores``.

    Returns the number of ranks where the ids differ (allowed swaps)."""
    gpu_ids = np.asarray(gpu_ids)
    ora_ids = np.asarray(ora_ids)
    nv_g = int((gpu_ids >= 0).sum())
    nv_o = int((ora_ids >= 0).sum())
    assert nv_g == nv_o, f"{what}: {nv_g} valid GPU entries vs {nv_o} oracle"
    assert (gpu_ids[:nv_g] >= 0).all() and (gpu_ids[nv_g:] == -1).all(), f"{what}: padding"
    assert np.isneginf(np.asarray(gpu_scores)[nv_g:]).all(), f"{what}: padded scores"
    if nv_g == 0:
        return 0
    g = gpu_ids[:nv_g]
    assert np.unique(g).shape[0] == nv_g, f"{what}: duplicate ids"
    s_ora_of_g = np.asarray(score_of(g), dtype=np.float64)
    os_ = np.asarray(ora_scores[:nv_o], dtype=np.float64)
    rank_err = np.abs(s_ora_of_g - os_)
    bad = rank_err > tol(os_)
    assert not bad.any(), (f"{what}: rank-wise score mismatch at ranks {np.flatnonzero(bad)[:5]}: "
                           f"gpu ids {g[bad][:5]} oracle ids {ora_ids[:nv_o][bad][:5]} "
                           f"err {rank_err[bad][:5]}")
    gs = np.asarray(gpu_scores[:nv_g], dtype=np.float64)
    serr = np.abs(gs - s_ora_of_g)
    bad = serr > tol(s_ora_of_g)
    assert not bad.any(), f"{what}: GPU score off by {serr.max():.3g} at ranks {np.flatnonzero(bad)[:5]}"
    return int((g != ora_ids[:nv_o]).sum())


def same_set(a, b):
    a = np.asarray(a)
    b = np.asarray(b)
    return np.array_equal(np.sort(a[a >= 0]), np.sort(b[b >= 0]))
