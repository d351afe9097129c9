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


def compare_search(index, arr, Q, k, L, reorder_num, lut_mode, qsel=None, max_leaf_mismatch=0.02,
                   max_cand_mismatch=0.05, orc=None):
    """Search all of Q on the GPU (one batch, as the benchmark launches it),
    then check the rows ``qsel`` stage by stage against the oracle.

    Returns a dict with the mismatch counts and the GPU/oracle outputs of the
    checked rows."""
    import torch
    from oracle import OracleIndex

    qsel = np.arange(Q.shape[0]) if qsel is None else np.asarray(qsel)
    qg = torch.from_numpy(np.ascontiguousarray(Q)).to(index.device)
    ids, scores, tr = index.search(qg, k, L, reorder_num, lut_mode, trace=True)
    index.sync_status()
    ids = ids.cpu().numpy()[qsel]
    scores = scores.cpu().numpy()[qsel]
    tr = {kk: v.cpu().numpy() for kk, v in tr.items()}
    tr = {kk: (v[qsel] if v.ndim >= 1 and v.shape[0] == Q.shape[0] else v) for kk, v in tr.items()}
    orc = orc or OracleIndex(arr)
    Qs = np.ascontiguousarray(Q[qsel])
    o = orc.search(Qs, k, L, reorder_num, lut_mode)
    n = arr["slot_ids"].shape[0]
    inv = np.empty(n, np.int64)
    inv[arr["slot_ids"]] = np.arange(n)
    leaf_mis = cand_mis = 0
    for i in range(Qs.shape[0]):
        q = Qs[i]
        cs = orc.centroid_scores(q)
        ranked_match(tr["leaf_ids"][i], tr["leaf_scores"][i], o["leaves"][i], o["leaf_scores"][i],
                     lambda g: cs[g], f"q{qsel[i]} leaves")
        if not same_set(tr["leaf_ids"][i], o["leaves"][i]):
            leaf_mis += 1
            continue
        assert tr["scanned"][i] == o["scanned"][i], f"q{qsel[i]} scanned"
        assert tr["ncand"][i] == o["ncand"][i], f"q{qsel[i]} ncand"
        gc = tr["cand_ids"][i]
        if lut_mode == 1:
            np.testing.assert_array_equal(gc, o["cand_ids"][i], err_msg=f"q{qsel[i]} u8 candidates")
            np.testing.assert_array_equal(tr["cand_sums"][i].astype(np.uint32), o["cand_sums"][i])
            np.testing.assert_array_equal(tr["cand_scores"][i], o["cand_scores"][i].astype(np.float32))
        else:
            ranked_match(gc, tr["cand_scores"][i], o["cand_ids"][i], o["cand_scores"][i],
                         lambda g: orc.point_scores(q, inv[g])[0], f"q{qsel[i]} candidates")
        if reorder_num > 0:
            exact_of = lambda g: orc.point_scores(q, inv[g])[1]
        elif lut_mode == 0:
            exact_of = lambda g: orc.point_scores(q, inv[g])[0]
        else:
            exact_of = None
        if not same_set(gc, o["cand_ids"][i]):
            cand_mis += 1
            nc = int((gc >= 0).sum())
            if exact_of is None:
                continue
            ex = exact_of(gc[:nc])
            order = np.lexsort((gc[:nc], -ex))[:k]
            ranked_match(ids[i], scores[i], np.pad(gc[:nc][order], (0, k - len(order)), constant_values=-1),
                         np.pad(ex[order], (0, k - len(order)), constant_values=-np.inf), exact_of,
                         f"q{qsel[i]} final*")
            continue
        if exact_of is None:
            np.testing.assert_array_equal(ids[i], o["ids"][i])
            np.testing.assert_array_equal(scores[i], o["scores"][i].astype(np.float32))
        else:
            ranked_match(ids[i], scores[i], o["ids"][i], o["scores"][i], exact_of, f"q{qsel[i]} final")
    nq = Qs.shape[0]
    assert leaf_mis <= max(1, max_leaf_mismatch * nq), f"{leaf_mis} queries with a different leaf set"
    assert cand_mis <= max(1, max_cand_mismatch * nq), f"{cand_mis} queries with a different candidate set"
    return dict(leaf_mismatch=leaf_mis, cand_mismatch=cand_mis, ids=ids, scores=scores, oracle=o, trace=tr)
