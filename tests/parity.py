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
                   max_cand_mismatch=0.05, orc=None, label=""):
    """Search all of Q on the GPU (one batch, as the benchmark launches it),
    then check the rows ``qsel`` stage by stage against the oracle.

    Every checked query is checked through every stage.  Leaves: ranked match
    with the oracle's own best L.  Where a near-tie at the L-th leaf makes the
    GPU's leaf set differ (a swap the ranked match allows), the later stages
    of that query are compared with the oracle run over the GPU's leaves
    (``OracleIndex.search_leaves``: the same arithmetic from the table on), so
    no query goes unchecked.  Candidates: ranked match (fp32 tables) or
    bit-exact ids, integer sums and scores (uint8 tables).  Final results:
    ranked match with the oracle's; where a near-tie at the R-th candidate
    makes the candidate sets differ, the GPU's final ids must be the best k of
    its own candidates by the oracle's scores.

    Returns a dict with the counts (checked queries, leaf-set swaps,
    candidate-set swaps) and the GPU/oracle outputs of the checked rows."""
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
    nq = Qs.shape[0]

    # 1. leaves, every query
    for i in range(nq):
        def leaf_scores_of(g, i=i):
            # the oracle's fp64 scores of the GPU's leaves: from its own list when
            # it holds them all, else every centroid scored afresh
            pos = {int(c): j for j, c in enumerate(o["leaves"][i])}
            if all(int(c) in pos for c in g):
                return o["leaf_scores"][i][[pos[int(c)] for c in g]]
            return orc.centroid_scores(Qs[i])[g]
        ranked_match(tr["leaf_ids"][i], tr["leaf_scores"][i], o["leaves"][i], o["leaf_scores"][i],
                     leaf_scores_of, f"{label} q{qsel[i]} leaves")
    swapped = np.array([i for i in range(nq) if not same_set(tr["leaf_ids"][i], o["leaves"][i])], np.int64)
    # the reference for the later stages: the oracle's own search, or for a
    # swapped leaf set the oracle over the GPU's leaves
    ref = {kk: o[kk].copy() for kk in ("ids", "scores", "cand_ids", "cand_scores", "cand_sums", "ncand", "scanned")}
    if swapped.shape[0]:
        o2 = orc.search_leaves(Qs[swapped], tr["leaf_ids"][swapped], k, reorder_num, lut_mode)
        for kk in ref:
            ref[kk][swapped] = o2[kk]

    # 2.-3. candidates and final results, every query
    cand_mis = 0
    for i in range(nq):
        q = Qs[i]
        what = f"{label} q{qsel[i]}"
        assert tr["scanned"][i] == ref["scanned"][i], f"{what} scanned {tr['scanned'][i]} vs {ref['scanned'][i]}"
        assert tr["ncand"][i] == ref["ncand"][i], f"{what} ncand"
        gc = tr["cand_ids"][i]
        if lut_mode == 1:
            np.testing.assert_array_equal(gc, ref["cand_ids"][i], err_msg=f"{what} u8 candidates")
            np.testing.assert_array_equal(tr["cand_sums"][i].astype(np.uint32), ref["cand_sums"][i],
                                          err_msg=f"{what} u8 sums")
            np.testing.assert_array_equal(tr["cand_scores"][i], ref["cand_scores"][i].astype(np.float32),
                                          err_msg=f"{what} u8 scores")
        else:
            ranked_match(gc, tr["cand_scores"][i], ref["cand_ids"][i], ref["cand_scores"][i],
                         lambda g: orc.point_scores(q, inv[g])[0], f"{what} candidates")
        if reorder_num > 0:
            exact_of = lambda g: orc.point_scores(q, inv[g])[1]
        elif lut_mode == 0:
            exact_of = lambda g: orc.point_scores(q, inv[g])[0]
        else:
            exact_of = None
        if not same_set(gc, ref["cand_ids"][i]):
            # only a near-tie at the R-th candidate (fp32 tables) gets here
            assert exact_of is not None, f"{what}: u8 candidate sets differ"
            cand_mis += 1
            nc = int((gc >= 0).sum())
            ex = exact_of(gc[:nc])
            order = np.lexsort((gc[:nc], -ex))[:k]
            ranked_match(ids[i], scores[i], np.pad(gc[:nc][order], (0, k - len(order)), constant_values=-1),
                         np.pad(ex[order], (0, k - len(order)), constant_values=-np.inf), exact_of,
                         f"{what} final (own candidates)")
            continue
        if exact_of is None:     # uint8 approximate ranking: bit-exact
            np.testing.assert_array_equal(ids[i], ref["ids"][i], err_msg=f"{what} u8 final ids")
            np.testing.assert_array_equal(scores[i], ref["scores"][i].astype(np.float32),
                                          err_msg=f"{what} u8 final scores")
        else:
            ranked_match(ids[i], scores[i], ref["ids"][i], ref["scores"][i], exact_of, f"{what} final")
    print(f"parity {label or ''}: {nq} queries checked through every stage, "
          f"{swapped.shape[0]} leaf-set swaps, {cand_mis} candidate-set swaps")
    assert swapped.shape[0] <= max(1, max_leaf_mismatch * nq), f"{swapped.shape[0]} queries with a different leaf set"
    assert cand_mis <= max(1, max_cand_mismatch * nq), f"{cand_mis} queries with a different candidate set"
    return dict(checked=nq, leaf_mismatch=int(swapped.shape[0]), cand_mismatch=cand_mis, ids=ids, scores=scores,
                oracle=o, ref=ref, trace=tr)
