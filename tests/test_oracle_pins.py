"""Pins for the CPU oracle: each test checks it against something other than
itself (numpy brute force, the reconstruction identity, an integer special case,
a hand-worked example, a quantisation error bound, the blog's worked-example
counts).  Source for every step: ScaNN blog post, "Three stages of a search".
"""
import os

import numpy as np
import pytest

from mips_ivf_centroid_b200 import datagen
from oracle import OracleIndex

HERE = os.path.dirname(os.path.abspath(__file__))


def _mini(n=1500, d=16, dpb=2, NL=12, L=4, nq=20, k=10, reorder_num=50, aniso=False, **kw):
    w = datagen.Workload(name="mini", n=n, d=d, dims_per_block=dpb, num_leaves=NL,
                         num_leaves_to_search=L, nq=nq, k=k, reorder_num=reorder_num,
                         n_means=8, sigma=0.3, training_sample_size=min(n, 2000),
                         code_loss="anisotropic" if aniso else "l2",
                         threshold_T=0.2 if aniso else None, **kw)
    X = datagen.make_data(w)
    Q = datagen.make_queries(w)
    ix = datagen.build_index(w, X, "cpu")
    return w, X, Q, ix, ix.numpy()


def _order(scores, ids):
    """Indices sorting by (score desc, id asc); an independent numpy restatement."""
    return np.lexsort((ids, -scores))


def _reconstruct(arr):
    """x~ per slot from the packed codes and codebook (numpy, its own unpacking)."""
    codes = arr["codes"]
    B = codes.shape[1] * 2
    idx = np.empty((codes.shape[0], B), np.int64)
    idx[:, 0::2] = codes & 0x0F
    idx[:, 1::2] = codes >> 4
    cb = arr["codebook"].astype(np.float64)
    return cb[np.arange(B)[None, :], idx].reshape(codes.shape[0], -1)


def test_leaves_match_numpy_fp64():
    w, X, Q, ix, arr = _mini()
    orc = OracleIndex(arr)
    out = orc.search(Q, w.k, w.num_leaves_to_search, w.reorder_num)
    s = Q.astype(np.float64) @ arr["centroids"].astype(np.float64).T
    for qi in range(Q.shape[0]):
        o = _order(s[qi], np.arange(w.num_leaves))[: w.num_leaves_to_search]
        np.testing.assert_array_equal(out["leaves"][qi], o)
        np.testing.assert_allclose(out["leaf_scores"][qi], s[qi][o], rtol=0, atol=1e-12)


def test_leaf_ties_go_to_lower_id():
    w, X, Q, ix, arr = _mini()
    arr = dict(arr)
    c = arr["centroids"].copy()
    c[7] = c[3]                       # leaves 3 and 7 now always score equal
    arr["centroids"] = c
    orc = OracleIndex(arr)
    out = orc.search(Q, w.k, w.num_leaves, w.reorder_num)
    for qi in range(Q.shape[0]):
        lv = list(out["leaves"][qi])
        assert lv.index(3) + 1 == lv.index(7)


def test_approximate_score_is_dot_with_reconstruction():
    # adding up the table entries a point's codes select gives q . x~ for its
    # reconstruction x~ ("Three stages of a search")
    w, X, Q, ix, arr = _mini(aniso=True)
    orc = OracleIndex(arr)
    out = orc.search(Q, w.k, w.num_leaves_to_search, w.reorder_num)
    xt = _reconstruct(arr)
    inv = np.empty(w.n, np.int64)
    inv[arr["slot_ids"]] = np.arange(w.n)
    for qi in range(Q.shape[0]):
        nc = out["ncand"][qi]
        slots = inv[out["cand_ids"][qi][:nc]]
        expect = xt[slots] @ Q[qi].astype(np.float64)
        np.testing.assert_allclose(out["cand_scores"][qi][:nc], expect, rtol=0, atol=1e-12)
        # and the R kept are the best R over the scanned leaves
        lv = out["leaves"][qi]
        scanned = np.concatenate([np.arange(arr["leaf_offsets"][c], arr["leaf_offsets"][c + 1])
                                  for c in lv])
        sc = xt[scanned] @ Q[qi].astype(np.float64)
        best = scanned[_order(sc, arr["slot_ids"][scanned])][:nc]
        np.testing.assert_array_equal(arr["slot_ids"][best], out["cand_ids"][qi][:nc])
        assert out["scanned"][qi] == scanned.shape[0]


def test_residual_score_is_dot_with_centroid_plus_reconstruction():
    # residual codes quantise x - c(leaf): the approximate point is c(leaf) + r~,
    # so the score is q . c(leaf) + the table sum over the residual codebook
    w, X, Q, ix, arr = _mini(aniso=True, residual=True)
    assert arr["residual"]
    orc = OracleIndex(arr)
    out = orc.search(Q, w.k, w.num_leaves_to_search, w.reorder_num)
    rt = _reconstruct(arr)
    leaf_of = np.repeat(np.arange(w.num_leaves), np.diff(arr["leaf_offsets"]))
    xt = rt + arr["centroids"].astype(np.float64)[leaf_of]
    inv = np.empty(w.n, np.int64)
    inv[arr["slot_ids"]] = np.arange(w.n)
    for qi in range(Q.shape[0]):
        nc = out["ncand"][qi]
        slots = inv[out["cand_ids"][qi][:nc]]
        expect = xt[slots] @ Q[qi].astype(np.float64)
        np.testing.assert_allclose(out["cand_scores"][qi][:nc], expect, rtol=0, atol=1e-12)
        lv = out["leaves"][qi]
        scanned = np.concatenate([np.arange(arr["leaf_offsets"][c], arr["leaf_offsets"][c + 1])
                                  for c in lv])
        sc = xt[scanned] @ Q[qi].astype(np.float64)
        best = scanned[_order(sc, arr["slot_ids"][scanned])][:nc]
        np.testing.assert_array_equal(arr["slot_ids"][best], out["cand_ids"][qi][:nc])
        a, _ = orc.point_scores(Q[qi], slots)
        np.testing.assert_allclose(a, expect, rtol=0, atol=1e-12)
    # the residual reconstruction is closer to the data than the plain one
    wp, Xp, _, _, arrp = _mini(aniso=True)
    err_res = np.linalg.norm(X[arr["slot_ids"]] - xt, axis=1).mean()
    err_plain = np.linalg.norm(Xp[arrp["slot_ids"]] - _reconstruct(arrp), axis=1).mean()
    assert err_res < err_plain


def test_residual_codes_reject_uint8_tables():
    w, X, Q, ix, arr = _mini(residual=True)
    orc = OracleIndex(arr)
    with pytest.raises(Exception):
        orc.search(Q, w.k, w.num_leaves_to_search, w.reorder_num, lut_mode=1)


def test_hand_worked_nibble_example():
    # One point, d = 4, dims_per_block = 1 (B = 4 blocks); codes bytes 0x21, 0x43
    # mean block 0 -> center 1, block 1 -> 2, block 2 -> 3, block 3 -> 4
    # (block 2i in the low nibble of byte i).  Centers: cb[b][j] = 10 b + j.
    # q = (1, 2, 3, 4): score = 1*1 + 2*12 + 3*23 + 4*34 = 1 + 24 + 69 + 136 = 230.
    cb = np.array([[[10.0 * b + j] for j in range(16)] for b in range(4)], np.float32)
    arr = dict(centroids=np.zeros((1, 4), np.float32), leaf_offsets=np.array([0, 1], np.int64),
               slot_ids=np.array([0], np.int32), codes=np.array([[0x21, 0x43]], np.uint8),
               codebook=cb, reorder_vecs=np.array([[5.0, 6.0, 7.0, 8.0]], np.float32))
    orc = OracleIndex(arr)
    q = np.array([[1, 2, 3, 4]], np.float32)
    out = orc.search(q, 1, 1, 0)
    assert out["ids"][0, 0] == 0 and out["scores"][0, 0] == 230.0
    out = orc.search(q, 1, 1, 1)          # exact: 5 + 12 + 21 + 32 = 70
    assert out["scores"][0, 0] == 70.0


def _brute_topk(X, Q, k):
    s = Q.astype(np.float64) @ X.astype(np.float64).T
    ids = np.empty((Q.shape[0], k), np.int64)
    sc = np.empty((Q.shape[0], k))
    for qi in range(Q.shape[0]):
        o = _order(s[qi], np.arange(X.shape[0]))[:k]
        ids[qi], sc[qi] = o, s[qi][o]
    return ids, sc


@pytest.mark.parametrize("nl", [1, 9])
def test_full_reorder_equals_brute_force_mips(nl):
    # L = NL and reorder_num = n: every point is rescored exactly.
    w, X, Q, ix, arr = _mini(n=1200, NL=nl, L=nl, k=10, reorder_num=1200)
    orc = OracleIndex(arr)
    out = orc.search(Q, 10, nl, 1200)
    ids, sc = _brute_topk(X, Q, 10)
    np.testing.assert_array_equal(out["ids"], ids)
    np.testing.assert_allclose(out["scores"], sc, rtol=0, atol=1e-12)


def test_exact_codes_make_ah_exact_integer_case():
    # Every block slice is one of 16 integer 2-vectors and the codebook is those
    # vectors, so x~ = x: without reorder the approximate top-k is the exact
    # top-k, with exact integer scores and id tie-breaks.
    rng = np.random.default_rng(11)
    n, d, B = 800, 12, 6
    cb = rng.integers(0, 16, size=(B, 16, 2)).astype(np.float32)
    codes = rng.integers(0, 16, size=(n, B))
    codes[5] = codes[2]; codes[9] = codes[2]          # planted exact ties
    X = cb[np.arange(B)[None, :], codes].reshape(n, d)
    perm = rng.permutation(n).astype(np.int32)        # slot order != id order
    packed = (codes[perm, 0::2] | (codes[perm, 1::2] << 4)).astype(np.uint8)
    arr = dict(centroids=np.zeros((1, d), np.float32), leaf_offsets=np.array([0, n], np.int64),
               slot_ids=perm, codes=packed, codebook=cb, reorder_vecs=X[perm])
    Q = rng.integers(-8, 9, size=(15, d)).astype(np.float32)
    Q[0] = 0.0                                          # all scores tie: ids 0..k-1
    orc = OracleIndex(arr)
    out = orc.search(Q, 10, 1, 0)
    ids, sc = _brute_topk(X, Q, 10)
    np.testing.assert_array_equal(out["ids"], ids)
    np.testing.assert_array_equal(out["scores"], sc)
    np.testing.assert_array_equal(out["ids"][0], np.arange(10))


def test_reorder_zero_returns_approximate_ranking():
    w, X, Q, ix, arr = _mini()
    orc = OracleIndex(arr)
    out = orc.search(Q, 10, 4, 0)
    np.testing.assert_array_equal(out["ids"], out["cand_ids"][:, :10])
    np.testing.assert_array_equal(out["scores"], out["cand_scores"][:, :10])


def test_reorder_rescores_candidates_exactly():
    w, X, Q, ix, arr = _mini()
    orc = OracleIndex(arr)
    out = orc.search(Q, 10, 4, 50)
    for qi in range(Q.shape[0]):
        cands = out["cand_ids"][qi][: out["ncand"][qi]]
        ex = X[cands].astype(np.float64) @ Q[qi].astype(np.float64)
        o = _order(ex, cands)[:10]
        np.testing.assert_array_equal(out["ids"][qi], cands[o])
        np.testing.assert_allclose(out["scores"][qi], ex[o], rtol=0, atol=1e-12)


def test_bf16_reorder_uses_stored_bf16_values():
    w, X, Q, ix, arr = _mini(reorder_dtype="bf16")
    assert arr["reorder_dtype"] == "bf16"
    orc = OracleIndex(arr)
    out = orc.search(Q, 10, 4, 50)
    bits = arr["reorder_vecs"].astype(np.uint32) << 16
    v = bits.view(np.float32).astype(np.float64)     # stored bf16 upcast
    inv = np.empty(w.n, np.int64)
    inv[arr["slot_ids"]] = np.arange(w.n)
    for qi in range(3):
        ex = v[inv[out["ids"][qi]]] @ Q[qi].astype(np.float64)
        np.testing.assert_allclose(out["scores"][qi], ex, rtol=0, atol=1e-12)


def test_short_results_are_padded():
    w, X, Q, ix, arr = _mini(n=1500, NL=300, L=1, k=10, reorder_num=0)
    sizes = np.diff(arr["leaf_offsets"])
    orc = OracleIndex(arr)
    out = orc.search(Q, 10, 1, 0)
    for qi in range(Q.shape[0]):
        m = sizes[out["leaves"][qi][0]]
        if m < 10:
            assert (out["ids"][qi][m:] == -1).all() and np.isneginf(out["scores"][qi][m:]).all()
        assert (out["ids"][qi][: min(m, 10)] >= 0).all()
    assert (sizes < 10).any()


def test_u8_table_definition_and_error_bound():
    w, X, Q, ix, arr = _mini(aniso=True)
    orc = OracleIndex(arr)
    xt = _reconstruct(arr)
    for qi in range(Q.shape[0]):
        lut8, delta, bias = orc.u8_table(Q[qi])
        assert (lut8.min(axis=1) == 0).all()          # every block's minimum maps to 0
        assert lut8.max() == 255                      # the widest block spans 0..255
        slots = np.arange(w.n)
        sums = orc.u8_sums(Q[qi], slots)
        approx = delta * sums.astype(np.float64) + bias
        exact = xt @ Q[qi].astype(np.float64)
        # each of B entries is off by at most delta/2, plus fp32 rounding of the table
        bound = w.blocks * delta / 2 + 1e-5
        assert np.max(np.abs(approx - exact)) <= bound


def test_u8_mode_orders_by_sum_then_id():
    w, X, Q, ix, arr = _mini()
    orc = OracleIndex(arr)
    out = orc.search(Q, 10, 4, 0, lut_mode=1)
    inv = np.empty(w.n, np.int64)
    inv[arr["slot_ids"]] = np.arange(w.n)
    for qi in range(Q.shape[0]):
        nc = out["ncand"][qi]
        ids = out["cand_ids"][qi][:nc]
        sums = out["cand_sums"][qi][:nc].astype(np.int64)
        np.testing.assert_array_equal(orc.u8_sums(Q[qi], inv[ids]), sums)
        key_ok = (np.diff(sums) < 0) | ((np.diff(sums) == 0) & (np.diff(ids) > 0))
        assert key_ok.all()
        lut8, delta, bias = orc.u8_table(Q[qi])
        want = (np.float32(delta) * sums[:10].astype(np.float32)).astype(np.float64)
        # score = fmaf(delta, sum, bias): compare within one fp32 ulp of the unfused form
        np.testing.assert_allclose(out["scores"][qi], want + bias, rtol=2e-7, atol=2e-7)


def test_invalid_arguments_rejected():
    w, X, Q, ix, arr = _mini()
    orc = OracleIndex(arr)
    for k, L, r, m in [(0, 4, 50, 0), (10, 0, 50, 0), (10, 13, 50, 0), (10, 4, 5, 0), (10, 4, 50, 2)]:
        with pytest.raises(ValueError):
            orc.search(Q, k, L, r, lut_mode=m)


def _golden(name):
    vals = {}
    for line in open(os.path.join(HERE, "golden", name)):
        line = line.strip()
        if line and not line.startswith("#"):
            k, v = line.split("=")
            vals[k.strip()] = int(v)
    return vals


def test_worked_example_operation_counts():
    # Balanced index of the worked example: 1,000 leaves of exactly 1,000 points.
    g = _golden("worked_example.txt")
    n, d, dpb, NL, L = g["n"], g["d"], g["dims_per_block"], g["num_leaves"], g["num_leaves_to_search"]
    B = d // dpb
    assert B == g["blocks"] and B // 2 == g["code_bytes_per_point"]
    assert n * (B // 2) == g["code_bytes_total"] and n * d * 4 == g["raw_vector_bytes"]
    assert NL * d == g["partition_macs"] and B * 16 * dpb == g["lut_macs"]
    assert g["reorder"] * d == g["reorder_macs"]
    rng = np.random.default_rng(5)
    arr = dict(centroids=rng.standard_normal((NL, d)).astype(np.float32),
               leaf_offsets=np.arange(0, n + 1, n // NL, dtype=np.int64),
               slot_ids=np.arange(n, dtype=np.int32),
               codes=rng.integers(0, 256, size=(n, B // 2), dtype=np.uint8),
               codebook=rng.standard_normal((B, 16, dpb)).astype(np.float32), reorder_vecs=None)
    assert arr["codes"].nbytes == g["code_bytes_total"]
    orc = OracleIndex(arr)
    q = rng.standard_normal((1, d)).astype(np.float32)
    out = orc.search(q, 10, L, 0)
    assert out["scanned"][0] == g["points_scanned"]
    assert out["scanned"][0] * B == g["lookups"]


# -- steps 2-5 over caller-given leaves (orc_search_leaves) --------------------

def test_search_leaves_with_own_leaves_equals_search():
    # the downstream arithmetic is the search's own: given the leaves step 1
    # picked, every output equals the full search's, in both table modes
    w, X, Q, ix, arr = _mini(aniso=True)
    orc = OracleIndex(arr)
    for mode in (0, 1):
        full = orc.search(Q, w.k, w.num_leaves_to_search, w.reorder_num, mode)
        part = orc.search_leaves(Q, full["leaves"], w.k, w.reorder_num, mode)
        for key in ("ids", "scores", "cand_ids", "cand_scores", "cand_sums", "ncand", "scanned"):
            np.testing.assert_array_equal(part[key], full[key], err_msg=key)


def test_search_leaves_matches_numpy_on_arbitrary_leaves():
    # leaves that are not the query's best (random distinct lists, in any
    # order): candidates are the best R of those leaves' points by q . x~
    # (numpy reconstruction), finals the best k of them by exact dot product
    w, X, Q, ix, arr = _mini(aniso=True)
    orc = OracleIndex(arr)
    rng = np.random.default_rng(7)
    L = 5
    leaves = np.stack([rng.permutation(w.num_leaves)[:L] for _ in range(Q.shape[0])]).astype(np.int32)
    out = orc.search_leaves(Q, leaves, w.k, w.reorder_num)
    xt = _reconstruct(arr)
    xs = X[arr["slot_ids"]].astype(np.float64)
    for qi in range(Q.shape[0]):
        scanned = np.concatenate([np.arange(arr["leaf_offsets"][c], arr["leaf_offsets"][c + 1])
                                  for c in leaves[qi]])
        assert out["scanned"][qi] == scanned.shape[0]
        q = Q[qi].astype(np.float64)
        sc = xt[scanned] @ q
        nc = min(w.reorder_num, scanned.shape[0])
        best = scanned[_order(sc, arr["slot_ids"][scanned])][:nc]
        assert out["ncand"][qi] == nc
        np.testing.assert_array_equal(out["cand_ids"][qi][:nc], arr["slot_ids"][best])
        np.testing.assert_allclose(out["cand_scores"][qi][:nc], xt[best] @ q, rtol=0, atol=1e-12)
        ex = xs[best] @ q
        fin = best[_order(ex, arr["slot_ids"][best])][: w.k]
        np.testing.assert_array_equal(out["ids"][qi][: len(fin)], arr["slot_ids"][fin])


def test_search_leaves_u8_sums_match_numpy():
    # uint8 tables: integer sums of the table entries the codes select (numpy's
    # own unpacking), best R by (sum desc, id asc) over the given leaves
    w, X, Q, ix, arr = _mini()
    orc = OracleIndex(arr)
    rng = np.random.default_rng(11)
    L = 3
    leaves = np.stack([rng.permutation(w.num_leaves)[:L] for _ in range(Q.shape[0])]).astype(np.int32)
    out = orc.search_leaves(Q, leaves, w.k, 0, 1)
    codes = arr["codes"]
    B = codes.shape[1] * 2
    idx = np.empty((codes.shape[0], B), np.int64)
    idx[:, 0::2] = codes & 0x0F
    idx[:, 1::2] = codes >> 4
    for qi in range(Q.shape[0]):
        lut8, delta, bias = orc.u8_table(Q[qi])
        scanned = np.concatenate([np.arange(arr["leaf_offsets"][c], arr["leaf_offsets"][c + 1])
                                  for c in leaves[qi]])
        sums = lut8.astype(np.int64)[np.arange(B)[None, :], idx[scanned]].sum(1)
        nc = min(w.k, scanned.shape[0])
        best = scanned[np.lexsort((arr["slot_ids"][scanned], -sums))][:nc]
        np.testing.assert_array_equal(out["cand_ids"][qi][:nc], arr["slot_ids"][best])
        np.testing.assert_array_equal(out["cand_sums"][qi][:nc],
                                      lut8.astype(np.int64)[np.arange(B)[None, :], idx[best]].sum(1))


def test_search_leaves_rejects_bad_leaf_ids():
    w, X, Q, ix, arr = _mini()
    orc = OracleIndex(arr)
    bad = np.full((Q.shape[0], 2), w.num_leaves, np.int32)
    with pytest.raises(ValueError):
        orc.search_leaves(Q, bad, w.k, w.reorder_num)
