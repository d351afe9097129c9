"""Parity of the CUDA search path (through the C ABI) with the CPU oracle.

Each search is compared stage by stage on the same seeded inputs:
  leaves      ranked match with the oracle's fp64 centroid scores;
  candidates  the best R by approximate score (fp32 mode: ranked match within
              tolerance; uint8 mode: ids, integer sums and fp32 scores
              bit-exact);
  final       ranked match with the oracle's exact (or approximate) scores.
A query whose leaf set differs from the oracle's (only possible through a
near-tie at the L-th leaf, which the ranked match checks) is checked for
validity downstream instead of equality; likewise for a near-tie at the R-th
candidate.  Such queries must stay rare.
"""
import numpy as np
import pytest
import torch

from mips_ivf_centroid_b200 import datagen
from oracle import OracleIndex

from parity import ranked_match, same_set

pytestmark = pytest.mark.gpu

_cache = {}


def _workload(name):
    """(workload, X, Q, index arrays on cuda, host arrays) for a named case."""
    if name in _cache:
        return _cache[name]
    W = datagen.WORKLOADS
    cases = {
        "tiny": W["tiny"],
        "glove-mini": W["glove"].scaled(n=60_000, num_leaves=300, num_leaves_to_search=24, nq=300,
                                        n_means=120, training_sample_size=60_000),
        "bigann-mini": W["bigann"].scaled(n=100_000, num_leaves=500, num_leaves_to_search=32, nq=200,
                                          n_means=400, training_sample_size=100_000),
        "openai-mini": W["openai"].scaled(n=20_000, num_leaves=100, num_leaves_to_search=10, nq=100,
                                          n_means=60, training_sample_size=20_000),
        "sweep-mini": W["sweep"].scaled(n=200_000, num_leaves=1000, num_leaves_to_search=64, nq=256,
                                        n_means=800, training_sample_size=200_000),
        "leaves-1500": W["glove"].scaled(n=30_000, d=32, num_leaves=1500, num_leaves_to_search=40, nq=128,
                                         n_means=100, training_sample_size=30_000),
        "leaves-3000": W["glove"].scaled(n=30_000, d=32, num_leaves=3000, num_leaves_to_search=64, nq=128,
                                         n_means=100, training_sample_size=30_000),
        "leaves-5000": W["glove"].scaled(n=50_000, d=32, num_leaves=5000, num_leaves_to_search=16, nq=128,
                                         n_means=100, training_sample_size=50_000),
        "gemm128-vec": W["glove"].scaled(n=40_000, d=64, num_leaves=2048, num_leaves_to_search=8, nq=2048,
                                         n_means=100, training_sample_size=40_000),
        "gemm128-scalar": W["glove"].scaled(n=40_000, d=34, dims_per_block=1, num_leaves=2048,
                                            num_leaves_to_search=8, nq=2048, n_means=100,
                                            training_sample_size=40_000),
        "glove-mini-residual": W["glove"].scaled(n=60_000, num_leaves=300, num_leaves_to_search=24, nq=300,
                                                 n_means=120, training_sample_size=60_000, residual=True),
        "tiny-leaves": W["glove"].scaled(n=3_000, d=16, num_leaves=2000, num_leaves_to_search=1500, nq=32,
                                         n_means=10, training_sample_size=3_000, code_loss="l2",
                                         threshold_T=None),
        "small-leaves": W["glove"].scaled(n=3_000, d=16, num_leaves=600, num_leaves_to_search=2, nq=64,
                                          n_means=10, training_sample_size=3_000, code_loss="l2",
                                          threshold_T=None),
    }
    w = cases[name]
    X = datagen.make_data(w)
    Q = datagen.make_queries(w)
    ix = datagen.build_index(w, X, "cuda")
    _cache[name] = (w, X, Q, ix, ix.numpy())
    return _cache[name]


@pytest.fixture(scope="module")
def Index():
    from mips_ivf_centroid_b200 import build
    build.build()
    from mips_ivf_centroid_b200 import Index as I
    return I


def compare(Index, name, k, L, reorder_num, lut_mode, max_leaf_mismatch=0.02, max_cand_mismatch=0.05,
            qsel=None):
    w, X, Q, ix, arr = _workload(name)
    index = Index(ix)
    Qs = Q if qsel is None else Q[qsel]
    qg = torch.from_numpy(Qs).cuda()
    ids, scores, tr = index.search(qg, k, L, reorder_num, lut_mode, trace=True)
    index.sync_status()
    ids, scores = ids.cpu().numpy(), scores.cpu().numpy()
    tr = {kk: v.cpu().numpy() for kk, v in tr.items()}
    orc = OracleIndex(arr)
    o = orc.search(Qs, k, L, reorder_num, lut_mode)
    inv = np.empty(w.n, np.int64)
    inv[arr["slot_ids"]] = np.arange(w.n)
    nq = Qs.shape[0]
    leaf_mis = cand_mis = 0
    for i in range(nq):
        q = Qs[i]
        cs = orc.centroid_scores(q)
        ranked_match(tr["leaf_ids"][i], tr["leaf_scores"][i], o["leaves"][i], o["leaf_scores"][i],
                     lambda g: cs[g], f"q{i} leaves")
        if not same_set(tr["leaf_ids"][i], o["leaves"][i]):
            leaf_mis += 1
            continue
        assert tr["scanned"][i] == o["scanned"][i]
        assert tr["ncand"][i] == o["ncand"][i]
        gc = tr["cand_ids"][i]
        if lut_mode == 1:
            np.testing.assert_array_equal(gc, o["cand_ids"][i], err_msg=f"q{i} u8 candidates")
            np.testing.assert_array_equal(tr["cand_sums"][i].astype(np.uint32), o["cand_sums"][i])
            np.testing.assert_array_equal(tr["cand_scores"][i], o["cand_scores"][i].astype(np.float32))
        else:
            ranked_match(gc, tr["cand_scores"][i], o["cand_ids"][i], o["cand_scores"][i],
                         lambda g: orc.point_scores(q, inv[g])[0], f"q{i} candidates")
        if reorder_num > 0:
            exact_of = lambda g: orc.point_scores(q, inv[g])[1]
        elif lut_mode == 0:
            exact_of = lambda g: orc.point_scores(q, inv[g])[0]
        else:
            exact_of = None
        if not same_set(gc, o["cand_ids"][i]):
            cand_mis += 1
            # valid: the final ids are the best k of the GPU's candidates
            nc = int((gc >= 0).sum())
            ex = exact_of(gc[:nc])
            order = np.lexsort((gc[:nc], -ex))[:k]
            ranked_match(ids[i], scores[i], np.pad(gc[:nc][order], (0, k - len(order)), constant_values=-1),
                         np.pad(ex[order], (0, k - len(order)), constant_values=-np.inf), exact_of, f"q{i} final*")
            continue
        if exact_of is None:     # uint8 approximate ranking: bit-exact
            np.testing.assert_array_equal(ids[i], o["ids"][i])
            np.testing.assert_array_equal(scores[i], o["scores"][i].astype(np.float32))
        else:
            ranked_match(ids[i], scores[i], o["ids"][i], o["scores"][i], exact_of, f"q{i} final")
    assert leaf_mis <= max(1, max_leaf_mismatch * nq), f"{leaf_mis} queries with a different leaf set"
    assert cand_mis <= max(1, max_cand_mismatch * nq), f"{cand_mis} queries with a different candidate set"
    index.close()
    return dict(leaf_mismatch=leaf_mis, cand_mismatch=cand_mis, ids=ids, scores=scores, oracle=o)


@pytest.mark.parametrize("lut_mode", [0, 1])
@pytest.mark.parametrize("reorder_num", [100, 0])
def test_tiny(Index, lut_mode, reorder_num):
    compare(Index, "tiny", 10, 1, reorder_num, lut_mode)


@pytest.mark.parametrize("lut_mode", [0, 1])
def test_glove_mini(Index, lut_mode):
    compare(Index, "glove-mini", 10, 24, 100, lut_mode)


def test_glove_mini_no_reorder(Index):
    compare(Index, "glove-mini", 10, 24, 0, 0)


def test_bigann_mini_integer_exact(Index):
    # integer data and queries: centroid scores and exact scores are integers
    # below 2^24, so both are computed exactly by fp32 and fp64 alike.
    r = compare(Index, "bigann-mini", 10, 32, 200, 0, max_leaf_mismatch=0.0)
    o = r["oracle"]
    assert r["leaf_mismatch"] == 0
    same = (r["ids"] == o["ids"]).all(axis=1)
    np.testing.assert_array_equal(r["scores"][same], o["scores"][same].astype(np.float32))


def test_openai_mini_bf16_reorder(Index):
    compare(Index, "openai-mini", 10, 10, 300, 0)


def test_openai_mini_u8(Index):
    compare(Index, "openai-mini", 10, 10, 0, 1)


def test_sweep_mini(Index):
    compare(Index, "sweep-mini", 10, 64, 100, 0)


@pytest.mark.parametrize("name,L", [("leaves-1500", 40), ("leaves-3000", 64), ("leaves-3000", 100),
                                    ("leaves-5000", 16)])
def test_many_centroids(Index, name, L):
    # more centroids than one warp holds in registers: two-stage warp selection
    # (two register widths, L <= 64), the block's register form (L > 64), and
    # beyond 4096 centroids the shared-memory radix
    compare(Index, name, 10, L, 100, 0)


@pytest.mark.parametrize("name", ["gemm128-vec", "gemm128-scalar"])
def test_large_batch_centroid_tiles(Index, name):
    # 2048 queries x 2048 centroids: the 128-wide centroid tiles (float4 operand
    # loads when d % 4 == 0, scalar ones otherwise); the whole batch is searched,
    # a sample of queries is checked stage by stage
    from parity import compare_search
    w, X, Q, ix, arr = _workload(name)
    index = Index(ix)
    compare_search(index, arr, Q, 10, w.num_leaves_to_search, 100, 0, qsel=np.arange(0, w.nq, 16))
    index.close()


@pytest.mark.parametrize("reorder_num", [100, 0])
def test_residual_codes(Index, reorder_num):
    # codes of x minus its leaf's centroid: scores add the query's centroid score
    compare(Index, "glove-mini-residual", 10, 24, reorder_num, 0)


def test_residual_codes_reject_uint8_tables(Index):
    from mips_ivf_centroid_b200 import AhError
    w, X, Q, ix, arr = _workload("glove-mini-residual")
    index = Index(ix)
    with pytest.raises(AhError) as e:
        index.search(torch.from_numpy(Q[:4]).cuda(), 10, 24, 100, 1)
    assert e.value.status == 2
    index.close()


@pytest.mark.parametrize("lut_mode", [0, 1])
def test_threshold_sample_over_hundreds_of_leaves(Index, lut_mode):
    # leaves of about 1.5 points, none empty: the threshold sample's segment
    # table fills (256 leaves, exactly at a warp round's end) before the
    # sample does, and the bound comes from that subset alone
    compare(Index, "tiny-leaves", 10, 1500, 100, lut_mode)


def _overflow_case():
    """Two leaves.  The better one by centroid score holds 2,000 points whose
    codes are all low (centers 0-3); the other holds 20,000 points whose codes
    are all high (centers 8-15), with every center a positive multiple of the
    all-ones vector and every query positive.  The filter bound comes from a
    sample of the first leaf, so every point of the second reaches it: about
    20,000 kept against a buffer of 8,192 (R = 100), and every query is
    rescanned with the bound taken from its stored candidates."""
    from mips_ivf_centroid_b200.datagen import IndexArrays
    key = "overflow"
    if key in _cache:
        return _cache[key]
    rng = np.random.default_rng(20261202)
    d, n0, n1, nq = 16, 2_000, 20_000, 16
    n = n0 + n1
    w = datagen.WORKLOADS["glove"].scaled(n=n, d=d, num_leaves=2, num_leaves_to_search=2, nq=nq,
                                          n_means=1, training_sample_size=n)
    B = d // w.dims_per_block
    nib = np.concatenate([rng.integers(0, 4, (n0, B)), rng.integers(8, 16, (n1, B))]).astype(np.uint8)
    codes = (nib[:, 0::2] | (nib[:, 1::2] << 4)).astype(np.uint8)
    codebook = np.broadcast_to((np.arange(16, dtype=np.float32) / 15)[None, :, None],
                               (B, 16, w.dims_per_block)).copy()
    centroids = np.stack([np.full(d, 10.0, np.float32), np.ones(d, np.float32)])
    X = rng.standard_normal((n, d)).astype(np.float32)
    Q = rng.uniform(0.5, 1.5, (nq, d)).astype(np.float32)
    slot_ids = rng.permutation(n).astype(np.int32)
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    ix = IndexArrays(workload=w, centroids=t(centroids), leaf_offsets=t(np.array([0, n0, n], np.int64)),
                     slot_ids=t(slot_ids), codes=t(codes), codebook=t(codebook), reorder_vecs=t(X[slot_ids]))
    _cache[key] = (w, X, Q, ix, ix.numpy())
    return _cache[key]


@pytest.mark.parametrize("lut_mode", [0, 1])
def test_candidate_buffer_overflow_rescans(Index, lut_mode):
    w, X, Q, ix, arr = _overflow_case()
    index = Index(ix)
    _, _, tr = index.search(torch.from_numpy(Q).cuda(), 10, 2, 100, lut_mode, trace=True)
    index.sync_status()
    index.close()
    assert int(tr["rescans"][0]) == w.nq
    assert (tr["passed"].cpu() > 8192).all()
    compare(Index, "overflow", 10, 2, 100, lut_mode, max_leaf_mismatch=0.0, max_cand_mismatch=0.0)


def test_all_leaves(Index):
    compare(Index, "glove-mini", 10, 300, 100, 0, qsel=slice(0, 40))


def test_single_query(Index):
    compare(Index, "glove-mini", 10, 24, 100, 0, qsel=slice(7, 8))


def test_padding_when_leaves_hold_fewer_than_k(Index):
    r = compare(Index, "small-leaves", 20, 1, 0, 0)
    assert (r["ids"] == -1).any()
    r = compare(Index, "small-leaves", 20, 2, 20, 1)


def test_R_above_points(Index):
    compare(Index, "small-leaves", 10, 2, 4096, 0)


def test_large_k(Index):
    compare(Index, "glove-mini", 1000, 24, 2000, 0, qsel=slice(0, 30))


def test_empty_leaves_selected(Index):
    # Extra leaves whose centroids copy a real centroid but hold no points.
    from mips_ivf_centroid_b200.datagen import IndexArrays
    w, X, Q, ix, arr = _workload("glove-mini")
    extra = 50
    cent = torch.cat([ix.centroids, ix.centroids[:extra] * 1.01])
    offs = torch.cat([ix.leaf_offsets, ix.leaf_offsets[-1:].repeat(extra)])
    ix2 = IndexArrays(workload=w, centroids=cent.contiguous(), leaf_offsets=offs.contiguous(),
                      slot_ids=ix.slot_ids, codes=ix.codes, codebook=ix.codebook, reorder_vecs=ix.reorder_vecs)
    key = "glove-mini-empty"
    arr2 = dict(arr)
    arr2["centroids"] = cent.cpu().numpy()
    arr2["leaf_offsets"] = offs.cpu().numpy()
    _cache[key] = (w.scaled(num_leaves=w.num_leaves + extra), X, Q, ix2, arr2)
    compare(Index, key, 10, 24, 100, 0)
    compare(Index, key, 10, 24, 100, 1)


def test_empty_batch_and_bad_args(Index):
    from mips_ivf_centroid_b200 import AhError
    w, X, Q, ix, arr = _workload("tiny")
    index = Index(ix)
    ids, scores = index.search(torch.empty((0, w.d), device="cuda"), 10, 1, 100)
    assert ids.shape == (0, 10)
    qg = torch.from_numpy(Q).cuda()
    for k, L, r, m in [(0, 1, 100, 0), (10, 2, 100, 0), (10, 1, 5, 0), (10, 1, 100, 3), (2000, 1, 2000, 0)]:
        with pytest.raises(AhError):
            index.search(qg, k, L, r, m)
    index.sync_status()


def test_host_entry_point_matches_device(Index):
    w, X, Q, ix, arr = _workload("glove-mini")
    index = Index(ix)
    qg = torch.from_numpy(Q).cuda()
    ids, scores = index.search(qg, 10, 24, 100)
    hq = torch.from_numpy(Q).pin_memory()
    hids, hscores = index.search_host(hq, 10, 24, 100)
    np.testing.assert_array_equal(hids.numpy(), ids.cpu().numpy())
    np.testing.assert_array_equal(hscores.numpy(), scores.cpu().numpy())


def test_repeatable_and_reentrant(Index):
    w, X, Q, ix, arr = _workload("glove-mini")
    index = Index(ix)
    qg = torch.from_numpy(Q).cuda()
    a = index.search(qg, 10, 24, 100)
    b = index.search(qg[:50], 10, 8, 0, 1)      # different knobs in between
    c = index.search(qg, 10, 24, 100)
    torch.testing.assert_close(a[0], c[0], rtol=0, atol=0)
    torch.testing.assert_close(a[1], c[1], rtol=0, atol=0)
    index.sync_status()


def test_worked_example_scan_counter(Index):
    # ScaNN blog, "Worked example": 100 of 1,000 equal leaves of 1,000 points,
    # 64 blocks per point -> 100,000 points and 6.4M table lookups per query.
    from mips_ivf_centroid_b200.datagen import IndexArrays
    n, d, NL, L = 1_000_000, 128, 1000, 100
    g = torch.Generator(device="cuda").manual_seed(0)
    w = datagen.Workload(name="worked", n=n, d=d, dims_per_block=2, num_leaves=NL, num_leaves_to_search=L,
                         nq=4, k=10, reorder_num=0)
    ix = IndexArrays(workload=w, centroids=torch.randn(NL, d, device="cuda", generator=g),
                     leaf_offsets=torch.arange(0, n + 1, n // NL, device="cuda", dtype=torch.int64),
                     slot_ids=torch.arange(n, device="cuda", dtype=torch.int32),
                     codes=torch.randint(0, 256, (n, 32), device="cuda", dtype=torch.uint8, generator=g),
                     codebook=torch.randn(64, 16, 2, device="cuda", generator=g), reorder_vecs=None)
    index = Index(ix)
    q = torch.randn(4, d, device="cuda", generator=g)
    _, _, tr = index.search(q, 10, L, 0, trace=True)
    info = index.last_search_info(points_scanned=True)
    assert (tr["scanned"].cpu().numpy() == 100_000).all()
    assert info["points_scanned"] == 4 * 100_000
    assert info["points_scanned"] // 4 * 64 == 6_400_000


@pytest.mark.parametrize("lut_mode", [0, 1])
def test_speed_knobs_do_not_change_results(Index, lut_mode):
    # progressive bound on/off, sample size and spread, scan chunk: same ids and scores
    w, X, Q, ix, arr = _workload("sweep-mini")
    index = Index(ix)
    qg = torch.from_numpy(Q).cuda()
    ref = index.search(qg, 10, 64, 100, lut_mode)
    for opt, val in [(Index.OPT_PROGRESSIVE_LEAVES, -1), (Index.OPT_PROGRESSIVE_LEAVES, 3),
                     (Index.OPT_THRESHOLD_SAMPLE, 64), (Index.OPT_THRESHOLD_LEAVES, 8),
                     (Index.OPT_SCAN_CHUNK_TILES, 3)]:
        index.set_option(opt, val)
        got = index.search(qg, 10, 64, 100, lut_mode)
        torch.testing.assert_close(got[0], ref[0], rtol=0, atol=0)
        torch.testing.assert_close(got[1], ref[1], rtol=0, atol=0)
    index.sync_status()
    index.close()
