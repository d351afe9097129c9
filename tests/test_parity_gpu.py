"""Parity of the CUDA search path (through the C ABI) with the CPU oracle.

Each search is compared stage by stage on the same seeded inputs:
  leaves      ranked match with the oracle's fp64 centroid scores;
  candidates  the best R by approximate score (fp32 mode: ranked match within
              tolerance; uint8 mode: ids, integer sums and fp32 scores
              bit-exact);
  final       ranked match with the oracle's exact (or approximate) scores.
Every query is checked through every stage: one whose leaf set differs from
the oracle's (a near-tie at the L-th leaf, which the ranked match allows) has
its later stages compared with the oracle run over the GPU's leaves; one whose
candidate set differs through a near-tie at the R-th candidate must return the
best k of its own candidates.  Such swaps must stay rare.
"""
import numpy as np
import pytest
import torch

from mips_ivf_centroid_b200 import datagen
from parity import compare_search

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
        "leaves-20000": W["glove"].scaled(n=100_000, d=16, num_leaves=20_000, num_leaves_to_search=40, nq=96,
                                          n_means=200, training_sample_size=100_000, code_loss="l2",
                                          threshold_T=None),
        "gemm128-vec": W["glove"].scaled(n=40_000, d=64, num_leaves=2048, num_leaves_to_search=8, nq=2048,
                                         n_means=100, training_sample_size=40_000),
        "gemm128-scalar": W["glove"].scaled(n=40_000, d=34, dims_per_block=1, num_leaves=2048,
                                            num_leaves_to_search=8, nq=2048, n_means=100,
                                            training_sample_size=40_000),
        "tc-ragged": W["glove"].scaled(n=60_000, d=36, num_leaves=3500, num_leaves_to_search=8, nq=300,
                                       n_means=150, training_sample_size=60_000, code_loss="l2", threshold_T=None),
        "tc-integer": W["bigann"].scaled(n=100_000, num_leaves=2000, num_leaves_to_search=16, nq=600,
                                         n_means=400, training_sample_size=100_000),
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
            qsel=None, options=()):
    """Search the case's queries (or the rows ``qsel`` of them) as one batch and
    check every query stage by stage against the oracle (parity.compare_search).
    ``options``: (option, value) pairs set on the index first."""
    w, X, Q, ix, arr = _workload(name)
    index = Index(ix)
    for opt, val in options:
        index.set_option(opt, val)
    Qs = Q if qsel is None else Q[qsel]
    r = compare_search(index, arr, Qs, k, L, reorder_num, lut_mode, max_leaf_mismatch=max_leaf_mismatch,
                       max_cand_mismatch=max_cand_mismatch, label=name)
    index.close()
    return r


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
                                    ("leaves-5000", 16), ("leaves-5000", 300), ("leaves-20000", 40)])
def test_many_centroids(Index, name, L):
    # more centroids than one warp holds in registers: two-stage warp selection
    # (two register widths, L <= 64), the 256-thread register form (L > 64),
    # the 1024-thread register form (4096 < centroids <= 16384), and beyond
    # that the shared-memory radix
    compare(Index, name, 10, L, 100, 0)


@pytest.mark.parametrize("L", [16, 300])
def test_many_centroids_small_batch(Index, L):
    # 40 queries over 5,000 centroids: the split top-L (segments of at most
    # 1,024 scores, then a merge) for L <= 256; beyond that the register form
    compare(Index, "leaves-5000", 10, L, 100, 0, qsel=slice(0, 40))


@pytest.mark.parametrize("name", ["gemm128-vec", "gemm128-scalar"])
def test_large_batch_centroid_tiles(Index, name):
    # 2048 queries x 2048 centroids: the 128-wide centroid tiles (float4 operand
    # loads when d % 4 == 0, scalar ones otherwise); the whole batch is searched
    # and every query checked stage by stage
    w, X, Q, ix, arr = _workload(name)
    compare(Index, name, 10, w.num_leaves_to_search, 100, 0)


def test_tensor_core_scores_ragged_tiles(Index):
    # 300 queries x 3,500 centroids x d = 36: the tensor-core centroid tiles
    # (128 x 256, K slices of 16) with a partial last tile in every dimension
    compare(Index, "tc-ragged", 10, 8, 100, 0)


def test_tensor_core_scores_integer_data_exact(Index):
    # integer coordinates 0..255 split with a zero low part, so the
    # tensor-core products and sums are exact: leaf scores bit-identical to
    # the oracle's fp64 scores
    r = compare(Index, "tc-integer", 10, 16, 200, 0, max_leaf_mismatch=0.0)
    np.testing.assert_array_equal(r["trace"]["leaf_scores"], r["oracle"]["leaf_scores"].astype(np.float32))


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
                     (Index.OPT_SCAN_CHUNK_TILES, 3), (Index.OPT_QUERY_MAJOR_SCAN, 1),
                     (Index.OPT_QUERY_MAJOR_SCAN, -1)]:
        index.set_option(opt, val)
        got = index.search(qg, 10, 64, 100, lut_mode)
        torch.testing.assert_close(got[0], ref[0], rtol=0, atol=0)
        torch.testing.assert_close(got[1], ref[1], rtol=0, atol=0)
    index.sync_status()
    index.close()


def test_speed_knobs_reject_values_out_of_range(Index):
    from mips_ivf_centroid_b200 import AhError
    w, X, Q, ix, arr = _workload("tiny")
    index = Index(ix)
    for opt, val in [(Index.OPT_QUERY_MAJOR_SCAN, 2), (Index.OPT_QUERY_MAJOR_SCAN, -2),
                     (Index.OPT_UINT8_TENSOR_CORES, 2), (Index.OPT_THRESHOLD_SAMPLE, 0),
                     (Index.OPT_SCAN_CHUNK_TILES, 2000), (99, 0)]:
        with pytest.raises(AhError) as e:
            index.set_option(opt, val)
        assert e.value.status == 1
    index.close()


@pytest.mark.skipif(not torch.cuda.is_available() or torch.cuda.device_count() < 2,
                    reason="needs two CUDA devices")
def test_search_refuses_a_device_other_than_the_index_device(Index):
    # the C entry points check the current device themselves (the binding's
    # own device guard is bypassed here by calling the library directly)
    import ctypes
    from mips_ivf_centroid_b200.index import load_library
    w, X, Q, ix, arr = _workload("glove-mini")
    index = Index(ix)
    lib = load_library()
    qg = torch.from_numpy(Q[:8]).cuda(0)
    ids = torch.empty((8, 10), dtype=torch.int32, device="cuda:0")
    sc = torch.empty((8, 10), dtype=torch.float32, device="cuda:0")
    with torch.cuda.device(1):
        torch.cuda.synchronize(1)
        free0, _ = torch.cuda.mem_get_info(1)
        st = lib.ah_search(index._h, ctypes.c_void_p(qg.data_ptr()), 8, 10, 24, 100, 0,
                           ctypes.c_void_p(ids.data_ptr()), ctypes.c_void_p(sc.data_ptr()), None)
        assert st == 1, lib.ah_last_error()
        st = lib.ah_reserve(index._h, 8, 10, 24, 100, 0)
        assert st == 1
        torch.cuda.synchronize(1)
        assert torch.cuda.mem_get_info(1)[0] == free0
    index.close()


QUERY_MAJOR_CASES = [("glove-mini", 24, 0, slice(0, 8), 0), ("glove-mini", 24, 1, slice(0, 8), 0),
                     ("glove-mini", 24, 0, None, 3), ("glove-mini-residual", 24, 0, slice(0, 8), 0),
                     ("openai-mini", 10, 0, slice(0, 5), 0), ("openai-mini", 10, 1, None, 2),
                     ("sweep-mini", 64, 0, slice(0, 3), 0), ("tiny", 1, 0, None, 0)]


@pytest.mark.parametrize("name,L,lut_mode,qsel,first", QUERY_MAJOR_CASES)
def test_query_major_scan(Index, name, L, lut_mode, qsel, first):
    # the query-major scan (CTAs split each query's tiles; chosen on its own
    # when queries seldom share a leaf) forced on: every query checked stage
    # by stage against the oracle, and the same candidates, sums and results
    # as the leaf-major scan forced on.  `first` > 0: scan phases over leaf
    # ranks [0, first), [first, 8 first), ..., so later phases start past rank 0
    prog = [(Index.OPT_PROGRESSIVE_LEAVES, first)] if first else []
    compare(Index, name, 10, L, 100, lut_mode, qsel=qsel, options=[(Index.OPT_QUERY_MAJOR_SCAN, 1)] + prog)
    w, X, Q, ix, arr = _workload(name)
    index = Index(ix)
    for opt, val in prog:
        index.set_option(opt, val)
    qg = torch.from_numpy(Q if qsel is None else Q[qsel]).cuda()
    out = {}
    for opt in (1, -1):
        index.set_option(Index.OPT_QUERY_MAJOR_SCAN, opt)
        out[opt] = index.search(qg, 10, L, 100, lut_mode, trace=True)
        index.sync_status()
    for x, y in zip(out[1][:2], out[-1][:2]):
        torch.testing.assert_close(x, y, rtol=0, atol=0)
    for key in ("cand_ids", "cand_sums", "ncand", "scanned"):
        torch.testing.assert_close(out[1][2][key], out[-1][2][key], rtol=0, atol=0)
    index.close()


@pytest.mark.parametrize("name,L", [("glove-mini", 24), ("openai-mini", 10), ("sweep-mini", 64), ("tiny-leaves", 1500)])
def test_uint8_tensor_core_scan_equals_lookup_scan(Index, name, L):
    # the int8 tensor-core scan sums the same integers as the table lookups:
    # both forms give identical candidates, sums and results (the lookup form,
    # the default, is checked against the oracle by the other tests)
    w, X, Q, ix, arr = _workload(name)
    index = Index(ix)
    qg = torch.from_numpy(Q).cuda()
    out = {}
    for opt in (0, 1):
        index.set_option(Index.OPT_UINT8_TENSOR_CORES, opt)
        out[opt] = index.search(qg, 10, L, 100, 1, trace=True)
        index.sync_status()
    for x, y in zip(out[0][:2], out[1][:2]):
        torch.testing.assert_close(x, y, rtol=0, atol=0)
    for key in ("cand_ids", "cand_sums", "ncand", "scanned"):
        torch.testing.assert_close(out[0][2][key], out[1][2][key], rtol=0, atol=0)
    index.close()
