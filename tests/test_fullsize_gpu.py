"""Parity at the five workloads' full sizes, in the benchmark's launch
configuration (the whole query batch in one search), checked against the
oracle query by query: whole batches for the tiny, GloVe-, BigANN- and
OpenAI-shaped workloads in both table modes, and on the sweep every batch
size and L (whole batches up to 256 queries, 64 queries of larger ones).  The pages' datasets are not available here;
seeded mixtures of the same shapes stand in for them (see datagen)."""
import gc

import numpy as np
import pytest
import torch

from mips_ivf_centroid_b200 import datagen

from parity import compare_search

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def Index():
    from mips_ivf_centroid_b200 import build
    build.build()
    from mips_ivf_centroid_b200 import Index as I
    return I


def _build(name):
    w = datagen.WORKLOADS[name]
    X = datagen.make_data(w)
    Q = datagen.make_queries(w)
    ix = datagen.build_index(w, X, "cuda")
    del X
    gc.collect()
    torch.cuda.empty_cache()
    return w, Q, ix, ix.numpy()


def _release(*objs):
    for o in objs:
        del o
    gc.collect()
    torch.cuda.empty_cache()


def test_tiny_full(Index):
    w, Q, ix, arr = _build("tiny")
    index = Index(ix)
    for mode in (0, 1):
        compare_search(index, arr, Q, w.k, w.num_leaves_to_search, w.reorder_num, mode)
    index.close()


def test_glove_full(Index):
    w, Q, ix, arr = _build("glove")
    index = Index(ix)
    from oracle import OracleIndex
    orc = OracleIndex(arr)
    for mode in (0, 1):                            # all 1,000 queries, both table modes
        compare_search(index, arr, Q, w.k, w.num_leaves_to_search, w.reorder_num, mode, orc=orc,
                       label=f"glove mode {mode}")
    index.close()
    _release(ix, arr, orc)


def test_bigann_full(Index):
    # integer data: centroid and exact scores are integers below 2^24, exact in fp32
    w, Q, ix, arr = _build("bigann")
    index = Index(ix)
    from oracle import OracleIndex
    orc = OracleIndex(arr)
    # all 10,000 queries (10,000 = 78 x 128 + 16: the last ones sit in the
    # partial row of 128-query centroid-score tiles)
    r = compare_search(index, arr, Q, w.k, w.num_leaves_to_search, w.reorder_num, 0, orc=orc,
                       max_leaf_mismatch=0.0, label="bigann mode 0")
    # integer scores are exact in fp32: leaf scores equal the oracle's, and
    # every final score of every query equals the oracle's exact score of the
    # same id, bit for bit
    np.testing.assert_array_equal(r["trace"]["leaf_scores"], r["oracle"]["leaf_scores"].astype(np.float32))
    inv = np.empty(w.n, np.int64)
    inv[arr["slot_ids"]] = np.arange(w.n)
    for i in range(w.nq):
        ex = orc.point_scores(Q[i], inv[r["ids"][i]])[1]
        np.testing.assert_array_equal(r["scores"][i], ex.astype(np.float32), err_msg=f"q{i} exact scores")
    compare_search(index, arr, Q, w.k, w.num_leaves_to_search, w.reorder_num, 1, orc=orc,
                   max_leaf_mismatch=0.0, label="bigann mode 1")
    index.close()
    _release(ix, arr, orc)


def test_openai_full(Index):
    w, Q, ix, arr = _build("openai")
    index = Index(ix)
    from oracle import OracleIndex
    orc = OracleIndex(arr)
    for mode in (0, 1):                            # all 10,000 queries, both table modes
        compare_search(index, arr, Q, w.k, w.num_leaves_to_search, w.reorder_num, mode, orc=orc,
                       label=f"openai mode {mode}")
    index.close()
    _release(ix, arr, orc)


def test_sweep_full(Index):
    # every sweep batch size at every L; whole batches up to 256 queries (64 of
    # them at L = 256), 64 queries spread over the larger batches; uint8
    # tables at L = 64
    w, Q, ix, arr = _build("sweep")
    index = Index(ix)
    from oracle import OracleIndex
    orc = OracleIndex(arr)
    for L in datagen.SWEEP_LEAVES:
        for nq in datagen.SWEEP_BATCHES:
            limit = 256 if L < 256 else 64
            sel = np.arange(nq) if nq <= limit else np.linspace(0, nq - 1, 64).astype(np.int64)
            for mode in ((0, 1) if L == 64 else (0,)):
                compare_search(index, arr, Q[:nq], w.k, L, w.reorder_num, mode, qsel=sel, orc=orc,
                               label=f"sweep nq {nq} L {L} mode {mode}")
    index.close()
    _release(ix, arr, orc)
