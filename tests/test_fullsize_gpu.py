"""Parity at the five workloads' full sizes, in the benchmark's launch
configuration (the whole query batch in one search), checked against the
oracle on a sample of queries.  The pages' datasets are not available here;
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
    sel = np.arange(0, w.nq, 5)                    # 200 of the 1,000 queries
    compare_search(index, arr, Q, w.k, w.num_leaves_to_search, w.reorder_num, 0, qsel=sel)
    compare_search(index, arr, Q, w.k, w.num_leaves_to_search, w.reorder_num, 1, qsel=sel[:100])
    index.close()
    _release(ix, arr)


def test_bigann_full(Index):
    # integer data: centroid and exact scores are integers below 2^24, exact in fp32
    w, Q, ix, arr = _build("bigann")
    index = Index(ix)
    # 40 of the 10,000 queries, and the last one: 10,000 = 78 x 128 + 16, so it
    # sits in the partial row of 128-query centroid-score tiles
    sel = np.r_[np.arange(0, w.nq, 250), w.nq - 1]
    r = compare_search(index, arr, Q, w.k, w.num_leaves_to_search, w.reorder_num, 0, qsel=sel,
                       max_leaf_mismatch=0.0)
    same = (r["ids"] == r["oracle"]["ids"]).all(axis=1)
    np.testing.assert_array_equal(r["scores"][same], r["oracle"]["scores"][same].astype(np.float32))
    np.testing.assert_array_equal(r["trace"]["leaf_scores"], r["oracle"]["leaf_scores"].astype(np.float32))
    index.close()
    _release(ix, arr)


def test_openai_full(Index):
    w, Q, ix, arr = _build("openai")
    index = Index(ix)
    sel = np.arange(0, w.nq, 400)                  # 25 of the 10,000 queries
    compare_search(index, arr, Q, w.k, w.num_leaves_to_search, w.reorder_num, 0, qsel=sel)
    index.close()
    _release(ix, arr)


def test_sweep_full(Index):
    w, Q, ix, arr = _build("sweep")
    index = Index(ix)
    from oracle import OracleIndex
    orc = OracleIndex(arr)
    for L in datagen.SWEEP_LEAVES:
        for nq in (1, 256, 16_384):
            sel = np.arange(0, nq, max(1, nq // 8))[:8]
            compare_search(index, arr, Q[:nq], w.k, L, w.reorder_num, 0, qsel=sel, orc=orc)
    index.close()
    _release(ix, arr, orc)
