"""The Python binding checks tensor extents before it passes pointers to the
library (which receives pointers and sizes only and so cannot check them):
index arrays against one another, and the queries and caller-provided outputs
of the search entry points.  Every check here raises before any CUDA call, so
the tests run without a GPU."""
import types

import pytest
import torch

from mips_ivf_centroid_b200.index import AhError, Index, _check_index_arrays


def _arrays(n=64, d=8, nl=3, dpb=2, reorder=torch.float32):
    B = d // dpb
    return types.SimpleNamespace(
        centroids=torch.zeros((nl, d), dtype=torch.float32),
        leaf_offsets=torch.tensor([0, 20, 40, n], dtype=torch.int64)[: nl + 1].contiguous(),
        slot_ids=torch.arange(n, dtype=torch.int32),
        codes=torch.zeros((n, B // 2), dtype=torch.uint8),
        codebook=torch.zeros((B, 16, dpb), dtype=torch.float32),
        reorder_vecs=None if reorder is None else torch.zeros((n, d), dtype=reorder),
        residual=False)


def test_consistent_arrays_pass():
    assert _check_index_arrays(_arrays()) == (64, 8, 3, 2)
    assert _check_index_arrays(_arrays(reorder=torch.bfloat16)) == (64, 8, 3, 2)
    assert _check_index_arrays(_arrays(reorder=None)) == (64, 8, 3, 2)


@pytest.mark.parametrize("field,bad", [
    ("leaf_offsets", torch.zeros(3, dtype=torch.int64)),            # NL entries, not NL + 1
    ("leaf_offsets", torch.zeros(4, dtype=torch.int32)),            # wrong type
    ("slot_ids", torch.zeros(64, dtype=torch.int64)),
    ("codes", torch.zeros((64, 4), dtype=torch.uint8)),             # B bytes, not B / 2
    ("codes", torch.zeros((63, 2), dtype=torch.uint8)),             # rows != n
    ("codebook", torch.zeros((4, 16, 1), dtype=torch.float32)),     # B * dpb != d
    ("codebook", torch.zeros((4, 8, 2), dtype=torch.float32)),      # 8 centers per block
    ("codebook", torch.zeros((3, 16, 2), dtype=torch.float32)),     # B * dpb != d
    ("reorder_vecs", torch.zeros((64, 7), dtype=torch.float32)),
    ("reorder_vecs", torch.zeros((64, 8), dtype=torch.float16)),
    ("centroids", torch.zeros((3, 8), dtype=torch.float64)),
    ("codes", torch.zeros((2, 64), dtype=torch.uint8).t()),         # not contiguous
])
def test_inconsistent_arrays_are_rejected(field, bad):
    a = _arrays()
    setattr(a, field, bad)
    with pytest.raises(AhError) as e:
        _check_index_arrays(a)
    assert e.value.status == 1


def test_odd_block_count_is_rejected():
    a = _arrays(d=6, dpb=2)             # B = 3
    with pytest.raises(AhError) as e:
        _check_index_arrays(a)
    assert e.value.status == 1


def _bare_index(device):
    ix = Index.__new__(Index)
    ix.d, ix.device, ix._lib, ix._h = 8, torch.device(device), None, None
    return ix


@pytest.mark.parametrize("call", [
    lambda ix: ix.search_host(torch.zeros((4, 7)), 10, 2, 100),                           # width != d
    lambda ix: ix.search_host(torch.zeros((4, 8), dtype=torch.float64), 10, 2, 100),
    lambda ix: ix.search_host(torch.zeros((4, 8)), 10, 2, 100,
                              out_ids=torch.zeros((4, 9), dtype=torch.int32)),              # k columns
    lambda ix: ix.search_host(torch.zeros((4, 8)), 10, 2, 100,
                              out_scores=torch.zeros((3, 10))),                             # nq rows
    lambda ix: ix.search_host(torch.zeros((4, 8)), 0, 2, 100),
])
def test_host_search_checks_before_copying(call):
    with pytest.raises(AhError) as e:
        call(_bare_index("cuda:0"))
    assert e.value.status == 1


@pytest.mark.parametrize("k,L,r", [(0, 2, 100), (10, 0, 100), (10, 2, -1)])
def test_search_checks_sizes_before_allocating(k, L, r):
    with pytest.raises(AhError) as e:
        _bare_index("cpu").search(torch.zeros((4, 8)), k, L, r)
    assert e.value.status == 1


@pytest.mark.parametrize("q,ids,scores", [
    ((4, 7), (4, 3), (4, 3)),            # query width
    ((4, 8), (4, 2), (4, 3)),            # leaf ids: L columns
    ((4, 8), (4, 3), (5, 3)),            # leaf scores: nq rows
])
def test_noalloc_checks_output_extents(q, ids, scores):
    ix = _bare_index("cpu")
    with pytest.raises(AhError) as e:
        ix.search_leaves_noalloc(torch.zeros(q), 3, torch.zeros(ids, dtype=torch.int32), torch.zeros(scores))
    assert e.value.status == 1
