"""Leaf-partitioned search, emulated on one GPU: G shard indexes (same
centroids and codebook, disjoint leaves' points) searched one after another,
their candidates merged by ah_merge_shards, must give exactly what one index
over all points gives (ids and scores bit for bit)."""
import numpy as np
import pytest
import torch

from mips_ivf_centroid_b200 import datagen

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def setup():
    from mips_ivf_centroid_b200 import build
    build.build()
    from mips_ivf_centroid_b200 import Index
    w = datagen.WORKLOADS["glove"].scaled(n=50_000, num_leaves=300, num_leaves_to_search=20, nq=256,
                                          n_means=100, training_sample_size=50_000)
    X = datagen.make_data(w)
    Q = torch.from_numpy(datagen.make_queries(w)).cuda()
    ix = datagen.build_index(w, X, "cuda")
    return w, Index, ix, Q


@pytest.mark.parametrize("G", [2, 3])
@pytest.mark.parametrize("lut_mode,reorder_num", [(0, 100), (0, 0), (1, 100), (1, 0)])
def test_merged_shards_equal_one_index(setup, G, lut_mode, reorder_num):
    from mips_ivf_centroid_b200 import shard
    w, Index, ix, Q = setup
    full = Index(ix)
    want_ids, want_scores = full.search(Q, 10, w.num_leaves_to_search, reorder_num, lut_mode)
    parts, held = [], []
    for g in range(G):
        sh = shard.shard_arrays(ix, G, g)
        assert int(sh.leaf_offsets[-1]) == sh.slot_ids.shape[0]
        index = Index(sh)
        held.append((sh, index))
        parts.append(shard.shard_candidates(index, Q, 10, w.num_leaves_to_search, reorder_num, lut_mode))
    ids, scores = shard.merge_local(parts, 10)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(ids.cpu().numpy(), want_ids.cpu().numpy())
    np.testing.assert_array_equal(scores.cpu().numpy(), want_scores.cpu().numpy())
    # the shards together scanned exactly the points one index scans
    assert sum(int(s.slot_ids.shape[0]) for s, _ in held) == w.n
    for _, index in held:
        index.close()
    full.close()


def test_merge_pads_short_lists(setup):
    from mips_ivf_centroid_b200 import merge_shards
    ids = torch.full((2, 3, 8), -1, dtype=torch.int32, device="cuda")
    approx = torch.full((2, 3, 8), float("-inf"), dtype=torch.float32, device="cuda")
    exact = torch.full((2, 3, 8), float("-inf"), dtype=torch.float32, device="cuda")
    ids[0, 0, :2] = torch.tensor([5, 7], dtype=torch.int32)
    approx[0, 0, :2] = torch.tensor([2.0, 1.0])
    exact[0, 0, :2] = torch.tensor([0.5, 0.9])
    ids[1, 0, :1] = 9
    approx[1, 0, :1] = 3.0
    exact[1, 0, :1] = 0.1
    out_ids, out_scores = merge_shards(ids, approx, exact, 4)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(out_ids.cpu().numpy()[0], [7, 5, 9, -1])
    np.testing.assert_allclose(out_scores.cpu().numpy()[0], [0.9, 0.5, 0.1, -np.inf])
    assert (out_ids.cpu().numpy()[1:] == -1).all()
