"""Index directories on the GPU: ah_save writes what numpy reads back exactly,
and an index loaded with ah_load searches bit-identically to the original."""
import os

import numpy as np
import pytest
import torch

from mips_ivf_centroid_b200 import datagen

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    from mips_ivf_centroid_b200 import build
    build.build()
    from mips_ivf_centroid_b200 import Index
    return Index


@pytest.mark.parametrize("reorder_dtype,residual", [("f32", False), ("bf16", False), ("f32", True)])
def test_save_load_round_trip(tmp_path, lib, reorder_dtype, residual):
    Index = lib
    w = datagen.WORKLOADS["glove"].scaled(n=40_000, d=64, num_leaves=200, num_leaves_to_search=12, nq=128,
                                          n_means=60, training_sample_size=40_000, reorder_dtype=reorder_dtype,
                                          residual=residual)
    X = datagen.make_data(w)
    Q = torch.from_numpy(datagen.make_queries(w)).cuda()
    ix = datagen.build_index(w, X, "cuda")
    arr = ix.numpy()
    a = Index(ix)
    a.save(str(tmp_path))
    # numpy reads back exactly the arrays the index borrows
    for k in ("centroids", "leaf_offsets", "slot_ids", "codes", "codebook", "reorder_vecs"):
        got = np.load(os.path.join(tmp_path, f"{k}.npy"))
        assert got.dtype == arr[k].dtype and got.shape == arr[k].shape, k
        np.testing.assert_array_equal(got, arr[k], err_msg=k)
    b = Index.load(str(tmp_path))
    assert (b.n, b.d, b.num_leaves, b.dims_per_block) == (w.n, w.d, w.num_leaves, w.dims_per_block)
    assert b.memory_bytes() >= sum(arr[k].nbytes for k in ("centroids", "leaf_offsets", "slot_ids", "codes",
                                                             "codebook", "reorder_vecs"))
    for mode in ((0,) if residual else (0, 1)):
        for R in (100, 0):
            ia, sa = a.search(Q, 10, w.num_leaves_to_search, R, mode)
            ib, sb = b.search(Q, 10, w.num_leaves_to_search, R, mode)
            torch.testing.assert_close(ib, ia, rtol=0, atol=0)
            torch.testing.assert_close(sb, sa, rtol=0, atol=0)
    a.sync_status()
    b.sync_status()
    b.close()
    a.close()


def test_load_errors(tmp_path, lib):
    from mips_ivf_centroid_b200 import AhError
    Index = lib
    with pytest.raises(AhError) as e:
        Index.load(str(tmp_path / "nothing_here"))
    assert e.value.status == 1
