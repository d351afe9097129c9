"""The no-allocation partition entry point (ah_search_leaves_noalloc).

It serves callers that cannot allocate device memory on the call path (a
serving process whose memory another allocator reserved up front, or a loop
that cannot take cudaMalloc's implicit synchronisation).  Its scratch lives in
a fixed device array inside the library.  Checked here: two calls in a row give
the leaves the regular traced search reports, and an over-size batch is
rejected before anything runs.  The file is named to be collected last.
"""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def setup():
    from mips_ivf_centroid_b200 import build, datagen
    build.build()
    from mips_ivf_centroid_b200 import Index
    w = datagen.WORKLOADS["glove"].scaled(n=40_000, num_leaves=400, num_leaves_to_search=16, nq=200,
                                          n_means=80, training_sample_size=40_000)
    X = datagen.make_data(w)
    Q = datagen.make_queries(w)
    ix = datagen.build_index(w, X, "cuda")
    index = Index(ix)
    yield w, index, torch.from_numpy(Q).cuda()
    index.close()


def test_noalloc_leaves_match_traced_search_twice(setup):
    w, index, qg = setup
    L = w.num_leaves_to_search
    _, _, tr = index.search(qg, 10, L, 100, trace=True)
    ref_ids = tr["leaf_ids"].cpu().numpy()
    ref_scores = tr["leaf_scores"].cpu().numpy()
    for _ in range(2):
        ids = torch.full((w.nq, L), -7, dtype=torch.int32, device="cuda")
        scores = torch.full((w.nq, L), float("nan"), dtype=torch.float32, device="cuda")
        index.search_leaves_noalloc(qg, L, ids, scores)
        index.sync_status()
        np.testing.assert_array_equal(ids.cpu().numpy(), ref_ids)
        np.testing.assert_allclose(scores.cpu().numpy(), ref_scores, rtol=0, atol=2e-5)


def test_noalloc_rejects_batches_beyond_the_scratch(setup):
    from mips_ivf_centroid_b200 import AhError
    w, index, qg = setup
    big = (8 << 20) // (4 * w.num_leaves) + 1          # nq * num_leaves scores no longer fit
    q = torch.zeros((big, w.d), dtype=torch.float32, device="cuda")
    ids = torch.empty((big, 4), dtype=torch.int32, device="cuda")
    sc = torch.empty((big, 4), dtype=torch.float32, device="cuda")
    with pytest.raises(AhError) as e:
        index.search_leaves_noalloc(q, 4, ids, sc)
    assert e.value.status == 2
    index.sync_status()
