"""The no-allocation partition entry point (ah_search_leaves_noalloc).

It serves callers that cannot allocate device memory on the call path (a
serving process whose memory another allocator reserved up front, or a loop
that cannot take cudaMalloc's implicit synchronisation).  Its scratch lives in
a fixed device array inside the library, whose address is looked up when the
index is built.  Checked here, with each of the top-L selection forms (one
warp per query up to 1,024 centroids, the two-stage warp form up to 4,096, the
1,024-thread register form up to 16,384, the shared-memory radix beyond): two
calls in a row give the leaves the regular
traced search reports and the oracle's leaves (ranked match), device memory is
unchanged by the calls, and an over-size batch is rejected before anything
runs.  The file is named to be collected last.
"""
import numpy as np
import pytest
import torch

from parity import ranked_match

pytestmark = pytest.mark.gpu

CASES = {
    # name: (num_leaves, num_leaves_to_search, n, d, nq)
    "warp-400": (400, 16, 40_000, 100, 128),
    "two-stage-1500": (1500, 40, 30_000, 32, 128),
    "register-5000": (5000, 16, 50_000, 32, 128),
    "radix-20000": (20_000, 24, 100_000, 16, 64),
}


@pytest.fixture(scope="module", params=sorted(CASES))
def setup(request):
    from mips_ivf_centroid_b200 import build, datagen
    build.build()
    from mips_ivf_centroid_b200 import Index
    nl, L, n, d, nq = CASES[request.param]
    w = datagen.WORKLOADS["glove"].scaled(n=n, d=d, num_leaves=nl, num_leaves_to_search=L, nq=nq,
                                          n_means=80, training_sample_size=n, code_loss="l2", threshold_T=None)
    X = datagen.make_data(w)
    Q = datagen.make_queries(w)
    ix = datagen.build_index(w, X, "cuda")
    index = Index(ix)
    yield w, index, torch.from_numpy(Q).cuda(), ix.numpy()
    index.close()


def test_noalloc_leaves_match_traced_search_and_oracle_twice(setup):
    from oracle import OracleIndex
    w, index, qg, arr = setup
    L = w.num_leaves_to_search
    _, _, tr = index.search(qg, 10, L, 100, trace=True)
    ref_ids = tr["leaf_ids"].cpu().numpy()
    ref_scores = tr["leaf_scores"].cpu().numpy()
    orc = OracleIndex(arr)
    Q = qg.cpu().numpy()
    o = orc.search(Q, 10, L, 0)
    for _ in range(2):
        ids = torch.full((w.nq, L), -7, dtype=torch.int32, device="cuda")
        scores = torch.full((w.nq, L), float("nan"), dtype=torch.float32, device="cuda")
        index.search_leaves_noalloc(qg, L, ids, scores)
        index.sync_status()
        gi, gs = ids.cpu().numpy(), scores.cpu().numpy()
        np.testing.assert_array_equal(gi, ref_ids)
        np.testing.assert_allclose(gs, ref_scores, rtol=0, atol=2e-5)
        for i in range(w.nq):
            cs = orc.centroid_scores(Q[i])
            ranked_match(gi[i], gs[i], o["leaves"][i], o["leaf_scores"][i], lambda g: cs[g], f"q{i} leaves")


def test_noalloc_calls_leave_device_memory_unchanged(setup):
    w, index, qg, arr = setup
    L = w.num_leaves_to_search
    ids = torch.empty((w.nq, L), dtype=torch.int32, device="cuda")
    scores = torch.empty((w.nq, L), dtype=torch.float32, device="cuda")
    index.search(qg, 10, L, 0)                 # the same kernels have run once in this process
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    for _ in range(2):
        index.search_leaves_noalloc(qg, L, ids, scores)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0, f"device free memory changed by {free0 - free1} bytes"


def test_noalloc_rejects_batches_beyond_the_scratch(setup):
    from mips_ivf_centroid_b200 import AhError
    w, index, qg, arr = setup
    big = (8 << 20) // (4 * w.num_leaves) + 1          # nq * num_leaves scores no longer fit
    q = torch.zeros((big, w.d), dtype=torch.float32, device="cuda")
    ids = torch.empty((big, 4), dtype=torch.int32, device="cuda")
    sc = torch.empty((big, 4), dtype=torch.float32, device="cuda")
    with pytest.raises(AhError) as e:
        index.search_leaves_noalloc(q, 4, ids, sc)
    assert e.value.status == 2
    index.sync_status()
