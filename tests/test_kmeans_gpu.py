"""GPU partition training (ah_kmeans_assign, ah_kmeans_update) against the
oracle's restatement: assignments, distances and new centroids bit-identical
(same fp64 operations in the same order on both sides)."""
import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def km():
    from mips_ivf_centroid_b200 import build
    build.build()
    from mips_ivf_centroid_b200 import kmeans_assign, kmeans_update
    return kmeans_assign, kmeans_update


def _data(n, d, k, seed):
    rng = np.random.default_rng(seed)
    C = rng.standard_normal((k, d)).astype(np.float32)
    X = (C[rng.integers(0, k, n)] + 0.5 * rng.standard_normal((n, d))).astype(np.float32)
    return X, C


@pytest.mark.parametrize("n,d,k", [(5000, 100, 200), (3001, 37, 65), (2000, 1536, 40), (777, 8, 1000)])
def test_assign_and_update_match_oracle(km, n, d, k):
    assign, update = km
    X, C = _data(n, d, k, seed=n + d + k)
    C[min(3, k - 1)] = C[0]                      # duplicate centroid: exact ties
    a_o, dist_o = oracle.kmeans_assign(X, C)
    a_g, dist_g = assign(torch.from_numpy(X).cuda(), torch.from_numpy(C).cuda())
    torch.cuda.synchronize()
    np.testing.assert_array_equal(a_g.cpu().numpy(), a_o)
    np.testing.assert_array_equal(dist_g.cpu().numpy(), dist_o)
    a_o = a_o.copy()
    a_o[a_o == 1] = 2                             # centroid 1 empty
    C_o, cnt_o = oracle.kmeans_update(X, a_o, C)
    C_g, cnt_g = update(torch.from_numpy(X).cuda(), torch.from_numpy(a_o).cuda(), torch.from_numpy(C).cuda())
    torch.cuda.synchronize()
    np.testing.assert_array_equal(cnt_g.cpu().numpy(), cnt_o)
    np.testing.assert_array_equal(C_g.cpu().numpy(), C_o)


def test_lloyd_iterations_match(km):
    assign, update = km
    X, C = _data(20000, 64, 300, 7)
    Xg, Cg = torch.from_numpy(X).cuda(), torch.from_numpy(C).cuda()
    Co = C
    for _ in range(3):
        a, _ = assign(Xg, Cg)
        Cg, _ = update(Xg, a, Cg)
        ao, _ = oracle.kmeans_assign(X, Co)
        Co, _ = oracle.kmeans_update(X, ao, Co)
    np.testing.assert_array_equal(Cg.cpu().numpy(), Co)


def test_kmeans_errors(km):
    from mips_ivf_centroid_b200 import AhError
    assign, update = km
    X, C = _data(10, 8, 4, 1)
    with pytest.raises(AhError) as e:
        assign(torch.from_numpy(X).cuda(), torch.from_numpy(C[:, :4].copy()).cuda())
    assert e.value.status == 1
    Xw = torch.zeros((4, 7000), dtype=torch.float32, device="cuda")
    with pytest.raises(AhError) as e:
        update(Xw, torch.zeros(4, dtype=torch.int32, device="cuda"), torch.zeros((2, 7000), device="cuda"))
    assert e.value.status == 2
