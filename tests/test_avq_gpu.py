"""GPU anisotropic center update (ah_avq_update) against the oracle's closed
form (oracle/avq.py center_updates), ScaNN blog post, "Training an anisotropic
codebook yourself" (Theorem 4.2 form).

The GPU solves each center's system by conjugate gradients in fp64 and rounds
the result to float; the oracle solves it by LU in fp64.  Both are accurate to
about the condition number (at most max(eta)/min(eta, 1), here below 5) times
the fp64 rounding unit (and the CG stopping tolerance), so the float results
agree to within 2 units in the last place of float32, plus 1e-12 of the
center's norm for components far smaller than it.
"""
import numpy as np
import pytest
import torch

from mips_ivf_centroid_b200 import datagen
from oracle import avq

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    from mips_ivf_centroid_b200 import build
    build.build()
    from mips_ivf_centroid_b200 import avq_update
    return avq_update


def _case(n, d, nl, T, sigma, seed):
    w = datagen.Workload(name="avq", n=n, d=d, dims_per_block=2, num_leaves=nl, num_leaves_to_search=1, nq=1,
                         k=1, reorder_num=0, n_means=nl, sigma=sigma, data_seed=seed)
    X = datagen.make_data(w)                                   # unit-norm mixture rows
    rng = np.random.default_rng(seed + 1)
    C0 = X[rng.choice(n, nl, replace=False)].astype(np.float64)
    d2 = (X.astype(np.float64) ** 2).sum(1)[:, None] - 2 * X.astype(np.float64) @ C0.T
    assign = d2.argmin(1).astype(np.int32)                     # nearest of the starting centers
    return X, assign, C0.astype(np.float32)


def _check(avq_update, X, assign, C_old, T):
    dev = "cuda"
    C, counts, iters = avq_update(torch.from_numpy(X).to(dev), torch.from_numpy(assign).to(dev),
                                  torch.from_numpy(C_old).to(dev), T)
    torch.cuda.synchronize()
    C, counts, iters = C.cpu().numpy(), counts.cpu().numpy(), iters.cpu().numpy()
    Co, co = avq.center_updates(X, assign, C_old, T)
    np.testing.assert_array_equal(counts, co)
    ref = Co.astype(np.float32)
    ulp = np.spacing(np.abs(ref).astype(np.float32)).astype(np.float64)
    err = np.abs(C.astype(np.float64) - Co)
    # the float rounding of each result, plus a norm-wise bound on the two fp64
    # solutions' difference (condition number times the CG stopping tolerance
    # 1e-14, for components far smaller than the row's norm)
    bound = 2 * ulp + 1e-12 * np.linalg.norm(Co, axis=1, keepdims=True)
    assert (err <= bound).all(), f"max error {err.max():.3g}, in ulps {(err / ulp).max():.2f}"
    assert (iters[co > 0] < 200).all() and (iters[co == 0] == 0).all()
    return C, iters


@pytest.mark.parametrize("n,d,nl,T", [(20_000, 100, 20, 0.2), (6_000, 1536, 6, 0.05)])
def test_avq_update_matches_oracle(lib, n, d, nl, T):
    X, assign, C_old = _case(n, d, nl, T, 0.4, 11)
    _, iters = _check(lib, X, assign, C_old, T)
    assert iters.max() > 3                                     # eta != 1: a real solve, not one step


def test_avq_update_eta_one_is_mean_and_empty_keeps_old(lib):
    X, assign, C_old = _case(5_000, 64, 12, 0.0, 0.4, 21)
    assign = assign.copy()
    assign[assign == 3] = -1                                   # center 3: no members
    assign[::97] = 12                                          # outside [0, nl): no center
    C, _ = _check(lib, X, assign, C_old, 0.0)
    np.testing.assert_array_equal(C[3], C_old[3])
    for c in (0, 5):
        np.testing.assert_allclose(C[c], X[assign == c].astype(np.float64).mean(0), rtol=0, atol=1e-6)


def test_avq_update_is_repeatable(lib):
    X, assign, C_old = _case(8_000, 100, 8, 0.2, 0.4, 31)
    dev = "cuda"
    args = (torch.from_numpy(X).to(dev), torch.from_numpy(assign).to(dev), torch.from_numpy(C_old).to(dev), 0.2)
    a = lib(*args)[0]
    b = lib(*args)[0]
    torch.testing.assert_close(a, b, rtol=0, atol=0)
