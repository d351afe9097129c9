"""Pins for the training-side formulas (oracle/avq.py) and the input generator.

Source: ScaNN blog post, "The loss in one paragraph" and "Training an
anisotropic codebook yourself".
"""
from fractions import Fraction

import numpy as np
import pytest
import torch

from mips_ivf_centroid_b200 import datagen
from oracle import avq


def test_eta_closed_forms():
    # unit norm: eta = (d-1) T^2 / (1 - T^2)
    # d = 100, T = 1/5:  99 * (1/25) / (24/25) = 99/24 = 4.125
    assert avq.eta_ratio(100, 0.2) == pytest.approx(float(Fraction(99, 24)), rel=1e-15)
    # d = 1536, T = 1/20: 1535 * (1/400) / (399/400) = 1535/399
    assert avq.eta_ratio(1536, 0.05) == pytest.approx(float(Fraction(1535, 399)), rel=1e-15)
    # the generator's workloads carry the same values
    assert datagen.WORKLOADS["glove"].eta == pytest.approx(99 / 24, rel=1e-15)
    assert datagen.WORKLOADS["openai"].eta == pytest.approx(1535 / 399, rel=1e-15)
    # non-unit norm: T/||x|| enters squared
    assert avq.eta_ratio(11, 1.0, norm=2.0) == pytest.approx(10 * 0.25 / 0.75, rel=1e-15)
    with pytest.raises(ValueError):
        avq.eta_ratio(10, 1.0, norm=1.0)


def test_loss_equals_weighted_parallel_plus_perpendicular():
    # (eta-1) r_par^2 + ||r||^2 == eta ||r_par||^2 + ||r_perp||^2, with r_par and
    # r_perp formed explicitly as the projection onto x and its remainder.
    rng = np.random.default_rng(0)
    x = rng.standard_normal((50, 9))
    xt = x + 0.3 * rng.standard_normal((50, 9))
    for eta in (0.3, 1.0, 4.125, 37.0):
        r = x - xt
        xhat = x / np.linalg.norm(x, axis=1, keepdims=True)
        r_par = np.einsum("ij,ij->i", r, xhat)[:, None] * xhat
        r_perp = r - r_par
        assert np.allclose(np.einsum("ij,ij->i", r_perp, xhat), 0.0, atol=1e-12)
        want = eta * np.sum(r_par ** 2, 1) + np.sum(r_perp ** 2, 1)
        np.testing.assert_allclose(avq.anisotropic_loss(x, xt, eta), want, rtol=1e-12, atol=1e-12)


def test_eta_one_center_update_is_mean():
    rng = np.random.default_rng(1)
    m = rng.standard_normal((23, 7))
    np.testing.assert_allclose(avq.center_update(m, 1.0), m.mean(axis=0), rtol=1e-12, atol=1e-12)


def test_center_update_minimises_member_loss():
    # The closed form is the minimiser of the members' summed anisotropic loss.
    rng = np.random.default_rng(2)
    m = rng.standard_normal((30, 6))
    m /= np.linalg.norm(m, axis=1, keepdims=True)
    eta = 4.125
    c = avq.center_update(m, eta)

    def total(cc):
        return avq.anisotropic_loss(m, np.repeat(cc[None, :], m.shape[0], 0), eta).sum()

    base = total(c)
    for _ in range(50):
        v = rng.standard_normal(6) * 1e-3
        assert total(c + v) > base and total(c - v) > base
    # and it differs from the plain mean when eta != 1
    assert np.linalg.norm(c - m.mean(0)) > 1e-6


def test_anisotropic_kmeans_at_eta_one_is_lloyd():
    # eta = 1 when T^2 = 1/d for unit data: one iteration equals one k-means step.
    rng = np.random.default_rng(3)
    X = rng.standard_normal((120, 4))
    X /= np.linalg.norm(X, axis=1, keepdims=True)
    T = 1 / np.sqrt(4)
    assert avq.eta_ratio(4, T) == pytest.approx(1.0)
    C, a = avq.anisotropic_kmeans(X, 5, T, iters=1, seed=7)
    C0 = X[np.random.default_rng(7).permutation(120)[:5]]     # the documented initial centers
    d2 = ((X[:, None, :] - C0[None]) ** 2).sum(-1)
    a_ref = d2.argmin(1)
    np.testing.assert_array_equal(a, a_ref)
    for j in range(5):
        if (a_ref == j).any():
            np.testing.assert_allclose(C[j], X[a_ref == j].mean(0), rtol=1e-9, atol=1e-12)


def test_generator_anisotropic_codes_never_worse_than_l2():
    # Descent invariant of the generator's coordinate descent, measured with the
    # oracle's loss: per point, loss(anisotropic codes) <= loss(L2 codes).
    w = datagen.Workload(name="aniso-mini", n=3000, d=20, dims_per_block=2, num_leaves=1,
                         num_leaves_to_search=1, nq=4, k=10, reorder_num=0, n_means=6,
                         sigma=0.4, code_loss="anisotropic", threshold_T=0.2,
                         training_sample_size=3000)
    X = datagen.make_data(w)
    ix = datagen.build_index(w, X, "cpu")
    Xs = X[ix.slot_ids.numpy()]
    cb = ix.codebook.numpy().astype(np.float64)
    B = w.blocks
    aniso = datagen.unpack_codes(ix.codes).numpy().astype(np.int64)
    l2 = datagen._l2_codes(torch.from_numpy(Xs), ix.codebook).numpy()
    rec = lambda c: cb[np.arange(B)[None, :], c].reshape(c.shape[0], -1)
    la = avq.anisotropic_loss(Xs, rec(aniso), w.eta)
    ll = avq.anisotropic_loss(Xs, rec(l2), w.eta)
    assert (la <= ll + 1e-12).all()
    assert (la < ll - 1e-9).mean() > 0.05        # it actually moves codes


def test_generator_l2_codes_are_nearest_centers():
    w = datagen.WORKLOADS["tiny"].scaled(n=2000, nq=5)
    X = datagen.make_data(w)
    ix = datagen.build_index(w, X, "cpu")
    Xs = X[ix.slot_ids.numpy()].astype(np.float64)
    cb = ix.codebook.numpy().astype(np.float64)
    codes = datagen.unpack_codes(ix.codes).numpy()
    B, dpb = cb.shape[0], cb.shape[2]
    for b in range(B):
        d2 = ((Xs[:, None, b * dpb:(b + 1) * dpb] - cb[b][None]) ** 2).sum(-1)
        chosen = d2[np.arange(len(Xs)), codes[:, b]]
        assert (chosen <= d2.min(1) + 1e-6).all()


def test_point_eta_rule():
    # eta_ratio at each row's norm; 1 where the weight is undefined
    rng = np.random.default_rng(4)
    X = rng.standard_normal((6, 100))
    X /= np.linalg.norm(X, axis=1, keepdims=True)
    np.testing.assert_allclose(avq.point_eta(X, 0.2), 99 / 24, rtol=1e-14)
    X2 = X * np.array([1, 2, 3, 0.5, 0.1, 0.0])[:, None]       # norms 1, 2, 3, 0.5, 0.1, 0
    e = avq.point_eta(X2, 0.2)
    np.testing.assert_allclose(e[:4], [99 * s / (1 - s) for s in (0.04, 0.01, 0.04 / 9, 0.16)], rtol=1e-13)
    assert e[4] == 1.0 and e[5] == 1.0                         # T above the norm; a zero row
    np.testing.assert_array_equal(avq.point_eta(X2, 0.0), 1.0)
    np.testing.assert_array_equal(avq.point_eta(X2, -1.0), 1.0)


def test_center_updates_at_eta_one_are_member_means():
    # T <= 0: every eta is 1 and each center is the plain mean of its members
    # (numpy); a center without members keeps its old value; assignments
    # outside [0, nl) belong to no center
    rng = np.random.default_rng(5)
    X = rng.standard_normal((300, 8))
    assign = rng.integers(-1, 7, 300)           # -1 and center 6 (of 6) are outside; center 5 left empty
    assign[assign == 5] = 4
    C_old = rng.standard_normal((6, 8))
    C, counts = avq.center_updates(X, assign, C_old, 0.0)
    for c in range(6):
        mem = X[assign == c]
        assert counts[c] == mem.shape[0]
        if mem.shape[0]:
            np.testing.assert_allclose(C[c], mem.mean(0), rtol=1e-12, atol=1e-13)
        else:
            np.testing.assert_array_equal(C[c], C_old[c])


def test_center_updates_minimise_each_members_loss():
    # T > 0: each center minimises its members' summed anisotropic loss, with
    # eta per member from its own norm
    rng = np.random.default_rng(6)
    X = rng.standard_normal((200, 6)) * rng.uniform(0.5, 2.0, (200, 1))
    assign = rng.integers(0, 3, 200)
    C, _ = avq.center_updates(X, assign, np.zeros((3, 6)), 0.3)
    for c in range(3):
        mem = X[assign == c]
        eta = avq.point_eta(mem, 0.3)
        assert (eta != 1.0).all()

        def total(cc):
            return avq.anisotropic_loss(mem, np.repeat(cc[None, :], mem.shape[0], 0), eta).sum()

        base = total(C[c])
        for _ in range(30):
            v = rng.standard_normal(6) * 1e-3
            assert total(C[c] + v) > base and total(C[c] - v) > base
