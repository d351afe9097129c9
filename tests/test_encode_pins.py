"""Pins for the oracle's anisotropic code assignment (``oracle.encode``).

Checked against things other than the function itself:
* T <= 0 (eta = 1): the loss is the plain squared error, blocks decouple, and
  the codes are the per-block nearest centers (numpy brute force).
* One live block (the other block's 16 centers identical, so its choice
  changes nothing): the descent must reach the exhaustive argmin of the
  anisotropic loss over that block's 16 centers, with the loss computed by
  ``avq.anisotropic_loss`` and eta by ``avq.eta_ratio`` (pinned in
  test_avq_pins.py) from each point's own norm.
* Converged codes are a coordinate-wise minimum: no single-block change
  lowers the independently computed loss.
* The descent never ends above the L2 codes' loss.
* A point whose norm does not exceed T gets plain L2 codes.
"""
import numpy as np
import pytest

import oracle
from oracle import avq


def _unpack(codes, B):
    out = np.empty((codes.shape[0], B), np.int64)
    out[:, 0::2] = codes & 15
    out[:, 1::2] = codes >> 4
    return out


def _recon(cb, codes):
    B, _, dpb = cb.shape
    return np.concatenate([cb[b][codes[:, b]] for b in range(B)], axis=1).astype(np.float64)


def _data(n, d, seed, unit=True):
    rng = np.random.default_rng(seed)
    X = rng.standard_normal((n, d)).astype(np.float32)
    if unit:
        X /= np.linalg.norm(X, axis=1, keepdims=True)
    return X


def test_eta_one_gives_per_block_nearest_centers():
    X = _data(400, 16, 1)
    cb = (np.random.default_rng(2).standard_normal((8, 16, 2)) * 0.4).astype(np.float32)
    codes, used = oracle.encode(X, cb, T=0.0, passes=5)
    got = _unpack(codes, 8)
    for b in range(8):
        err = ((X[:, None, 2 * b:2 * b + 2].astype(np.float64) - cb[b][None].astype(np.float64)) ** 2).sum(-1)
        np.testing.assert_array_equal(got[:, b], np.argmin(err, axis=1))
    assert (used == 1).all()           # one pass, nothing to change


def test_single_live_block_reaches_exhaustive_argmin():
    d, T = 4, 0.3
    X = _data(500, d, 3, unit=False) * np.float32(0.8)       # norms vary: eta per point
    rng = np.random.default_rng(4)
    cb = np.empty((2, 16, 2), np.float32)
    cb[0] = rng.standard_normal((16, 2)) * 0.5
    cb[1] = rng.standard_normal((1, 2)) * 0.5                  # 16 identical centers
    norms = np.linalg.norm(X.astype(np.float64), axis=1)
    keep = norms > T * 1.01
    X, norms = X[keep], norms[keep]
    codes, used = oracle.encode(X, cb, T=T, passes=10)
    got = _unpack(codes, 2)
    eta = avq.eta_ratio(d, T, norms)
    losses = np.empty((X.shape[0], 16))
    for j in range(16):
        xt = _recon(cb, np.stack([np.full(X.shape[0], j), got[:, 1]], axis=1))
        losses[:, j] = avq.anisotropic_loss(X, xt, eta)
    want = np.argmin(losses, axis=1)
    srt = np.sort(losses, axis=1)
    clear = (srt[:, 1] - srt[:, 0]) > 1e-9 * (1 + srt[:, 0])  # skip exact near-ties
    assert clear.mean() > 0.95
    np.testing.assert_array_equal(got[clear, 0], want[clear])
    assert (got[:, 1] == 0).all()      # irrelevant block keeps its first center


@pytest.mark.parametrize("dpb", [1, 2, 4])
def test_converged_codes_are_coordinatewise_minima(dpb):
    d, T = 16, 0.2
    X = _data(300, d, 5 + dpb)
    B = d // dpb
    cb = (np.random.default_rng(6).standard_normal((B, 16, dpb)) * 0.3).astype(np.float32)
    codes, used = oracle.encode(X, cb, T=T, passes=100)
    assert (used < 100).all()          # every point converged
    got = _unpack(codes, B)
    eta = avq.eta_ratio(d, T, np.linalg.norm(X.astype(np.float64), axis=1))
    base = avq.anisotropic_loss(X, _recon(cb, got), eta)
    for b in range(B):
        for j in range(16):
            alt = got.copy()
            alt[:, b] = j
            la = avq.anisotropic_loss(X, _recon(cb, alt), eta)
            assert (la >= base - 1e-10 * (1 + base)).all(), (b, j)
    # and never worse than the L2 codes
    l2codes, _ = oracle.encode(X, cb, T=0.0, passes=0)
    l2 = avq.anisotropic_loss(X, _recon(cb, _unpack(l2codes, B)), eta)
    assert (base <= l2 + 1e-12).all()
    assert (base < l2 - 1e-9).any()    # the descent does change codes here


def test_norm_at_or_below_threshold_gets_l2_codes():
    X = _data(50, 8, 7) * np.float32(0.1)        # norms 0.1 <= T
    cb = (np.random.default_rng(8).standard_normal((4, 16, 2)) * 0.05).astype(np.float32)
    a, _ = oracle.encode(X, cb, T=0.2, passes=10)
    b, _ = oracle.encode(X, cb, T=0.0, passes=10)
    np.testing.assert_array_equal(a, b)


def test_zero_passes_is_l2_start():
    X = _data(100, 8, 9)
    cb = (np.random.default_rng(10).standard_normal((4, 16, 2)) * 0.4).astype(np.float32)
    a, used = oracle.encode(X, cb, T=0.5, passes=0)
    b, _ = oracle.encode(X, cb, T=0.0, passes=3)
    np.testing.assert_array_equal(a, b)
    assert (used == 0).all()
