"""The seeded input generator: shapes, determinism and index-array invariants."""
import numpy as np
import torch

from mips_ivf_centroid_b200 import datagen


def _small():
    return datagen.WORKLOADS["glove"].scaled(n=5000, num_leaves=40, nq=30, n_means=25,
                                             training_sample_size=5000)


def test_shapes_and_invariants():
    w = _small()
    X, Q, ix = datagen.make_workload(w)
    assert X.shape == (w.n, w.d) and X.dtype == np.float32
    assert Q.shape == (w.nq, w.d)
    np.testing.assert_allclose(np.linalg.norm(X, axis=1), 1.0, atol=1e-5)
    a = ix.numpy()
    assert a["centroids"].shape == (w.num_leaves, w.d)
    off = a["leaf_offsets"]
    assert off[0] == 0 and off[-1] == w.n and (np.diff(off) >= 0).all()
    assert np.array_equal(np.sort(a["slot_ids"]), np.arange(w.n))
    assert a["codes"].shape == (w.n, w.code_bytes) and a["codes"].dtype == np.uint8
    assert a["codebook"].shape == (w.blocks, 16, w.dims_per_block)
    np.testing.assert_array_equal(a["reorder_vecs"], X[a["slot_ids"]])
    # every slot sits in the leaf of its nearest centroid
    Xs = X[a["slot_ids"]].astype(np.float64)
    C = a["centroids"].astype(np.float64)
    leaf = np.repeat(np.arange(w.num_leaves), np.diff(off))
    d2 = ((Xs[:, None, :] - C[None]) ** 2).sum(-1)
    assert (d2[np.arange(w.n), leaf] <= d2.min(1) + 1e-5).all()
    # queries are fresh draws, not indexed rows
    assert (np.abs(Q @ X.T).max(axis=1) < 0.9999).all()


def test_deterministic():
    w = _small()
    X1, Q1 = datagen.make_data(w), datagen.make_queries(w)
    X2, Q2 = datagen.make_data(w), datagen.make_queries(w)
    np.testing.assert_array_equal(X1, X2)
    np.testing.assert_array_equal(Q1, Q2)
    a1 = datagen.build_index(w, X1).numpy()
    a2 = datagen.build_index(w, X2).numpy()
    for k in ("centroids", "leaf_offsets", "slot_ids", "codes", "codebook"):
        np.testing.assert_array_equal(a1[k], a2[k])


def test_integer_workload_values():
    w = datagen.WORKLOADS["bigann"].scaled(n=3000, num_leaves=20, nq=10, n_means=15,
                                           training_sample_size=3000)
    X = datagen.make_data(w)
    assert X.min() >= 0 and X.max() <= 255 and np.array_equal(X, np.rint(X))
    Q = datagen.make_queries(w)
    assert np.array_equal(Q, np.rint(Q))


def test_pack_roundtrip_and_bf16_copy():
    c = torch.randint(0, 16, (100, 12))
    np.testing.assert_array_equal(datagen.unpack_codes(datagen.pack_codes(c)).numpy(), c.numpy())
    p = datagen.pack_codes(c).numpy()
    assert (p[:, 0] & 0x0F == c[:, 0].numpy()).all() and (p[:, 0] >> 4 == c[:, 1].numpy()).all()
    w = _small().scaled(reorder_dtype="bf16")
    X = datagen.make_data(w)
    a = datagen.build_index(w, X).numpy()
    assert a["reorder_dtype"] == "bf16"
    want = torch.from_numpy(X[a["slot_ids"]]).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(a["reorder_vecs"], want)
