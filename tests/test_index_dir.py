"""Index directories: the .npy layout ah_inspect / ah_load read (no GPU here).

The directory is written with numpy's own np.save, so the library's header
parser is checked against numpy's writer; a saved directory written by the
library is read back with numpy in the GPU test."""
import os

import numpy as np
import pytest

from mips_ivf_centroid_b200 import datagen


def _write(path, arr, reorder="f32", residual=None):
    os.makedirs(path, exist_ok=True)
    for k in ("centroids", "leaf_offsets", "slot_ids", "codes", "codebook"):
        np.save(os.path.join(path, f"{k}.npy"), arr[k])
    if reorder is not None:
        np.save(os.path.join(path, "reorder_vecs.npy"), arr["reorder_vecs"])
    with open(os.path.join(path, "ah_index.txt"), "w") as f:
        f.write(f"ah-index 1\nreorder_dtype {reorder or 'none'}\n")
        if residual is not None:
            f.write(f"residual {residual}\n")


@pytest.fixture(scope="module")
def arrays():
    w = datagen.WORKLOADS["glove"].scaled(n=3000, d=20, num_leaves=30, nq=5, n_means=10,
                                          training_sample_size=3000)
    X = datagen.make_data(w)
    return w, datagen.build_index(w, X, "cpu").numpy()


def _status(fn):
    from mips_ivf_centroid_b200.index import AhError
    with pytest.raises(AhError) as e:
        fn()
    return e.value.status, str(e.value)


def test_inspect_reads_numpy_written_directory(tmp_path, arrays):
    from mips_ivf_centroid_b200 import inspect
    w, arr = arrays
    _write(tmp_path, arr)
    info = inspect(str(tmp_path))
    assert info == dict(n=3000, d=20, num_leaves=30, dims_per_block=2, reorder_dtype="f32", residual=False)


def test_inspect_bf16_and_no_reorder_copy(tmp_path, arrays):
    from mips_ivf_centroid_b200 import inspect
    w, arr = arrays
    a = dict(arr)
    bits = (arr["reorder_vecs"].view(np.uint32) >> 16).astype(np.uint16)
    a["reorder_vecs"] = bits
    _write(tmp_path / "b", a, reorder="bf16")
    assert inspect(str(tmp_path / "b"))["reorder_dtype"] == "bf16"
    _write(tmp_path / "n", arr, reorder=None)
    assert inspect(str(tmp_path / "n"))["reorder_dtype"] is None


def test_inspect_reads_format_2_headers(tmp_path, arrays):
    # numpy writes format 2.0 (4-byte header length) when asked; the reader takes both
    from mips_ivf_centroid_b200 import inspect
    w, arr = arrays
    _write(tmp_path, arr)
    for k in ("centroids", "codes", "reorder_vecs"):
        with open(os.path.join(tmp_path, f"{k}.npy"), "wb") as f:
            np.lib.format.write_array(f, arr[k], version=(2, 0))
    assert inspect(str(tmp_path))["n"] == 3000


def test_inspect_residual_line(tmp_path, arrays):
    from mips_ivf_centroid_b200 import inspect
    w, arr = arrays
    _write(tmp_path / "r1", arr, residual=1)
    assert inspect(str(tmp_path / "r1"))["residual"] is True
    _write(tmp_path / "r0", arr, residual=0)
    assert inspect(str(tmp_path / "r0"))["residual"] is False
    _write(tmp_path / "bad", arr, residual=2)
    st, msg = _status(lambda: inspect(str(tmp_path / "bad")))
    assert st == 1 and "ah_index.txt" in msg


@pytest.mark.parametrize("case", ["missing", "dtype", "offsets", "codes", "truncated", "fortran", "meta",
                                  "bf16_as_f32", "codebook", "huge_shape"])
def test_inspect_rejects_malformed(tmp_path, arrays, case):
    from mips_ivf_centroid_b200 import inspect
    w, arr = arrays
    a = dict(arr)
    reorder = "f32"
    if case == "dtype":
        a["slot_ids"] = arr["slot_ids"].astype(np.int64)
    elif case == "offsets":
        a["leaf_offsets"] = arr["leaf_offsets"][:-1]
    elif case == "codes":
        a["codes"] = arr["codes"][:, :-1]
    elif case == "fortran":
        a["centroids"] = np.asfortranarray(arr["centroids"])
    elif case == "bf16_as_f32":
        reorder = "bf16"                       # but the file holds <f4
    elif case == "codebook":
        a["codebook"] = arr["codebook"][:, :8]
    _write(tmp_path, a, reorder=reorder)
    if case == "missing":
        os.remove(tmp_path / "codes.npy")
    elif case == "truncated":
        p = tmp_path / "reorder_vecs.npy"
        data = p.read_bytes()
        p.write_bytes(data[:-100])
    elif case == "meta":
        (tmp_path / "ah_index.txt").write_text("something else\n")
    elif case == "huge_shape":
        # 2^33 x 2^33 elements: the element count wraps to 0 in int64, so only
        # a bound on the product keeps the length check meaningful
        with open(tmp_path / "reorder_vecs.npy", "wb") as f:
            np.lib.format.write_array_header_1_0(f, {"descr": "<f4", "fortran_order": False,
                                                     "shape": (2 ** 33, 2 ** 33)})
            f.write(b"\0" * 64)
    st, msg = _status(lambda: inspect(str(tmp_path)))
    assert st == 1, msg
    if case == "huge_shape":
        assert "shape too large" in msg, msg
    want = {"missing": "codes.npy", "dtype": "slot_ids.npy", "offsets": "leaf_offsets.npy", "codes": "codes.npy",
            "truncated": "reorder_vecs.npy", "fortran": "centroids.npy", "meta": "ah_index.txt",
            "bf16_as_f32": "reorder_vecs.npy", "codebook": "codebook.npy", "huge_shape": "reorder_vecs.npy"}[case]
    assert want in msg, msg
