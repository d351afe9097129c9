"""The C ABI library builds for sm_100a, loads without a GPU, exports every
entry point include/ah.h declares, and rejects bad arguments on the host
before touching CUDA."""
import ctypes
import os
import re

import pytest

from mips_ivf_centroid_b200 import build as ahbuild
from mips_ivf_centroid_b200 import index as ahindex

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "ah.h")).read()
    return sorted(set(re.findall(r"AH_API\s+[\w\s\*]*?\b(ah_\w+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    ahbuild.build()
    return ahindex.load_library()


def test_header_declares_the_boundary():
    names = _declared()
    for need in ("ah_build_index_views", "ah_search", "ah_destroy", "ah_status_string"):
        assert need in names
    assert len(names) >= 14


def test_every_declared_symbol_is_exported(lib):
    for name in _declared():
        assert hasattr(lib, name), name


def test_status_strings(lib):
    assert lib.ah_status_string(0) == b"ok"
    assert lib.ah_status_string(1) == b"invalid argument"
    assert lib.ah_status_string(5) == b"device-side error"
    assert lib.ah_status_string(99) == b"unknown status"


def _views(**kw):
    base = dict(n=1000, d=16, num_leaves=4, dims_per_block=2, centroids=8, leaf_offsets=8, slot_ids=8,
                codes=8, codebook=8, reorder_vecs=None, reorder_dtype=0)
    base.update(kw)
    return ahindex.Views(**base)


@pytest.mark.parametrize("kw, text", [
    (dict(n=0), b"n outside"),
    (dict(d=15), b"d not divisible"),
    (dict(dims_per_block=0), b"non-positive"),
    (dict(num_leaves=0), b"non-positive"),
    (dict(codes=None), b"NULL index array"),
    (dict(reorder_dtype=7), b"unknown reorder_dtype"),
])
def test_build_rejects_bad_views_on_host(lib, kw, text):
    out = ctypes.c_void_p(123)
    st = lib.ah_build_index_views(ctypes.byref(_views(**kw)), None, ctypes.byref(out))
    assert st == 1
    assert out.value is None
    assert text in lib.ah_last_error()


def test_build_rejects_unsupported_sizes(lib):
    out = ctypes.c_void_p()
    st = lib.ah_build_index_views(ctypes.byref(_views(d=16384, dims_per_block=2)), None, ctypes.byref(out))
    assert st == 2


def test_null_arguments(lib):
    assert lib.ah_build_index_views(None, None, None) == 1
    assert lib.ah_search(None, None, 1, 10, 1, 0, 0, None, None, None) == 1
    assert lib.ah_sync_status(None, None) == 1
    assert lib.ah_set_profiling(None, 1) == 1
    assert lib.ah_index_memory(None, None) == 1
    lib.ah_destroy(None)     # no-op
    assert lib.ah_stage_name(0) == b"centroid_scores"
    assert lib.ah_stage_name(99) == b""


def test_library_is_sm100a_only():
    log = open(os.path.join(ahbuild.BUILD, "ptxas.log")).read()
    assert "sm_100a" in log
    assert "compute_100a,code=sm_100a" in " ".join(ahbuild.NVCC_FLAGS)


def test_missing_library_fails_loudly(tmp_path):
    # the package has no other way to search: without the CUDA library it raises
    with pytest.raises(ahindex.AhError) as e:
        ahindex.load_library(str(tmp_path / "libah.so"))
    assert e.value.status == 4
    assert "not built" in str(e.value)
