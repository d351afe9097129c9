"""Python binding of the C ABI in ``include/ah.h`` (ctypes; marshalling only).

Every step of a search runs in the CUDA library ``_build/libah.so``; this module
only passes device pointers, sizes and the current torch stream, and allocates
output tensors.  There is no fallback: without the library, or without a CUDA
device, constructing an ``Index`` raises ``AhError``.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import numpy as np
import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "_build", "libah.so")

AH_OK = 0
_STATUS = {0: "AH_OK", 1: "AH_ERR_INVALID_ARG", 2: "AH_ERR_UNSUPPORTED", 3: "AH_ERR_OOM",
           4: "AH_ERR_CUDA", 5: "AH_ERR_DEVICE", 6: "AH_ERR_TIMEOUT"}
AH_F32, AH_BF16 = 0, 1

_lib = None


class AhError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{_STATUS.get(status, status)}: {msg}")
        self.status = status


class Views(ctypes.Structure):
    _fields_ = [
        ("n", ctypes.c_int64),
        ("d", ctypes.c_int32),
        ("num_leaves", ctypes.c_int32),
        ("dims_per_block", ctypes.c_int32),
        ("centroids", ctypes.c_void_p),
        ("leaf_offsets", ctypes.c_void_p),
        ("slot_ids", ctypes.c_void_p),
        ("codes", ctypes.c_void_p),
        ("codebook", ctypes.c_void_p),
        ("reorder_vecs", ctypes.c_void_p),
        ("reorder_dtype", ctypes.c_int32),
        ("residual", ctypes.c_int32),
    ]


class Trace(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("leaf_ids", "leaf_scores", "cand_ids", "cand_scores", "cand_sums", "ncand", "scanned",
                 "passed", "rescans", "cand_exact")]


def load_library(path: Optional[str] = None) -> ctypes.CDLL:
    """Load ``libah.so`` and declare the prototypes of ``include/ah.h``."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise AhError(4, f"CUDA library not built: {p} (run python -m mips_ivf_centroid_b200.build)")
    lib = ctypes.CDLL(p)
    P, I32, I64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
    sig = {
        "ah_build_index_views": (I32, [P, P, ctypes.POINTER(P)]),
        "ah_search": (I32, [P, P, I32, I32, I32, I32, I32, P, P, P]),
        "ah_search_traced": (I32, [P, P, I32, I32, I32, I32, I32, P, P, P, P]),
        "ah_search_host": (I32, [P, P, I32, I32, I32, I32, I32, P, P, P]),
        "ah_reserve": (I32, [P, I32, I32, I32, I32, I32]),
        "ah_sync_status": (I32, [P, P]),
        "ah_set_profiling": (I32, [P, I32]),
        "ah_stage_times": (I32, [P, P, I32, P]),
        "ah_stage_name": (ctypes.c_char_p, [I32]),
        "ah_last_search_info": (I32, [P, P, P]),
        "ah_index_memory": (I32, [P, P]),
        "ah_destroy": (None, [P]),
        "ah_status_string": (ctypes.c_char_p, [I32]),
        "ah_last_error": (ctypes.c_char_p, []),
        "ah_search_leaves_noalloc": (I32, [P, P, I32, I32, P, P, P]),
        "ah_encode": (I32, [P, I64, I32, I32, P, ctypes.c_double, I32, P, P, P]),
        "ah_kmeans_assign": (I32, [P, I64, I32, P, I32, P, P, P]),
        "ah_kmeans_update": (I32, [P, I64, I32, P, I32, P, P, P, P]),
        "ah_avq_update": (I32, [P, I64, I32, P, I32, P, ctypes.c_double, I32, ctypes.c_double, P, P, P, P]),
        "ah_save": (I32, [P, ctypes.c_char_p]),
        "ah_merge_shards": (I32, [I32, I32, I32, I32, P, P, P, P, P, P]),
        "ah_inspect": (I32, [ctypes.c_char_p, P]),
        "ah_load": (I32, [ctypes.c_char_p, P, ctypes.POINTER(P)]),
        "ah_set_option": (I32, [P, I32, I64]),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    if path is None:
        _lib = lib
    return lib


def _check(lib, st: int):
    if st != AH_OK:
        raise AhError(st, lib.ah_last_error().decode())


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _need(t, name: str, dtype, shape, device=None):
    """AhError(1) unless ``t`` is a contiguous ``dtype`` tensor of ``shape``
    (None matches any extent), on ``device`` when one is given.  The library
    receives pointers and sizes only, so extents are checked here."""
    ok = (isinstance(t, torch.Tensor) and t.dtype == dtype and t.is_contiguous() and t.dim() == len(shape)
          and all(e is None or t.shape[i] == e for i, e in enumerate(shape))
          and (device is None or t.device == device))
    if not ok:
        want = "[" + ", ".join("*" if e is None else str(e) for e in shape) + "]"
        raise AhError(1, f"{name}: need contiguous {dtype} {want}" + ("" if device is None else f" on {device}"))


def _check_index_arrays(arrays):
    """Extents of the index arrays against one another: centroids [NL, d],
    leaf_offsets [NL + 1], slot_ids [n], codes [n, B / 2], codebook [B, 16,
    dpb] with B * dpb = d and B even, reorder_vecs [n, d] or None.  Returns
    (n, d, NL, dpb)."""
    c, cb = arrays.centroids, arrays.codebook
    if not isinstance(c, torch.Tensor) or c.dim() != 2:
        raise AhError(1, "centroids: need [num_leaves, d]")
    nl, d = c.shape
    if not isinstance(cb, torch.Tensor) or cb.dim() != 3 or cb.shape[1] != 16 or cb.shape[0] * cb.shape[2] != d:
        raise AhError(1, "codebook: need [d / dims_per_block, 16, dims_per_block]")
    B, dpb = cb.shape[0], cb.shape[2]
    if B % 2:
        raise AhError(1, "codebook: need an even number of blocks (d a multiple of 2 * dims_per_block)")
    dev = c.device
    _need(c, "centroids", torch.float32, (nl, d))
    _need(arrays.leaf_offsets, "leaf_offsets", torch.int64, (nl + 1,), dev)
    _need(arrays.slot_ids, "slot_ids", torch.int32, (None,), dev)
    n = arrays.slot_ids.shape[0]
    _need(arrays.codes, "codes", torch.uint8, (n, B // 2), dev)
    _need(cb, "codebook", torch.float32, (B, 16, dpb), dev)
    rv = arrays.reorder_vecs
    if rv is not None:
        if not isinstance(rv, torch.Tensor) or rv.dtype not in (torch.float32, torch.bfloat16):
            raise AhError(1, "reorder_vecs: need float32 or bfloat16")
        _need(rv, "reorder_vecs", rv.dtype, (n, d), dev)
    return n, d, nl, dpb


def encode(X: torch.Tensor, codebook: torch.Tensor, T: float, passes: int = 10, stream=None,
           out: Optional[torch.Tensor] = None, passes_used: Optional[torch.Tensor] = None):
    """Anisotropic codes of the rows of X (index build, ``ah_encode``).

    X [n, d] float32 and codebook [B, 16, dpb] float32 on one CUDA device.
    Returns (codes [n, B/2] uint8, passes_used [n] int32), asynchronous on the
    stream."""
    lib = load_library()
    if X.dtype != torch.float32 or X.dim() != 2 or not X.is_contiguous() or X.device.type != "cuda":
        raise AhError(1, "X: need contiguous float32 [n, d] on a CUDA device")
    if codebook.dtype != torch.float32 or codebook.dim() != 3 or not codebook.is_contiguous() \
            or codebook.device != X.device:
        raise AhError(1, "codebook: need contiguous float32 [B, 16, dpb] on X's device")
    n, d = X.shape
    B, _, dpb = codebook.shape
    if B * dpb != d or codebook.shape[1] != 16:
        raise AhError(1, "codebook: need [d / dims_per_block, 16, dims_per_block]")
    if out is None:
        out = torch.empty((n, B // 2), dtype=torch.uint8, device=X.device)
    _need(out, "out", torch.uint8, (n, B // 2), X.device)
    if passes_used is None:
        passes_used = torch.empty((n,), dtype=torch.int32, device=X.device)
    _need(passes_used, "passes_used", torch.int32, (n,), X.device)
    with torch.cuda.device(X.device):
        _check(lib, lib.ah_encode(_ptr(X), n, d, dpb, _ptr(codebook), float(T), int(passes), _ptr(out),
                                  _ptr(passes_used), _stream(stream)))
    return out, passes_used


def _f32_2d(t: torch.Tensor, name: str, dev=None):
    if t.dtype != torch.float32 or t.dim() != 2 or not t.is_contiguous() or t.device.type != "cuda" \
            or (dev is not None and t.device != dev):
        raise AhError(1, f"{name}: need contiguous float32 2-D CUDA tensor" + (f" on {dev}" if dev else ""))


def kmeans_assign(X: torch.Tensor, C: torch.Tensor, stream=None):
    """Nearest centroid of every row of X (``ah_kmeans_assign``): (assign [n]
    int32, squared distance [n] float64), asynchronous on the stream."""
    lib = load_library()
    _f32_2d(X, "X")
    _f32_2d(C, "C", X.device)
    if C.shape[1] != X.shape[1]:
        raise AhError(1, "C: need [nl, d] with X's d")
    n, d = X.shape
    a = torch.empty((n,), dtype=torch.int32, device=X.device)
    dist = torch.empty((n,), dtype=torch.float64, device=X.device)
    with torch.cuda.device(X.device):
        _check(lib, lib.ah_kmeans_assign(_ptr(X), n, d, _ptr(C), C.shape[0], _ptr(a), _ptr(dist), _stream(stream)))
    return a, dist


def kmeans_update(X: torch.Tensor, assign: torch.Tensor, C_old: torch.Tensor, stream=None):
    """Centroid means over each centroid's members (``ah_kmeans_update``):
    (C_new [nl, d] float32, counts [nl] int64), asynchronous on the stream."""
    lib = load_library()
    _f32_2d(X, "X")
    _f32_2d(C_old, "C_old", X.device)
    if assign.dtype != torch.int32 or assign.dim() != 1 or assign.shape[0] != X.shape[0] \
            or assign.device != X.device or not assign.is_contiguous():
        raise AhError(1, "assign: need contiguous int32 [n] on X's device")
    n, d = X.shape
    if C_old.shape[1] != d:
        raise AhError(1, "C_old: need [nl, d] with X's d")
    nl = C_old.shape[0]
    C_new = torch.empty_like(C_old)
    counts = torch.empty((nl,), dtype=torch.int64, device=X.device)
    with torch.cuda.device(X.device):
        _check(lib, lib.ah_kmeans_update(_ptr(X), n, d, _ptr(assign), nl, _ptr(C_old), _ptr(C_new), _ptr(counts),
                                         _stream(stream)))
    return C_new, counts


def avq_update(X: torch.Tensor, assign: torch.Tensor, C_old: torch.Tensor, T: float, max_iters: int = 200,
               tol: float = 1e-14, stream=None):
    """Anisotropic center update over each center's members (``ah_avq_update``):
    (C_new [nl, d] float32, counts [nl] int64, iters [nl] int32), asynchronous
    on the stream.  eta per point from the threshold T and the point's norm."""
    lib = load_library()
    _f32_2d(X, "X")
    _f32_2d(C_old, "C_old", X.device)
    if assign.dtype != torch.int32 or assign.dim() != 1 or assign.shape[0] != X.shape[0] \
            or assign.device != X.device or not assign.is_contiguous():
        raise AhError(1, "assign: need contiguous int32 [n] on X's device")
    n, d = X.shape
    if C_old.shape[1] != d:
        raise AhError(1, "C_old: need [nl, d] with X's d")
    nl = C_old.shape[0]
    C_new = torch.empty_like(C_old)
    counts = torch.empty((nl,), dtype=torch.int64, device=X.device)
    iters = torch.empty((nl,), dtype=torch.int32, device=X.device)
    with torch.cuda.device(X.device):
        _check(lib, lib.ah_avq_update(_ptr(X), n, d, _ptr(assign), nl, _ptr(C_old), float(T), int(max_iters),
                                      float(tol), _ptr(C_new), _ptr(counts), _ptr(iters), _stream(stream)))
    return C_new, counts, iters


def merge_shards(cand_ids: torch.Tensor, cand_approx: torch.Tensor, cand_exact: Optional[torch.Tensor], k: int,
                 stream=None):
    """Exact merge of a leaf-partitioned search (``ah_merge_shards``).

    cand_ids [G, nq, R] int32, cand_approx [G, nq, R] float32 (descending =
    approximate ranking), cand_exact [G, nq, R] float32 or None (searched
    without reorder), all on one CUDA device.  Returns (ids [nq, k] int32,
    scores [nq, k] float32)."""
    lib = load_library()
    if cand_ids.dtype != torch.int32 or cand_ids.dim() != 3 or not cand_ids.is_contiguous() \
            or cand_ids.device.type != "cuda":
        raise AhError(1, "cand_ids: need contiguous int32 [G, nq, R] on a CUDA device")
    if cand_approx is None:
        raise AhError(1, "cand_approx: required")
    if k < 1:
        raise AhError(1, "need k >= 1")
    for name, t in (("cand_approx", cand_approx), ("cand_exact", cand_exact)):
        if t is not None and (t.dtype != torch.float32 or t.shape != cand_ids.shape or not t.is_contiguous()
                              or t.device != cand_ids.device):
            raise AhError(1, f"{name}: need contiguous float32 like cand_ids")
    G, nq, R = cand_ids.shape
    ids = torch.empty((nq, k), dtype=torch.int32, device=cand_ids.device)
    scores = torch.empty((nq, k), dtype=torch.float32, device=cand_ids.device)
    with torch.cuda.device(cand_ids.device):
        _check(lib, lib.ah_merge_shards(G, nq, R, k, _ptr(cand_ids), _ptr(cand_approx), _ptr(cand_exact), _ptr(ids),
                                        _ptr(scores), _stream(stream)))
    return ids, scores


def inspect(path: str) -> dict:
    """Sizes of an index directory written by ``Index.save`` (no GPU needed):
    n, d, num_leaves, dims_per_block, reorder_dtype ("f32", "bf16" or None)."""
    lib = load_library()
    v = Views()
    _check(lib, lib.ah_inspect(os.fsencode(path), ctypes.byref(v)))
    rdt = {AH_F32: "f32", AH_BF16: "bf16"}.get(v.reorder_dtype)
    return dict(n=v.n, d=v.d, num_leaves=v.num_leaves, dims_per_block=v.dims_per_block, reorder_dtype=rdt,
                residual=bool(v.residual))


class Index:
    """A searchable index over borrowed device arrays.

    ``arrays`` is a ``datagen.IndexArrays`` (or any object with the same
    attributes) whose tensors live on one CUDA device; the index keeps a
    reference to them for its lifetime.
    """

    def __init__(self, arrays, stream=None):
        self._lib = load_library()
        if not torch.cuda.is_available():
            raise AhError(4, "no CUDA device")
        self.arrays = arrays
        c = arrays.centroids
        dev = c.device
        if dev.type != "cuda":
            raise AhError(1, "index arrays must be CUDA tensors")
        req = dict(centroids=torch.float32, leaf_offsets=torch.int64, slot_ids=torch.int32,
                   codes=torch.uint8, codebook=torch.float32)
        for k, dt in req.items():
            t = getattr(arrays, k)
            if t.dtype != dt or not t.is_contiguous() or t.device != dev:
                raise AhError(1, f"{k}: need contiguous {dt} on {dev}")
        rv = arrays.reorder_vecs
        if rv is not None and (not rv.is_contiguous() or rv.device != dev or rv.dtype not in (torch.float32, torch.bfloat16)):
            raise AhError(1, "reorder_vecs: need contiguous float32/bfloat16 on the index device")
        _check_index_arrays(arrays)
        self.device = dev
        self.n = arrays.slot_ids.shape[0]
        self.d = c.shape[1]
        self.num_leaves = c.shape[0]
        self.dims_per_block = arrays.codebook.shape[2]
        v = Views(self.n, self.d, self.num_leaves, self.dims_per_block, c.data_ptr(),
                  arrays.leaf_offsets.data_ptr(), arrays.slot_ids.data_ptr(), arrays.codes.data_ptr(),
                  arrays.codebook.data_ptr(), rv.data_ptr() if rv is not None else None,
                  AH_BF16 if (rv is not None and rv.dtype == torch.bfloat16) else AH_F32,
                  1 if getattr(arrays, "residual", False) else 0)
        h = ctypes.c_void_p()
        with torch.cuda.device(dev):
            _check(self._lib, self._lib.ah_build_index_views(ctypes.byref(v), _stream(stream), ctypes.byref(h)))
        self._h = h

    # -- index directories -----------------------------------------------------
    def save(self, path: str):
        """Write the index arrays to directory ``path`` (created if missing) as
        .npy files plus ``ah_index.txt``; synchronous."""
        os.makedirs(path, exist_ok=True)
        with torch.cuda.device(self.device):
            _check(self._lib, self._lib.ah_save(self._h, os.fsencode(path)))

    @classmethod
    def load(cls, path: str, device=None, stream=None) -> "Index":
        """An index loaded from a directory written by ``save``; its arrays are
        owned by the library (device memory freed by ``close``)."""
        self = cls.__new__(cls)
        self._lib = load_library()
        if not torch.cuda.is_available():
            raise AhError(4, "no CUDA device")
        info = inspect(path)
        dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
        h = ctypes.c_void_p()
        with torch.cuda.device(dev):
            _check(self._lib, self._lib.ah_load(os.fsencode(path), _stream(stream), ctypes.byref(h)))
        self._h = h
        self.arrays = None
        self.device = dev
        self.n, self.d = info["n"], info["d"]
        self.num_leaves, self.dims_per_block = info["num_leaves"], info["dims_per_block"]
        return self

    # -- search ---------------------------------------------------------------
    def search(self, queries: torch.Tensor, k: int, num_leaves_to_search: int, reorder_num: int,
               lut_mode: int = 0, stream=None, trace: bool = False):
        """(ids int32 [nq,k], scores float32 [nq,k]) on the index device.

        With ``trace`` a third element holds the intermediate results (leaf ids
        and scores, best-R candidates, points scanned per query).
        """
        q = queries
        if q.device != self.device or q.dtype != torch.float32 or not q.is_contiguous() or q.dim() != 2 \
                or q.shape[1] != self.d:
            raise AhError(1, f"queries: need contiguous float32 [nq, {self.d}] on {self.device}")
        if k < 1 or num_leaves_to_search < 1 or reorder_num < 0:
            raise AhError(1, "need k >= 1, num_leaves_to_search >= 1, reorder_num >= 0")
        nq = q.shape[0]
        ids = torch.empty((nq, k), dtype=torch.int32, device=self.device)
        scores = torch.empty((nq, k), dtype=torch.float32, device=self.device)
        with torch.cuda.device(self.device):
            s = _stream(stream)
            if not trace:
                _check(self._lib, self._lib.ah_search(self._h, _ptr(q), nq, k, num_leaves_to_search, reorder_num,
                                                      lut_mode, _ptr(ids), _ptr(scores), s))
                return ids, scores
            R = max(reorder_num, k)
            L = num_leaves_to_search
            t = dict(leaf_ids=torch.empty((nq, L), dtype=torch.int32, device=self.device),
                     leaf_scores=torch.empty((nq, L), dtype=torch.float32, device=self.device),
                     cand_ids=torch.empty((nq, R), dtype=torch.int32, device=self.device),
                     cand_scores=torch.empty((nq, R), dtype=torch.float32, device=self.device),
                     cand_sums=torch.empty((nq, R), dtype=torch.int32, device=self.device),
                     ncand=torch.empty((nq,), dtype=torch.int32, device=self.device),
                     scanned=torch.empty((nq,), dtype=torch.int64, device=self.device),
                     passed=torch.empty((nq,), dtype=torch.int32, device=self.device),
                     rescans=torch.zeros((1,), dtype=torch.int32, device=self.device),
                     cand_exact=torch.full((nq, R), float("-inf"), dtype=torch.float32, device=self.device))
            tr = Trace(*[t[n].data_ptr() for n, _ in Trace._fields_])
            _check(self._lib, self._lib.ah_search_traced(self._h, _ptr(q), nq, k, num_leaves_to_search, reorder_num,
                                                         lut_mode, _ptr(ids), _ptr(scores), ctypes.byref(tr), s))
            return ids, scores, t

    def search_host(self, queries, k: int, num_leaves_to_search: int, reorder_num: int, lut_mode: int = 0,
                    out_ids=None, out_scores=None, stream=None):
        """Search host queries (numpy or CPU tensor, ideally pinned); returns
        host (ids, scores).  The copies in and out happen inside the call."""
        if isinstance(queries, np.ndarray):
            queries = torch.from_numpy(np.ascontiguousarray(queries, dtype=np.float32))
        if queries.device.type != "cpu" or queries.dtype != torch.float32 or not queries.is_contiguous() \
                or queries.dim() != 2 or queries.shape[1] != self.d:
            raise AhError(1, f"queries: need a contiguous float32 host tensor [nq, {self.d}]")
        if k < 1:
            raise AhError(1, "need k >= 1")
        nq = queries.shape[0]
        cpu = torch.device("cpu")
        if out_ids is None:
            out_ids = torch.empty((nq, k), dtype=torch.int32, pin_memory=queries.is_pinned())
        _need(out_ids, "out_ids", torch.int32, (nq, k), cpu)
        if out_scores is None:
            out_scores = torch.empty((nq, k), dtype=torch.float32, pin_memory=queries.is_pinned())
        _need(out_scores, "out_scores", torch.float32, (nq, k), cpu)
        with torch.cuda.device(self.device):
            _check(self._lib, self._lib.ah_search_host(self._h, _ptr(queries), nq, k, num_leaves_to_search,
                                                       reorder_num, lut_mode, _ptr(out_ids), _ptr(out_scores),
                                                       _stream(stream)))
        return out_ids, out_scores

    def reserve(self, max_nq: int, k: int, num_leaves_to_search: int, reorder_num: int, lut_mode: int = 0):
        with torch.cuda.device(self.device):
            _check(self._lib, self._lib.ah_reserve(self._h, max_nq, k, num_leaves_to_search, reorder_num, lut_mode))

    def sync_status(self, stream=None):
        with torch.cuda.device(self.device):
            _check(self._lib, self._lib.ah_sync_status(self._h, _stream(stream)))

    OPT_THRESHOLD_SAMPLE = 1
    OPT_SCAN_CHUNK_TILES = 2
    OPT_THRESHOLD_LEAVES = 3
    OPT_PROGRESSIVE_LEAVES = 4
    OPT_UINT8_TENSOR_CORES = 5
    OPT_QUERY_MAJOR_SCAN = 6

    def set_option(self, option: int, value: int):
        """Tuning knob (ah_set_option): results are unchanged, only speed."""
        _check(self._lib, self._lib.ah_set_option(self._h, option, value))

    # -- instrumentation ------------------------------------------------------
    def set_profiling(self, on=True):
        """0/False off, 1/True every stage, 2 the scan phases only."""
        _check(self._lib, self._lib.ah_set_profiling(self._h, int(on)))

    def stage_times(self) -> dict:
        ms = (ctypes.c_float * 16)()
        n = ctypes.c_int32()
        _check(self._lib, self._lib.ah_stage_times(self._h, ms, 16, ctypes.byref(n)))
        return {self._lib.ah_stage_name(i).decode(): float(ms[i]) for i in range(n.value)}

    def last_search_info(self, points_scanned: bool = False) -> dict:
        launches = ctypes.c_int32()
        pts = ctypes.c_int64()
        _check(self._lib, self._lib.ah_last_search_info(self._h, ctypes.byref(launches),
                                                        ctypes.byref(pts) if points_scanned else None))
        out = {"launches": launches.value}
        if points_scanned:
            out["points_scanned"] = pts.value
        return out

    def memory_bytes(self) -> int:
        b = ctypes.c_int64()
        _check(self._lib, self._lib.ah_index_memory(self._h, ctypes.byref(b)))
        return b.value

    def search_leaves_noalloc(self, queries: torch.Tensor, num_leaves_to_search: int, out_leaf_ids: torch.Tensor,
                              out_leaf_scores: torch.Tensor, stream=None):
        """Partition stage into caller-provided outputs, with no device
        allocation anywhere on the call path (see ah_search_leaves_noalloc in
        include/ah.h for the scratch limit and the sharing rules)."""
        _need(queries, "queries", torch.float32, (None, self.d), self.device)
        nq, L = queries.shape[0], num_leaves_to_search
        if L < 1:
            raise AhError(1, "need num_leaves_to_search >= 1")
        _need(out_leaf_ids, "out_leaf_ids", torch.int32, (nq, L), self.device)
        _need(out_leaf_scores, "out_leaf_scores", torch.float32, (nq, L), self.device)
        with torch.cuda.device(self.device):
            _check(self._lib, self._lib.ah_search_leaves_noalloc(
                self._h, _ptr(queries), queries.shape[0], num_leaves_to_search, _ptr(out_leaf_ids),
                _ptr(out_leaf_scores), _stream(stream)))

    def close(self):
        if getattr(self, "_h", None):
            self._lib.ah_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
