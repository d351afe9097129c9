"""CPU oracle for the anisotropic-AH search path: TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  It shares no code with the CUDA library
(``mips_ivf_centroid_b200``) and never imports it.

* ``ah_oracle.c``: the search, step by step, in plain C (fp64), following the
  ScaNN blog post, "Three stages of a search".
* ``avq.py``: the training-side formulas the pages print: the eta ratio, the
  anisotropic loss and its closed-form center update ("The loss in one
  paragraph", "Training an anisotropic codebook yourself").
* ``encode`` (``orc_encode`` in ah_oracle.c): anisotropic code assignment by
  coordinate descent, the index-build step before the search.
* ``kmeans_assign`` / ``kmeans_update``: partition training (nearest centroid,
  centroid means), the other index-build step.

Parity pins: every function here is checked against something other than
itself: the search in ``tests/test_oracle_pins.py`` (numpy brute force, the
reconstruction identity, residual codes, an integer special case, hand-worked
values, the blog's operation counts), the training formulas in
``tests/test_avq_pins.py``, the code assignment in ``tests/test_encode_pins.py``
(eta = 1 gives the per-block nearest centers; with one live block the result is
the exhaustive argmin of the loss as ``avq.py`` computes it; converged codes
are coordinate-wise minima; never worse than the L2 codes) and partition
training in ``tests/test_kmeans_pins.py`` (numpy argmin and means, exact ties,
Lloyd monotonicity).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_BUILD = os.path.join(_HERE, "_build")
_SO = os.path.join(_BUILD, "libahoracle.so")
_SRC = os.path.join(_HERE, "ah_oracle.c")

_lib = None


def build(force: bool = False) -> str:
    """Compile ``ah_oracle.c`` with gcc into ``oracle/_build/libahoracle.so``."""
    os.makedirs(_BUILD, exist_ok=True)
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        tmp = _SO + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math", "-std=c11",
               "-Wall", "-shared", "-fPIC", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _SO)
    return _SO


class _Index(ctypes.Structure):
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
        ("reorder_is_bf16", ctypes.c_int32),
        ("residual", ctypes.c_int32),
    ]


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        lib.orc_search.restype = ctypes.c_int
        lib.orc_search.argtypes = [P, P, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                   ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                   P, P, P, P, P, P, P, P, P]
        lib.orc_search_leaves.restype = ctypes.c_int
        lib.orc_search_leaves.argtypes = [P, P, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, P,
                                          ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                          P, P, P, P, P, P, P]
        lib.orc_centroid_scores.argtypes = [P, P, P]
        lib.orc_point_scores.argtypes = [P, P, ctypes.c_int64, P, P, P]
        lib.orc_u8_table.argtypes = [P, P, P, P, P]
        lib.orc_u8_sums.argtypes = [P, P, ctypes.c_int64, P, P]
        lib.orc_max_threads.restype = ctypes.c_int
        lib.orc_encode.argtypes = [P, ctypes.c_int64, ctypes.c_int, ctypes.c_int, P, ctypes.c_double,
                                   ctypes.c_int, P, P]
        lib.orc_kmeans_assign.argtypes = [P, ctypes.c_int64, ctypes.c_int, P, ctypes.c_int, P, P]
        lib.orc_kmeans_update.argtypes = [P, ctypes.c_int64, ctypes.c_int, P, ctypes.c_int, P, P, P]
        _lib = lib
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


class OracleIndex:
    """Host copies of the index arrays, held for the oracle's C code.

    ``arrays``: dict with centroids [NL,d] f32, leaf_offsets [NL+1] i64,
    slot_ids [n] i32, codes [n,B/2] u8, codebook [B,16,dpb] f32,
    reorder_vecs [n,d] (f32, or bf16 bits as u16; None if never reordered),
    reorder_dtype and residual (codes of x minus its leaf's centroid; the
    approximate score then adds q . centroid to the table sum).
    """

    def __init__(self, arrays: dict):
        a = {}
        a["centroids"] = np.ascontiguousarray(arrays["centroids"], dtype=np.float32)
        a["leaf_offsets"] = np.ascontiguousarray(arrays["leaf_offsets"], dtype=np.int64)
        a["slot_ids"] = np.ascontiguousarray(arrays["slot_ids"], dtype=np.int32)
        a["codes"] = np.ascontiguousarray(arrays["codes"], dtype=np.uint8)
        a["codebook"] = np.ascontiguousarray(arrays["codebook"], dtype=np.float32)
        bf16 = arrays.get("reorder_dtype", "f32") == "bf16"
        rv = arrays.get("reorder_vecs")   # may be None when only reorder_num = 0 is searched
        a["reorder_vecs"] = None if rv is None else np.ascontiguousarray(
            rv, dtype=np.uint16 if bf16 else np.float32)
        self.arrays = a
        nl, d = a["centroids"].shape
        B, centers, dpb = a["codebook"].shape
        assert centers == 16 and B * dpb == d and a["codes"].shape[1] * 2 == B
        self.n, self.d, self.num_leaves, self.dpb, self.blocks = a["slot_ids"].shape[0], d, nl, dpb, B
        self._s = _Index(self.n, d, nl, dpb, _ptr(a["centroids"]), _ptr(a["leaf_offsets"]),
                         _ptr(a["slot_ids"]), _ptr(a["codes"]), _ptr(a["codebook"]),
                         _ptr(a["reorder_vecs"]), 1 if bf16 else 0, 1 if arrays.get("residual") else 0)

    @property
    def ref(self):
        return ctypes.byref(self._s)

    def search(self, Q: np.ndarray, k: int, num_leaves_to_search: int, reorder_num: int,
               lut_mode: int = 0, nthreads: int = 0, trace: bool = True) -> dict:
        """Run the oracle search on host queries Q [nq, d] (float32).

        Returns ids/scores [nq,k]; with ``trace`` also leaves/leaf_scores
        [nq,L], cand_ids/cand_scores/cand_sums [nq,R], ncand and scanned [nq].
        Scores are fp64 (uint8 mode: the fp32 values it defines, widened).
        """
        lib = _load()
        Q = np.ascontiguousarray(Q, dtype=np.float32)
        nq = Q.shape[0]
        L = num_leaves_to_search
        R = max(reorder_num, k)
        out = {"ids": np.empty((nq, k), np.int32), "scores": np.empty((nq, k), np.float64)}
        if trace:
            out.update(leaves=np.empty((nq, L), np.int32), leaf_scores=np.empty((nq, L), np.float64),
                       cand_ids=np.empty((nq, R), np.int32), cand_scores=np.empty((nq, R), np.float64),
                       cand_sums=np.empty((nq, R), np.uint32), ncand=np.empty(nq, np.int32),
                       scanned=np.empty(nq, np.int64))
        g = out.get
        rc = lib.orc_search(self.ref, _ptr(Q), nq, k, L, reorder_num, lut_mode, nthreads,
                            _ptr(out["ids"]), _ptr(out["scores"]), _ptr(g("leaves")),
                            _ptr(g("leaf_scores")), _ptr(g("cand_ids")), _ptr(g("cand_scores")),
                            _ptr(g("cand_sums")), _ptr(g("ncand")), _ptr(g("scanned")))
        if rc != 0:
            raise ValueError("oracle: invalid search arguments")
        return out

    def search_leaves(self, Q: np.ndarray, leaves: np.ndarray, k: int, reorder_num: int, lut_mode: int = 0,
                      nthreads: int = 0) -> dict:
        """Steps 2-5 of the search over caller-given leaves [nq, L] (int32,
        distinct ids per row) instead of each query's own best L; the same
        arithmetic as ``search``.  Returns ids/scores [nq,k], cand_ids/
        cand_scores/cand_sums [nq,R], ncand and scanned [nq]."""
        lib = _load()
        Q = np.ascontiguousarray(Q, dtype=np.float32)
        leaves = np.ascontiguousarray(leaves, dtype=np.int32)
        nq = Q.shape[0]
        if leaves.ndim != 2 or leaves.shape[0] != nq:
            raise ValueError("oracle: leaves must be [nq, L]")
        L = leaves.shape[1]
        R = max(reorder_num, k)
        out = {"ids": np.empty((nq, k), np.int32), "scores": np.empty((nq, k), np.float64),
               "cand_ids": np.empty((nq, R), np.int32), "cand_scores": np.empty((nq, R), np.float64),
               "cand_sums": np.empty((nq, R), np.uint32), "ncand": np.empty(nq, np.int32),
               "scanned": np.empty(nq, np.int64)}
        rc = lib.orc_search_leaves(self.ref, _ptr(Q), nq, k, L, _ptr(leaves), reorder_num, lut_mode, nthreads,
                                   _ptr(out["ids"]), _ptr(out["scores"]), _ptr(out["cand_ids"]),
                                   _ptr(out["cand_scores"]), _ptr(out["cand_sums"]), _ptr(out["ncand"]),
                                   _ptr(out["scanned"]))
        if rc != 0:
            raise ValueError("oracle: invalid search arguments")
        return out

    def centroid_scores(self, q: np.ndarray) -> np.ndarray:
        q = np.ascontiguousarray(q, dtype=np.float32)
        out = np.empty(self.num_leaves, np.float64)
        _load().orc_centroid_scores(self.ref, _ptr(q), _ptr(out))
        return out

    def point_scores(self, q: np.ndarray, slots) -> tuple:
        """(approximate fp64-table scores, exact scores) of one query at ``slots``."""
        q = np.ascontiguousarray(q, dtype=np.float32)
        slots = np.ascontiguousarray(slots, dtype=np.int64)
        ah = np.empty(slots.shape[0], np.float64)
        ex = np.empty(slots.shape[0], np.float64)
        _load().orc_point_scores(self.ref, _ptr(q), slots.shape[0], _ptr(slots), _ptr(ah), _ptr(ex))
        return ah, ex

    def u8_table(self, q: np.ndarray) -> tuple:
        q = np.ascontiguousarray(q, dtype=np.float32)
        lut8 = np.empty((self.blocks, 16), np.uint8)
        delta = np.empty(1, np.float32)
        bias = np.empty(1, np.float32)
        _load().orc_u8_table(self.ref, _ptr(q), _ptr(lut8), _ptr(delta), _ptr(bias))
        return lut8, float(delta[0]), float(bias[0])

    def u8_sums(self, q: np.ndarray, slots) -> np.ndarray:
        q = np.ascontiguousarray(q, dtype=np.float32)
        slots = np.ascontiguousarray(slots, dtype=np.int64)
        out = np.empty(slots.shape[0], np.uint32)
        _load().orc_u8_sums(self.ref, _ptr(q), slots.shape[0], _ptr(slots), _ptr(out))
        return out


def encode(X, codebook, T: float, passes: int):
    """Anisotropic code assignment (index build), ``orc_encode`` in ah_oracle.c.

    X [n, d] float32, codebook [B, 16, dpb] float32; eta per point from T and
    the point's norm (T <= 0: plain L2 codes).  Returns (codes [n, B/2] uint8
    nibble-packed, passes_used [n] int32)."""
    X = np.ascontiguousarray(X, dtype=np.float32)
    cb = np.ascontiguousarray(codebook, dtype=np.float32)
    n, d = X.shape
    B, _, dpb = cb.shape
    if B * dpb != d or B % 2:
        raise ValueError("codebook shape does not match d (B must be even)")
    codes = np.empty((n, B // 2), np.uint8)
    used = np.empty(n, np.int32)
    _load().orc_encode(_ptr(X), n, d, dpb, _ptr(cb), float(T), int(passes), _ptr(codes), _ptr(used))
    return codes, used


def kmeans_assign(X, C):
    """Nearest centroid of every row of X (``orc_kmeans_assign``): (assign [n]
    int32, squared distance [n] float64)."""
    X = np.ascontiguousarray(X, dtype=np.float32)
    C = np.ascontiguousarray(C, dtype=np.float32)
    n, d = X.shape
    a = np.empty(n, np.int32)
    dist = np.empty(n, np.float64)
    _load().orc_kmeans_assign(_ptr(X), n, d, _ptr(C), C.shape[0], _ptr(a), _ptr(dist))
    return a, dist


def kmeans_update(X, assign, C_old):
    """Centroid means (``orc_kmeans_update``): (C_new [nl, d] float32, counts [nl] int64)."""
    X = np.ascontiguousarray(X, dtype=np.float32)
    a = np.ascontiguousarray(assign, dtype=np.int32)
    C_old = np.ascontiguousarray(C_old, dtype=np.float32)
    n, d = X.shape
    nl = C_old.shape[0]
    C_new = np.empty_like(C_old)
    counts = np.empty(nl, np.int64)
    _load().orc_kmeans_update(_ptr(X), n, d, _ptr(a), nl, _ptr(C_old), _ptr(C_new), _ptr(counts))
    return C_new, counts


def max_threads() -> int:
    return int(_load().orc_max_threads())
