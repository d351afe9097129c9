"""B200-native anisotropic-AH maximum inner product search.

The search path (centroid scoring -> top-L leaves -> per-query lookup tables ->
4-bit code scan -> top-R -> exact reorder -> top-k) runs in hand-written sm_100a
CUDA kernels behind the C ABI declared in ``include/ah.h``; this package is the
thin Python binding over that library: ``Index`` (search, save/load),
``encode``, ``kmeans_assign``/``kmeans_update`` and ``avq_update`` (index
build), ``merge_shards`` and the ``shard`` module (leaf-partitioned search),
plus the seeded input generator ``datagen``.  Importing the package does not load the
CUDA library; the first call that needs it does, and raises if it is missing.
"""
from __future__ import annotations

__all__ = ["Index", "AhError", "load_library", "inspect", "encode", "kmeans_assign", "kmeans_update", "avq_update", "merge_shards", "LUT_F32", "LUT_U8"]

LUT_F32 = 0
LUT_U8 = 1


def __getattr__(name):
    if name in ("Index", "AhError", "load_library", "inspect", "encode", "kmeans_assign", "kmeans_update",
                "avq_update", "merge_shards"):
        from . import index as _index
        return getattr(_index, name)
    raise AttributeError(name)
