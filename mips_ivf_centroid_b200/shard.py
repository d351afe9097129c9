"""Leaf-partitioned search over several GPUs (or several indexes on one).

Every shard holds the same centroids and codebook and the points of its own
leaves (leaf c belongs to shard c mod G; the others are empty there), so each
shard picks the same L leaves for a query and scans its own points of them.
Each shard's best R by approximate score, with their exact scores, is gathered
and merged by ``merge_shards`` (``ah_merge_shards``): the best R of the union
by approximate score, then the best k of those by exact score, which is what
one index over all points returns.

This module only moves data: slicing index arrays (torch indexing) and
gathering candidate tensors (``torch.distributed``); the search and the merge
run in the CUDA library.
"""
from __future__ import annotations

import dataclasses
import torch

from .index import AhError, merge_shards


def shard_arrays(arrays, G: int, g: int):
    """The index arrays of shard g of G: all centroids and the codebook; the
    points of leaves c with c % G == g, in the same slot order; other leaves
    empty.  ``arrays`` is a ``datagen.IndexArrays`` (or alike)."""
    if not (0 <= g < G):
        raise AhError(1, "need 0 <= g < G")
    offs = arrays.leaf_offsets
    nl = offs.shape[0] - 1
    sizes = offs[1:] - offs[:-1]
    owned = (torch.arange(nl, device=offs.device) % G) == g
    leaf_of_slot = torch.repeat_interleave(torch.arange(nl, device=offs.device), sizes)
    keep = owned[leaf_of_slot].nonzero().squeeze(1)
    new_sizes = torch.where(owned, sizes, torch.zeros_like(sizes))
    new_offs = torch.zeros_like(offs)
    new_offs[1:] = torch.cumsum(new_sizes, 0)
    fields = {f.name: getattr(arrays, f.name) for f in dataclasses.fields(arrays)}
    fields.update(leaf_offsets=new_offs, slot_ids=arrays.slot_ids[keep].contiguous(),
                  codes=arrays.codes[keep].contiguous(),
                  reorder_vecs=None if arrays.reorder_vecs is None else arrays.reorder_vecs[keep].contiguous())
    return type(arrays)(**fields)


def shard_candidates(index, queries: torch.Tensor, k: int, num_leaves_to_search: int, reorder_num: int,
                     lut_mode: int = 0, stream=None):
    """One shard's best R (ids, approximate ranking values, final ranking
    values or None), each [nq, R], from a traced search of ``index``.

    With uint8 tables the approximate ranking is by the integer sums (exact);
    without reorder the final values are then the fp32 scores the search
    reports, so the merged scores equal one index's (the order of two
    candidates whose different sums round to the same fp32 score follows id
    there)."""
    _, _, tr = index.search(queries, k, num_leaves_to_search, reorder_num, lut_mode, stream=stream, trace=True)
    approx = tr["cand_scores"] if lut_mode == 0 else tr["cand_sums"].to(torch.float32)
    if reorder_num > 0:
        final = tr["cand_exact"]
    else:
        final = None if lut_mode == 0 else tr["cand_scores"]
    return tr["cand_ids"], approx, final


def merge_local(parts, k: int, stream=None):
    """Merge a list of per-shard (ids, approx, exact) on this device."""
    ids = torch.stack([p[0] for p in parts]).contiguous()
    approx = torch.stack([p[1] for p in parts]).contiguous()
    exact = None if parts[0][2] is None else torch.stack([p[2] for p in parts]).contiguous()
    return merge_shards(ids, approx, exact, k, stream=stream)


def gather_candidates(local, group=None):
    """All ranks' (ids, approx, exact) stacked in rank order: [G, nq, R] each
    (exact None if the ranks searched without reorder)."""
    import torch.distributed as dist
    G = dist.get_world_size(group)
    out = []
    for t in local:
        if t is None:
            out.append(None)
            continue
        parts = [torch.empty_like(t) for _ in range(G)]
        dist.all_gather(parts, t.contiguous(), group=group)
        out.append(torch.stack(parts).contiguous())
    return tuple(out)


def merge_gathered(gathered, k: int, stream=None):
    ids, approx, exact = gathered
    return merge_shards(ids, approx, exact, k, stream=stream)
