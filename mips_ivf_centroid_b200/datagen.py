"""Seeded synthetic inputs for anisotropic-AH maximum inner product search.

Everything a search reads is produced here, deterministically from a workload
spec and fixed seeds:

* the datapoints X and the queries Q, drawn from Gaussian mixtures whose shapes
  follow the workloads the ScaNN blog post discusses ("Worked example: cost of
  one query": normalised float32 embeddings, d = 128, ~1M points), scaled to the
  five workloads in ``WORKLOADS``;
* the trained index arrays a search borrows: partition centroids, the
  leaf-sorted slot order, the per-block 16-center codebook, the nibble-packed
  4-bit codes and the reorder copy of the vectors.

Training an index is outside the search path (ScaNN blog, "Training an
anisotropic codebook yourself"; "Three stages of a search" starts from a built
index).  This module therefore holds no step of the search: it never scores a
query against centroids, never builds a query lookup table, never scans codes
and never selects or reorders candidates.  The CPU oracle and the CUDA library
both consume its arrays unchanged.

Random draws use ``numpy.random.default_rng`` (PCG64): the component means
and labels from the workload's seed, the noise of each 1M-row chunk from a
generator seeded with (seed-derived key, chunk index).  Heavy index-build
arithmetic (nearest-centroid assignment, Lloyd iterations, code assignment) runs
in torch on whatever device is given, so the large workloads build in seconds on
a GPU; the results are inputs, so the device used does not affect parity.
"""
from __future__ import annotations

import dataclasses
import os
from concurrent.futures import ThreadPoolExecutor
from typing import Optional

import numpy as np
import torch

NUM_CENTERS = 16  # 4-bit codes: 16 learned centers per block (ScaNN blog, "Three stages of a search")


@dataclasses.dataclass(frozen=True)
class Workload:
    """Shape of one synthetic search workload.

    n, d: datapoints and dimension.  dims_per_block (dpb): dimensions per AH
    block, B = d / dpb blocks, B / 2 code bytes per point.  num_leaves (NL):
    partitions; num_leaves_to_search (L); nq queries; k final neighbours;
    reorder_num: candidates rescored exactly (0 = no reorder).
    """

    name: str
    n: int
    d: int
    dims_per_block: int
    num_leaves: int
    num_leaves_to_search: int
    nq: int
    k: int
    reorder_num: int
    data_kind: str = "unit_mixture"       # "unit_mixture" | "int255_mixture"
    n_means: int = 20
    sigma: float = 0.3
    code_loss: str = "l2"                 # "l2" | "anisotropic"
    threshold_T: Optional[float] = None   # anisotropic_quantization_threshold
    reorder_dtype: str = "f32"            # "f32" | "bf16"
    query_kind: str = "mixture"           # "mixture" | "gaussian"
    codebook_train: bool = True           # Lloyd-train codebook (False: sampled slices only)
    data_seed: int = 0
    centroid_seed: int = 1
    query_seed: int = 2
    codebook_seed: int = 3
    training_sample_size: int = 250_000
    lloyd_iters: int = 10
    aniso_passes: int = 10
    residual: bool = False                # codes of x - (its leaf's centroid) instead of x

    @property
    def blocks(self) -> int:
        return self.d // self.dims_per_block

    @property
    def code_bytes(self) -> int:
        return self.blocks // 2

    @property
    def eta(self) -> Optional[float]:
        """Large-d, unit-norm weight ratio eta = (d-1) T^2 / (1 - T^2).

        ScaNN blog, "The loss in one paragraph" (Theorem 3.4 limit, unit-norm form).
        """
        if self.code_loss != "anisotropic":
            return None
        T = self.threshold_T
        return (self.d - 1) * T * T / (1.0 - T * T)

    def scaled(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The five workloads (shapes of GloVe-100, BigANN, OpenAI-1536 and a 50M sweep).
WORKLOADS = {
    "tiny": Workload(
        name="tiny", n=10_000, d=32, dims_per_block=2, num_leaves=1,
        num_leaves_to_search=1, nq=100, k=10, reorder_num=100,
        data_kind="unit_mixture", n_means=20, sigma=0.3, code_loss="l2",
        query_kind="gaussian", codebook_train=False, codebook_seed=1),
    "glove": Workload(
        name="glove", n=1_000_000, d=100, dims_per_block=2, num_leaves=1_000,
        num_leaves_to_search=32, nq=1_000, k=10, reorder_num=100,
        data_kind="unit_mixture", n_means=1_000, sigma=0.4,
        code_loss="anisotropic", threshold_T=0.2),
    "bigann": Workload(
        name="bigann", n=10_000_000, d=128, dims_per_block=2, num_leaves=4_000,
        num_leaves_to_search=64, nq=10_000, k=10, reorder_num=200,
        data_kind="int255_mixture", n_means=4_000, sigma=20.0, code_loss="l2"),
    "openai": Workload(
        name="openai", n=2_000_000, d=1536, dims_per_block=4, num_leaves=2_000,
        num_leaves_to_search=40, nq=10_000, k=10, reorder_num=300,
        data_kind="unit_mixture", n_means=2_000, sigma=0.5,
        code_loss="anisotropic", threshold_T=0.05, reorder_dtype="bf16"),
    "sweep": Workload(
        name="sweep", n=50_000_000, d=96, dims_per_block=2, num_leaves=10_000,
        num_leaves_to_search=64, nq=16_384, k=10, reorder_num=100,
        data_kind="unit_mixture", n_means=10_000, sigma=0.4, code_loss="l2",
        reorder_dtype="bf16"),
}

SWEEP_BATCHES = (1, 16, 256, 4_096, 16_384)
SWEEP_LEAVES = (16, 64, 256)

_CHUNK_ROWS = 1_000_000
_ELEM_BUDGET = 1 << 27   # elements per temporary in the index-build steps (CPU)
_ELEM_BUDGET_CUDA = 1 << 29


def _budget(device) -> int:
    return _ELEM_BUDGET_CUDA if torch.device(device).type == "cuda" else _ELEM_BUDGET


# --------------------------------------------------------------------------
# raw data and queries
# --------------------------------------------------------------------------

def _normalise_rows(a: np.ndarray) -> None:
    """In-place L2 normalisation of float32 rows (float32 arithmetic)."""
    for s in range(0, a.shape[0], _CHUNK_ROWS):
        blk = a[s:s + _CHUNK_ROWS]
        nrm = np.sqrt(np.einsum("ij,ij->i", blk, blk, dtype=np.float32))
        nrm[nrm == 0] = 1.0
        blk /= nrm[:, None]


def _draw_means(w: Workload, rng: np.random.Generator) -> np.ndarray:
    if w.data_kind == "int255_mixture":
        return rng.uniform(0.0, 255.0, size=(w.n_means, w.d)).astype(np.float32)
    return rng.standard_normal((w.n_means, w.d), dtype=np.float32)


def _mixture_rows(w: Workload, means: np.ndarray, rng: np.random.Generator, n: int, stream_key: int) -> np.ndarray:
    """Mixture draws: component labels (uniform) from ``rng``; then, per chunk
    of 1M rows, noise from the chunk's own generator seeded with
    (``stream_key``, chunk index), so chunks can be drawn in parallel and the
    result does not depend on the thread count."""
    labels = rng.integers(0, means.shape[0], size=n)
    out = np.empty((n, w.d), dtype=np.float32)
    sig = np.float32(w.sigma)

    def work(c: int) -> None:
        s = c * _CHUNK_ROWS
        e = min(n, s + _CHUNK_ROWS)
        g = np.random.default_rng([stream_key, c])
        noise = g.standard_normal((e - s, w.d), dtype=np.float32)
        noise *= sig
        noise += means[labels[s:e]]
        if w.data_kind == "int255_mixture":
            np.clip(noise, 0.0, 255.0, out=noise)
            np.rint(noise, out=noise)
        else:
            _normalise_rows(noise)
        out[s:e] = noise

    chunks = (n + _CHUNK_ROWS - 1) // _CHUNK_ROWS
    if chunks == 1:
        work(0)
    else:
        with ThreadPoolExecutor(max_workers=min(chunks, os.cpu_count() or 1)) as ex:
            list(ex.map(work, range(chunks)))
    return out


def make_data(w: Workload) -> np.ndarray:
    """Datapoints X [n, d] float32 (seed ``w.data_seed``: means, labels; noise
    per chunk from (data_seed, chunk))."""
    rng = np.random.default_rng(w.data_seed)
    means = _draw_means(w, rng)
    return _mixture_rows(w, means, rng, w.n, 1_000_003 * w.data_seed + 11)


def make_queries(w: Workload, nq: Optional[int] = None) -> np.ndarray:
    """Queries Q [nq, d] float32, never drawn from the indexed rows.

    "gaussian": unit-normalised N(0, I).  "mixture": fresh draws around the
    data's own component means (re-derived from the data seed), with labels and
    noise from ``w.query_seed``; normalised when the data is.
    """
    nq = w.nq if nq is None else nq
    rng = np.random.default_rng(w.query_seed)
    if w.query_kind == "gaussian":
        q = rng.standard_normal((nq, w.d), dtype=np.float32)
        _normalise_rows(q)
        return q
    means = _draw_means(w, np.random.default_rng(w.data_seed))
    return _mixture_rows(w, means, rng, nq, 1_000_003 * w.query_seed + 17)


# --------------------------------------------------------------------------
# index arrays
# --------------------------------------------------------------------------

@dataclasses.dataclass
class IndexArrays:
    """The arrays a search borrows.  All tensors live on one device.

    centroids [NL, d] f32; leaf_offsets [NL+1] int64 (CSR over slots);
    slot_ids [n] int32 (original datapoint id of each slot); codes [n, B/2]
    uint8 in slot order, block 2i in the low nibble and block 2i+1 in the high
    nibble of byte i; codebook [B, 16, dpb] f32; reorder_vecs [n, d] in slot
    order, float32 or bfloat16 (round-to-nearest-even copy of X).
    """

    workload: Workload
    centroids: torch.Tensor
    leaf_offsets: torch.Tensor
    slot_ids: torch.Tensor
    codes: torch.Tensor
    codebook: torch.Tensor
    reorder_vecs: torch.Tensor
    residual: bool = False

    def to(self, device) -> "IndexArrays":
        f = {k: (v.to(device) if isinstance(v, torch.Tensor) else v)
             for k, v in dataclasses.asdict(self).items() if k != "workload"}
        return IndexArrays(workload=self.workload, **f)

    def numpy(self) -> dict:
        """Host copies; bf16 reorder vectors are returned as their uint16 bits."""
        out = {}
        for k in ("centroids", "leaf_offsets", "slot_ids", "codes", "codebook"):
            out[k] = getattr(self, k).cpu().numpy()
        rv = self.reorder_vecs.cpu()
        if rv.dtype == torch.bfloat16:
            out["reorder_vecs"] = rv.view(torch.int16).numpy().view(np.uint16)
            out["reorder_dtype"] = "bf16"
        else:
            out["reorder_vecs"] = rv.numpy()
            out["reorder_dtype"] = "f32"
        out["residual"] = bool(self.residual)
        return out


def _nearest_rows(x: torch.Tensor, c: torch.Tensor) -> torch.Tensor:
    """argmin_j ||x_i - c_j||^2 by chunks; ties go to the lower j (first minimum)."""
    chunk = max(1024, _budget(x.device) // max(1, c.shape[0]))
    cn = (c.double() * c.double()).sum(1).float()
    out = torch.empty(x.shape[0], dtype=torch.int64, device=x.device)
    for s in range(0, x.shape[0], chunk):
        xb = x[s:s + chunk]
        dist = cn[None, :] - 2.0 * (xb @ c.T)
        out[s:s + chunk] = torch.argmin(dist, dim=1)
    return out


def _train_codebook(w: Workload, X: torch.Tensor) -> torch.Tensor:
    """Per-block 16-center codebook [B, 16, dpb].

    Initialisation: for each block in order, 16 distinct rows sampled from one
    seeded stream, their block slices taken as centers.  When ``codebook_train``
    is set, the sample is a ``training_sample_size`` subset (ScaNN blog, builder
    ``training_sample_size``) and each block then runs ``lloyd_iters`` plain
    squared-L2 k-means iterations; an empty center keeps its value.
    """
    dev = X.device
    n, d, dpb, B = w.n, w.d, w.dims_per_block, w.blocks
    rng = np.random.default_rng(w.codebook_seed)
    if w.codebook_train:
        s_idx = np.sort(rng.choice(n, size=min(n, w.training_sample_size), replace=False))
        S = X[torch.from_numpy(s_idx).to(dev)]
    else:
        S = X
    cb = torch.empty((B, NUM_CENTERS, dpb), dtype=torch.float32, device=dev)
    for b in range(B):
        rows = rng.choice(S.shape[0], size=NUM_CENTERS, replace=False)
        cb[b] = S[torch.from_numpy(rows).to(dev), b * dpb:(b + 1) * dpb]
    if not w.codebook_train:
        return cb
    Sb = S.view(S.shape[0], B, dpb).transpose(0, 1).contiguous()        # [B, m, dpb]
    m = Sb.shape[1]
    bstep = max(1, _budget(dev) // (m * NUM_CENTERS * max(dpb, 2)))
    for _ in range(w.lloyd_iters):
        new = cb.clone()
        for b0 in range(0, B, bstep):
            sb, cbb = Sb[b0:b0 + bstep], cb[b0:b0 + bstep]
            dist = (sb[:, :, None, :] - cbb[:, None, :, :]).pow(2).sum(-1)  # [b, m, 16]
            a = torch.argmin(dist, dim=2)                                  # [b, m]
            # member sums as a one-hot product (deterministic, unlike atomic scatter-adds)
            onehot = torch.nn.functional.one_hot(a, NUM_CENTERS).to(torch.float64)   # [b, m, 16]
            sums = torch.bmm(onehot.transpose(1, 2), sb.double())                    # [b, 16, dpb]
            cnt = onehot.sum(1)                                                      # [b, 16]
            new[b0:b0 + bstep] = torch.where((cnt > 0)[:, :, None],
                                             (sums / cnt.clamp(min=1)[:, :, None]).float(), cbb)
        cb = new
    return cb


def _l2_codes(X: torch.Tensor, cb: torch.Tensor) -> torch.Tensor:
    """Per block nearest of 16 centers by squared L2 (ties -> lower j). [n, B] int64."""
    n = X.shape[0]
    B, _, dpb = cb.shape
    chunk = max(1024, _budget(X.device) // (B * NUM_CENTERS * dpb))
    codes = torch.empty((n, B), dtype=torch.int64, device=X.device)
    for s in range(0, n, chunk):
        xb = X[s:s + chunk].view(-1, B, dpb)
        dist = (xb[:, :, None, :] - cb[None, :, :, :]).pow(2).sum(-1)   # [m, B, 16]
        codes[s:s + chunk] = torch.argmin(dist, dim=2)
    return codes


def _anisotropic_codes(X: torch.Tensor, cb: torch.Tensor, codes: torch.Tensor,
                       eta: float, passes: int) -> torch.Tensor:
    """Coordinate descent on the anisotropic loss, block by block.

    Loss of a reconstruction x~ of x: (eta - 1) (r . u)^2 + ||r||^2 with
    r = x - x~ and u = x / ||x|| (ScaNN blog, "Training an anisotropic codebook
    yourself", the loss rewrite).  Blocks couple through r . u, so codes are
    refined iteratively (same post, last paragraph of that section): starting
    from the L2 codes, each pass visits b = 0..B-1 and picks, with the other
    blocks fixed, the center of least loss; ties keep the current code, then
    the lower index.  Stops after ``passes`` passes or a pass with no change.
    Arithmetic in float64.
    """
    n = X.shape[0]
    B, _, dpb = cb.shape
    cbd = cb.double()
    out = codes.clone()
    e1 = float(eta) - 1.0
    chunk = max(1024, _budget(X.device) // (4 * B * dpb))
    for s in range(0, n, chunk):
        x = X[s:s + chunk].double()
        m = x.shape[0]
        u = x / x.norm(dim=1, keepdim=True).clamp(min=1e-300)
        cd = out[s:s + chunk].clone()
        rows = torch.arange(m, device=X.device)
        for _ in range(passes):
            xt = cbd[torch.arange(B, device=X.device)[None, :], cd]       # [m, B, dpb]
            r = x - xt.reshape(m, -1)
            rpar = (r * u).sum(1)
            rn2 = (r * r).sum(1)
            changed = 0
            for b in range(B):
                sl = slice(b * dpb, (b + 1) * dpb)
                xb, ub = x[:, sl], u[:, sl]
                cur = cd[:, b]
                xtb = cbd[b][cur]                                        # [m, dpb]
                cj = cbd[b]                                              # [16, dpb]
                rpar_j = rpar[:, None] + (xtb * ub).sum(1)[:, None] - ub @ cj.T
                rn2_j = (rn2 - ((xb - xtb) ** 2).sum(1))[:, None] + \
                    ((xb[:, None, :] - cj[None, :, :]) ** 2).sum(-1)
                loss = e1 * rpar_j * rpar_j + rn2_j                       # [m, 16]
                best = torch.argmin(loss, dim=1)
                lb = loss[rows, best]
                lc = loss[rows, cur]
                take = lb < lc
                if bool(take.any()):
                    changed += int(take.sum())
                    nb = torch.where(take, best, cur)
                    rpar = torch.where(take, rpar_j[rows, nb], rpar)
                    rn2 = torch.where(take, rn2_j[rows, nb], rn2)
                    cd[:, b] = nb
            if changed == 0:
                break
        out[s:s + chunk] = cd
    return out


def pack_codes(codes: torch.Tensor) -> torch.Tensor:
    """[n, B] center indices -> [n, B/2] bytes; block 2i low nibble, 2i+1 high."""
    c = codes.to(torch.uint8)
    return (c[:, 0::2] | (c[:, 1::2] << 4)).contiguous()


def unpack_codes(packed: torch.Tensor) -> torch.Tensor:
    lo = packed & 0x0F
    hi = packed >> 4
    return torch.stack([lo, hi], dim=2).reshape(packed.shape[0], -1)


def build_index(w: Workload, X: np.ndarray, device="cpu") -> IndexArrays:
    """Train the index arrays for workload ``w`` on datapoints ``X``.

    Partition (ScaNN builder ``.tree``): NL distinct datapoints chosen with
    ``centroid_seed`` are the centroids; each point joins its nearest centroid
    by squared L2 (ties -> lower leaf).  NL = 1 is "no partitioning": one leaf
    holds every point and its centroid is the data mean.  Slots are the points
    stably sorted by leaf.  Codebook and codes as in ``_train_codebook``,
    ``_l2_codes`` and ``_anisotropic_codes``.
    """
    dev = torch.device(device)
    n, d = X.shape
    assert n == w.n and d == w.d and d % (2 * w.dims_per_block) == 0
    Xt = torch.from_numpy(X).to(dev)
    if w.num_leaves == 1:
        cent = Xt.double().mean(0, keepdim=True).float()
        assign = torch.zeros(n, dtype=torch.int64, device=dev)
    else:
        rng = np.random.default_rng(w.centroid_seed)
        cidx = rng.choice(n, size=w.num_leaves, replace=False)
        cent = Xt[torch.from_numpy(cidx).to(dev)].clone()
        assign = _nearest_rows(Xt, cent)
    order = torch.sort(assign, stable=True).indices
    counts = torch.bincount(assign, minlength=w.num_leaves)
    offs = torch.zeros(w.num_leaves + 1, dtype=torch.int64, device=dev)
    offs[1:] = torch.cumsum(counts, 0)
    Xs = Xt[order]
    del Xt
    # residual codes quantise x minus its leaf's centroid (one codebook for all
    # leaves); the approximate score then adds q . centroid to the table sum
    Ys = Xs - cent[assign[order]] if w.residual else Xs
    cb = _train_codebook(w, Ys)
    codes = _l2_codes(Ys, cb)
    if w.code_loss == "anisotropic":
        codes = _anisotropic_codes(Ys, cb, codes, w.eta, w.aniso_passes)
    del Ys
    packed = pack_codes(codes)
    del codes
    rv = Xs.to(torch.bfloat16) if w.reorder_dtype == "bf16" else Xs
    return IndexArrays(workload=w, centroids=cent.contiguous(), leaf_offsets=offs,
                       slot_ids=order.to(torch.int32), codes=packed, codebook=cb.contiguous(),
                       reorder_vecs=rv.contiguous(), residual=w.residual)


def make_workload(w: Workload, device="cpu", nq: Optional[int] = None):
    """(X, Q, IndexArrays) for ``w``; the index tensors are on ``device``."""
    X = make_data(w)
    Q = make_queries(w, nq)
    ix = build_index(w, X, device)
    return X, Q, ix
