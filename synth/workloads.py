"""Synthetic routing, gate weights and hidden states for the five workloads.

The pages measure on real routing of trained MoE models (Megatron-LM
pretraining runs in "Expert Coupling in MoE Pretraining", abstract;
GLM-4.5-Air in "Cobalt", "Key Observation").  Neither the weights nor the
data exist here, so these generators stand in for them with the structure
the pages describe: experts that tokens tend to pick jointly (clusters of
experts chosen together by a token) and next-layer experts that are
predictable from this layer's (cluster persistence across layers), with a
skewed (Zipf) popularity of clusters.  The DODOCO abstract warns that Zipf
mock tokens overstate routing imbalance; these are stand-ins, not a model of
real routing.

Recipe (draw order is part of the definition, so both sides of a test see the
same bits):

* ``numpy.random.Generator(PCG64)`` streams seeded with ``SeedSequence``:
  ``[layout_seed, 0]`` draws the per-layer cluster layout -- the stand-in for
  the trained router, shared by every batch of one workload, so it defaults to
  the workload's seed -- ``[seed, 0, 1 + b]`` the routing of token block b
  (65536 tokens per block), ``[seed, 1]`` the gate logits and ``[seed, 2, b]``
  hidden-state row block b (4096 rows per block).  A calibration batch is the
  same workload with another token seed;
* per layer l a random permutation pi_l of the E expert ids, cut into
  ``n_clusters`` clusters of ``cluster_size`` (so clusters are never runs of
  contiguous ids);
* layer 0: each token draws a cluster from ``cluster_probs`` (Zipf:
  P(c) proportional to (c+1)^-s);
* layer l+1: with probability ``persistence`` the token's cluster becomes
  sigma_l(c) (sigma_l = identity for ``next_cluster == "keep"``, a fixed random
  permutation drawn once per layer pair for ``"perm"``), otherwise it is
  redrawn from the cluster law;
* k picks without repeats: each pick, with probability ``p_in``, is uniform
  over the token's not yet chosen in-cluster experts; otherwise, or when those
  are exhausted, uniform over all not yet chosen experts (rejection sampling,
  which is exactly uniform over the remaining set);
* gate weights: softmax over the k chosen experts of N(0,1) logits, fp32;
* stand-in experts (for the receiver-side pre-reduced combine): expert e of
  layer l scales its input row by a factor drawn uniformly from [0.5, 1.5]
  (fp32, stream ``[seed, 3]``);
* hidden states: N(0,1) fp32, rounded to bf16 (round to nearest even) where
  the workload is bf16.
"""
from __future__ import annotations

from dataclasses import dataclass, replace
from typing import Optional, Tuple

import numpy as np

STREAM_ROUTING = 0
STREAM_GATES = 1
STREAM_HIDDEN = 2
STREAM_EXPERTS = 3


@dataclass(frozen=True)
class Workload:
    name: str
    T: int                      # tokens
    E: int                      # experts per layer
    k: int                      # experts per token (top-k)
    L: int                      # MoE layers
    G: int                      # logical EP ranks (0: statistics-only workload)
    rpn: int                    # ranks per node
    d: int                      # hidden size (0: no hidden states)
    dtype: str                  # "f32" | "bf16" | "" (no hidden states)
    n_clusters: int
    cluster_size: int
    p_in: float                 # probability that a pick is in-cluster
    persistence: float          # probability the cluster carries to the next layer
    next_cluster: str = "keep"  # "keep" (sigma = id) or "perm" (fixed permutation)
    zipf_s: Optional[float] = None
    cluster_probs: Optional[Tuple[float, ...]] = None
    seed: int = 0
    sweep_G: Tuple[int, ...] = ()

    def probs(self) -> np.ndarray:
        if self.cluster_probs is not None:
            p = np.asarray(self.cluster_probs, dtype=np.float64)
        else:
            c = np.arange(self.n_clusters, dtype=np.float64)
            p = (c + 1.0) ** (-float(self.zipf_s))
        return p / p.sum()

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)

    @property
    def elem_bytes(self) -> int:
        return {"f32": 4, "bf16": 2}.get(self.dtype, 0)


# The five workloads, with the shapes, sizes and structure stated for them.
# Where a workload states no cluster persistence ("ep32"), the next layer's
# cluster is drawn afresh (persistence 0): the plainest reading of a
# description that gives no layer-to-layer relation.
WORKLOADS = {
    "tiny": Workload("tiny", T=4096, E=8, k=2, L=2, G=4, rpn=2, d=128, dtype="f32",
                     n_clusters=2, cluster_size=4, cluster_probs=(0.5, 0.5),
                     p_in=0.8, persistence=0.7, next_cluster="keep"),
    "one_node": Workload("one_node", T=16384, E=64, k=2, L=2, G=8, rpn=8, d=2048, dtype="bf16",
                         n_clusters=16, cluster_size=4, zipf_s=1.1,
                         p_in=0.85, persistence=0.75, next_cluster="perm"),
    "ep32": Workload("ep32", T=65536, E=64, k=6, L=2, G=32, rpn=8, d=4096, dtype="bf16",
                     n_clusters=8, cluster_size=8, zipf_s=1.0,
                     p_in=0.7, persistence=0.0, next_cluster="keep"),
    "large_ep64": Workload("large_ep64", T=131072, E=256, k=8, L=4, G=64, rpn=8, d=7168, dtype="bf16",
                           n_clusters=32, cluster_size=8, zipf_s=1.2,
                           p_in=0.75, persistence=0.6, next_cluster="keep"),
    "stats_sweep": Workload("stats_sweep", T=1048576, E=128, k=8, L=8, G=0, rpn=8, d=0, dtype="",
                            n_clusters=16, cluster_size=8, zipf_s=1.1,
                            p_in=0.8, persistence=0.7, next_cluster="keep",
                            sweep_G=(8, 32, 64)),
}


def _rng(seed: int, stream: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([int(seed), int(stream)])))


def _draw_clusters(rng: np.random.Generator, p: np.ndarray, n: int) -> np.ndarray:
    # inverse-CDF draw; ties at the boundaries are measure-zero
    cdf = np.cumsum(p)
    cdf[-1] = 1.0
    u = rng.random(n)
    return np.searchsorted(cdf, u, side="right").astype(np.int64)


def _pick_without_repeats(rng, ids, j, idx, draw):
    """Fill ids[idx, j] by rejection: redraw where the candidate repeats an earlier pick."""
    while idx.size:
        cand = draw(idx)
        if j:
            clash = (ids[idx, :j] == cand[:, None]).any(axis=1)
        else:
            clash = np.zeros(idx.size, dtype=bool)
        ok = ~clash
        ids[idx[ok], j] = cand[ok]
        idx = idx[clash]


def _layout(w: Workload, seed: int):
    """Per-layer cluster members and layer-pair cluster maps sigma_l."""
    rng = _rng(seed, STREAM_ROUTING)
    E, L, nc, cs = w.E, w.L, w.n_clusters, w.cluster_size
    members, cluster_of, sigmas = [], [], [np.arange(nc, dtype=np.int64)]
    for l in range(L):
        perm = rng.permutation(E).astype(np.int32)
        m = perm[: nc * cs].reshape(nc, cs)
        co = np.full(E, -1, dtype=np.int64)
        for q in range(nc):
            co[m[q]] = q
        members.append(m)
        cluster_of.append(co)
        if l > 0:
            if w.next_cluster == "perm":
                sigmas.append(rng.permutation(nc).astype(np.int64))
            else:
                sigmas.append(np.arange(nc, dtype=np.int64))
    return members, cluster_of, sigmas


def _routing_block(w: Workload, seed: int, block: int, n: int, layout) -> np.ndarray:
    members, cluster_of, sigmas = layout
    E, k, L, cs = w.E, w.k, w.L, w.cluster_size
    rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence([int(seed), STREAM_ROUTING, 1 + block])))
    p = w.probs()
    out = np.empty((L, n, k), dtype=np.int32)
    cl = None
    for l in range(L):
        if l == 0:
            cl = _draw_clusters(rng, p, n)
        else:
            keep = rng.random(n) < w.persistence
            fresh = _draw_clusters(rng, p, n)
            cl = np.where(keep, sigmas[l][cl], fresh)
        m, co = members[l], cluster_of[l]
        ids = np.full((n, k), -1, dtype=np.int32)
        n_in = np.zeros(n, dtype=np.int64)
        for j in range(k):
            want_in = rng.random(n) < w.p_in
            use_in = want_in & (n_in < cs)
            idx_in = np.nonzero(use_in)[0]
            idx_all = np.nonzero(~use_in)[0]
            _pick_without_repeats(
                rng, ids, j, idx_in,
                lambda ii: m[cl[ii], rng.integers(0, cs, ii.size)].astype(np.int32))
            _pick_without_repeats(
                rng, ids, j, idx_all,
                lambda ii: rng.integers(0, E, ii.size).astype(np.int32))
            n_in += co[ids[:, j]] == cl
        out[l] = ids
    return out


TOKENS_PER_BLOCK = 65536


def _parallel(fn, nblocks):
    if nblocks == 1:
        return [fn(0)]
    from concurrent.futures import ThreadPoolExecutor
    import os
    with ThreadPoolExecutor(max_workers=min(nblocks, os.cpu_count() or 1)) as ex:
        return list(ex.map(fn, range(nblocks)))


def make_routing(w: Workload, seed: Optional[int] = None, T: Optional[int] = None,
                 layout_seed: Optional[int] = None) -> np.ndarray:
    """Top-k expert ids, int32 [L][T][k], k distinct ids per token and layer.

    Tokens are drawn in blocks of TOKENS_PER_BLOCK, each from its own
    generator, so the result does not depend on the thread count.  The
    cluster layout comes from ``layout_seed`` (default: the workload's seed).
    """
    seed = w.seed if seed is None else seed
    layout_seed = w.seed if layout_seed is None else layout_seed
    T = w.T if T is None else T
    if w.n_clusters * w.cluster_size > w.E:
        raise ValueError("clusters do not fit in E")
    if w.k > w.E:
        raise ValueError("k > E")
    layout = _layout(w, layout_seed)
    nb = max(1, -(-T // TOKENS_PER_BLOCK))
    parts = _parallel(lambda b: _routing_block(
        w, seed, b, min(T, (b + 1) * TOKENS_PER_BLOCK) - b * TOKENS_PER_BLOCK, layout), nb)
    return np.ascontiguousarray(np.concatenate(parts, axis=1))


def make_gates(w: Workload, seed: Optional[int] = None, T: Optional[int] = None) -> np.ndarray:
    """Gate weights, fp32 [L][T][k]: softmax over the k chosen experts of N(0,1) logits."""
    seed = w.seed if seed is None else seed
    T = w.T if T is None else T
    rng = _rng(seed, STREAM_GATES)
    z = rng.standard_normal((w.L, T, w.k), dtype=np.float32)
    z = z - z.max(axis=-1, keepdims=True)
    e = np.exp(z, dtype=np.float32)
    return (e / e.sum(axis=-1, keepdims=True, dtype=np.float32)).astype(np.float32)


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (nearest, ties to even); returns the uint16 bit patterns."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    r = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def make_hidden(w: Workload, seed: Optional[int] = None, T: Optional[int] = None,
                rows_per_block: int = 4096) -> np.ndarray:
    """Hidden states x [T][d]: float32 array for "f32", uint16 bf16 bits for "bf16".

    Rows are drawn in blocks of ``rows_per_block``, block b from generator
    SeedSequence([seed, 2, b]), so any block can be regenerated on its own.
    """
    seed = w.seed if seed is None else seed
    T = w.T if T is None else T
    if w.d <= 0:
        raise ValueError("workload has no hidden states")
    bf16 = w.dtype == "bf16"
    out = np.empty((T, w.d), dtype=np.uint16 if bf16 else np.float32)

    def fill(b):
        r0 = b * rows_per_block
        r1 = min(T, r0 + rows_per_block)
        rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence([int(seed), STREAM_HIDDEN, b])))
        v = rng.standard_normal((r1 - r0, w.d), dtype=np.float32)
        out[r0:r1] = f32_to_bf16_bits(v) if bf16 else v

    _parallel(fill, max(1, -(-T // rows_per_block)))
    return out


def make_expert_scales(w: Workload, seed: Optional[int] = None) -> np.ndarray:
    """Per-expert scale factors of the stand-in experts, fp32 [L][E] in [0.5, 1.5)."""
    seed = w.seed if seed is None else seed
    rng = _rng(seed, STREAM_EXPERTS)
    return (0.5 + rng.random((w.L, w.E))).astype(np.float32)
