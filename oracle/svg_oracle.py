"""CPU oracle for semantic-aware top-p sparse attention (test infrastructure).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this module.  The CUDA library
never calls it, and it shares no code with the CUDA library.

Plain, slow, float64 restatement of the method described on the page
"Sparse VideoGen2: Accelerate Video Generation with Sparse Attention via
Semantic-Aware Permutation" (technical summary, section 2 "Methodology"):

  (a) Semantic-aware permutation -- "Clustering": Q and K tokens of a head
      are clustered independently with k-means into C_q and C_k clusters;
      "Permutation": tokens are reordered so that every cluster is contiguous;
      "Mathematical equivalence": the permutations pi_q, pi_k leave the
      attention output unchanged once it is permuted back.
  (b) Centroid-based top-p selection -- "Centroid approximation": scores are
      computed between cluster centroids instead of tokens; "Top-p strategy":
      clusters are sorted by estimated score and taken in order until their
      cumulative score reaches p.
  (c) System co-design -- "Centroid cache": k-means starts from the previous
      denoising step's centroids; "Customized attention kernel": attention
      over variable-size (q-cluster, k-cluster) blocks.

Readings taken where the page is silent:
  * k-means uses squared Euclidean distance; ties go to the lowest cluster
    index; an empty cluster keeps its previous centroid; the returned
    assignment is the one of the last assign step and the returned centroids
    are the means of exactly that assignment.
  * The score of k-cluster j for q-cluster i is the attention mass the
    centroid pair stands for: w_ij = n_kj * exp(mu_q_i . mu_k_j * scale),
    normalised over the k-clusters of the row (one row per q-cluster).
  * "reaches p" means cumulative normalised score >= p; p >= 1 keeps every
    non-empty k-cluster; empty k-clusters are never selected.
  * scale = 1/sqrt(D); no causal mask (video DiTs attend bidirectionally);
    V is permuted with K's permutation.

All arithmetic is float64.  Inputs are the bfloat16-valued float32 arrays of
``synth``, so the oracle sees exactly the GPU's input values.
"""
from __future__ import annotations

import math
from dataclasses import dataclass
from typing import List, Optional, Sequence, Tuple

import numpy as np

# ---------------------------------------------------------------------------
# (a) k-means  -- section 2(a) "Clustering"; section 2(c) "Centroid cache"
# ---------------------------------------------------------------------------


def sq_distances(x: np.ndarray, mu: np.ndarray) -> np.ndarray:
    """Squared Euclidean distance of every token to every centroid, [N, C].

    ||x - mu||^2 is evaluated as ||x||^2 - 2 x.mu + ||mu||^2 with a float64
    matrix product (a library step); the identity is exact in real
    arithmetic and float64 keeps its rounding far below float32's.
    """
    x = np.asarray(x, np.float64)
    mu = np.asarray(mu, np.float64)
    xx = np.einsum("nd,nd->n", x, x)
    mm = np.einsum("cd,cd->c", mu, mu)
    return xx[:, None] - 2.0 * (x @ mu.T) + mm[None, :]


def kmeans_assign(x: np.ndarray, mu: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """Assign step: a_n = argmin_c ||x_n - mu_c||^2 (ties -> lowest c).

    Returns (assign [N] int64, gap [N] float64) where gap is the distance of
    the second-nearest centroid minus the nearest one (inf when C == 1); a
    small gap marks a token whose assignment a float32 path may legitimately
    flip.
    """
    d = sq_distances(x, mu)
    a = np.argmin(d, axis=1)                       # first minimum = lowest index
    if d.shape[1] == 1:
        return a, np.full(d.shape[0], np.inf)
    part = np.partition(d, 1, axis=1)
    return a, part[:, 1] - part[:, 0]


def kmeans_update(x: np.ndarray, assign: np.ndarray, mu_prev: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """Update step: mu_c = mean of the tokens assigned to c; empty c keeps mu_prev[c]."""
    x = np.asarray(x, np.float64)
    C = mu_prev.shape[0]
    counts = np.bincount(assign, minlength=C)
    sums = np.zeros((C, x.shape[1]), np.float64)
    np.add.at(sums, assign, x)
    mu = np.array(mu_prev, np.float64, copy=True)
    nz = counts > 0
    mu[nz] = sums[nz] / counts[nz, None]
    return mu, counts


def kmeans(x: np.ndarray, mu0: np.ndarray, iters: int):
    """Lloyd's k-means for one head.

    x [N, D]; mu0 [C, D] initial centroids (seeding tokens, or the cached
    centroids of the previous denoising step); iters >= 1 rounds of
    (assign, update).  Returns (mu [C, D] float64, assign [N], counts [C],
    gap [N] of the last assign step).
    """
    if iters < 1:
        raise ValueError("iters must be >= 1")
    mu = np.asarray(mu0, np.float64)
    for _ in range(iters):
        a, gap = kmeans_assign(x, mu)
        mu, counts = kmeans_update(x, a, mu)
    return mu, a, counts, gap


def lloyd_objective(x: np.ndarray, mu: np.ndarray, assign: np.ndarray) -> float:
    """sum_n ||x_n - mu_{a_n}||^2, written out directly."""
    diff = np.asarray(x, np.float64) - np.asarray(mu, np.float64)[assign]
    return float(np.sum(diff * diff))


# ---------------------------------------------------------------------------
# (b) permutation -- section 2(a) "Permutation", "Mathematical equivalence"
# ---------------------------------------------------------------------------


def permutation(assign: np.ndarray, C: int) -> Tuple[np.ndarray, np.ndarray]:
    """Stable sort of token indices by cluster id.

    Returns (perm [N], offsets [C+1]): row r of the permuted tensor is token
    perm[r]; cluster c occupies rows [offsets[c], offsets[c+1]); inside a
    cluster tokens keep ascending index order.
    """
    assign = np.asarray(assign)
    perm = np.argsort(assign, kind="stable")
    counts = np.bincount(assign, minlength=C)
    offsets = np.concatenate([[0], np.cumsum(counts)])
    return perm.astype(np.int64), offsets.astype(np.int64)


def gather_rows(x: np.ndarray, perm: np.ndarray) -> np.ndarray:
    """Permuted tensor: xp[r] = x[perm[r]]."""
    return np.asarray(x)[perm]


def scatter_rows(xp: np.ndarray, perm: np.ndarray) -> np.ndarray:
    """Inverse permutation: x[perm[r]] = xp[r]."""
    out = np.empty_like(xp)
    out[perm] = xp
    return out


# ---------------------------------------------------------------------------
# (c) centroid scores and top-p -- section 2(b)
# ---------------------------------------------------------------------------


def centroid_weights(mu_q_i: np.ndarray, mu_k: np.ndarray, n_k: np.ndarray, scale: float) -> np.ndarray:
    """Normalised score of every k-cluster for one q-cluster (0 for empty k-clusters).

    logit_j = mu_q_i . mu_k_j * scale;  w_j = n_kj exp(logit_j - max) / sum.
    """
    logits = (np.asarray(mu_k, np.float64) @ np.asarray(mu_q_i, np.float64)) * float(scale)
    live = np.asarray(n_k) > 0
    w = np.zeros(len(logits), np.float64)
    if not live.any():
        return w
    m = logits[live].max()
    w[live] = np.asarray(n_k, np.float64)[live] * np.exp(logits[live] - m)
    return w / w.sum()


# Unit roundoff of float64.
U64 = 2.0 ** -53
# Two weights closer than this (relative) are treated as equal at the cut: a
# float64 evaluation of either weight may order them either way.
TIE_REL = 2.0 ** -38


def selection_band(mu_q_i: np.ndarray, mu_k: np.ndarray, n_k: np.ndarray, scale: float) -> float:
    """How far two float64 evaluations of one row's normalised prefix masses can differ.

    The top-p cut of a row is a comparison of prefix masses with p; both this
    oracle and a float64 kernel evaluate them with rounding.  Bound (standard
    forward error analysis, u = 2^-53, gamma_n = n u / (1 - n u)):
      * logit_j = scale * mu_q . mu_k_j over D channels: error at most
        scale * gamma_D * sum_d |mu_q_d mu_k_jd| + u |logit_j|; the row max
        shifts by at most the same amount;
      * a weight n_j exp(logit_j - max) then carries a relative error
        rho <= 2 * max_j (logit error) + 4u (exp and the product);
      * a normalised prefix C_k / S moves by at most 2 rho from the weights
        plus 2 gamma_(n + 8) from the two sums over n live clusters, and the
        threshold p * S by u.
    The band covers both evaluations (twice one evaluation's bound).
    """
    mu_q_i = np.asarray(mu_q_i, np.float64)
    mu_k = np.asarray(mu_k, np.float64)
    live = np.asarray(n_k) > 0
    if not live.any():
        return 0.0
    D = mu_q_i.shape[0]
    gamma_d = D * U64 / (1.0 - D * U64)
    absdot = np.abs(mu_k[live]) @ np.abs(mu_q_i)
    logits = (mu_k[live] @ mu_q_i) * float(scale)
    dl = float(scale) * gamma_d * float(absdot.max()) + U64 * float(np.abs(logits).max())
    rho = 2.0 * dl + 4.0 * U64
    n = int(live.sum())
    gamma_n = (n + 8) * U64 / (1.0 - (n + 8) * U64)
    return 2.0 * (2.0 * rho + 2.0 * gamma_n + U64)


@dataclass
class RowSelection:
    cols: np.ndarray          # selected k-cluster ids, ascending
    order: np.ndarray         # all live k-clusters by descending weight (ties: lower id)
    weights: np.ndarray       # normalised weights [Ck]
    undecided: bool           # the cut sits within `band` of p, or between near-equal weights
    band: float = 0.0         # the band the row was decided with


def select_row(weights: np.ndarray, p: float, tol: float,
               live_mask: Optional[np.ndarray] = None) -> RowSelection:
    """Smallest prefix of the descending-score order whose mass reaches p.

    ``live_mask`` marks the non-empty k-clusters (default: weight > 0).
    ``tol`` is the row's rounding band (``selection_band``): the row is marked
    undecided when a prefix mass next to the cut lies within ``tol`` of p, or
    when the last kept and the first dropped weights are equal within TIE_REL.
    """
    w = np.asarray(weights, np.float64)
    live = np.nonzero(w > 0 if live_mask is None else np.asarray(live_mask))[0]
    if len(live) == 0:
        return RowSelection(np.zeros(0, np.int64), live, w, False, tol)
    # descending weight, ties -> lower index (stable sort of ascending index list)
    order = live[np.argsort(-w[live], kind="stable")]
    if p >= 1.0:
        return RowSelection(np.sort(order), order, w, False, tol)
    csum = np.cumsum(w[order])
    k = int(np.searchsorted(csum, p, side="left")) + 1     # first prefix with csum >= p
    k = min(k, len(order))
    undecided = abs(csum[k - 1] - p) < tol or (k >= 2 and abs(csum[k - 2] - p) < tol)
    if k < len(order):
        wl, wn = w[order[k - 1]], w[order[k]]
        undecided = undecided or (wl - wn) <= TIE_REL * wl
    return RowSelection(np.sort(order[:k]), order, w, bool(undecided), tol)


def select_topp(mu_q: np.ndarray, n_q: np.ndarray, mu_k: np.ndarray, n_k: np.ndarray,
                p: float, scale: float) -> List[RowSelection]:
    """Per q-cluster top-p block selection for one head.  Empty q-clusters select nothing."""
    rows = []
    for i in range(mu_q.shape[0]):
        if n_q[i] == 0:
            rows.append(RowSelection(np.zeros(0, np.int64), np.zeros(0, np.int64),
                                     np.zeros(mu_k.shape[0]), False, 0.0))
            continue
        band = selection_band(mu_q[i], mu_k, n_k, scale)
        rows.append(select_row(centroid_weights(mu_q[i], mu_k, n_k, scale), p, band,
                               np.asarray(n_k) > 0))
    return rows


def selection_is_valid(gpu_cols: Sequence[int], weights: np.ndarray, p: float, tol: float) -> bool:
    """Whether a selection is an acceptable minimal top-p set up to rounding.

    ``tol`` is the row's band (``selection_band``).  Accepts the set when
    (i) it only holds live clusters, (ii) every selected weight is at least
    every unselected weight (within TIE_REL relative), (iii) its mass reaches
    p - tol, and (iv) without its lightest member it stays below p + tol.
    """
    w = np.asarray(weights, np.float64)
    sel = np.asarray(sorted(set(int(c) for c in gpu_cols)), np.int64)
    if len(sel) == 0 or np.any(w[sel] <= 0):
        return False
    live = np.nonzero(w > 0)[0]
    if p >= 1.0:
        return np.array_equal(sel, live)
    uns = np.setdiff1d(live, sel)
    if len(uns) and w[sel].min() < w[uns].max() * (1 - TIE_REL):
        return False
    mass = w[sel].sum()
    if mass < p - tol:
        return False
    return mass - w[sel].min() < p + tol


# ---------------------------------------------------------------------------
# (d) attention over the selected blocks -- section 2(a) "Mathematical
#     equivalence", section 2(c) "Customized attention kernel"
# ---------------------------------------------------------------------------


def key_rows(k_off: np.ndarray, cols: Sequence[int]) -> np.ndarray:
    """Permuted key rows covered by a set of k-clusters."""
    parts = [np.arange(k_off[j], k_off[j + 1]) for j in cols]
    return np.concatenate(parts) if parts else np.zeros(0, np.int64)


def softmax_attention_rows(q_rows: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float):
    """Exact softmax attention of some query rows over a key/value set (float64).

    Returns (out [R, D], lse [R]) with lse the natural-log sum of
    exp(scale * q.k) over the keys.
    """
    q_rows = np.asarray(q_rows, np.float64)
    s = (q_rows @ np.asarray(k, np.float64).T) * float(scale)
    m = s.max(axis=1, keepdims=True)
    e = np.exp(s - m)
    l = e.sum(axis=1, keepdims=True)
    out = (e @ np.asarray(v, np.float64)) / l
    return out, (m + np.log(l))[:, 0]


def sparse_attention(qp: np.ndarray, kp: np.ndarray, vp: np.ndarray, q_off: np.ndarray,
                     k_off: np.ndarray, selection: Sequence[Sequence[int]], scale: float,
                     rows: Optional[np.ndarray] = None):
    """Block-sparse attention on permuted tensors of one head.

    Query rows of q-cluster i attend to the union of the key rows of the
    k-clusters selected for i.  ``rows`` restricts the computation to some
    permuted query rows (sampled checks); other rows are returned as NaN.
    Returns (op [N, D] float64, lse [N] float64).
    """
    N, D = qp.shape
    op = np.full((N, vp.shape[1]), np.nan)
    lse = np.full(N, np.nan)
    want = np.ones(N, bool) if rows is None else np.isin(np.arange(N), rows)
    for i, cols in enumerate(selection):
        r0, r1 = int(q_off[i]), int(q_off[i + 1])
        rr = np.arange(r0, r1)[want[r0:r1]]
        if len(rr) == 0:
            continue
        kr = key_rows(k_off, cols)
        if len(kr) == 0:
            raise ValueError(f"q-cluster {i} has rows but selects no keys")
        o, l = softmax_attention_rows(qp[rr], kp[kr], vp[kr], scale)
        op[rr], lse[rr] = o, l
    return op, lse


def dense_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float,
                    rows: Optional[np.ndarray] = None) -> np.ndarray:
    """Textbook softmax attention, one query row at a time (no blocking)."""
    rows = np.arange(q.shape[0]) if rows is None else rows
    k64 = np.asarray(k, np.float64)
    v64 = np.asarray(v, np.float64)
    out = np.empty((len(rows), v.shape[1]), np.float64)
    for t, r in enumerate(rows):
        s = k64 @ np.asarray(q[r], np.float64) * float(scale)
        e = np.exp(s - s.max())
        out[t] = (e / e.sum()) @ v64
    return out


# ---------------------------------------------------------------------------
# the whole layer, one head at a time
# ---------------------------------------------------------------------------


@dataclass
class HeadResult:
    mu_q: np.ndarray
    mu_k: np.ndarray
    assign_q: np.ndarray
    assign_k: np.ndarray
    gap_q: np.ndarray
    gap_k: np.ndarray
    n_q: np.ndarray
    n_k: np.ndarray
    perm_q: np.ndarray
    perm_k: np.ndarray
    q_off: np.ndarray
    k_off: np.ndarray
    selection: List[RowSelection]
    out: Optional[np.ndarray]          # un-permuted output [N, D] (NaN outside sampled rows)
    lse: Optional[np.ndarray]


def svg_head(q: np.ndarray, k: np.ndarray, v: np.ndarray, mu_q0: np.ndarray, mu_k0: np.ndarray,
             iters: int, p: float, scale: Optional[float] = None, attn_rows: Optional[np.ndarray] = None,
             attention: bool = True) -> HeadResult:
    """One head of the layer: k-means(Q), k-means(K), permute, select, attend, un-permute.

    ``attn_rows`` (original token indices) restricts the attention stage to
    those query tokens.
    """
    D = q.shape[1]
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    mu_q, a_q, n_q, g_q = kmeans(q, mu_q0, iters)
    mu_k, a_k, n_k, g_k = kmeans(k, mu_k0, iters)
    perm_q, q_off = permutation(a_q, mu_q.shape[0])
    perm_k, k_off = permutation(a_k, mu_k.shape[0])
    sel = select_topp(mu_q, n_q, mu_k, n_k, p, scale)
    out = lse = None
    if attention:
        qp, kp, vp = gather_rows(q, perm_q), gather_rows(k, perm_k), gather_rows(v, perm_k)
        prow = None
        if attn_rows is not None:
            inv = np.empty_like(perm_q)
            inv[perm_q] = np.arange(len(perm_q))
            prow = np.sort(inv[np.asarray(attn_rows)])
        op, lsep = sparse_attention(qp, kp, vp, q_off, k_off, [s.cols for s in sel], scale, prow)
        out, lse = scatter_rows(op, perm_q), scatter_rows(lsep, perm_q)
    return HeadResult(mu_q, mu_k, a_q, a_k, g_q, g_k, n_q, n_k, perm_q, perm_k, q_off, k_off, sel, out, lse)


def density(q_off: np.ndarray, k_off: np.ndarray, selection: Sequence[Sequence[int]]) -> Tuple[float, float]:
    """(selected query-key pairs, fraction of N^2) for one head."""
    nq = np.diff(q_off)
    nk = np.diff(k_off)
    pairs = float(sum(nq[i] * nk[np.asarray(c, np.int64)].sum() for i, c in enumerate(selection) if len(c)))
    N = float(q_off[-1])
    return pairs, pairs / (N * N)
