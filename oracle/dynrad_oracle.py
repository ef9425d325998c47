"""CPU oracle for DynamicRad block masks (test infrastructure).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this module.  The CUDA library
never calls it, and it shares no code with the CUDA library.

Plain float64 restatement of the mask generation on the page "DynamicRad:
Content-Adaptive Sparse Attention for Long Video Diffusion", technical summary
section 2(a) "Unified candidate set and dual-mode selection":

  * a hardware-friendly candidate set derived from a radial locality prior
    (attention mass between blocks fades with their spatial and temporal
    distance);
  * static-ratio mode (throughput first): a retention ratio fixed by the
    temporal distance, no content-dependent scoring, a fixed share of the
    candidate set is kept;
  * dynamic-threshold mode (quality first): pre-softmax attention logits as a
    light importance proxy, one global threshold keeps the high-scoring pairs;
    a block left empty by the filter keeps its highest-scoring pair.

The page names the hyper-parameters (decay factor gamma, block size B_s,
thresholds theta) but gives no formulas.  Readings taken:
  * tokens are frame-major, token n = t * S + s with S = N / frames tokens per
    frame (raster order inside a frame);
  * a block is B consecutive tokens of one frame: a frame has
    nb = ceil(S / B) blocks (the last one ragged) and block id c = t * nb + b
    covers tokens [t S + b B, t S + min((b + 1) B, S));
  * radial candidate set: key block (t2, b2) is a candidate of query block
    (t1, b1) iff |b1 - b2| <= w(|t1 - t2|), with the spatial window
    w(d) = floor(w0 * gamma^d) in blocks; w(d) >= 0 always keeps the
    co-located block of every frame (the long-range link);
  * gamma^d is formed by d successive float64 multiplications (w0 * gamma *
    gamma * ...), so every implementation rounds it identically;
  * static-ratio mode: in every key frame, the k = max(1, ceil(rho(d) * m))
    candidates nearest to b1 are kept (|b2 - b1| ascending, ties to the lower
    b2), where m is the number of candidates in that frame and
    rho(d) = min(1, rho0 * gamma^d);
  * dynamic-threshold mode: the proxy of a candidate pair is the pre-softmax
    logit of the block means, scale * mean(q rows of block i) . mean(k rows of
    block j); candidates with proxy >= theta are kept; a query block that
    keeps none keeps its highest-proxy candidate (ties to the lower id);
  * selected key blocks are listed in ascending id order; scale = 1/sqrt(D).

All arithmetic is float64 unless a reading above says otherwise.
"""
from __future__ import annotations

import math
from dataclasses import dataclass
from typing import List, Tuple

import numpy as np

U64 = 2.0 ** -53


def block_layout(N: int, frames: int, B: int) -> Tuple[np.ndarray, int]:
    """Block offsets [Cb + 1] and blocks per frame nb (frame-major token order)."""
    if frames < 1 or N % frames != 0 or B < 1:
        raise ValueError("frames must divide N and B >= 1")
    S = N // frames
    nb = -(-S // B)
    offs = [t * S + min(b * B, S) for t in range(frames) for b in range(nb)]
    offs.append(N)
    return np.asarray(offs, np.int64), nb


def decayed(x0: float, gamma: float, d: int) -> float:
    """x0 * gamma^d by d successive float64 multiplications."""
    v = float(x0)
    for _ in range(d):
        v = v * float(gamma)
    return v


def window(d: int, w0: float, gamma: float) -> int:
    """Spatial window (in blocks) at temporal distance d."""
    return int(math.floor(decayed(w0, gamma, d)))


def candidates(frames: int, nb: int, w0: float, gamma: float) -> List[np.ndarray]:
    """Radial candidate set: per query block, its candidate key block ids, ascending."""
    out = []
    for t1 in range(frames):
        for b1 in range(nb):
            ids = []
            for t2 in range(frames):
                w = window(abs(t1 - t2), w0, gamma)
                for b2 in range(nb):
                    if abs(b1 - b2) <= w:
                        ids.append(t2 * nb + b2)
            out.append(np.asarray(ids, np.int64))
    return out


def static_select(frames: int, nb: int, w0: float, gamma: float, rho0: float) -> List[np.ndarray]:
    """Static-ratio mode: per key frame, the nearest share rho(d) of the candidates."""
    out = []
    for t1 in range(frames):
        for b1 in range(nb):
            ids = []
            for t2 in range(frames):
                d = abs(t1 - t2)
                w = window(d, w0, gamma)
                cand = [b2 for b2 in range(nb) if abs(b1 - b2) <= w]
                rho = min(1.0, decayed(rho0, gamma, d))
                k = max(1, int(math.ceil(rho * len(cand))))
                nearest = sorted(cand, key=lambda b2: (abs(b2 - b1), b2))[:k]
                ids.extend(t2 * nb + b2 for b2 in sorted(nearest))
            out.append(np.asarray(ids, np.int64))
    return out


def block_means(x: np.ndarray, offsets: np.ndarray) -> np.ndarray:
    """Mean row of every block [Cb, D] (float64)."""
    x = np.asarray(x, np.float64)
    return np.stack([x[offsets[c]:offsets[c + 1]].mean(axis=0) for c in range(len(offsets) - 1)])


@dataclass
class DynRow:
    cols: np.ndarray           # kept key block ids, ascending
    proxies: np.ndarray        # proxy logit of every candidate (candidate order)
    band: float                # float64 rounding band of the proxies (two evaluations)
    fallback: bool             # nothing reached theta: the top candidate was kept


def proxy_band(mq_i: np.ndarray, mk: np.ndarray, scale: float) -> float:
    """How far two float64 evaluations of the proxies of one row can differ.

    The block means are exact sums of bf16 values divided once (identical on
    every implementation); the dot product over D channels in another order
    differs by at most gamma_D * sum_d |a_d b_d| (standard forward error
    bound, u = 2^-53), the scaling adds u |proxy|.  Twice that covers two
    evaluations."""
    D = mq_i.shape[0]
    gamma_d = D * U64 / (1.0 - D * U64)
    absdot = np.abs(mk) @ np.abs(mq_i)
    prox = (mk @ mq_i) * scale
    return 2.0 * (scale * gamma_d * float(absdot.max()) + U64 * float(np.abs(prox).max()) + U64)


def dynamic_select(q: np.ndarray, k: np.ndarray, offsets: np.ndarray, frames: int, nb: int, w0: float,
                   gamma: float, theta: float, scale: float) -> List[DynRow]:
    """Dynamic-threshold mode on one head: q, k [N, D]."""
    mq, mk = block_means(q, offsets), block_means(k, offsets)
    rows = []
    for i, cand in enumerate(candidates(frames, nb, w0, gamma)):
        prox = (mk[cand] @ mq[i]) * float(scale)
        keep = prox >= float(theta)
        fallback = not keep.any()
        if fallback:
            keep = np.zeros_like(keep)
            keep[int(np.argmax(prox))] = True      # first maximum = lowest id
        rows.append(DynRow(cand[keep], prox, proxy_band(mq[i], mk[cand], float(scale)), fallback))
    return rows


def dynamic_row_is_valid(gpu_cols: np.ndarray, cand: np.ndarray, row: DynRow, theta: float) -> Tuple[bool, bool]:
    """(valid, decided) for a GPU row of the dynamic mode.

    Decided: no proxy lies within the band of theta and, for a fallback row,
    the top proxy beats the runner-up by more than the band.  A decided row
    must equal the oracle's row.  An undecided row must list candidates in
    ascending order and keep every candidate clearly above theta and none
    clearly below; with none clearly above it keeps either a non-empty subset
    of the candidates near theta or (its own fallback) exactly one candidate
    within the band of the maximum."""
    gpu = np.asarray(gpu_cols, np.int64)
    prox, band = row.proxies, row.band
    above = prox > theta + band
    below = prox < theta - band
    near = ~above & ~below
    decided = not near.any()
    if row.fallback and len(prox) > 1:
        top = np.sort(prox)[::-1]
        decided = decided and (top[0] - top[1] > band)
    if decided:
        return bool(np.array_equal(gpu, row.cols)), True
    if len(gpu) == 0 or not np.all(np.diff(gpu) > 0) or not np.all(np.isin(gpu, cand)):
        return False, False
    pos = {int(c): j for j, c in enumerate(cand)}
    kept = np.zeros(len(cand), bool)
    kept[[pos[int(c)] for c in gpu]] = True
    if above.any():
        return bool(np.all(kept[above]) and not np.any(kept & below)), False
    subset_of_near = not np.any(kept & ~near)
    one_top = kept.sum() == 1 and bool(prox[kept][0] >= prox.max() - band)
    return bool(subset_of_near or one_top), False


def attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, offsets: np.ndarray, sel: List[np.ndarray],
              scale: float) -> Tuple[np.ndarray, np.ndarray]:
    """Exact softmax attention of every query block over its selected key blocks (token order in and out)."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    out = np.zeros_like(q)
    lse = np.zeros(q.shape[0])
    for i, cols in enumerate(sel):
        r0, r1 = offsets[i], offsets[i + 1]
        if r1 <= r0:
            continue
        keys = np.concatenate([np.arange(offsets[j], offsets[j + 1]) for j in cols])
        s = (q[r0:r1] @ k[keys].T) * scale
        m = s.max(axis=1, keepdims=True)
        e = np.exp(s - m)
        l = e.sum(axis=1, keepdims=True)
        out[r0:r1] = (e @ v[keys]) / l
        lse[r0:r1] = (m + np.log(l))[:, 0]
    return out, lse


def density(offsets: np.ndarray, sel: List[np.ndarray]) -> Tuple[int, float]:
    """(selected query-key token pairs, their share of all N^2 pairs)."""
    sizes = np.diff(offsets)
    pairs = int(sum(int(sizes[i]) * int(sizes[np.asarray(cols, np.int64)].sum()) for i, cols in enumerate(sel)))
    N = int(offsets[-1])
    return pairs, pairs / float(N) / float(N)
