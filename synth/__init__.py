"""Seeded synthetic inputs shaped like video-DiT self-attention layers.

This module only draws data: Q, K, V for one attention layer and the token
indices that seed k-means.  It holds none of the sparse-attention method's
arithmetic, so both the CPU oracle (``oracle/``) and the CUDA path read their
inputs from here and nothing else is shared between them.

Workload shapes follow the token counts quoted for Wan-class video DiTs on
the "long video generation, six approaches" page (section "VRAM wall":
about 32.7K latent tokens for an 81-frame clip, about 65.5K for 165 frames)
and the 480p/720p HunyuanVideo / Wan 2.1 settings of the Sparse VideoGen2
page (section 4, experimental results).  Latent grids use 4x temporal and
16x spatial compression: 81 frames at 480x832 -> 21x30x52 = 32,760 tokens.

Value recipe (one independent stream per tensor and head):
  * the (t, h, w) grid is cut into R_t x R_h x R_w contiguous regions;
  * every head draws one N(0, I_D) centre per region;  Q and K of a token are
    that region's centre plus isotropic Gaussian noise (the centre set is
    shared by Q and K: "region-correlated");
  * V is either centre + noise from its own centre set (tiny case) or i.i.d.
    N(0, 1);
  * the drifting variant moves every centre linearly along t;
  * every value is rounded to bfloat16 (round to nearest even) here, so the
    CPU oracle and the GPU see bit-identical inputs.

k-means seeding: C distinct token indices per head, drawn without
replacement; the initial centroids are those tokens' rows.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Dict, Optional, Sequence, Tuple

import numpy as np

# stream tags: one independent random stream per (seed, tag, head)
TAG_CENTRES, TAG_QNOISE, TAG_KNOISE, TAG_V, TAG_INIT_Q, TAG_INIT_K, TAG_VCENTRES, TAG_DRIFT = range(8)


@dataclass(frozen=True)
class Workload:
    name: str
    heads: int
    head_dim: int
    grid: Tuple[int, int, int]            # latent (t, h, w)
    regions: Tuple[int, int, int]         # regions along (t, h, w); (0,0,0) = no structure
    qk_noise: float                       # std of the per-token noise around the centre
    v_mode: str                           # "centre" | "iid"
    cq: int
    ck: int
    iters: int
    top_p: Tuple[float, ...]
    drift: float = 0.0                    # std of the per-region drift vector (0 = static)
    warm_iters: int = 0                   # >0: a second, warm-started call with these iterations
    seed: int = 0
    noise_seeds: Tuple[int, int] = (1, 2)
    warm_noise_seeds: Tuple[int, int] = (11, 12)

    @property
    def tokens(self) -> int:
        t, h, w = self.grid
        return t * h * w

    @property
    def bh(self) -> int:
        return self.heads


WORKLOADS: Dict[str, Workload] = {
    # 1 head, d=64, 4x16x32 tokens in 8 octant regions, noise 0.3
    "tiny": Workload("tiny", 1, 64, (4, 16, 32), (2, 2, 2), 0.3, "centre", 32, 64, 10, (0.9, 1.0)),
    # 480p, 5 s: 81 frames -> 21x30x52 latent tokens
    "480p-5s": Workload("480p-5s", 40, 128, (21, 30, 52), (4, 4, 4), 0.5, "iid", 100, 500, 5, (0.9,)),
    # 720p, 5 s: 21x45x80 latent tokens, top-p sweep
    "720p-5s": Workload("720p-5s", 40, 128, (21, 45, 80), (4, 4, 4), 0.5, "iid", 200, 1000, 5,
                        (0.5, 0.75, 0.9, 0.95)),
    # 480p, 10 s: 41x30x52 tokens, drifting centres, warm start from the first call
    "480p-10s": Workload("480p-10s", 40, 128, (41, 30, 52), (4, 4, 4), 0.5, "iid", 200, 1000, 5, (0.9,),
                         drift=0.5, warm_iters=2),
    # dense anchors: no cluster structure, top-p = 1
    "dense-d128": Workload("dense-d128", 40, 128, (21, 30, 52), (0, 0, 0), 1.0, "iid", 100, 500, 5, (1.0,)),
    "dense-d64": Workload("dense-d64", 80, 64, (21, 30, 52), (0, 0, 0), 1.0, "iid", 100, 500, 5, (1.0,)),
}


def _rng(seed: int, tag: int, head: int) -> np.random.Generator:
    return np.random.default_rng(np.random.SeedSequence([int(seed), int(tag), int(head)]))


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bfloat16 (ties to even); returns float32."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    b = x.view(np.uint32).astype(np.uint64)
    b = (b + 0x7FFF + ((b >> 16) & 1)) & 0xFFFF0000
    return b.astype(np.uint32).view(np.float32)


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """Upper 16 bits of float32 values that are already bfloat16-representable."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    bits = x.view(np.uint32)
    if np.any(bits & 0xFFFF):
        raise ValueError("values are not bfloat16-representable; call round_bf16 first")
    return (bits >> 16).astype(np.uint16)


def region_of_tokens(grid: Sequence[int], regions: Sequence[int]) -> np.ndarray:
    """Region id of every token of a row-major (t, h, w) grid."""
    T, Hh, W = grid
    Rt, Rh, Rw = regions
    t = np.arange(T)[:, None, None]
    h = np.arange(Hh)[None, :, None]
    w = np.arange(W)[None, None, :]
    r = ((t * Rt) // T) * (Rh * Rw) + ((h * Rh) // Hh) * Rw + (w * Rw) // W
    return np.broadcast_to(r, (T, Hh, W)).reshape(-1)


@dataclass
class LayerInputs:
    workload: Workload
    q: np.ndarray                    # [BH, N, D] float32, bfloat16-valued
    k: np.ndarray
    v: np.ndarray
    init_q_idx: np.ndarray           # [BH, Cq] int64 token indices
    init_k_idx: np.ndarray           # [BH, Ck] int64
    extra: Dict[str, np.ndarray] = field(default_factory=dict)

    def init_centroids(self, which: str) -> np.ndarray:
        """Rows of the seeding tokens: [BH, C, D] float32."""
        x = self.q if which == "q" else self.k
        idx = self.init_q_idx if which == "q" else self.init_k_idx
        return np.take_along_axis(x, idx[:, :, None], axis=1).astype(np.float32)


def make_layer(name_or_wl, heads: Optional[int] = None, call: int = 0) -> LayerInputs:
    """Draw one layer's inputs.

    ``heads`` limits the draw to the first ``heads`` heads (the values of a head
    do not depend on how many heads are drawn).  ``call`` selects the noise of
    the first (0) or the warm-started second (1) call of a drifting workload;
    the centres, drift and seeding indices are the same for both calls.
    """
    wl = WORKLOADS[name_or_wl] if isinstance(name_or_wl, str) else name_or_wl
    H = wl.heads if heads is None else int(heads)
    N, D = wl.tokens, wl.head_dim
    qs, ks = (wl.noise_seeds if call == 0 else wl.warm_noise_seeds)
    q = np.empty((H, N, D), np.float32)
    k = np.empty((H, N, D), np.float32)
    v = np.empty((H, N, D), np.float32)
    iq = np.empty((H, wl.cq), np.int64)
    ik = np.empty((H, wl.ck), np.int64)
    structured = all(r > 0 for r in wl.regions)
    region = region_of_tokens(wl.grid, wl.regions) if structured else None
    nreg = int(np.prod(wl.regions)) if structured else 0
    for h in range(H):
        if structured:
            centres = _rng(wl.seed, TAG_CENTRES, h).standard_normal((nreg, D), dtype=np.float32)
            drift = None
            if wl.drift > 0:
                drift = np.float32(wl.drift) * _rng(wl.seed, TAG_DRIFT, h).standard_normal(
                    (nreg, D), dtype=np.float32)
            nq = _rng(qs, TAG_QNOISE, h).standard_normal((N, D), dtype=np.float32)
            nk = _rng(ks, TAG_KNOISE, h).standard_normal((N, D), dtype=np.float32)
            q[h] = centres[region] + np.float32(wl.qk_noise) * nq
            k[h] = centres[region] + np.float32(wl.qk_noise) * nk
            if drift is not None:
                T = wl.grid[0]
                frac = (np.repeat(np.arange(T), wl.grid[1] * wl.grid[2]).astype(np.float32)
                        / np.float32(max(T - 1, 1)))
                q[h] += frac[:, None] * drift[region]
                k[h] += frac[:, None] * drift[region]
            if wl.v_mode == "centre":
                vc = _rng(wl.seed, TAG_VCENTRES, h).standard_normal((nreg, D), dtype=np.float32)
                nv = _rng(wl.seed, TAG_V, h).standard_normal((N, D), dtype=np.float32)
                v[h] = vc[region] + np.float32(wl.qk_noise) * nv
            else:
                v[h] = _rng(wl.seed, TAG_V, h).standard_normal((N, D), dtype=np.float32)
        else:
            q[h] = _rng(qs, TAG_QNOISE, h).standard_normal((N, D), dtype=np.float32)
            k[h] = _rng(ks, TAG_KNOISE, h).standard_normal((N, D), dtype=np.float32)
            v[h] = _rng(wl.seed, TAG_V, h).standard_normal((N, D), dtype=np.float32)
        iq[h] = np.sort(_rng(wl.seed + 4, TAG_INIT_Q, h).choice(N, wl.cq, replace=False))
        ik[h] = np.sort(_rng(wl.seed + 4, TAG_INIT_K, h).choice(N, wl.ck, replace=False))
    return LayerInputs(wl, round_bf16(q), round_bf16(k), round_bf16(v), iq, ik)


def small_workload(base: str, tokens_grid: Tuple[int, int, int], heads: int, cq: int, ck: int,
                   iters: Optional[int] = None, head_dim: Optional[int] = None) -> Workload:
    """A reduced copy of a named workload (same value recipe, fewer tokens/heads)."""
    wl = WORKLOADS[base]
    return Workload(f"{base}-small", heads, head_dim or wl.head_dim, tokens_grid, wl.regions,
                    wl.qk_noise, wl.v_mode, cq, ck, iters if iters is not None else wl.iters, wl.top_p,
                    drift=wl.drift, warm_iters=wl.warm_iters, seed=wl.seed, noise_seeds=wl.noise_seeds,
                    warm_noise_seeds=wl.warm_noise_seeds)


def sample_rows(n_rows: int, count: int, seed: int) -> np.ndarray:
    """Sorted distinct row indices used by sampled parity checks."""
    count = min(count, n_rows)
    return np.sort(_rng(seed, 99, 0).choice(n_rows, count, replace=False))
