"""Shared helpers for the GPU parity tests (host<->device marshalling and the
comparison rules; the expected values always come from oracle/)."""
import numpy as np
import torch

import synth

# Attention tolerance (bf16 GPU inputs/outputs vs float64 oracle), per output tensor.
ATTN_REL_L2 = 1e-2
ATTN_MAX_ABS = 2e-2
# k-means: fraction of tokens whose final assignment must agree after T rounds.
KMEANS_AGREE = 0.999


def as_f32(p: float) -> float:
    """The float32 value a float argument of the C ABI carries (e.g. top-p)."""
    return float(np.float32(p))


def dev_bf16(x: np.ndarray) -> torch.Tensor:
    """bfloat16-valued float32 array -> bit-identical CUDA bf16 tensor."""
    bits = synth.bf16_bits(x).view(np.int16)
    return torch.from_numpy(bits).view(torch.bfloat16).cuda()


def host_f32(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy()


def dev_i32(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).cuda()


def dev_f32(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()


def rel_l2(a, b) -> float:
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30))


def check_attention(got, want, what=""):
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    r = rel_l2(got, want)
    m = float(np.max(np.abs(got - want))) if got.size else 0.0
    assert r <= ATTN_REL_L2, f"{what}: rel L2 {r:.3e} > {ATTN_REL_L2}"
    assert m <= ATTN_MAX_ABS, f"{what}: max abs {m:.3e} > {ATTN_MAX_ABS}"
    return r, m


def selection_lists(sel_count: torch.Tensor, sel_cols: torch.Tensor):
    """Device block list -> per head, per q-cluster sorted column lists."""
    cnt = sel_count.cpu().numpy()
    cols = sel_cols.cpu().numpy()
    return [[cols[h, i, :cnt[h, i]].astype(np.int64) for i in range(cnt.shape[1])] for h in range(cnt.shape[0])]


def assignment_gap_tolerance(x: np.ndarray, mu: np.ndarray) -> np.ndarray:
    """Per-token bound below which a float32 tensor-core assign may pick the runner-up.

    The GPU scores ||mu||^2 - 2 x.mu with the centroid split into two bf16
    parts (|residual| <= 2^-17 |mu| per channel) and fp32 accumulation; a flip
    needs the two distances to differ by less than twice the score error.
    Bound used: 2^-12 * ||x|| * max||mu|| + 2^-20 * max||mu||^2 (about 16x the
    worst-case sum of those error terms at D <= 128).
    """
    xn = np.linalg.norm(np.asarray(x, np.float64), axis=1)
    mn = float(np.max(np.linalg.norm(np.asarray(mu, np.float64), axis=1)))
    return 2.0 ** -12 * xn * mn + 2.0 ** -20 * mn * mn
