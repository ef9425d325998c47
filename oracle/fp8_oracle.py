"""CPU oracle for attention with 8-bit floating-point Q and K (test infrastructure).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this module.  The CUDA library
never calls it, and it shares no code with the CUDA library.

The page "TurboDiffusion" (section "SageAttention: low-bit quantization")
says attention is computed at reduced precision, through low-bit
quantisation, to cut memory traffic and compute while keeping accuracy; it
gives no format, no scales and no formulas.  Readings taken:
  * Q and K are quantised to FP8 E4M3 (1 sign, 4 exponent bits with bias 7,
    3 mantissa bits; largest finite value 448, smallest subnormal 2^-9, no
    infinities), rounding to nearest with ties to the even mantissa and
    saturating to +-448 (the tensor cores' E4M3 input format);
  * Q has one scale per token row, s_q = amax|q_row| / 448, and K one scale
    per head, s_k = amax|k| / 448 (one value for every key row, so a key tile
    gathered from any rows shares it); both are float32, a zero amax gives
    scale 1; the quantised value is E4M3(x / s) with the division in float32;
  * the logits are scale * (q8 . k8) * s_q * s_k; P and V stay bf16/exact as
    in the bf16 path (only Q K^T is 8-bit).

Arithmetic after quantisation is float64 (the products of E4M3 values are
exact there).
"""
from __future__ import annotations

from typing import Sequence, Tuple

import numpy as np

from oracle import svg_oracle as so

E4M3_MAX = 448.0
E4M3_MIN_NORMAL = 2.0 ** -6
E4M3_SUBNORMAL_QUANTUM = 2.0 ** -9


def e4m3(x) -> np.ndarray:
    """Round to the nearest E4M3 value (ties to even mantissa), saturating at +-448."""
    x = np.asarray(x, np.float64)
    out = np.zeros_like(x)
    a = np.abs(x)
    normal = a >= E4M3_MIN_NORMAL
    # quantum of the binade of a: 2^(e - 3) for a in [2^e, 2^(e+1))
    _, e = np.frexp(np.where(normal, a, 1.0))          # a = m 2^e with m in [0.5, 1)
    quantum = np.where(normal, np.ldexp(1.0, e - 4), E4M3_SUBNORMAL_QUANTUM)
    q = np.round(a / quantum) * quantum                 # numpy rounds halves to even
    q = np.minimum(q, E4M3_MAX)
    out = np.copysign(q, x)
    return out


def all_e4m3_values() -> np.ndarray:
    """Every finite E4M3 value, from its bit fields (the NaN patterns excluded)."""
    vals = []
    for bits in range(256):
        s, ex, m = bits >> 7, (bits >> 3) & 15, bits & 7
        if ex == 15 and m == 7:
            continue                                     # NaN
        v = (m / 8.0) * 2.0 ** -6 if ex == 0 else (1.0 + m / 8.0) * 2.0 ** (ex - 7)
        vals.append(-v if s else v)
    return np.asarray(vals)


def _scale(amax: np.ndarray) -> np.ndarray:
    amax = np.asarray(amax, np.float32)
    s = amax / np.float32(E4M3_MAX)                     # float32 division
    return np.where(amax > 0, s, np.float32(1.0)).astype(np.float32)


def quantize_rows(x: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """Per-row scales and E4M3 values: (q8 [R, D] as float64 values, s [R] float32)."""
    x32 = np.asarray(x, np.float32)
    s = _scale(np.abs(x32).max(axis=1))
    q8 = e4m3((x32 / s[:, None]).astype(np.float32))
    return q8, s


def quantize_tensor(x: np.ndarray) -> Tuple[np.ndarray, np.float32]:
    """One scale for the whole tensor (a head's keys): (k8 as float64 values, s float32)."""
    x32 = np.asarray(x, np.float32)
    s = _scale(np.abs(x32).max())
    return e4m3((x32 / s).astype(np.float32)), np.float32(s)


def sparse_attention_fp8(qp: np.ndarray, kp: np.ndarray, vp: np.ndarray, q_off: np.ndarray,
                         k_off: np.ndarray, selection: Sequence[Sequence[int]], scale: float,
                         rows=None):
    """Block-sparse attention of one head with E4M3 Q and K (see the module readings).

    Equal to the bf16-path oracle run on the dequantised Q and K: the per-row
    Q scale and the head's K scale multiply the logits."""
    q8, sq = quantize_rows(qp)
    k8, sk = quantize_tensor(kp)
    qd = q8 * sq.astype(np.float64)[:, None]
    kd = k8 * float(sk)
    return so.sparse_attention(qd, kd, vp, q_off, k_off, selection, scale, rows=rows)
