"""Python binding of libsvg.so (semantic-aware top-p sparse attention, B200).

Argument marshalling only: every step of the path runs in the CUDA kernels
of libsvg.so, reached through its C ABI (include/svg.h) with ctypes.
PyTorch supplies device memory and the current CUDA stream.  There is no
CPU fallback: importing works without a GPU, but every call needs the built
library and a CUDA device and raises otherwise.

Stages (Sparse VideoGen2, section 2): ``kmeans`` -> ``permute`` ->
``select_topp`` -> ``sparse_attn`` -> ``unpermute``; ``svg_attention`` runs
the whole layer.  Options: ``sparse_attn_gather`` (K/V rows fetched through
the K permutation), ``dynrad_select`` (DynamicRad block masks),
``quantize_e4m3`` + ``sparse_attn_fp8`` (Q K^T on 8-bit tensor cores).
"""
from __future__ import annotations

import ctypes
import math
import os
from dataclasses import dataclass
from typing import Optional, Sequence, Tuple

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsvg.so")

STATUS = {0: "SVG_OK", 1: "SVG_ERR_INVALID_ARG", 2: "SVG_ERR_UNSUPPORTED", 3: "SVG_ERR_WORKSPACE",
          4: "SVG_ERR_CUDA", 5: "SVG_ERR_TIMEOUT", 6: "SVG_ERR_DEVICE_CHECK"}

# name -> (restype, argtypes)
_P = ctypes.c_void_p
_I = ctypes.c_int
_F = ctypes.c_float
_SZ = ctypes.c_size_t
SIGNATURES = {
    "svg_status_string": (ctypes.c_char_p, [_I]),
    "svg_version": (ctypes.c_char_p, []),
    "svg_last_cuda_error": (ctypes.c_char_p, []),
    "svg_set_wait_timeout_ns": (None, [ctypes.c_uint64]),
    "svg_debug_set_fault": (None, [_I]),
    "svg_get_error": (_I, [_P]),
    "svg_get_error_detail": (_I, [_P, _P, _P]),
    "svg_kmeans_workspace_size": (_SZ, [_I, _I, _I, _I]),
    "svg_kmeans": (_I, [_P, _I, _I, _I, _I, _I, _P, _P, _P, _P, _SZ, _P]),
    "svg_permute_workspace_size": (_SZ, [_I, _I, _I]),
    "svg_permute": (_I, [_P, _I, _I, _I, _P, _P, _I, _P, _P, _I, _P, _SZ, _P]),
    "svg_select_topp": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _F, _F, _P, _P, _P]),
    "svg_sparse_attn_workspace_size": (_SZ, [_I, _I, _I]),
    "svg_sparse_attn": (_I, [_P, _P, _P, _I, _I, _I, _P, _I, _P, _I, _P, _P, _F, _P, _P, _P, _SZ, _P]),
    "svg_sparse_attn_unpermuted": (_I, [_P, _P, _P, _I, _I, _I, _P, _I, _P, _I, _P, _P, _F, _P, _P, _P, _P,
                                        _SZ, _P]),
    "svg_sparse_attn_gather": (_I, [_P, _P, _P, _P, _I, _I, _I, _P, _I, _P, _I, _P, _P, _F, _P, _P, _P, _P,
                                    _SZ, _P]),
    "svg_unpermute": (_I, [_P, _P, _I, _I, _I, _P, _P]),
    "svg_quantize_e4m3": (_I, [_P, _P, _I, _I, _I, _I, _P, _P, _P]),
    "svg_sparse_attn_fp8": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _P, _I, _P, _I, _P, _P, _F, _P, _P, _P, _P, _SZ,
                                 _P]),
    "svg_dynrad_num_blocks": (_I, [_I, _I, _I]),
    "svg_dynrad_workspace_size": (_SZ, [_I, _I, _I, _I, _I]),
    "svg_dynrad_select": (_I, [_P, _P, _I, _I, _I, _I, _I, _I, _F, _F, _F, _F, _F, _P, _P, _P, _P, _SZ, _P]),
    "svg_sparse_attn_noalloc": (_I, [_P, _P, _P, _I, _I, _I, _P, _I, _P, _I, _P, _P, _F, _P, _P, _P]),
    "svg_profile_enable": (_I, [_I]),
    "svg_profile_read": (_I, [_I, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_int),
                              ctypes.POINTER(ctypes.c_int)]),
    "svg_profile_attn_pairs": (_I, [ctypes.POINTER(ctypes.c_uint64)]),
}

PROFILE_KERNELS = {"kmeans_assign": 0, "sparse_attn": 1}

NOALLOC_SCRATCH_BYTES = 4 << 20   # SVG_NOALLOC_SCRATCH_BYTES in include/svg.h

_lib = None


class SvgError(RuntimeError):
    def __init__(self, fn: str, status: int, detail: str = ""):
        msg = f"{fn} failed: {STATUS.get(status, status)}"
        super().__init__(f"{msg} ({detail})" if detail else msg)
        self.status = status


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Loads libsvg.so (no CUDA device needed) and declares every ABI symbol."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with `python -m sparse_attention_long_svg_b200.build` "
                           "(or __graft_entry__.build()); there is no CPU fallback")
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    _lib = lib
    return lib


def _check(name: str, status: int):
    if status != 0:
        detail = ""
        if status == 4 and _lib is not None:      # SVG_ERR_CUDA: say which call failed
            detail = (_lib.svg_last_cuda_error() or b"").decode(errors="replace")
        raise SvgError(name, status, detail)


def _stream(stream=None) -> ctypes.c_void_p:
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t: Optional[torch.Tensor]) -> ctypes.c_void_p:
    return ctypes.c_void_p(0 if t is None else t.data_ptr())


def _need(t: torch.Tensor, name: str, dtype, dims: int):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if t.dim() != dims:
        raise ValueError(f"{name} must have {dims} dims, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _ws(nbytes: int, device) -> torch.Tensor:
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def get_error(stream=None) -> int:
    """Synchronises the stream and returns (and clears) the device error word."""
    return load_library().svg_get_error(_stream(stream))


ERROR_SITES = {0: "none", 1: "attention producer", 2: "attention MMA issuer", 3: "attention softmax",
               4: "attention drain", 5: "attention planning", 6: "permute range", 7: "k-means MMA issuer",
               8: "k-means epilogue", 9: "k-means range", 10: "k-means drain"}


def get_error_detail(stream=None) -> Tuple[int, str, int]:
    """Like get_error, also naming where the error was recorded: (status, site, CTA index)."""
    site, block = ctypes.c_int32(), ctypes.c_int32()
    st = load_library().svg_get_error_detail(_stream(stream), ctypes.byref(site), ctypes.byref(block))
    return st, ERROR_SITES.get(site.value, str(site.value)), block.value


def set_wait_timeout_ns(ns: int):
    load_library().svg_set_wait_timeout_ns(int(ns))


def profile_enable(on: bool = True):
    """Live timing of the k-means assign and attention kernels (see svg_profile_enable)."""
    _check("svg_profile_enable", load_library().svg_profile_enable(1 if on else 0))


def profile_read(kernel: str) -> Tuple[float, int, int]:
    """(summed ms, timed launches, untimed launches) of a kernel since the last read."""
    ms, n, dropped = ctypes.c_double(), ctypes.c_int(), ctypes.c_int()
    _check("svg_profile_read", load_library().svg_profile_read(PROFILE_KERNELS[kernel], ctypes.byref(ms),
                                                               ctypes.byref(n), ctypes.byref(dropped)))
    return ms.value, n.value, dropped.value


def profile_attn_pairs() -> int:
    """(query tile, key tile) pairs the attention kernel issued MMAs for since the last call."""
    v = ctypes.c_uint64()
    _check("svg_profile_attn_pairs", load_library().svg_profile_attn_pairs(ctypes.byref(v)))
    return int(v.value)


ATTN_TILE = 128   # query rows and keys per (query tile, key tile) pair


# --------------------------------------------------------------------- stages

def kmeans(x: torch.Tensor, centroids: torch.Tensor, iters: int, assign: Optional[torch.Tensor] = None,
           counts: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None, stream=None):
    """k-means of every head of x [BH, N, D] bf16, updating centroids [BH, C, D] fp32 in place.

    Returns (centroids, assign [BH, N] int32, counts [BH, C] int32).
    """
    lib = load_library()
    _need(x, "x", torch.bfloat16, 3)
    _need(centroids, "centroids", torch.float32, 3)
    BH, N, D = x.shape
    C = centroids.shape[1]
    if assign is None:
        assign = torch.empty((BH, N), dtype=torch.int32, device=x.device)
    if counts is None:
        counts = torch.empty((BH, C), dtype=torch.int32, device=x.device)
    nbytes = lib.svg_kmeans_workspace_size(BH, N, D, C)
    if workspace is None:
        workspace = _ws(nbytes, x.device)
    _check("svg_kmeans", lib.svg_kmeans(_ptr(x), BH, N, D, C, int(iters), _ptr(centroids), _ptr(assign),
                                        _ptr(counts), _ptr(workspace), workspace.numel(), _stream(stream)))
    return centroids, assign, counts


def permute(assign: torch.Tensor, C: int, tensors: Sequence[torch.Tensor] = (),
            out: Optional[Sequence[torch.Tensor]] = None, perm: Optional[torch.Tensor] = None,
            offsets: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None, stream=None):
    """Stable counting sort by cluster and row gather of up to 3 [BH, N, D] bf16 tensors.

    Returns (perm [BH, N] int32, offsets [BH, C+1] int32, permuted tensors).
    """
    lib = load_library()
    _need(assign, "assign", torch.int32, 2)
    BH, N = assign.shape
    dev = assign.device
    tensors = list(tensors)
    if out is None:
        out = [torch.empty_like(t) for t in tensors]
    out = list(out)
    D = tensors[0].shape[2] if tensors else 64
    for t in tensors + out:
        _need(t, "tensor", torch.bfloat16, 3)
    if perm is None:
        perm = torch.empty((BH, N), dtype=torch.int32, device=dev)
    if offsets is None:
        offsets = torch.empty((BH, C + 1), dtype=torch.int32, device=dev)
    if workspace is None:
        workspace = _ws(lib.svg_permute_workspace_size(BH, N, C), dev)
    n = len(tensors)
    src = (ctypes.c_void_p * max(n, 1))(*[t.data_ptr() for t in tensors])
    dst = (ctypes.c_void_p * max(n, 1))(*[t.data_ptr() for t in out])
    _check("svg_permute", lib.svg_permute(_ptr(assign), BH, N, int(C), _ptr(perm), _ptr(offsets), n,
                                          ctypes.cast(src, ctypes.c_void_p), ctypes.cast(dst, ctypes.c_void_p),
                                          int(D), _ptr(workspace), workspace.numel(), _stream(stream)))
    return perm, offsets, out


def select_topp(mu_q: torch.Tensor, n_q: torch.Tensor, mu_k: torch.Tensor, n_k: torch.Tensor, p: float,
                scale: float = 0.0, sel_count: Optional[torch.Tensor] = None,
                sel_cols: Optional[torch.Tensor] = None, stream=None):
    """Top-p (q-cluster, k-cluster) block selection.  Returns (sel_count [BH, Cq], sel_cols [BH, Cq, Ck])."""
    lib = load_library()
    _need(mu_q, "mu_q", torch.float32, 3)
    _need(mu_k, "mu_k", torch.float32, 3)
    _need(n_q, "n_q", torch.int32, 2)
    _need(n_k, "n_k", torch.int32, 2)
    BH, Cq, D = mu_q.shape
    Ck = mu_k.shape[1]
    if sel_count is None:
        sel_count = torch.empty((BH, Cq), dtype=torch.int32, device=mu_q.device)
    if sel_cols is None:
        sel_cols = torch.empty((BH, Cq, Ck), dtype=torch.int32, device=mu_q.device)
    _check("svg_select_topp", lib.svg_select_topp(_ptr(mu_q), _ptr(n_q), _ptr(mu_k), _ptr(n_k), BH, Cq, Ck, D,
                                                  float(p), float(scale), _ptr(sel_count), _ptr(sel_cols),
                                                  _stream(stream)))
    return sel_count, sel_cols


def sparse_attn(qp, kp, vp, q_off, k_off, sel_count, sel_cols, scale: float = 0.0, op=None,
                want_lse: bool = False, lse=None, workspace=None, stream=None, perm_q=None):
    """Attention over the selected blocks of permuted Q/K/V.  Returns (op, lse or None).

    With ``perm_q`` (the Q permutation) the un-permutation is fused into the
    kernel's store: ``op`` (and ``lse``) come back in the original token order.
    """
    lib = load_library()
    for t, n in ((qp, "qp"), (kp, "kp"), (vp, "vp")):
        _need(t, n, torch.bfloat16, 3)
    BH, N, D = qp.shape
    Cq = q_off.shape[1] - 1
    Ck = k_off.shape[1] - 1
    if op is None:
        op = torch.empty_like(qp)
    if want_lse and lse is None:
        lse = torch.empty((BH, N), dtype=torch.float32, device=qp.device)
    if workspace is None:
        workspace = _ws(lib.svg_sparse_attn_workspace_size(BH, N, Cq), qp.device)
    if perm_q is not None:
        _need(perm_q, "perm_q", torch.int32, 2)
        _check("svg_sparse_attn_unpermuted", lib.svg_sparse_attn_unpermuted(
            _ptr(qp), _ptr(kp), _ptr(vp), BH, N, D, _ptr(q_off), Cq, _ptr(k_off), Ck, _ptr(sel_count),
            _ptr(sel_cols), float(scale), _ptr(perm_q), _ptr(op), _ptr(lse), _ptr(workspace),
            workspace.numel(), _stream(stream)))
        return op, lse
    _check("svg_sparse_attn", lib.svg_sparse_attn(
        _ptr(qp), _ptr(kp), _ptr(vp), BH, N, D, _ptr(q_off), Cq, _ptr(k_off), Ck, _ptr(sel_count),
        _ptr(sel_cols), float(scale), _ptr(op), _ptr(lse), _ptr(workspace), workspace.numel(), _stream(stream)))
    return op, lse


def sparse_attn_gather(qp, k, v, perm_k, q_off, k_off, sel_count, sel_cols, scale: float = 0.0, op=None,
                       want_lse: bool = False, lse=None, workspace=None, stream=None, perm_q=None):
    """Attention over the selected blocks with K and V in token order: the kernel
    fetches key rows through ``perm_k`` (the K permutation), so no permuted K/V
    copy exists.  Q is permuted.  With ``perm_q`` the output (and lse) come back
    in token order, else in the Q-permuted order.  Returns (op, lse or None).
    """
    lib = load_library()
    for t, n in ((qp, "qp"), (k, "k"), (v, "v")):
        _need(t, n, torch.bfloat16, 3)
    _need(perm_k, "perm_k", torch.int32, 2)
    BH, N, D = qp.shape
    Cq = q_off.shape[1] - 1
    Ck = k_off.shape[1] - 1
    if op is None:
        op = torch.empty_like(qp)
    if want_lse and lse is None:
        lse = torch.empty((BH, N), dtype=torch.float32, device=qp.device)
    if workspace is None:
        workspace = _ws(lib.svg_sparse_attn_workspace_size(BH, N, Cq), qp.device)
    if perm_q is not None:
        _need(perm_q, "perm_q", torch.int32, 2)
    _check("svg_sparse_attn_gather", lib.svg_sparse_attn_gather(
        _ptr(qp), _ptr(k), _ptr(v), _ptr(perm_k), BH, N, D, _ptr(q_off), Cq, _ptr(k_off), Ck, _ptr(sel_count),
        _ptr(sel_cols), float(scale), _ptr(perm_q), _ptr(op), _ptr(lse), _ptr(workspace), workspace.numel(),
        _stream(stream)))
    return op, lse


def quantize_e4m3(x, per_row: bool, x8=None, scales=None, stream=None, perm=None):
    """E4M3 copy of x [BH, N, D] bf16 and its float32 scales (svg_quantize_e4m3):
    per_row -> scales [BH, N] (one per row, for Q), else [BH] (one per head, for K).
    With ``perm`` [BH, N] int32 the rows are gathered on the way: row i of head h
    is quantised from row perm[h, i].  Returns (x8 as torch.float8_e4m3fn, scales)."""
    lib = load_library()
    _need(x, "x", torch.bfloat16, 3)
    if perm is not None:
        _need(perm, "perm", torch.int32, 2)
    BH, N, D = x.shape
    if x8 is None:
        x8 = torch.empty((BH, N, D), dtype=torch.float8_e4m3fn, device=x.device)
    if scales is None:
        scales = torch.empty((BH, N) if per_row else (BH,), dtype=torch.float32, device=x.device)
    _check("svg_quantize_e4m3", lib.svg_quantize_e4m3(_ptr(x), _ptr(perm), BH, N, D, 1 if per_row else 0,
                                                      _ptr(x8), _ptr(scales), _stream(stream)))
    return x8, scales


def sparse_attn_fp8(q8, q_scale, k8, k_scale, vp, q_off, k_off, sel_count, sel_cols, scale: float = 0.0, op=None,
                    want_lse: bool = False, lse=None, workspace=None, stream=None, perm_q=None):
    """Attention over the selected blocks with E4M3 Q and K (quantize_e4m3 of the
    permuted qp, per row, and kp, per head) and bf16 V.  With ``perm_q`` the output
    (and lse) come back in token order.  Returns (op, lse or None)."""
    lib = load_library()
    _need(q8, "q8", torch.float8_e4m3fn, 3)
    _need(k8, "k8", torch.float8_e4m3fn, 3)
    _need(vp, "vp", torch.bfloat16, 3)
    BH, N, D = q8.shape
    if q_scale.dtype != torch.float32 or q_scale.numel() != BH * N or not q_scale.is_contiguous():
        raise ValueError("q_scale must be a contiguous float32 tensor of BH * N values")
    if k_scale.dtype != torch.float32 or k_scale.numel() != BH or not k_scale.is_contiguous():
        raise ValueError("k_scale must be a contiguous float32 tensor of BH values")
    Cq = q_off.shape[1] - 1
    Ck = k_off.shape[1] - 1
    if op is None:
        op = torch.empty((BH, N, D), dtype=torch.bfloat16, device=q8.device)
    if want_lse and lse is None:
        lse = torch.empty((BH, N), dtype=torch.float32, device=q8.device)
    if workspace is None:
        workspace = _ws(lib.svg_sparse_attn_workspace_size(BH, N, Cq), q8.device)
    if perm_q is not None:
        _need(perm_q, "perm_q", torch.int32, 2)
    _check("svg_sparse_attn_fp8", lib.svg_sparse_attn_fp8(
        _ptr(q8), _ptr(q_scale), _ptr(k8), _ptr(k_scale), _ptr(vp), BH, N, D, _ptr(q_off), Cq, _ptr(k_off), Ck,
        _ptr(sel_count), _ptr(sel_cols), float(scale), _ptr(perm_q), _ptr(op), _ptr(lse), _ptr(workspace),
        workspace.numel(), _stream(stream)))
    return op, lse


DYNRAD_MODES = {"candidates": 0, "static": 1, "dynamic": 2}


def dynrad_select(q, k, frames: int, block: int, mode: str, w0: float, gamma: float, rho0: float = 1.0,
                  theta: float = 0.0, scale: float = 0.0, offsets=None, sel_count=None, sel_cols=None,
                  workspace=None, stream=None):
    """DynamicRad block masks (svg_dynrad_select) for q, k [BH, N, D] bf16 in token order.

    Returns (offsets [BH, Cb+1], sel_count [BH, Cb], sel_cols [BH, Cb, Cb]): the
    block list svg_sparse_attn consumes with q_off = k_off = offsets.
    """
    lib = load_library()
    _need(q, "q", torch.bfloat16, 3)
    _need(k, "k", torch.bfloat16, 3)
    BH, N, D = q.shape
    Cb = lib.svg_dynrad_num_blocks(N, frames, block)
    if Cb <= 0:
        raise ValueError(f"frames {frames} must divide N {N} and block must be positive")
    i32 = dict(dtype=torch.int32, device=q.device)
    if offsets is None:
        offsets = torch.empty((BH, Cb + 1), **i32)
    if sel_count is None:
        sel_count = torch.empty((BH, Cb), **i32)
    if sel_cols is None:
        sel_cols = torch.empty((BH, Cb, Cb), **i32)
    if workspace is None:
        workspace = _ws(lib.svg_dynrad_workspace_size(BH, N, D, frames, block), q.device)
    _check("svg_dynrad_select", lib.svg_dynrad_select(
        _ptr(q), _ptr(k), BH, N, D, int(frames), int(block), DYNRAD_MODES[mode], float(w0), float(gamma),
        float(rho0), float(theta), float(scale), _ptr(offsets), _ptr(sel_count), _ptr(sel_cols), _ptr(workspace),
        workspace.numel(), _stream(stream)))
    return offsets, sel_count, sel_cols


def dynrad_attention(q, k, v, frames: int, block: int, mode: str, w0: float, gamma: float, rho0: float = 1.0,
                     theta: float = 0.0, scale: float = 0.0, out=None, want_lse: bool = False, stream=None):
    """One attention layer with DynamicRad block masks (token order in and out, no permutation).

    Returns (out, lse or None, (offsets, sel_count, sel_cols))."""
    blocks = dynrad_select(q, k, frames, block, mode, w0, gamma, rho0, theta, scale, stream=stream)
    offsets, sel_count, sel_cols = blocks
    out, lse = sparse_attn(q, k, v, offsets, offsets, sel_count, sel_cols, scale, out, want_lse=want_lse,
                           stream=stream)
    return out, lse, blocks


def sparse_attn_noalloc(qp, kp, vp, q_off, k_off, sel_count, sel_cols, scale: float = 0.0, op=None,
                       want_lse: bool = False, lse=None, stream=None):
    """sparse_attn for callers that cannot provide device scratch memory.

    Same inputs and result as ``sparse_attn``; the library uses a fixed scratch
    array of its own instead of a workspace (see svg_sparse_attn_noalloc in
    include/svg.h: size limit, one shared array, calls must not overlap).
    """
    lib = load_library()
    for t, n in ((qp, "qp"), (kp, "kp"), (vp, "vp")):
        _need(t, n, torch.bfloat16, 3)
    BH, N, D = qp.shape
    Cq = q_off.shape[1] - 1
    Ck = k_off.shape[1] - 1
    if op is None:
        op = torch.empty_like(qp)
    if want_lse and lse is None:
        lse = torch.empty((BH, N), dtype=torch.float32, device=qp.device)
    _check("svg_sparse_attn_noalloc", lib.svg_sparse_attn_noalloc(
        _ptr(qp), _ptr(kp), _ptr(vp), BH, N, D, _ptr(q_off), Cq, _ptr(k_off), Ck, _ptr(sel_count),
        _ptr(sel_cols), float(scale), _ptr(op), _ptr(lse), _stream(stream)))
    return op, lse


def unpermute(xp: torch.Tensor, perm: torch.Tensor, out: Optional[torch.Tensor] = None, stream=None):
    """x[h, perm[h, r]] = xp[h, r]."""
    lib = load_library()
    _need(xp, "xp", torch.bfloat16, 3)
    BH, N, D = xp.shape
    if out is None:
        out = torch.empty_like(xp)
    _check("svg_unpermute", lib.svg_unpermute(_ptr(xp), _ptr(perm), BH, N, D, _ptr(out), _stream(stream)))
    return out


# --------------------------------------------------------------------- the layer

@dataclass
class LayerState:
    """Everything one layer call produces; centroids are the next call's warm start."""
    mu_q: torch.Tensor
    mu_k: torch.Tensor
    assign_q: torch.Tensor
    assign_k: torch.Tensor
    n_q: torch.Tensor
    n_k: torch.Tensor
    perm_q: torch.Tensor
    perm_k: torch.Tensor
    q_off: torch.Tensor
    k_off: torch.Tensor
    sel_count: torch.Tensor
    sel_cols: torch.Tensor
    qp: Optional[torch.Tensor]     # permuted Q; None with qk_fp8 (Q quantised while gathered)
    kp: Optional[torch.Tensor]     # permuted K; None with kv_gather (rows fetched through perm_k) or qk_fp8
    vp: Optional[torch.Tensor]     # permuted V; None with kv_gather
    op: Optional[torch.Tensor]     # permuted output; None when the un-permutation was fused


class SvgLayer:
    """Preallocated buffers for repeated layer calls of one shape (no allocation per call)."""

    def __init__(self, BH: int, N: int, D: int, Cq: int, Ck: int, device="cuda"):
        lib = load_library()
        self.shape = (BH, N, D, Cq, Ck)
        i32 = dict(dtype=torch.int32, device=device)
        bf = dict(dtype=torch.bfloat16, device=device)
        self.assign_q = torch.empty((BH, N), **i32)
        self.assign_k = torch.empty((BH, N), **i32)
        self.n_q = torch.empty((BH, Cq), **i32)
        self.n_k = torch.empty((BH, Ck), **i32)
        self.perm_q = torch.empty((BH, N), **i32)
        self.perm_k = torch.empty((BH, N), **i32)
        self.q_off = torch.empty((BH, Cq + 1), **i32)
        self.k_off = torch.empty((BH, Ck + 1), **i32)
        self.sel_count = torch.empty((BH, Cq), **i32)
        self.sel_cols = torch.empty((BH, Cq, Ck), **i32)
        self.qp = torch.empty((BH, N, D), **bf)
        self.kp = torch.empty((BH, N, D), **bf)
        self.vp = torch.empty((BH, N, D), **bf)
        self.op = torch.empty((BH, N, D), **bf)
        ws = max(lib.svg_kmeans_workspace_size(BH, N, D, Cq), lib.svg_kmeans_workspace_size(BH, N, D, Ck),
                 lib.svg_permute_workspace_size(BH, N, max(Cq, Ck)),
                 lib.svg_sparse_attn_workspace_size(BH, N, Cq))
        self.workspace = _ws(ws, device)
        self.fp8 = None     # (q8, q_scale, k8, k_scale), made by the first call with qk_fp8

    def __call__(self, q, k, v, mu_q, mu_k, iters: int, p: float, scale: float = 0.0, out=None, stream=None,
                 fused_unpermute: bool = True, kv_gather: bool = False, qk_fp8: bool = False):
        """One layer; with ``fused_unpermute`` the attention kernel stores rows in token order
        (no permuted output copy, ``LayerState.op`` is None), else attention + svg_unpermute.
        With ``kv_gather`` K and V are not permuted: the attention kernel fetches their rows
        through the K permutation (``LayerState.kp``/``vp`` are None); requires fused_unpermute.
        With ``qk_fp8`` Q and K are quantised to E4M3 (per-row / per-head scales) while they are
        gathered into permuted order (no bf16 permuted copies: ``LayerState.qp``/``kp`` are None)
        and S = Q K^T runs on 8-bit operands; D must be 128."""
        if qk_fp8 and kv_gather:
            raise ValueError("qk_fp8 and kv_gather cannot be combined")
        kmeans(q, mu_q, iters, self.assign_q, self.n_q, self.workspace, stream)
        kmeans(k, mu_k, iters, self.assign_k, self.n_k, self.workspace, stream)
        Cq, Ck = mu_q.shape[1], mu_k.shape[1]
        if qk_fp8:     # Q and K are gathered by the quantisation below; only V is moved here
            permute(self.assign_q, Cq, [], [], self.perm_q, self.q_off, self.workspace, stream)
            permute(self.assign_k, Ck, [v], [self.vp], self.perm_k, self.k_off, self.workspace, stream)
        else:
            permute(self.assign_q, Cq, [q], [self.qp], self.perm_q, self.q_off, self.workspace, stream)
            if kv_gather:
                if not fused_unpermute:
                    raise ValueError("kv_gather requires fused_unpermute")
                permute(self.assign_k, Ck, [], [], self.perm_k, self.k_off, self.workspace, stream)
            else:
                permute(self.assign_k, Ck, [k, v], [self.kp, self.vp], self.perm_k, self.k_off, self.workspace,
                        stream)
        select_topp(mu_q, self.n_q, mu_k, self.n_k, p, scale, self.sel_count, self.sel_cols, stream)
        if kv_gather:
            if out is None:
                out = torch.empty_like(q)
            sparse_attn_gather(self.qp, k, v, self.perm_k, self.q_off, self.k_off, self.sel_count,
                               self.sel_cols, scale, out, workspace=self.workspace, stream=stream,
                               perm_q=self.perm_q)
            return out, LayerState(mu_q, mu_k, self.assign_q, self.assign_k, self.n_q, self.n_k, self.perm_q,
                                   self.perm_k, self.q_off, self.k_off, self.sel_count, self.sel_cols, self.qp,
                                   None, None, None)
        if qk_fp8:
            if self.fp8 is None:
                BH, N, D = self.qp.shape
                f8 = dict(dtype=torch.float8_e4m3fn, device=self.qp.device)
                f32 = dict(dtype=torch.float32, device=self.qp.device)
                self.fp8 = (torch.empty((BH, N, D), **f8), torch.empty((BH, N), **f32),
                            torch.empty((BH, N, D), **f8), torch.empty((BH,), **f32))
            q8, sq, k8, sk = self.fp8
            quantize_e4m3(q, True, q8, sq, stream, perm=self.perm_q)
            quantize_e4m3(k, False, k8, sk, stream, perm=self.perm_k)
            if fused_unpermute:
                if out is None:
                    out = torch.empty_like(q)
                sparse_attn_fp8(q8, sq, k8, sk, self.vp, self.q_off, self.k_off, self.sel_count, self.sel_cols,
                                scale, out, workspace=self.workspace, stream=stream, perm_q=self.perm_q)
                op = None
            else:
                sparse_attn_fp8(q8, sq, k8, sk, self.vp, self.q_off, self.k_off, self.sel_count, self.sel_cols,
                                scale, self.op, workspace=self.workspace, stream=stream)
                out = unpermute(self.op, self.perm_q, out, stream)
                op = self.op
            return out, LayerState(mu_q, mu_k, self.assign_q, self.assign_k, self.n_q, self.n_k, self.perm_q,
                                   self.perm_k, self.q_off, self.k_off, self.sel_count, self.sel_cols, None, None,
                                   self.vp, op)
        if fused_unpermute:
            if out is None:
                out = torch.empty_like(q)
            sparse_attn(self.qp, self.kp, self.vp, self.q_off, self.k_off, self.sel_count, self.sel_cols, scale,
                        out, workspace=self.workspace, stream=stream, perm_q=self.perm_q)
            op = None
        else:
            sparse_attn(self.qp, self.kp, self.vp, self.q_off, self.k_off, self.sel_count, self.sel_cols, scale,
                        self.op, workspace=self.workspace, stream=stream)
            out = unpermute(self.op, self.perm_q, out, stream)
            op = self.op
        return out, LayerState(mu_q, mu_k, self.assign_q, self.assign_k, self.n_q, self.n_k, self.perm_q,
                               self.perm_k, self.q_off, self.k_off, self.sel_count, self.sel_cols, self.qp,
                               self.kp, self.vp, op)


class LayerGraph:
    """One SvgLayer call recorded as a CUDA graph: replay() re-runs the whole layer
    (k-means from the given initial centroids, permute, select, attention) on the
    same device buffers with one launch from the host.

    The captured call reads q, k, v and the initial centroids mu_q0 / mu_k0 from
    the tensors given at capture time (refill them in place between replays) and
    writes ``out``; mu_q / mu_k receive the final centroids.  The layer's own
    kernels do no allocation and no host synchronisation, which is what makes
    the capture valid.
    """

    def __init__(self, layer: "SvgLayer", q, k, v, mu_q0, mu_k0, iters: int, p: float, scale: float = 0.0,
                 kv_gather: bool = False, qk_fp8: bool = False):
        self.mu_q = torch.empty_like(mu_q0)
        self.mu_k = torch.empty_like(mu_k0)
        self.out = torch.empty_like(q)
        args = (layer, q, k, v, mu_q0, mu_k0, iters, p, scale, kv_gather, qk_fp8)
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):        # one eager call: warms every kernel before capture
            self._call(*args)
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph):
            self._call(*args)

    def _call(self, layer, q, k, v, mu_q0, mu_k0, iters, p, scale, kv_gather, qk_fp8):
        self.mu_q.copy_(mu_q0)
        self.mu_k.copy_(mu_k0)
        layer(q, k, v, self.mu_q, self.mu_k, iters, p, scale, self.out, kv_gather=kv_gather, qk_fp8=qk_fp8)

    def replay(self):
        self.graph.replay()
        return self.out


def svg_attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, mu_q: torch.Tensor, mu_k: torch.Tensor,
                  iters: int, p: float, scale: float = 0.0):
    """One SVG2 attention layer: returns (out [BH, N, D] bf16, LayerState).

    mu_q / mu_k [BH, C, D] fp32 hold the initial centroids (seeding tokens or
    the previous step's cache) and are updated in place.
    """
    BH, N, D = q.shape
    layer = SvgLayer(BH, N, D, mu_q.shape[1], mu_k.shape[1], q.device)
    return layer(q, k, v, mu_q, mu_k, iters, p, scale)


def default_scale(D: int) -> float:
    return 1.0 / math.sqrt(D)
