"""C-ABI checks that need no GPU: the library loads, exports every function
include/svg.h declares, and rejects bad arguments on the host before any
launch (these calls return before touching the CUDA runtime)."""
import ctypes
import os
import re

import pytest

import sparse_attention_long_svg_b200 as svg
from sparse_attention_long_svg_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return svg.load_library()


def declared_functions():
    text = open(os.path.join(ROOT, "include", "svg.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(svg_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_the_five_stages():
    names = declared_functions()
    for stage in ("svg_kmeans", "svg_permute", "svg_select_topp", "svg_sparse_attn", "svg_unpermute"):
        assert stage in names


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert names
    for n in names:
        assert hasattr(lib, n), n
        assert n in svg.SIGNATURES, f"binding lacks {n}"


def test_status_strings(lib):
    for code, name in svg.STATUS.items():
        assert lib.svg_status_string(code).decode() == name
    assert lib.svg_version().decode().startswith("svg-b200")
    assert lib.svg_last_cuda_error().decode() == ""      # no CUDA call has failed in this process


def test_workspace_sizes_are_positive_and_monotone(lib):
    a = lib.svg_kmeans_workspace_size(40, 32760, 128, 500)
    b = lib.svg_kmeans_workspace_size(40, 75600, 128, 1000)
    assert 0 < a < b
    assert lib.svg_permute_workspace_size(1, 2048, 64) > 0
    assert lib.svg_sparse_attn_workspace_size(40, 32760, 100) > 0
    assert lib.svg_kmeans_workspace_size(0, 10, 64, 4) == 0


def _p(v):
    return ctypes.c_void_p(v)


FAKE = 0x10000  # 256-byte aligned, never dereferenced: every call below fails its host checks


def test_dynrad_block_counts(lib):
    assert lib.svg_dynrad_num_blocks(30, 3, 4) == 9          # frames of 10 tokens: blocks of 4, 4, 2
    assert lib.svg_dynrad_num_blocks(32760, 21, 256) == 147  # 480p: 1,560 tokens per frame, 7 blocks
    assert lib.svg_dynrad_num_blocks(31, 3, 4) == 0
    assert lib.svg_dynrad_num_blocks(30, 3, 0) == 0
    assert lib.svg_dynrad_workspace_size(40, 32760, 128, 21, 256) == 2 * 40 * 147 * 128 * 8


def test_invalid_arguments_are_rejected_before_launch(lib):
    nul = _p(0)
    f = _p(FAKE)
    # k-means: null pointer, C > N, iters < 1, unsupported D, too many clusters, small workspace
    assert lib.svg_kmeans(nul, 1, 16, 64, 4, 1, f, f, f, f, 1 << 20, nul) == 1
    assert lib.svg_kmeans(f, 1, 16, 64, 17, 1, f, f, f, f, 1 << 20, nul) == 1
    assert lib.svg_kmeans(f, 1, 16, 64, 4, 0, f, f, f, f, 1 << 20, nul) == 1
    assert lib.svg_kmeans(f, 1, 16, 96, 4, 1, f, f, f, f, 1 << 20, nul) == 2
    assert lib.svg_kmeans(f, 1, 4096, 64, 2000, 1, f, f, f, f, 1 << 30, nul) == 2
    assert lib.svg_kmeans(f, 1, 4096, 64, 64, 1, f, f, f, f, 16, nul) == 3
    # misaligned bf16 pointer
    assert lib.svg_kmeans(_p(FAKE + 2), 1, 16, 64, 4, 1, f, f, f, f, 1 << 20, nul) == 1
    # permute: more than 3 tensors, aliasing src == dst
    assert lib.svg_permute(f, 1, 16, 4, f, f, 4, f, f, 64, f, 1 << 20, nul) == 1
    ptrs = (ctypes.c_void_p * 1)(FAKE)
    arr = ctypes.cast(ptrs, ctypes.c_void_p)
    assert lib.svg_permute(f, 1, 16, 4, f, f, 1, arr, arr, 64, f, 1 << 20, nul) == 1
    # select: p <= 0, NaN p, Ck too large
    assert lib.svg_select_topp(f, f, f, f, 1, 4, 8, 64, 0.0, 0.0, f, f, nul) == 1
    assert lib.svg_select_topp(f, f, f, f, 1, 4, 8, 64, float("nan"), 0.0, f, f, nul) == 1
    assert lib.svg_select_topp(f, f, f, f, 1, 4, 2048, 64, 0.9, 0.0, f, f, nul) == 2
    # attention: unsupported D, more than 1024 k-clusters, workspace too small
    assert lib.svg_sparse_attn(f, f, f, 1, 16, 80, f, 2, f, 2, f, f, 0.0, f, nul, f, 1 << 20, nul) == 2
    assert lib.svg_sparse_attn(f, f, f, 1, 4096, 64, f, 2, f, 1025, f, f, 0.0, f, nul, f, 1 << 20, nul) == 2
    assert lib.svg_sparse_attn(f, f, f, 1, 4096, 64, f, 2, f, 2, f, f, 0.0, f, nul, f, 8, nul) == 3
    # fused attention + un-permute: missing perm_q, output aliasing an input, small workspace
    g = _p(FAKE + 4096)
    assert lib.svg_sparse_attn_unpermuted(f, f, f, 1, 16, 64, f, 2, f, 2, f, f, 0.0, nul, g, nul, f,
                                          1 << 20, nul) == 1
    assert lib.svg_sparse_attn_unpermuted(f, g, g, 1, 16, 64, f, 2, f, 2, f, f, 0.0, g, f, nul, g,
                                          1 << 20, nul) == 1
    assert lib.svg_sparse_attn_unpermuted(f, f, f, 1, 4096, 64, f, 2, f, 2, f, f, 0.0, f, g, nul, f,
                                          8, nul) == 3
    # unpermute: aliasing
    assert lib.svg_unpermute(f, f, 1, 16, 64, f, nul) == 1
    # gathered-K/V attention: missing perm_k, output aliasing K
    assert lib.svg_sparse_attn_gather(f, f, f, nul, 1, 16, 64, f, 2, f, 2, f, f, 0.0, nul, g, nul, f,
                                      1 << 20, nul) == 1
    assert lib.svg_sparse_attn_gather(f, g, f, f, 1, 16, 64, f, 2, f, 2, f, f, 0.0, nul, g, nul, f,
                                      1 << 20, nul) == 1
    # DynamicRad masks: frames not dividing N, more than 1024 blocks, bad mode, negative window,
    # static ratio <= 0, dynamic mode without q/k, unsupported D, small workspace
    dyn = lambda q, N, D, fr, blk, mode, w0=2.0, gamma=0.5, rho0=0.5, ws=1 << 20: lib.svg_dynrad_select(
        q, q, 1, N, D, fr, blk, mode, w0, gamma, rho0, 0.0, 0.0, f, f, f, f, ws, nul)
    assert dyn(f, 30, 64, 4, 4, 1) == 1
    assert dyn(f, 2048, 64, 1, 1, 1) == 2
    assert dyn(f, 30, 64, 3, 4, 3) == 1
    assert dyn(f, 30, 64, 3, 4, 1, w0=-1.0) == 1
    assert dyn(f, 30, 64, 3, 4, 1, rho0=0.0) == 1
    assert dyn(nul, 30, 64, 3, 4, 2) == 1
    assert dyn(f, 30, 96, 3, 4, 2) == 2
    assert dyn(f, 30, 64, 3, 4, 2, ws=8) == 3
    # E4M3 quantisation: unsupported D, per_row not 0/1, x8 aliasing x, null scales, misaligned x
    assert lib.svg_quantize_e4m3(f, nul, 1, 16, 96, 1, g, f, nul) == 2
    assert lib.svg_quantize_e4m3(f, nul, 1, 16, 64, 2, g, f, nul) == 1
    assert lib.svg_quantize_e4m3(f, nul, 1, 16, 64, 1, f, g, nul) == 1
    assert lib.svg_quantize_e4m3(f, nul, 1, 16, 64, 0, g, nul, nul) == 1
    assert lib.svg_quantize_e4m3(_p(FAKE + 2), nul, 1, 16, 64, 0, g, f, nul) == 1
    # 8-bit Q K^T attention: missing scales, D other than 128, small workspace
    fp8 = lambda qs, ks, N, D, ws: lib.svg_sparse_attn_fp8(f, qs, f, ks, f, 1, N, D, f, 2, f, 2, f, f, 0.0, nul,
                                                           g, nul, f, ws, nul)
    assert fp8(nul, f, 16, 128, 1 << 20) == 1
    assert fp8(f, nul, 16, 128, 1 << 20) == 1
    assert fp8(f, f, 16, 64, 1 << 20) == 2
    assert fp8(f, f, 4096, 128, 8) == 3
    # nothing above reached CUDA
    assert lib.svg_last_cuda_error().decode() == ""
