"""The attention entry point for callers that cannot allocate device memory.

svg_sparse_attn_noalloc exists for callers with no way to hand the library a
scratch buffer (a plug-in inside a framework that owns every allocation, a
serving loop with a memory budget fixed at start-up, a runtime that forbids
device allocation after initialisation).  It uses a scratch array compiled
into the library instead of a caller workspace.  These tests call it through
the C ABI and compare it with svg_sparse_attn on the same inputs, on two calls
in a row with different shapes (the shared array keeps the first call's
contents when the second one runs).

This file is named so that pytest collects it last.
"""
import pytest
import torch

import synth
from tests.helpers import dev_bf16, dev_f32

pytestmark = pytest.mark.gpu

svg = pytest.importorskip("sparse_attention_long_svg_b200")


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from sparse_attention_long_svg_b200 import build
    build.build()
    svg.load_library()


def layer_inputs(wl):
    """Clustered, permuted and selected inputs produced by the library's own stages."""
    L = synth.make_layer(wl)
    layer = svg.SvgLayer(*L.q.shape, wl.cq, wl.ck)
    q, k, v = dev_bf16(L.q), dev_bf16(L.k), dev_bf16(L.v)
    _, st = layer(q, k, v, dev_f32(L.init_centroids("q")), dev_f32(L.init_centroids("k")), wl.iters, wl.top_p[0])
    return st


def test_noalloc_matches_workspace_entry_point_on_two_calls():
    cases = [synth.small_workload("480p-5s", (5, 12, 20), heads=3, cq=6, ck=40, iters=3),
             synth.small_workload("dense-d64", (3, 10, 41), heads=2, cq=8, ck=30, iters=2)]
    for wl in cases:
        st = layer_inputs(wl)
        args = (st.qp, st.kp, st.vp, st.q_off, st.k_off, st.sel_count, st.sel_cols)
        ref, ref_lse = svg.sparse_attn(*args, want_lse=True)
        got, got_lse = svg.sparse_attn_noalloc(*args, want_lse=True)
        torch.cuda.synchronize()
        assert svg.get_error() == 0
        # the same kernel on the same inputs: every row is computed by one CTA
        # over a fixed sequence of key tiles, so the results are bit-identical
        assert torch.equal(got, ref), f"no-alloc vs workspace ({wl.name})"
        assert torch.equal(got_lse, ref_lse), f"no-alloc vs workspace lse ({wl.name})"


def test_noalloc_rejects_sizes_beyond_its_scratch():
    lib = svg.load_library()
    big_bh, big_n, big_cq = 200, 200000, 1000
    assert lib.svg_sparse_attn_workspace_size(big_bh, big_n, big_cq) > svg.NOALLOC_SCRATCH_BYTES
    f = svg.ctypes.c_void_p(0x10000)
    status = lib.svg_sparse_attn_noalloc(f, f, f, big_bh, big_n, 128, f, big_cq, f, 64, f, f, 0.0, f,
                                         svg.ctypes.c_void_p(0), svg.ctypes.c_void_p(0))
    assert status == 3   # SVG_ERR_WORKSPACE, returned before any launch
