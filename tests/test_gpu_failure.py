"""Failure detection without a GPU fault.

A host-set flag (svg_debug_set_fault) makes the attention kernel skip its
query-tile loads, so the barrier they would complete never completes (a
flag that nothing sets).  With a short wait limit every role's bounded wait
runs out; the kernel must record SVG_ERR_TIMEOUT in the device error word,
drain its own copies, free its tensor memory and return, leaving the
context usable: the next normal launch must reproduce the reference output.
"""
import numpy as np
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


ATTN_SITES = {"attention producer", "attention MMA issuer", "attention softmax", "attention drain"}


@pytest.mark.parametrize("gather", [False, True], ids=["permuted-kv", "gathered-kv"])
def test_timeout_is_reported_and_context_stays_usable(gather):
    lib = svg.load_library()
    wl = synth.small_workload("480p-5s", (5, 12, 20), heads=3, cq=6, ck=40, iters=3)
    L = synth.make_layer(wl)
    layer = svg.SvgLayer(*L.q.shape, wl.cq, wl.ck)
    k, v = dev_bf16(L.k), dev_bf16(L.v)
    _, st = layer(dev_bf16(L.q), k, v, dev_f32(L.init_centroids("q")), dev_f32(L.init_centroids("k")),
                  wl.iters, 0.9)
    blocks = (st.q_off, st.k_off, st.sel_count, st.sel_cols)

    def attend():
        if gather:
            return svg.sparse_attn_gather(st.qp, k, v, st.perm_k, *blocks)
        return svg.sparse_attn(st.qp, st.kp, st.vp, *blocks)
    ref, _ = attend()
    ref = ref.clone()
    assert svg.get_error() == 0
    try:
        svg.set_wait_timeout_ns(20_000_000)          # 20 ms
        lib.svg_debug_set_fault(1)
        attend()                                     # the launch itself succeeds
        status, site, cta = svg.get_error_detail()
    finally:
        lib.svg_debug_set_fault(0)
        svg.set_wait_timeout_ns(0)                   # default bound
    assert status == 5, svg.STATUS.get(status, status)   # SVG_ERR_TIMEOUT
    assert site in ATTN_SITES, site
    assert 0 <= cta < 160
    assert svg.get_error() == 0                      # the word was cleared
    again, _ = attend()
    torch.cuda.synchronize()
    assert svg.get_error() == 0
    assert torch.equal(again, ref)


def test_device_check_reports_bad_block_list():
    """A cluster id out of range in the block list is flagged, not dereferenced."""
    wl = synth.small_workload("480p-5s", (5, 12, 20), heads=1, cq=6, ck=40, iters=2)
    L = synth.make_layer(wl)
    layer = svg.SvgLayer(*L.q.shape, wl.cq, wl.ck)
    _, st = layer(dev_bf16(L.q), dev_bf16(L.k), dev_bf16(L.v), dev_f32(L.init_centroids("q")),
                  dev_f32(L.init_centroids("k")), wl.iters, 0.9)
    cols = st.sel_cols.clone()
    i = int(np.nonzero(st.sel_count.cpu().numpy()[0] > 0)[0][0])
    cols[0, i, 0] = 10_000                           # out of range, in a row that is read
    svg.sparse_attn(st.qp, st.kp, st.vp, st.q_off, st.k_off, st.sel_count, cols)
    assert svg.get_error() == 6                      # SVG_ERR_DEVICE_CHECK
    assert svg.get_error() == 0


def test_device_check_reports_block_count_beyond_the_row():
    """A block count above Ck is clamped to the row (no read past it) and flagged."""
    wl = synth.small_workload("480p-5s", (5, 12, 20), heads=1, cq=6, ck=40, iters=2)
    L = synth.make_layer(wl)
    layer = svg.SvgLayer(*L.q.shape, wl.cq, wl.ck)
    _, st = layer(dev_bf16(L.q), dev_bf16(L.k), dev_bf16(L.v), dev_f32(L.init_centroids("q")),
                  dev_f32(L.init_centroids("k")), wl.iters, 0.9)
    cnt = st.sel_count.clone()
    cols = torch.arange(wl.ck, dtype=torch.int32, device=cnt.device).expand_as(st.sel_cols).contiguous()
    i = int(np.nonzero(cnt.cpu().numpy()[0] > 0)[0][-1])   # the last non-empty row: nothing follows it
    cnt[0, i] = wl.ck + 1
    svg.sparse_attn(st.qp, st.kp, st.vp, st.q_off, st.k_off, cnt, cols)
    assert svg.get_error() == 6                      # SVG_ERR_DEVICE_CHECK
    assert svg.get_error() == 0
