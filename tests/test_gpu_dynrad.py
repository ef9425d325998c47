"""GPU parity of the DynamicRad block masks (svg_dynrad_select) and of the
attention kernel running them, against oracle/dynrad_oracle.py.

  * block offsets, candidate-set and static-ratio selections: bit-exact;
  * dynamic-threshold selection: bit-exact on rows the oracle marks decided
    (no proxy within the float64 rounding band of theta, fallback maximum
    separated by more than the band); any valid row elsewhere, and the number
    of such rows is asserted to be zero on the seeded cases;
  * attention on those masks: relative L2 <= 1e-2, max abs <= 2e-2 against
    float64 (all rows on the small cases, seeded sampled rows at full size).
"""
import math

import numpy as np
import pytest
import torch

import synth
from oracle import dynrad_oracle as dr
from tests.helpers import as_f32, check_attention, dev_bf16, host_f32, selection_lists

pytestmark = pytest.mark.gpu

svg = pytest.importorskip("sparse_attention_long_svg_b200")


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from sparse_attention_long_svg_b200 import build
    build.build()
    svg.load_library()
    yield
    assert svg.get_error() == 0


# (workload, block, w0, gamma, rho0, thetas)
CASES = {
    "small-d128": (synth.small_workload("480p-5s", (5, 12, 20), heads=3, cq=6, ck=40, iters=2), 32, 2.5, 0.6, 0.5,
                   (0.5, 3.0)),
    "small-d64": (synth.small_workload("dense-d64", (3, 10, 41), heads=2, cq=8, ck=30, iters=2), 64, 1.8, 0.5, 0.4,
                  (0.25, 2.0)),
}
FULL = ("480p-5s", 256, 3.0, 0.5, 0.5, 1.0)   # the bench's settings


def _params(w0, gamma, rho0, theta):
    return as_f32(w0), as_f32(gamma), as_f32(rho0), as_f32(theta)


def check_dynamic(got_rows, q, k, offs, frames, nb, w0, gamma, theta, scale):
    """Per-row validity against the oracle; returns the number of undecided rows."""
    rows = dr.dynamic_select(q, k, offs, frames, nb, w0, gamma, theta, scale)
    cand = dr.candidates(frames, nb, w0, gamma)
    undecided = 0
    for i, (g, r) in enumerate(zip(got_rows, rows)):
        ok, decided = dr.dynamic_row_is_valid(g, cand[i], r, theta)
        assert ok, f"row {i}: gpu {g.tolist()} oracle {r.cols.tolist()}"
        undecided += not decided
    return undecided


@pytest.mark.parametrize("name", list(CASES))
def test_candidates_and_static_bit_exact(name):
    wl, B, w0, gamma, rho0, _ = CASES[name]
    L = synth.make_layer(wl)
    H, N, D = L.q.shape
    frames = wl.grid[0]
    w0, gamma, rho0, _ = _params(w0, gamma, rho0, 0.0)
    q, k = dev_bf16(L.q), dev_bf16(L.k)
    offs, nb = dr.block_layout(N, frames, B)
    for mode, want in (("candidates", dr.candidates(frames, nb, w0, gamma)),
                       ("static", dr.static_select(frames, nb, w0, gamma, rho0))):
        o, cnt, cols = svg.dynrad_select(q, k, frames, B, mode, w0, gamma, rho0)
        torch.cuda.synchronize()
        assert svg.get_error() == 0
        assert np.array_equal(o.cpu().numpy(), np.tile(offs, (H, 1)))
        got = selection_lists(cnt, cols)
        for h in range(H):
            assert [x.tolist() for x in got[h]] == [x.tolist() for x in want], f"{name} {mode} head {h}"


@pytest.mark.parametrize("name", list(CASES))
def test_dynamic_matches_oracle(name):
    wl, B, w0, gamma, rho0, thetas = CASES[name]
    L = synth.make_layer(wl)
    H, N, D = L.q.shape
    frames = wl.grid[0]
    offs, nb = dr.block_layout(N, frames, B)
    q, k = dev_bf16(L.q), dev_bf16(L.k)
    for theta in thetas:
        w0f, gf, _, tf = _params(w0, gamma, rho0, theta)
        _, cnt, cols = svg.dynrad_select(q, k, frames, B, "dynamic", w0f, gf, theta=tf)
        torch.cuda.synchronize()
        assert svg.get_error() == 0
        got = selection_lists(cnt, cols)
        undecided = sum(check_dynamic(got[h], L.q[h], L.k[h], offs, frames, nb, w0f, gf, tf, 1.0 / math.sqrt(D))
                        for h in range(H))
        print(f"dynrad {name} theta {theta}: {undecided} undecided rows")
        assert undecided == 0


@pytest.mark.parametrize("name", list(CASES))
@pytest.mark.parametrize("mode", ["static", "dynamic"])
def test_attention_on_dynrad_masks(name, mode):
    wl, B, w0, gamma, rho0, thetas = CASES[name]
    L = synth.make_layer(wl)
    H, N, D = L.q.shape
    frames = wl.grid[0]
    w0f, gf, rf, tf = _params(w0, gamma, rho0, thetas[0])
    out, lse, (o, cnt, cols) = svg.dynrad_attention(dev_bf16(L.q), dev_bf16(L.k), dev_bf16(L.v), frames, B, mode,
                                                    w0f, gf, rf, tf, want_lse=True)
    torch.cuda.synchronize()
    assert svg.get_error() == 0
    offs = o.cpu().numpy()[0].astype(np.int64)
    sel = selection_lists(cnt, cols)
    got, got_lse = host_f32(out), lse.cpu().numpy()
    for h in range(H):
        want, want_lse = dr.attention(L.q[h], L.k[h], L.v[h], offs, sel[h], 1.0 / math.sqrt(D))
        check_attention(got[h], want, f"{name} {mode} head {h}")
        assert np.max(np.abs(got_lse[h] - want_lse)) < 1e-3


def _sampled_attention(q, k, v, offs, sel, rows, scale):
    """Oracle attention of single query rows (float64), from the block list."""
    owner = np.searchsorted(offs, rows, side="right") - 1
    out = np.zeros((len(rows), q.shape[1]))
    for n, (r, i) in enumerate(zip(rows, owner)):
        keys = np.concatenate([np.arange(offs[j], offs[j + 1]) for j in sel[i]])
        s = (k[keys].astype(np.float64) @ q[r].astype(np.float64)) * scale
        e = np.exp(s - s.max())
        out[n] = (e @ v[keys].astype(np.float64)) / e.sum()
    return out


@pytest.mark.parametrize("mode", ["static", "dynamic"])
def test_full_size_480p(mode):
    """The bench's DynamicRad settings on the full 480p-5s layer: every head's
    selection against the oracle, attention on seeded sampled rows of two heads."""
    name, B, w0, gamma, rho0, theta = FULL
    wl = synth.WORKLOADS[name]
    L = synth.make_layer(wl)
    H, N, D = L.q.shape
    frames = wl.grid[0]
    offs, nb = dr.block_layout(N, frames, B)
    w0f, gf, rf, tf = _params(w0, gamma, rho0, theta)
    q, k, v = dev_bf16(L.q), dev_bf16(L.k), dev_bf16(L.v)
    out, _, (o, cnt, cols) = svg.dynrad_attention(q, k, v, frames, B, mode, w0f, gf, rf, tf)
    torch.cuda.synchronize()
    assert svg.get_error() == 0
    assert np.array_equal(o.cpu().numpy(), np.tile(offs, (H, 1)))
    sel = selection_lists(cnt, cols)
    scale = 1.0 / math.sqrt(D)
    if mode == "static":
        want = [x.tolist() for x in dr.static_select(frames, nb, w0f, gf, rf)]
        for h in range(H):
            assert [x.tolist() for x in sel[h]] == want, f"head {h}"
    else:
        undecided = sum(check_dynamic(sel[h], L.q[h], L.k[h], offs, frames, nb, w0f, gf, tf, scale)
                        for h in range(H))
        assert undecided == 0
    got = host_f32(out)
    for h in (0, H - 1):
        rows = synth.sample_rows(N, 256, seed=100 + h)
        want = _sampled_attention(L.q[h], L.k[h], L.v[h], offs, sel[h], rows, scale)
        check_attention(got[h][rows], want, f"480p {mode} head {h} sampled rows")
