"""Pins of the DynamicRad mask oracle (CPU only).

Each pin checks oracle/dynrad_oracle.py against something other than itself:
hand-derived values from the definitions (tests/golden/hand_cases.json),
brute force written differently (vectorised masks, explicit loops), limits
that reduce to the candidate set, and textbook masked dense attention.  The
mutation test at the end plants typical mistakes and checks that a pin fails
for each.
"""
import math

import numpy as np
import pytest
import torch

from oracle import dynrad_oracle as dr


def _brute_candidates(frames, nb, w0, gamma):
    """Candidate mask by broadcasting over (t1, b1, t2, b2) with numpy's power."""
    t = np.repeat(np.arange(frames), nb)
    b = np.tile(np.arange(nb), frames)
    dt = np.abs(t[:, None] - t[None, :])
    db = np.abs(b[:, None] - b[None, :])
    w = np.floor(w0 * np.power(gamma, dt.astype(np.float64)))
    return db <= w


def test_golden_layout_candidates_static(golden):
    g = golden["dynrad_layout"]
    offs, nb = dr.block_layout(g["N"], g["frames"], g["block"])
    assert offs.tolist() == g["offsets"] and nb == g["blocks_per_frame"]
    assert [dr.window(d, g["w0"], g["gamma"]) for d in range(g["frames"])] == g["windows"]
    assert [c.tolist() for c in dr.candidates(g["frames"], nb, g["w0"], g["gamma"])] == g["candidates"]
    got = dr.static_select(g["frames"], nb, g["w0"], g["gamma"], g["rho0"])
    assert [c.tolist() for c in got] == g["static"]


def test_golden_dynamic(golden):
    g = golden["dynrad_dynamic"]
    offs, nb = dr.block_layout(g["N"], g["frames"], g["block"])
    assert [c.tolist() for c in dr.candidates(g["frames"], nb, g["w0"], g["gamma"])] == g["candidates"]
    q, k = np.asarray(g["q"], np.float64), np.asarray(g["k"], np.float64)
    for case in g["cases"]:
        rows = dr.dynamic_select(q, k, offs, g["frames"], nb, g["w0"], g["gamma"], case["theta"], g["scale"])
        assert [r.cols.tolist() for r in rows] == case["cols"], case["why"]
        assert [r.fallback for r in rows] == case["fallback"]


@pytest.mark.parametrize("frames,S,B", [(5, 37, 8), (3, 64, 16), (1, 50, 7)])
def test_layout_brute_force(frames, S, B):
    offs, nb = dr.block_layout(frames * S, frames, B)
    owner = np.full(frames * S, -1)
    for c in range(len(offs) - 1):
        owner[offs[c]:offs[c + 1]] = c
    for n in range(frames * S):                       # token n = t S + s lies in block t nb + s // B
        assert owner[n] == (n // S) * nb + (n % S) // B
    assert nb == math.ceil(S / B)


@pytest.mark.parametrize("w0,gamma", [(2.7, 0.6), (5.3, 0.8), (1.2, 0.3)])
def test_candidates_match_brute_force(w0, gamma):
    frames, nb = 6, 9
    mask = _brute_candidates(frames, nb, w0, gamma)
    got = dr.candidates(frames, nb, w0, gamma)
    for i in range(frames * nb):
        assert got[i].tolist() == np.flatnonzero(mask[i]).tolist()


def test_candidates_symmetric_and_reflexive():
    frames, nb = 7, 6
    cand = dr.candidates(frames, nb, 3.1, 0.55)
    m = np.zeros((frames * nb, frames * nb), bool)
    for i, c in enumerate(cand):
        m[i, c] = True
    assert np.array_equal(m, m.T)
    assert m.diagonal().all()
    for i in range(frames * nb):                      # the co-located block of every frame is a candidate
        b1 = i % nb
        assert all(m[i, t2 * nb + b1] for t2 in range(frames))


def test_static_ratio_one_keeps_every_candidate():
    frames, nb = 5, 8                                # rho(d) = min(1, rho0 gamma^d) = 1 at every distance
    a = dr.candidates(frames, nb, 3.6, 0.7)
    b = dr.static_select(frames, nb, 3.6, 0.7, 1e9)
    assert [x.tolist() for x in a] == [x.tolist() for x in b]


def test_static_keeps_the_nearest_share_of_every_frame():
    frames, nb, w0, gamma, rho0 = 6, 11, 4.4, 0.75, 0.6
    cand = dr.candidates(frames, nb, w0, gamma)
    got = dr.static_select(frames, nb, w0, gamma, rho0)
    for i in range(frames * nb):
        t1, b1 = divmod(i, nb)
        for t2 in range(frames):
            c = [j % nb for j in cand[i] if j // nb == t2]
            kept = [j % nb for j in got[i] if j // nb == t2]
            rho = min(1.0, rho0 * gamma ** abs(t1 - t2))
            assert len(kept) == max(1, math.ceil(rho * len(c) - 1e-12))
            dropped = [x for x in c if x not in kept]
            if dropped:                                # every kept block is at least as near as every dropped one
                assert max(abs(x - b1) for x in kept) <= min(abs(x - b1) for x in dropped)


def test_block_means_brute_force():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((45, 4))
    offs, _ = dr.block_layout(45, 3, 4)
    got = dr.block_means(x, offs)
    for c in range(len(offs) - 1):
        rows = [x[n] for n in range(offs[c], offs[c + 1])]
        want = [sum(r[d] for r in rows) / len(rows) for d in range(4)]
        assert np.allclose(got[c], want, rtol=0, atol=1e-15)


def test_dynamic_limits():
    rng = np.random.default_rng(5)
    frames, S, B, D = 4, 24, 5, 8
    q, k = rng.standard_normal((frames * S, D)), rng.standard_normal((frames * S, D))
    offs, nb = dr.block_layout(frames * S, frames, B)
    cand = dr.candidates(frames, nb, 2.5, 0.6)
    every = dr.dynamic_select(q, k, offs, frames, nb, 2.5, 0.6, -math.inf, 0.5)
    assert [r.cols.tolist() for r in every] == [c.tolist() for c in cand]
    none = dr.dynamic_select(q, k, offs, frames, nb, 2.5, 0.6, math.inf, 0.5)
    mq = [q[offs[c]:offs[c + 1]].mean(0) for c in range(len(offs) - 1)]
    mk = [k[offs[c]:offs[c + 1]].mean(0) for c in range(len(offs) - 1)]
    for i, r in enumerate(none):                      # all rows fall back to their best candidate
        scores = [0.5 * float(np.dot(mq[i], mk[j])) for j in cand[i]]
        assert r.fallback and r.cols.tolist() == [int(cand[i][int(np.argmax(scores))])]


def test_dynamic_proxies_match_brute_force():
    rng = np.random.default_rng(9)
    frames, S, B, D = 3, 23, 6, 5                      # ragged blocks of 6, 6, 6, 5
    q, k = rng.standard_normal((frames * S, D)), rng.standard_normal((frames * S, D))
    offs, nb = dr.block_layout(frames * S, frames, B)
    rows = dr.dynamic_select(q, k, offs, frames, nb, 1.5, 0.5, 0.0, 0.3)
    for i, (r, cand) in enumerate(zip(rows, dr.candidates(frames, nb, 1.5, 0.5))):
        qi = [sum(q[n][d] for n in range(offs[i], offs[i + 1])) / (offs[i + 1] - offs[i]) for d in range(D)]
        for p, j in zip(r.proxies, cand):
            kj = [sum(k[n][d] for n in range(offs[j], offs[j + 1])) / (offs[j + 1] - offs[j]) for d in range(D)]
            assert abs(p - 0.3 * sum(a * b for a, b in zip(qi, kj))) < 1e-13


def test_proxy_band_bounds_reordered_sums():
    rng = np.random.default_rng(7)
    for _ in range(20):
        a, b = rng.standard_normal(64), rng.standard_normal((5, 64))
        band = dr.proxy_band(a, b, 0.125)
        for j in range(5):
            fwd = 0.0
            for d in range(64):
                fwd += a[d] * b[j, d]
            rev = 0.0
            for d in reversed(range(64)):
                rev += a[d] * b[j, d]
            assert abs(fwd * 0.125 - rev * 0.125) <= band


def test_attention_equals_masked_dense():
    rng = np.random.default_rng(11)
    frames, S, B, D = 3, 20, 6, 16
    N = frames * S
    q, k, v = (rng.standard_normal((N, D)) for _ in range(3))
    offs, nb = dr.block_layout(N, frames, B)
    Cb = len(offs) - 1                                 # an asymmetric block list: a random subset per row
    sel = [np.sort(rng.choice(Cb, size=int(rng.integers(1, Cb + 1)), replace=False)) for _ in range(Cb)]
    got, lse = dr.attention(q, k, v, offs, sel, 1.0 / math.sqrt(D))
    mask = torch.full((N, N), -math.inf, dtype=torch.float64)
    for i, cols in enumerate(sel):
        for j in cols:
            mask[offs[i]:offs[i + 1], offs[j]:offs[j + 1]] = 0.0
    t = lambda a: torch.from_numpy(a)[None, None]
    want = torch.nn.functional.scaled_dot_product_attention(t(q), t(k), t(v), attn_mask=mask)[0, 0].numpy()
    assert np.allclose(got, want, rtol=1e-12, atol=1e-12)
    logits = (q @ k.T) / math.sqrt(D) + mask.numpy()
    assert np.allclose(lse, np.log(np.exp(logits - logits.max(1, keepdims=True)).sum(1)) + logits.max(1), atol=1e-12)


def test_validity_rejects_wrong_rows():
    row = dr.DynRow(np.array([2, 5]), np.array([0.1, 3.0, 0.2, 2.5]), 1e-12, False)
    cand = np.array([1, 2, 4, 5])
    assert dr.dynamic_row_is_valid(np.array([2, 5]), cand, row, 1.0) == (True, True)
    assert dr.dynamic_row_is_valid(np.array([2]), cand, row, 1.0)[0] is False
    assert dr.dynamic_row_is_valid(np.array([1, 2, 5]), cand, row, 1.0)[0] is False
    near = dr.DynRow(np.array([2]), np.array([0.1, 1.0 + 1e-14, 0.2, 0.3]), 1e-12, False)
    assert dr.dynamic_row_is_valid(np.array([2]), cand, near, 1.0) == (True, False)
    assert dr.dynamic_row_is_valid(np.array([1]), cand, near, 1.0)[0] is False


# ----------------------------------------------------------------- planted mistakes

def _expect_failure(fn, *args):
    with pytest.raises(AssertionError):
        fn(*args)


def test_pins_catch_planted_mistakes(monkeypatch, golden):
    # 1. window one frame too far (d + 1)
    with monkeypatch.context() as m:
        orig = dr.window
        m.setattr(dr, "window", lambda d, w0, g: orig(d + 1, w0, g))
        _expect_failure(test_golden_layout_candidates_static, golden)
        _expect_failure(test_candidates_match_brute_force, 2.7, 0.6)
    # 2. static mode keeps the farthest candidates
    with monkeypatch.context() as m:
        def farthest(frames, nb, w0, gamma, rho0):
            out = []
            for t1 in range(frames):
                for b1 in range(nb):
                    ids = []
                    for t2 in range(frames):
                        d = abs(t1 - t2)
                        cand = [b2 for b2 in range(nb) if abs(b1 - b2) <= dr.window(d, w0, gamma)]
                        kk = max(1, int(math.ceil(min(1.0, dr.decayed(rho0, gamma, d)) * len(cand))))
                        ids.extend(t2 * nb + b2 for b2 in sorted(sorted(cand, key=lambda x: -abs(x - b1))[:kk]))
                    out.append(np.asarray(ids, np.int64))
            return out
        m.setattr(dr, "static_select", farthest)
        _expect_failure(test_golden_layout_candidates_static, golden)
        _expect_failure(test_static_keeps_the_nearest_share_of_every_frame)
    # 3. dynamic fallback keeps the lowest-scoring candidate
    with monkeypatch.context() as m:
        orig_sel = dr.dynamic_select

        def worst(q, k, offsets, frames, nb, w0, gamma, theta, scale):
            rows = orig_sel(q, k, offsets, frames, nb, w0, gamma, theta, scale)
            cand = dr.candidates(frames, nb, w0, gamma)
            for r, c in zip(rows, cand):
                if r.fallback:
                    r.cols = c[[int(np.argmin(r.proxies))]]
            return rows
        m.setattr(dr, "dynamic_select", worst)
        _expect_failure(test_golden_dynamic, golden)
        _expect_failure(test_dynamic_limits)
    # 4. block means summed instead of averaged
    with monkeypatch.context() as m:
        m.setattr(dr, "block_means", lambda x, offs: np.stack(
            [np.asarray(x, np.float64)[offs[c]:offs[c + 1]].sum(0) for c in range(len(offs) - 1)]))
        _expect_failure(test_block_means_brute_force)
        _expect_failure(test_dynamic_proxies_match_brute_force)
    # 5. attention over the transposed block list (key blocks as query blocks)
    with monkeypatch.context() as m:
        orig_att = dr.attention

        def transposed(q, k, v, offsets, sel, scale):
            tr = [[] for _ in sel]
            for i, cols in enumerate(sel):
                for j in cols:
                    tr[int(j)].append(i)
            return orig_att(q, k, v, offsets, [np.asarray(sorted(c), np.int64) for c in tr], scale)
        m.setattr(dr, "attention", transposed)
        _expect_failure(test_attention_equals_masked_dense)
