"""Pins for the CPU oracle: hand-derived worked examples, closed forms,
invariants and brute force on tiny inputs (no GPU).

Each pin checks the oracle against something other than itself: values
derived by hand from the definitions on the Sparse VideoGen2 page
(tests/golden/hand_cases.json), pure-Python brute force, closed forms
(one cluster = the mean; one cluster per token = a fixed point), textbook or
library routines (dense softmax attention, torch's scaled-dot-product
attention) and invariants of the method (permutation is a bijection and
leaves attention unchanged; top-p set reaches p and is minimal).
The mutation tests at the end plant typical mistakes in a copy of the oracle
and check that a pin catches each one.
"""
import math

import numpy as np
import pytest

import oracle
import synth
from oracle import svg_oracle as so


# ----------------------------------------------------------------- helpers

def brute_assign(x, mu):
    """argmin_c sum_d (x_nd - mu_cd)^2 by pure-Python loops (ties: lowest c)."""
    out, gaps = [], []
    for xn in x.tolist():
        ds = []
        for mc in mu.tolist():
            ds.append(sum((a - b) * (a - b) for a, b in zip(xn, mc)))
        best = min(range(len(ds)), key=lambda c: (ds[c], c))
        out.append(best)
        rest = sorted(ds)
        gaps.append(rest[1] - rest[0] if len(rest) > 1 else math.inf)
    return np.array(out), np.array(gaps)


def brute_softmax_row(q, keys, vals, scale):
    logits = [scale * sum(a * b for a, b in zip(q, k)) for k in keys]
    m = max(logits)
    e = [math.exp(s - m) for s in logits]
    tot = sum(e)
    out = [sum(e[j] * vals[j][d] for j in range(len(keys))) / tot for d in range(len(vals[0]))]
    return out, m + math.log(tot)


# Band used with hand-made weight vectors (a float64-sized rounding band).
BAND = 1e-12


def rnd(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


# ----------------------------------------------------------------- k-means

def test_assign_matches_brute_force():
    x, mu = rnd((60, 5), 1), rnd((7, 5), 2)
    a, gap = so.kmeans_assign(x, mu)
    ba, bg = brute_assign(x, mu)
    assert np.array_equal(a, ba)
    assert np.allclose(gap, bg, rtol=1e-9, atol=1e-9)


def test_assign_tie_goes_to_lowest_index():
    x = rnd((20, 3), 3)
    mu = rnd((4, 3), 4)
    mu[3] = mu[1]                        # duplicate centroid: exact ties
    mu[2] = mu[0]
    a, _ = so.kmeans_assign(x, mu)
    assert set(a.tolist()) <= {0, 1}


def test_golden_kmeans_1d(golden):
    g = golden["kmeans_1d"]
    x, mu = np.array(g["x"]), np.array(g["mu0"])
    for step in g["after_iter"]:
        mu_new, a, counts, _ = so.kmeans(x, mu, 1)
        assert a.tolist() == step["assign"]
        assert np.allclose(mu_new, step["mu"], rtol=0, atol=1e-12)
        mu = mu_new
    mu3, a3, _, _ = so.kmeans(x, np.array(g["mu0"]), 3)
    assert np.allclose(mu3, g["after_iter"][-1]["mu"], atol=1e-12)


def test_golden_empty_cluster_keeps_centroid(golden):
    g = golden["kmeans_empty_cluster"]
    mu, a, counts, _ = so.kmeans(np.array(g["x"]), np.array(g["mu0"]), 1)
    assert a.tolist() == g["assign"]
    assert counts.tolist() == g["counts"]
    assert np.allclose(mu, g["mu"], atol=1e-12)


def test_one_cluster_is_the_mean():
    x = rnd((37, 6), 5)
    mu, a, counts, _ = so.kmeans(x, x[:1], 2)
    mean = [sum(col) / len(col) for col in zip(*x.tolist())]     # closed form, written out
    assert np.allclose(mu[0], mean, atol=1e-12)
    assert counts.tolist() == [37]


def test_every_token_its_own_cluster_is_a_fixed_point():
    x = rnd((25, 4), 6)
    mu, a, counts, _ = so.kmeans(x, x.copy(), 3)
    assert np.array_equal(a, np.arange(25))
    assert np.array_equal(mu, x)
    assert np.all(counts == 1)


def test_objective_non_increasing_tiny_workload():
    L = synth.make_layer("tiny")
    for x, mu0 in ((L.q[0], L.init_centroids("q")[0]), (L.k[0], L.init_centroids("k")[0])):
        mu = mu0.astype(np.float64)
        prev = math.inf
        for _ in range(10):
            a, _ = so.kmeans_assign(x, mu)
            cur = so.lloyd_objective(x, mu, a)       # objective after assign
            assert cur <= prev + 1e-9 * abs(prev if prev < math.inf else 1)
            mu, _ = so.kmeans_update(x, a, mu)
            after = so.lloyd_objective(x, mu, a)     # update can only lower it
            assert after <= cur + 1e-9 * cur
            prev = after


def test_lloyd_objective_matches_brute_force():
    x, mu = rnd((23, 4), 24), rnd((5, 4), 25)
    a = np.random.default_rng(26).integers(0, 5, 23)
    brute = 0.0
    for n in range(23):
        for d in range(4):
            diff = x[n, d] - mu[a[n], d]
            brute += diff * diff
    assert abs(so.lloyd_objective(x, mu, a) - brute) <= 1e-12 * brute


def test_separated_mixture_recovers_regions():
    rng = np.random.default_rng(7)
    centres = rng.standard_normal((6, 16)) * 10.0
    labels = rng.integers(0, 6, 300)
    x = centres[labels] + 0.1 * rng.standard_normal((300, 16))
    init = np.stack([x[np.nonzero(labels == r)[0][0]] for r in range(6)])
    mu, a, counts, _ = so.kmeans(x, init, 4)
    assert np.array_equal(a, labels)        # init one token per region -> labels line up


def test_returned_centroids_are_means_of_returned_assignment():
    L = synth.make_layer("tiny")
    x = L.k[0]
    mu, a, counts, _ = so.kmeans(x, L.init_centroids("k")[0], 3)
    for c in range(mu.shape[0]):
        members = [x[n].tolist() for n in range(len(a)) if a[n] == c]
        assert counts[c] == len(members)
        if members:
            mean = [sum(col) / len(members) for col in zip(*members)]
            assert np.allclose(mu[c], mean, atol=1e-9)


# ----------------------------------------------------------------- permutation

def test_golden_permutation(golden):
    g = golden["permutation"]
    perm, off = so.permutation(np.array(g["assign"]), g["C"])
    assert perm.tolist() == g["perm"]
    assert off.tolist() == g["offsets"]


def test_permutation_invariants():
    rng = np.random.default_rng(8)
    a = rng.integers(0, 13, 500)
    perm, off = so.permutation(a, 13)
    assert np.array_equal(np.sort(perm), np.arange(500))          # bijection
    ids = a[perm]
    assert np.all(np.diff(ids) >= 0)                              # clusters contiguous
    for c in range(13):
        seg = perm[off[c]:off[c + 1]]
        assert np.all(a[seg] == c)
        assert np.all(np.diff(seg) > 0)                           # stable
        assert off[c + 1] - off[c] == int(np.sum(a == c))
    x = rng.standard_normal((500, 3)).astype(np.float32)
    assert np.array_equal(so.scatter_rows(so.gather_rows(x, perm), perm), x)


# ----------------------------------------------------------------- top-p selection

@pytest.mark.parametrize("case", ["select_equal_logits", "select_logits"])
def test_golden_select(golden, case):
    g = golden[case]
    mu_q, mu_k, n_k = np.array(g["mu_q"]), np.array(g["mu_k"]), np.array(g["n_k"])
    w = so.centroid_weights(mu_q[0], mu_k, n_k, g["scale"])
    assert np.allclose(w, g["weights"], atol=1e-12)
    for c in g["cases"]:
        rows = so.select_topp(mu_q, np.array([1]), mu_k, n_k, c["p"], g["scale"])
        assert rows[0].cols.tolist() == c["cols"], c


def test_weights_match_brute_force():
    mq, mk = rnd((1, 8), 9), rnd((11, 8), 10)
    nk = np.random.default_rng(11).integers(0, 9, 11)
    nk[3] = 0
    scale = 0.3
    w = so.centroid_weights(mq[0], mk, nk, scale)
    logits = [scale * sum(a * b for a, b in zip(mq[0], r)) for r in mk.tolist()]
    live = [j for j in range(11) if nk[j] > 0]
    m = max(logits[j] for j in live)
    raw = [nk[j] * math.exp(logits[j] - m) if nk[j] > 0 else 0.0 for j in range(11)]
    tot = sum(raw)
    assert np.allclose(w, [r / tot for r in raw], atol=1e-12)


def test_selection_reaches_p_and_is_minimal():
    rng = np.random.default_rng(12)
    for trial in range(200):
        w = rng.random(30) ** 4
        w[rng.integers(0, 30, 3)] = 0
        w /= w.sum()
        p = float(rng.uniform(0.05, 0.99))
        r = so.select_row(w, p, BAND)
        sel = r.cols
        mass = w[sel].sum()
        assert mass >= p - 1e-12
        assert mass - w[sel].min() < p                   # minimal
        uns = np.setdiff1d(np.nonzero(w > 0)[0], sel)
        if len(uns):
            assert w[sel].min() >= w[uns].max()          # exactly the top-|S|
        assert so.selection_is_valid(sel, w, p, BAND)


def test_p_one_keeps_every_live_cluster_and_empty_rows_select_nothing():
    mu_q, mu_k = rnd((3, 4), 13), rnd((6, 4), 14)
    n_q = np.array([5, 0, 2])
    n_k = np.array([1, 0, 3, 2, 0, 7])
    rows = so.select_topp(mu_q, n_q, mu_k, n_k, 1.0, 0.5)
    assert rows[0].cols.tolist() == [0, 2, 3, 5]
    assert rows[1].cols.tolist() == []
    assert rows[2].cols.tolist() == [0, 2, 3, 5]
    rows = so.select_topp(mu_q, n_q, mu_k, n_k, 0.3, 0.5)
    for i in (0, 2):
        assert len(rows[i].cols) >= 1 and not set(rows[i].cols.tolist()) & {1, 4}


def test_one_token_per_cluster_is_token_level_top_p():
    """C_q = C_k = N: centroid scores are the exact attention probabilities."""
    rng = np.random.default_rng(15)
    N, D, scale, p = 12, 4, 0.7, 0.8
    q, k = rng.standard_normal((N, D)), rng.standard_normal((N, D))
    rows = so.select_topp(q, np.ones(N, int), k, np.ones(N, int), p, scale)
    for i in range(N):
        logits = [scale * sum(a * b for a, b in zip(q[i], kk)) for kk in k.tolist()]
        m = max(logits)
        e = [math.exp(s - m) for s in logits]
        probs = [v / sum(e) for v in e]
        order = sorted(range(N), key=lambda j: (-probs[j], j))
        acc, chosen = 0.0, []
        for j in order:
            chosen.append(j)
            acc += probs[j]
            if acc >= p:
                break
        assert rows[i].cols.tolist() == sorted(chosen)


def test_selection_validator_rejects_wrong_sets():
    w = np.array([0.5, 0.3, 0.15, 0.05])
    assert so.selection_is_valid([0, 1], w, 0.75, BAND)
    assert not so.selection_is_valid([0], w, 0.75, BAND)           # mass too small
    assert not so.selection_is_valid([0, 1, 2], w, 0.75, BAND)     # not minimal
    assert not so.selection_is_valid([0, 2], w, 0.6, BAND)         # skips a heavier cluster
    # a cut one cluster short is rejected even when its mass misses p by only 1e-9
    w2 = np.array([0.5, 0.4 - 1e-9, 0.1 + 1e-9])
    assert not so.selection_is_valid([0, 1], w2, 0.9, BAND)
    assert so.selection_is_valid([0, 1, 2], w2, 0.9, BAND)


def _exact_prefix_masses(mu_q_i, mu_k, n_k, scale, order):
    """Normalised prefix masses along `order`, from exact rational logits and 50-digit exp."""
    from decimal import Decimal, localcontext
    from fractions import Fraction
    with localcontext() as ctx:
        ctx.prec = 50
        sc = Fraction(scale)
        logits = {}
        for j in range(len(n_k)):
            if n_k[j] > 0:
                dot = sum(Fraction(float(a)) * Fraction(float(b)) for a, b in zip(mu_q_i, mu_k[j]))
                f = dot * sc
                logits[j] = Decimal(f.numerator) / Decimal(f.denominator)
        m = max(logits.values())
        w = {j: Decimal(int(n_k[j])) * (logits[j] - m).exp() for j in logits}
        tot = sum(w.values())
        out, acc = [], Decimal(0)
        for j in order:
            acc += w[j]
            out.append(float(acc / tot))
        return np.array(out)


def test_selection_band_bounds_the_float64_error():
    """The band (twice one evaluation's bound) covers the oracle's own float64
    prefix masses against 50-digit arithmetic, on rows with large centroids."""
    rng = np.random.default_rng(31)
    for trial in range(12):
        D = (64, 128)[trial % 2]
        C = int(rng.integers(20, 120))
        mag = (1.0, 4.0, 12.0)[trial % 3]
        mu_q = (rng.standard_normal(D) * mag).astype(np.float32).astype(np.float64)
        mu_k = (rng.standard_normal((C, D)) * mag).astype(np.float32).astype(np.float64)
        n_k = rng.integers(0, 90, C)
        n_k[0] = 5
        scale = 1.0 / math.sqrt(D)
        band = so.selection_band(mu_q, mu_k, n_k, scale)
        assert 0 < band < 1e-9                   # float64-sized, not a float32-sized band
        w = so.centroid_weights(mu_q, mu_k, n_k, scale)
        r = so.select_row(w, 0.9, band, n_k > 0)
        exact = _exact_prefix_masses(mu_q, mu_k, n_k, scale, r.order)
        got = np.cumsum(w[r.order])
        assert np.max(np.abs(got - exact)) <= band / 2, (trial, np.max(np.abs(got - exact)), band)


def test_golden_density(golden):
    g = golden["density"]
    pairs, frac = so.density(np.array(g["q_off"]), np.array(g["k_off"]), g["selection"])
    assert pairs == g["pairs"] and frac == g["fraction"]


# ----------------------------------------------------------------- attention

def test_golden_attention(golden):
    g = golden["attention_two_keys"]
    q, k, v = (np.array(g[n]) for n in ("q", "k", "v"))
    out, lse = so.softmax_attention_rows(q, k, v, g["scale"])
    assert np.allclose(out, g["out"], atol=1e-12)
    assert np.allclose(lse, g["lse"], atol=1e-12)


def test_attention_rows_match_brute_force():
    q, k, v = rnd((5, 6), 16), rnd((9, 6), 17), rnd((9, 3), 18)
    out, lse = so.softmax_attention_rows(q, k, v, 0.4)
    for r in range(5):
        bo, bl = brute_softmax_row(q[r].tolist(), k.tolist(), v.tolist(), 0.4)
        assert np.allclose(out[r], bo, atol=1e-12) and abs(lse[r] - bl) < 1e-12


def test_dense_attention_matches_torch_sdpa():
    torch = pytest.importorskip("torch")
    q, k, v = rnd((40, 16), 19), rnd((55, 16), 20), rnd((55, 16), 21)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None], torch.from_numpy(k)[None], torch.from_numpy(v)[None])[0].numpy()
    assert np.allclose(so.dense_attention(q, k, v, 1 / 4.0), ref, atol=1e-12)


def test_sparse_attention_equals_masked_dense():
    rng = np.random.default_rng(22)
    N, D, Cq, Ck = 64, 8, 5, 7
    qp, kp, vp = rng.standard_normal((3, N, D))
    q_off = np.array([0, 10, 10, 30, 50, 64])
    k_off = np.array([0, 3, 20, 21, 40, 41, 60, 64])
    sel = [[0, 3], [], [6], [1, 2, 4, 5], [0, 1, 2, 3, 4, 5, 6]]
    out, lse = so.sparse_attention(qp, kp, vp, q_off, k_off, sel, 0.5)
    for i in range(Cq):
        allowed = np.zeros(N, bool)
        for j in sel[i]:
            allowed[k_off[j]:k_off[j + 1]] = True
        for r in range(q_off[i], q_off[i + 1]):
            s = kp @ qp[r] * 0.5
            s[~allowed] = -np.inf
            e = np.exp(s - s.max())
            assert np.allclose(out[r], (e / e.sum()) @ vp, atol=1e-12)


def test_single_key_row_returns_that_value_row():
    rng = np.random.default_rng(23)
    qp, kp, vp = rng.standard_normal((3, 10, 4))
    out, _ = so.sparse_attention(qp, kp, vp, np.array([0, 10]), np.array([0, 6, 7, 10]), [[1]], 1.0)
    assert np.allclose(out, np.broadcast_to(vp[6], (10, 4)), atol=1e-14)


def test_layer_at_p_one_equals_dense_attention():
    """Mathematical equivalence: permute -> attend over all blocks -> un-permute == dense."""
    L = synth.make_layer("tiny")
    q, k, v = L.q[0], L.k[0], L.v[0]
    r = so.svg_head(q, k, v, L.init_centroids("q")[0], L.init_centroids("k")[0], 10, 1.0)
    rows = synth.sample_rows(q.shape[0], 64, 0)
    dense = so.dense_attention(q, k, v, 1 / 8.0, rows)
    assert np.allclose(r.out[rows], dense, atol=1e-10)


def test_layer_tiny_top_p_is_sparse_and_close():
    L = synth.make_layer("tiny")
    q, k, v = L.q[0], L.k[0], L.v[0]
    r = so.svg_head(q, k, v, L.init_centroids("q")[0], L.init_centroids("k")[0], 10, 0.9)
    pairs, dens = so.density(r.q_off, r.k_off, [s.cols for s in r.selection])
    assert 0.02 < dens < 0.5
    dense = so.dense_attention(q, k, v, 1 / 8.0)
    err = np.linalg.norm(r.out - dense) / np.linalg.norm(dense)
    assert err < 0.1                    # region-structured input: top-p 0.9 keeps most of the mass


# ----------------------------------------------------------------- planted mistakes

def _expect_failure(fn, *args):
    with pytest.raises(AssertionError):
        fn(*args)


def test_pins_catch_planted_mistakes(monkeypatch, golden):
    # 1. dropped ||mu||^2 term in the distance
    orig = so.sq_distances
    monkeypatch.setattr(so, "sq_distances",
                        lambda x, mu: orig(x, mu) - np.einsum("cd,cd->c", mu, mu)[None, :])
    _expect_failure(test_assign_matches_brute_force)
    monkeypatch.setattr(so, "sq_distances", orig)
    # 2. weights without the cluster-size factor
    origw = so.centroid_weights
    monkeypatch.setattr(so, "centroid_weights",
                        lambda mq, mk, nk, s: origw(mq, mk, (np.asarray(nk) > 0).astype(int), s))
    _expect_failure(test_golden_select, golden, "select_equal_logits")
    monkeypatch.setattr(so, "centroid_weights", origw)
    # 3. top-p cut one element late (cumsum > p instead of >= p)
    origr = so.select_row

    def late(w, p, tol, live_mask=None):
        r = origr(w, p, tol, live_mask)
        if p < 1 and len(r.cols) < len(r.order):
            r.cols = np.sort(r.order[:len(r.cols) + 1])
        return r
    monkeypatch.setattr(so, "select_row", late)
    _expect_failure(test_selection_reaches_p_and_is_minimal)
    monkeypatch.setattr(so, "select_row", origr)
    # 4. transposed value operand / wrong scale in attention
    origa = so.softmax_attention_rows
    monkeypatch.setattr(so, "softmax_attention_rows", lambda q, k, v, s: origa(q, k, v, 1.0))
    _expect_failure(test_attention_rows_match_brute_force)
    monkeypatch.setattr(so, "softmax_attention_rows", origa)
    # 5. un-permute applied as a second gather instead of a scatter
    origs = so.scatter_rows
    monkeypatch.setattr(so, "scatter_rows", lambda xp, perm: np.asarray(xp)[perm])
    _expect_failure(test_permutation_invariants)
    monkeypatch.setattr(so, "scatter_rows", origs)
    # 6. objective with unsquared differences
    monkeypatch.setattr(so, "lloyd_objective", lambda x, mu, a: float(np.sum(
        np.abs(np.asarray(x, np.float64) - np.asarray(mu, np.float64)[a]))))
    _expect_failure(test_lloyd_objective_matches_brute_force)
    # 7. density counting k-cluster sizes only (q-cluster size dropped)
    monkeypatch.setattr(so, "density", lambda qo, ko, sel: (
        float(sum(np.diff(ko)[np.asarray(c, np.int64)].sum() for c in sel if len(c))), 0.0))
    _expect_failure(test_golden_density, golden)
    # 8. a float32-sized rounding band (u = 2^-24) would swallow decided cuts
    monkeypatch.setattr(so, "U64", 2.0 ** -24)
    _expect_failure(test_selection_band_bounds_the_float64_error)
