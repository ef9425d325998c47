"""GPU parity: every stage of the CUDA path against the float64 oracle.

Stage tests feed both sides identical inputs (the oracle's clustering,
offsets and selection), so each kernel is checked in isolation; the layer
tests run the whole path.  Comparison rules:
  * permutation, offsets, counts, gathered rows: bit-exact;
  * block selection: bit-exact on rows the oracle marks decided; a row is
    undecided only when its top-p cut sits within the float64 rounding band
    of p (oracle.selection_band, about 1e-12) or between weights equal to
    2^-38; there any valid minimal set is accepted (oracle.selection_is_valid),
    and the number of such rows is asserted to be zero on the seeded cases;
  * k-means one round: assignment equal except on tokens whose two nearest
    centroids are within the float32 error bound; centroids equal to the
    float32 rounding of the exact means of the GPU's own assignment;
  * k-means T rounds: >= 99.9 % of tokens agree;
  * attention: relative L2 <= 1e-2 and max abs <= 2e-2 (bf16 vs float64).
"""
import math

import numpy as np
import pytest
import torch

import synth
from oracle import svg_oracle as so
from tests.helpers import (KMEANS_AGREE, as_f32, assignment_gap_tolerance, check_attention, dev_bf16, dev_f32,
                           dev_i32, host_f32, selection_lists)

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


# Small cases: several q-tiles and key tiles each, ragged N, both head dims.
CASES = {
    "tiny": (synth.WORKLOADS["tiny"], None),
    "small-d128": (synth.small_workload("480p-5s", (5, 12, 20), heads=3, cq=6, ck=40, iters=5), None),
    "small-d64-dense": (synth.small_workload("dense-d64", (3, 10, 41), heads=2, cq=8, ck=30, iters=3), None),
    "small-drift": (synth.small_workload("480p-10s", (9, 10, 14), heads=2, cq=10, ck=48, iters=5), None),
}


def oracle_layer(L, p, iters=None, attention=True, rows=None):
    wl = L.workload
    T = wl.iters if iters is None else iters
    out = []
    for h in range(L.q.shape[0]):
        out.append(so.svg_head(L.q[h], L.k[h], L.v[h], L.init_centroids("q")[h], L.init_centroids("k")[h], T, p,
                               attention=attention, attn_rows=rows))
    return out


def top_p_of(wl):
    return wl.top_p[0]


@pytest.fixture(scope="module")
def case_data():
    cache = {}

    def get(name):
        if name not in cache:
            wl, _ = CASES[name]
            L = synth.make_layer(wl)
            cache[name] = (L, oracle_layer(L, top_p_of(wl)))
        return cache[name]
    return get


# ------------------------------------------------------------------ permutation

@pytest.mark.parametrize("name", list(CASES))
def test_permute_and_unpermute_bit_exact(name, case_data):
    L, ref = case_data(name)
    H, N, D = L.q.shape
    for which in ("q", "k"):
        C = ref[0].mu_q.shape[0] if which == "q" else ref[0].mu_k.shape[0]
        assign = np.stack([r.assign_q if which == "q" else r.assign_k for r in ref])
        x = L.q if which == "q" else L.k
        perm, off, (xp,) = svg.permute(dev_i32(assign), C, [dev_bf16(x)])
        perm, off = perm.cpu().numpy(), off.cpu().numpy()
        for h in range(H):
            p_ref, o_ref = so.permutation(assign[h], C)
            assert np.array_equal(perm[h], p_ref)
            assert np.array_equal(off[h], o_ref)
        xp_h = host_f32(xp)
        for h in range(H):
            assert np.array_equal(xp_h[h], so.gather_rows(x[h], perm[h]))
        back = svg.unpermute(xp, torch.from_numpy(perm).cuda())
        assert np.array_equal(host_f32(back), x)


def test_permute_three_tensors_and_ragged_sizes():
    rng = np.random.default_rng(5)
    for (H, N, D, C) in ((2, 1000, 128, 37), (3, 2049, 64, 1), (1, 5000, 128, 1024), (1, 77, 64, 77)):
        assign = rng.integers(0, C, (H, N))
        xs = [synth.round_bf16(rng.standard_normal((H, N, D)).astype(np.float32)) for _ in range(3)]
        perm, off, outs = svg.permute(dev_i32(assign), C, [dev_bf16(x) for x in xs])
        perm = perm.cpu().numpy()
        for h in range(H):
            p_ref, o_ref = so.permutation(assign[h], C)
            assert np.array_equal(perm[h], p_ref)
            assert np.array_equal(off.cpu().numpy()[h], o_ref)
        for x, o in zip(xs, outs):
            got = host_f32(o)
            for h in range(H):
                assert np.array_equal(got[h], x[h][perm[h]])


# ------------------------------------------------------------------ selection

def check_selection(got_lists, ref_rows_per_head, p):
    """Decided rows bit-exact, undecided rows valid; returns the undecided count."""
    undecided = 0
    for h, rows in enumerate(ref_rows_per_head):
        for i, r in enumerate(rows):
            got = got_lists[h][i]
            if r.undecided:
                undecided += 1
                assert so.selection_is_valid(got, r.weights, p, r.band), (h, i)
            else:
                assert np.array_equal(got, r.cols), (h, i, got, r.cols)
    return undecided


@pytest.mark.parametrize("name", list(CASES))
def test_select_matches_oracle(name, case_data):
    L, ref = case_data(name)
    p = top_p_of(L.workload)
    D = L.q.shape[2]
    scale = 1.0 / math.sqrt(D)
    mu_q = np.stack([r.mu_q for r in ref]).astype(np.float32)
    mu_k = np.stack([r.mu_k for r in ref]).astype(np.float32)
    n_q = np.stack([r.n_q for r in ref])
    n_k = np.stack([r.n_k for r in ref])
    for pp in sorted({p, 0.5, 0.9, 0.99, 1.0}):
        cnt, cols = svg.select_topp(dev_f32(mu_q), dev_i32(n_q), dev_f32(mu_k), dev_i32(n_k), pp)
        p32 = as_f32(pp)          # the kernel decides with the float32 value of p
        ref_rows = [so.select_topp(mu_q[h].astype(np.float64), n_q[h], mu_k[h].astype(np.float64), n_k[h], p32,
                                   scale) for h in range(len(ref))]
        undecided = check_selection(selection_lists(cnt, cols), ref_rows, p32)
        print(f"select {name} p={pp}: undecided rows {undecided}")
        assert undecided == 0


def test_select_hand_cases(golden):
    for case in ("select_equal_logits", "select_logits"):
        g = golden[case]
        # pad the 1- and 2-channel examples to D = 64 with zeros (dot products unchanged)
        mu_q = np.zeros((1, 1, 64), np.float32)
        mu_q[0, :, :len(g["mu_q"][0])] = g["mu_q"]
        mk = np.array(g["mu_k"], np.float32)
        mu_k = np.zeros((1, mk.shape[0], 64), np.float32)
        mu_k[0, :, :mk.shape[1]] = mk
        n_k = np.array([g["n_k"]], np.int32)
        for c in g["cases"]:
            cnt, cols = svg.select_topp(dev_f32(mu_q), dev_i32(np.ones((1, 1))), dev_f32(mu_k), dev_i32(n_k),
                                        c["p"], g["scale"])
            got = selection_lists(cnt, cols)[0][0].tolist()
            p32 = as_f32(c["p"])
            ref = so.select_topp(mu_q[0].astype(np.float64), np.ones(1), mu_k[0].astype(np.float64), n_k[0], p32,
                                 g["scale"])[0]
            # p landing exactly on a cumulative sum is a rounding boundary: there either cut is valid
            if ref.undecided:
                assert so.selection_is_valid(got, ref.weights, p32, ref.band), (case, c, got)
            else:
                assert got == ref.cols.tolist() == c["cols"], (case, c, got)


# ------------------------------------------------------------------ attention

def run_attention_from_oracle(L, ref, want_lse=True):
    H, N, D = L.q.shape
    qp = np.stack([so.gather_rows(L.q[h], ref[h].perm_q) for h in range(H)])
    kp = np.stack([so.gather_rows(L.k[h], ref[h].perm_k) for h in range(H)])
    vp = np.stack([so.gather_rows(L.v[h], ref[h].perm_k) for h in range(H)])
    q_off = np.stack([r.q_off for r in ref])
    k_off = np.stack([r.k_off for r in ref])
    Cq, Ck = q_off.shape[1] - 1, k_off.shape[1] - 1
    cnt = np.zeros((H, Cq), np.int32)
    cols = np.full((H, Cq, Ck), -1, np.int32)
    for h in range(H):
        for i, s in enumerate(ref[h].selection):
            cnt[h, i] = len(s.cols)
            cols[h, i, :len(s.cols)] = s.cols
    op, lse = svg.sparse_attn(dev_bf16(qp), dev_bf16(kp), dev_bf16(vp), dev_i32(q_off), dev_i32(k_off),
                              dev_i32(cnt), dev_i32(cols), want_lse=want_lse)
    return qp, kp, vp, q_off, k_off, op, lse


@pytest.mark.parametrize("name", list(CASES))
def test_sparse_attention_matches_oracle(name, case_data):
    L, ref = case_data(name)
    H, N, D = L.q.shape
    qp, kp, vp, q_off, k_off, op, lse = run_attention_from_oracle(L, ref)
    got = host_f32(op)
    got_lse = lse.cpu().numpy()
    for h in range(H):
        want, want_lse = so.sparse_attention(qp[h], kp[h], vp[h], q_off[h], k_off[h],
                                             [s.cols for s in ref[h].selection], 1.0 / math.sqrt(D))
        check_attention(got[h], want, f"{name} head {h}")
        assert np.max(np.abs(got_lse[h] - want_lse)) < 1e-3


@pytest.mark.parametrize("name", list(CASES))
def test_fused_unpermute_equals_separate_pass(name, case_data):
    """svg_sparse_attn_unpermuted == svg_sparse_attn then svg_unpermute, bit for bit (lse too)."""
    L, ref = case_data(name)
    qp, kp, vp, q_off, k_off, op, lse = run_attention_from_oracle(L, ref)
    perm = dev_i32(np.stack([r.perm_q for r in ref]))
    want = svg.unpermute(op, perm)
    H, N, D = L.q.shape
    cnt = np.zeros((H, q_off.shape[1] - 1), np.int32)
    cols = np.full((H, q_off.shape[1] - 1, k_off.shape[1] - 1), -1, np.int32)
    for h in range(H):
        for i, s in enumerate(ref[h].selection):
            cnt[h, i] = len(s.cols)
            cols[h, i, :len(s.cols)] = s.cols
    o, lse_o = svg.sparse_attn(dev_bf16(qp), dev_bf16(kp), dev_bf16(vp), dev_i32(q_off), dev_i32(k_off),
                               dev_i32(cnt), dev_i32(cols), want_lse=True, perm_q=perm)
    torch.cuda.synchronize()
    assert svg.get_error() == 0
    assert torch.equal(o, want)
    lse_want = torch.empty_like(lse)
    lse_want.scatter_(1, perm.long(), lse)
    assert torch.equal(lse_o, lse_want)


def oracle_blocks(ref, Cq, Ck):
    """The oracle's selection as (sel_count [H, Cq], sel_cols [H, Cq, Ck]) arrays."""
    H = len(ref)
    cnt = np.zeros((H, Cq), np.int32)
    cols = np.full((H, Cq, Ck), -1, np.int32)
    for h in range(H):
        for i, s in enumerate(ref[h].selection):
            cnt[h, i] = len(s.cols)
            cols[h, i, :len(s.cols)] = s.cols
    return cnt, cols


@pytest.mark.parametrize("name", list(CASES))
def test_gather_kv_equals_permuted_kv(name, case_data):
    """svg_sparse_attn_gather (K, V in token order, key rows fetched through perm_k) equals
    svg_sparse_attn on permuted K, V bit for bit, with and without the fused
    un-permutation (lse too); the latter is checked against the oracle above."""
    L, ref = case_data(name)
    qp, kp, vp, q_off, k_off, op, lse = run_attention_from_oracle(L, ref)
    cnt, cols = oracle_blocks(ref, q_off.shape[1] - 1, k_off.shape[1] - 1)
    perm_k = dev_i32(np.stack([r.perm_k for r in ref]))
    perm_q = dev_i32(np.stack([r.perm_q for r in ref]))
    args = (dev_i32(q_off), dev_i32(k_off), dev_i32(cnt), dev_i32(cols))
    k, v = dev_bf16(L.k), dev_bf16(L.v)
    og, lg = svg.sparse_attn_gather(dev_bf16(qp), k, v, perm_k, *args, want_lse=True)
    torch.cuda.synchronize()
    assert svg.get_error() == 0
    assert torch.equal(og, op)
    assert torch.equal(lg, lse)
    ou, lu = svg.sparse_attn_gather(dev_bf16(qp), k, v, perm_k, *args, want_lse=True, perm_q=perm_q)
    torch.cuda.synchronize()
    assert svg.get_error() == 0
    assert torch.equal(ou, svg.unpermute(op, perm_q))
    lse_want = torch.empty_like(lse)
    lse_want.scatter_(1, perm_q.long(), lse)
    assert torch.equal(lu, lse_want)


@pytest.mark.parametrize("name", list(CASES))
def test_layer_kv_gather_equals_permuted_layer(name, case_data):
    """The layer with K/V gathered inside attention gives the same output, bit for bit."""
    L, _ = case_data(name)
    H, N, D = L.q.shape
    wl = L.workload
    outs = []
    for gather in (False, True):
        layer = svg.SvgLayer(H, N, D, wl.cq, wl.ck)
        mu_q, mu_k = dev_f32(L.init_centroids("q")), dev_f32(L.init_centroids("k"))
        out, st = layer(dev_bf16(L.q), dev_bf16(L.k), dev_bf16(L.v), mu_q, mu_k, wl.iters, top_p_of(wl),
                        kv_gather=gather)
        torch.cuda.synchronize()
        assert svg.get_error() == 0
        assert (st.kp is None) == gather
        outs.append(out)
    assert torch.equal(outs[0], outs[1])


@pytest.mark.parametrize("name", ["tiny", "small-d128"])
def test_layer_graph_replay_equals_eager(name, case_data):
    """The layer recorded as a CUDA graph and replayed gives the eager layer's output, bit for bit."""
    L, _ = case_data(name)
    H, N, D = L.q.shape
    wl = L.workload
    q, k, v = dev_bf16(L.q), dev_bf16(L.k), dev_bf16(L.v)
    mq0, mk0 = dev_f32(L.init_centroids("q")), dev_f32(L.init_centroids("k"))
    layer = svg.SvgLayer(H, N, D, wl.cq, wl.ck)
    want, _ = layer(q, k, v, mq0.clone(), mk0.clone(), wl.iters, top_p_of(wl))
    want = want.clone()
    graph = svg.LayerGraph(layer, q, k, v, mq0, mk0, wl.iters, top_p_of(wl))
    for _ in range(2):                       # replays start from the same initial centroids
        got = graph.replay()
        torch.cuda.synchronize()
        assert svg.get_error() == 0
        assert torch.equal(got, want)


def test_sparse_attention_all_blocks_equals_dense(case_data):
    L, ref = case_data("tiny")
    H, N, D = L.q.shape
    C = ref[0].k_off.shape[0] - 1
    full = [so.RowSelection(np.nonzero(np.diff(ref[0].k_off) > 0)[0], None, None, False) for _ in ref[0].selection]
    ref_full = [so.HeadResult(**{**ref[0].__dict__, "selection": full})]
    qp, kp, vp, q_off, k_off, op, _ = run_attention_from_oracle(L, ref_full)
    got = svg.unpermute(op, dev_i32(np.stack([ref[0].perm_q])))
    dense = so.dense_attention(L.q[0], L.k[0], L.v[0], 1.0 / math.sqrt(D))
    check_attention(host_f32(got)[0], dense, "all blocks vs dense")


# ------------------------------------------------------------------ k-means

@pytest.mark.parametrize("name", list(CASES))
def test_kmeans_one_round(name, case_data):
    L, _ = case_data(name)
    H, N, D = L.q.shape
    for which, x in (("q", L.q), ("k", L.k)):
        mu0 = L.init_centroids(which)
        mu = dev_f32(mu0)
        _, assign, counts = svg.kmeans(dev_bf16(x), mu, 1)
        a_gpu, n_gpu, mu_gpu = assign.cpu().numpy(), counts.cpu().numpy(), mu.cpu().numpy()
        for h in range(H):
            a_ref, gap = so.kmeans_assign(x[h], mu0[h])
            tol = assignment_gap_tolerance(x[h], mu0[h])
            diff = a_gpu[h] != a_ref
            assert np.all(gap[diff] <= tol[diff]), f"{name}/{which}: flips beyond the float32 bound"
            assert diff.mean() < 1e-3
            # the update is the exact mean of the GPU's own assignment, rounded to float32
            mean_ref, cnt_ref = so.kmeans_update(x[h], a_gpu[h], mu0[h])
            assert np.array_equal(n_gpu[h], cnt_ref)
            assert np.array_equal(mu_gpu[h], mean_ref.astype(np.float32))


@pytest.mark.parametrize("name", list(CASES))
def test_kmeans_rounds_agree(name, case_data):
    L, ref = case_data(name)
    H = L.q.shape[0]
    T = L.workload.iters
    for which, x in (("q", L.q), ("k", L.k)):
        mu = dev_f32(L.init_centroids(which))
        _, assign, counts = svg.kmeans(dev_bf16(x), mu, T)
        a_gpu = assign.cpu().numpy()
        a_ref = np.stack([r.assign_q if which == "q" else r.assign_k for r in ref])
        agree = (a_gpu == a_ref).mean()
        assert agree >= KMEANS_AGREE, f"{name}/{which}: {agree:.5f}"


# ------------------------------------------------------------------ whole layer

@pytest.mark.parametrize("name", list(CASES))
def test_layer_end_to_end(name, case_data):
    L, ref = case_data(name)
    H, N, D = L.q.shape
    wl = L.workload
    p = top_p_of(wl)
    mu_q, mu_k = dev_f32(L.init_centroids("q")), dev_f32(L.init_centroids("k"))
    out, st = svg.svg_attention(dev_bf16(L.q), dev_bf16(L.k), dev_bf16(L.v), mu_q, mu_k, wl.iters, p)
    got = host_f32(out)
    sel = selection_lists(st.sel_count, st.sel_cols)
    perm_q, perm_k = st.perm_q.cpu().numpy(), st.perm_k.cpu().numpy()
    q_off, k_off = st.q_off.cpu().numpy(), st.k_off.cpu().numpy()
    oracle_clustering_checked = 0
    for h in range(H):
        # isolate: oracle attention on the GPU's own clustering and selection
        qp = so.gather_rows(L.q[h], perm_q[h])
        kp = so.gather_rows(L.k[h], perm_k[h])
        vp = so.gather_rows(L.v[h], perm_k[h])
        op, _ = so.sparse_attention(qp, kp, vp, q_off[h], k_off[h], sel[h], 1.0 / math.sqrt(D))
        check_attention(got[h], so.scatter_rows(op, perm_q[h]), f"{name} head {h} (GPU clustering)")
        # end to end against the oracle's own clustering
        if np.array_equal(st.assign_q.cpu().numpy()[h], ref[h].assign_q) and \
                np.array_equal(st.assign_k.cpu().numpy()[h], ref[h].assign_k):
            check_attention(got[h], ref[h].out, f"{name} head {h} (oracle clustering)")
            oracle_clustering_checked += 1
    print(f"layer {name}: {oracle_clustering_checked} of {H} heads also matched the oracle's own clustering")
    if name == "tiny":          # well-separated regions: the clustering must agree exactly
        assert oracle_clustering_checked == H


def test_layer_top_p_one_equals_dense():
    L = synth.make_layer("tiny")
    D = L.q.shape[2]
    out, _ = svg.svg_attention(dev_bf16(L.q), dev_bf16(L.k), dev_bf16(L.v), dev_f32(L.init_centroids("q")),
                               dev_f32(L.init_centroids("k")), 3, 1.0)
    dense = so.dense_attention(L.q[0], L.k[0], L.v[0], 1.0 / math.sqrt(D))
    check_attention(host_f32(out)[0], dense, "top-p 1.0 vs dense")


# ------------------------------------------------------------------ edge cases

def run_layer_and_check(q, k, v, mu_q0, mu_k0, iters, p, what):
    out, st = svg.svg_attention(dev_bf16(q), dev_bf16(k), dev_bf16(v), dev_f32(mu_q0), dev_f32(mu_k0), iters, p)
    H, N, D = q.shape
    got = host_f32(out)
    sel = selection_lists(st.sel_count, st.sel_cols)
    for h in range(H):
        perm_q, perm_k = st.perm_q.cpu().numpy()[h], st.perm_k.cpu().numpy()[h]
        op, _ = so.sparse_attention(so.gather_rows(q[h], perm_q), so.gather_rows(k[h], perm_k),
                                    so.gather_rows(v[h], perm_k), st.q_off.cpu().numpy()[h],
                                    st.k_off.cpu().numpy()[h], sel[h], 1.0 / math.sqrt(D))
        check_attention(got[h], so.scatter_rows(op, perm_q), what)
    return st


def rand_bf16(shape, seed):
    return synth.round_bf16(np.random.default_rng(seed).standard_normal(shape).astype(np.float32))


def test_edge_single_cluster_is_dense():
    q, k, v = (rand_bf16((2, 700, 64), s) for s in (1, 2, 3))
    st = run_layer_and_check(q, k, v, q[:, :1], k[:, :1], 2, 0.9, "one cluster")
    assert st.sel_count.cpu().numpy().tolist() == [[1], [1]]
    out, _ = svg.svg_attention(dev_bf16(q), dev_bf16(k), dev_bf16(v), dev_f32(q[:, :1]), dev_f32(k[:, :1]), 1, 0.5)
    for h in range(2):
        check_attention(host_f32(out)[h], so.dense_attention(q[h], k[h], v[h], 1 / 8.0), "one cluster vs dense")


def test_edge_one_token_per_cluster():
    q, k, v = (rand_bf16((1, 96, 128), s) for s in (4, 5, 6))
    st = run_layer_and_check(q, k, v, q.copy(), k.copy(), 2, 0.7, "C = N")
    assert np.array_equal(st.assign_q.cpu().numpy()[0], np.arange(96))
    assert np.all(st.n_k.cpu().numpy() == 1)


def test_edge_empty_clusters_and_tiny_p():
    q, k, v = (rand_bf16((2, 1500, 128), s) for s in (7, 8, 9))
    mu_q0 = np.repeat(q[:, :5], 4, axis=1)        # duplicated seeds -> empty clusters
    mu_k0 = np.repeat(k[:, :9], 3, axis=1)
    st = run_layer_and_check(q, k, v, mu_q0, mu_k0, 3, 0.01, "empty clusters, p=0.01")
    n_q = st.n_q.cpu().numpy()
    assert (n_q == 0).any()
    cnt = st.sel_count.cpu().numpy()
    assert np.all(cnt[n_q == 0] == 0) and np.all(cnt[n_q > 0] >= 1)


def test_edge_max_clusters_and_ragged_tail():
    q, k, v = (rand_bf16((1, 4100, 64), s) for s in (10, 11, 12))
    st = run_layer_and_check(q, k, v, q[:, :1024], k[:, :1024], 1, 0.9, "C = 1024")
    assert st.n_k.cpu().numpy().sum() == 4100


def test_warm_start_zero_drift_is_fixed_point():
    """Centroid cache: restarting from converged centroids on the same tokens keeps them."""
    L = synth.make_layer("tiny")
    x = dev_bf16(L.k)
    mu = dev_f32(L.init_centroids("k"))
    svg.kmeans(x, mu, 50)
    mu1 = mu.clone()
    _, a1, _ = svg.kmeans(x, mu, 1)
    _, a2, _ = svg.kmeans(x, mu, 1)
    assert torch.equal(a1, a2)
    assert torch.equal(mu, mu1)
