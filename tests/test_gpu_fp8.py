"""GPU parity of the 8-bit Q K^T path (svg_quantize_e4m3, svg_sparse_attn_fp8)
against oracle/fp8_oracle.py.

  * quantisation: E4M3 values and float32 scales bit-exact (per row and per
    head; zero rows, wide dynamic ranges, saturation);
  * attention on the oracle's clustering and selection: relative L2 <= 1e-2,
    max abs <= 2e-2 against the float64 attention of the dequantised Q and K
    (the same bound as the bf16 path: P and O are bf16 either way), lse within
    1e-3; the fused un-permutation equals a separate pass bit for bit;
  * the layer with qk_fp8 equals its stages run one by one, bit for bit, and
    its CUDA-graph replay equals the eager call;
  * accuracy against exact attention (bf16 Q and K, no quantisation) is
    reported, and held to the bound the oracle itself reaches on the seeded
    case (relative L2 <= 0.08);
  * the full 480p-5s layer: sampled rows of four heads against the oracle, on
    the GPU's clustering and selection.
"""
import math

import numpy as np
import pytest
import torch

import synth
from oracle import fp8_oracle as f8
from oracle import svg_oracle as so
from tests.helpers import check_attention, dev_bf16, dev_f32, dev_i32, host_f32, rel_l2, selection_lists

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


def bf16_values(x: np.ndarray) -> np.ndarray:
    """float32 array rounded to bf16 values (what the device tensor holds)."""
    return synth.round_bf16(np.asarray(x, np.float32))


def awkward_rows(R: int, D: int, seed: int) -> np.ndarray:
    """Rows spanning many binades: per-row magnitudes 1e-4 .. 1e3, a zero row,
    rows with one dominant entry (the rest falls into E4M3's subnormal range)."""
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((R, D)) * (10.0 ** rng.uniform(-4, 3, (R, 1)))
    x[0] = 0.0
    x[1] = rng.standard_normal(D) * 1e-3
    x[1, 5] = 300.0
    x[2, :] = 2.0 ** -130      # bf16 subnormal inputs
    x[3, 7] = -np.abs(x[3]).max() * 4
    return bf16_values(x)


@pytest.mark.parametrize("D", [128, 64])
def test_quantize_rows_bit_exact(D):
    BH, N = 3, 301
    x = awkward_rows(BH * N, D, seed=D).reshape(BH, N, D)
    x8, s = svg.quantize_e4m3(dev_bf16(x), per_row=True)
    torch.cuda.synchronize()
    assert svg.get_error() == 0
    want8, want_s = f8.quantize_rows(x.reshape(BH * N, D))
    got_s = s.cpu().numpy().reshape(-1)
    assert np.array_equal(got_s, want_s)
    got8 = x8.float().cpu().numpy().reshape(BH * N, D)
    assert np.array_equal(got8, want8), np.argwhere(got8 != want8)[:5]


@pytest.mark.parametrize("D", [128, 64])
def test_quantize_heads_bit_exact(D):
    BH, N = 4, 517
    x = awkward_rows(BH * N, D, seed=10 + D).reshape(BH, N, D)
    x[2] = 0.0                 # an all-zero head: scale 1
    x[3] *= 1e-6
    x = bf16_values(x)
    x8, s = svg.quantize_e4m3(dev_bf16(x), per_row=False)
    torch.cuda.synchronize()
    assert svg.get_error() == 0
    got8 = x8.float().cpu().numpy()
    for h in range(BH):
        want8, want_s = f8.quantize_tensor(x[h])
        assert s[h].item() == want_s, h
        assert np.array_equal(got8[h], want8), (h, np.argwhere(got8[h] != want8)[:5])


@pytest.mark.parametrize("per_row", [True, False])
def test_quantize_gathered_equals_quantize_of_gathered_rows(per_row):
    """Quantising through a permutation equals gathering the rows first, bit for bit;
    a permutation entry out of range gives a zero row and the device check."""
    BH, N, D = 3, 517, 128
    x = awkward_rows(BH * N, D, seed=7).reshape(BH, N, D)
    rng = np.random.default_rng(8)
    perm = np.stack([rng.permutation(N) for _ in range(BH)]).astype(np.int32)
    xg = np.stack([x[h][perm[h]] for h in range(BH)])
    dx, dp = dev_bf16(x), dev_i32(perm)
    a8, sa = svg.quantize_e4m3(dx, per_row=per_row, perm=dp)
    b8, sb = svg.quantize_e4m3(dev_bf16(xg), per_row=per_row)
    torch.cuda.synchronize()
    assert svg.get_error() == 0
    assert torch.equal(a8.view(torch.uint8), b8.view(torch.uint8)) and torch.equal(sa, sb)
    bad = perm.copy()
    bad[1, 5] = N + 3
    c8, sc = svg.quantize_e4m3(dx, per_row=per_row, perm=dev_i32(bad))
    torch.cuda.synchronize()
    assert svg.get_error() == 6                  # SVG_ERR_DEVICE_CHECK
    assert torch.count_nonzero(c8[1, 5].view(torch.uint8)).item() == 0
    if per_row:
        assert sc[1, 5].item() == 1.0


def test_quantize_rejects_bad_arguments():
    lib = svg.load_library()
    x = torch.zeros((2, 8, 128), dtype=torch.bfloat16, device="cuda")
    x8 = torch.empty((2, 8, 128), dtype=torch.uint8, device="cuda")
    s = torch.empty(16, dtype=torch.float32, device="cuda")
    P = svg._ptr
    assert lib.svg_quantize_e4m3(P(x), None, 2, 8, 96, 1, P(x8), P(s), None) == 2        # D unsupported
    assert lib.svg_quantize_e4m3(P(x), None, 2, 8, 128, 2, P(x8), P(s), None) == 1       # per_row not 0/1
    assert lib.svg_quantize_e4m3(P(x), None, 2, 8, 128, 1, P(x), P(s), None) == 1        # x8 aliases x
    assert lib.svg_quantize_e4m3(None, None, 2, 8, 128, 1, P(x8), P(s), None) == 1


CASES = {
    "small-d128": synth.small_workload("480p-5s", (5, 12, 20), heads=3, cq=6, ck=40, iters=5),
    "small-drift": synth.small_workload("480p-10s", (9, 10, 14), heads=2, cq=10, ck=48, iters=5),
}


@pytest.fixture(scope="module")
def case_data():
    cache = {}

    def get(name):
        if name not in cache:
            wl = CASES[name]
            L = synth.make_layer(wl)
            ref = [so.svg_head(L.q[h], L.k[h], L.v[h], L.init_centroids("q")[h], L.init_centroids("k")[h], wl.iters,
                               wl.top_p[0], attention=False) for h in range(L.q.shape[0])]
            cache[name] = (L, ref)
        return cache[name]
    return get


def permuted_inputs(L, ref):
    H = L.q.shape[0]
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
    return qp, kp, vp, q_off, k_off, cnt, cols


def run_fp8(qp, kp, vp, q_off, k_off, cnt, cols, perm_q=None):
    q8, sq = svg.quantize_e4m3(dev_bf16(qp), per_row=True)
    k8, sk = svg.quantize_e4m3(dev_bf16(kp), per_row=False)
    op, lse = svg.sparse_attn_fp8(q8, sq, k8, sk, dev_bf16(vp), dev_i32(q_off), dev_i32(k_off), dev_i32(cnt),
                                  dev_i32(cols), want_lse=True, perm_q=perm_q)
    torch.cuda.synchronize()
    assert svg.get_error() == 0
    return op, lse


@pytest.mark.parametrize("name", list(CASES))
def test_fp8_attention_matches_oracle(name, case_data):
    L, ref = case_data(name)
    H, N, D = L.q.shape
    qp, kp, vp, q_off, k_off, cnt, cols = permuted_inputs(L, ref)
    op, lse = run_fp8(qp, kp, vp, q_off, k_off, cnt, cols)
    got, got_lse = host_f32(op), lse.cpu().numpy()
    errs = []
    for h in range(H):
        sel = [s.cols for s in ref[h].selection]
        want, want_lse = f8.sparse_attention_fp8(qp[h], kp[h], vp[h], q_off[h], k_off[h], sel, 1.0 / math.sqrt(D))
        check_attention(got[h], want, f"{name} head {h}")
        assert np.max(np.abs(got_lse[h] - want_lse)) < 1e-3
        exact, _ = so.sparse_attention(qp[h], kp[h], vp[h], q_off[h], k_off[h], sel, 1.0 / math.sqrt(D))
        errs.append(rel_l2(got[h], exact))
    print(f"{name}: fp8 Q K^T vs exact attention, relative L2 per head {['%.4f' % e for e in errs]}")
    assert max(errs) <= 0.08


@pytest.mark.parametrize("name", list(CASES))
def test_fp8_fused_unpermute_equals_separate_pass(name, case_data):
    L, ref = case_data(name)
    args = permuted_inputs(L, ref)
    op, lse = run_fp8(*args)
    perm = dev_i32(np.stack([r.perm_q for r in ref]))
    o, lse_o = run_fp8(*args, perm_q=perm)
    assert torch.equal(o, svg.unpermute(op, perm))
    lse_want = torch.empty_like(lse)
    lse_want.scatter_(1, perm.long(), lse)
    assert torch.equal(lse_o, lse_want)


def test_fp8_rejects_bad_arguments(case_data):
    L, ref = case_data("small-d128")
    qp, kp, vp, q_off, k_off, cnt, cols = permuted_inputs(L, ref)
    lib = svg.load_library()
    H, N, D = qp.shape
    q8, sq = svg.quantize_e4m3(dev_bf16(qp), per_row=True)
    k8, sk = svg.quantize_e4m3(dev_bf16(kp), per_row=False)
    v = dev_bf16(vp)
    o = torch.empty_like(v)
    ws = torch.empty(lib.svg_sparse_attn_workspace_size(H, N, q_off.shape[1] - 1), dtype=torch.uint8, device="cuda")
    P = svg._ptr
    qo, ko, c, cl = dev_i32(q_off), dev_i32(k_off), dev_i32(cnt), dev_i32(cols)

    def call(sq_, sk_, D_):
        return lib.svg_sparse_attn_fp8(P(q8), P(sq_), P(k8), P(sk_), P(v), H, N, D_, P(qo), q_off.shape[1] - 1,
                                       P(ko), k_off.shape[1] - 1, P(c), P(cl), 0.0, None, P(o), None, P(ws),
                                       ws.numel(), None)
    assert call(None, sk, D) == 1
    assert call(sq, None, D) == 1
    assert call(sq, sk, 64) == 2


def test_fp8_layer_equals_stages_and_graph(case_data):
    L, _ = case_data("small-d128")
    H, N, D = L.q.shape
    wl = CASES["small-d128"]
    q, k, v = dev_bf16(L.q), dev_bf16(L.k), dev_bf16(L.v)
    mq0, mk0 = dev_f32(L.init_centroids("q")), dev_f32(L.init_centroids("k"))
    layer = svg.SvgLayer(H, N, D, wl.cq, wl.ck)
    out, st = layer(q, k, v, mq0.clone(), mk0.clone(), wl.iters, wl.top_p[0], qk_fp8=True)
    out = out.clone()
    torch.cuda.synchronize()
    assert svg.get_error() == 0
    assert st.qp is None and st.kp is None      # Q and K were quantised while gathered
    q8, sq = svg.quantize_e4m3(q, per_row=True, perm=st.perm_q)
    k8, sk = svg.quantize_e4m3(k, per_row=False, perm=st.perm_k)
    want, _ = svg.sparse_attn_fp8(q8, sq, k8, sk, st.vp, st.q_off, st.k_off, st.sel_count, st.sel_cols,
                                  perm_q=st.perm_q)
    torch.cuda.synchronize()
    assert torch.equal(out, want)
    graph = svg.LayerGraph(layer, q, k, v, mq0, mk0, wl.iters, wl.top_p[0], qk_fp8=True)
    for _ in range(2):
        got = graph.replay()
        torch.cuda.synchronize()
        assert svg.get_error() == 0
        assert torch.equal(got, out)


def test_fp8_full_size_480p():
    """The full 480p-5s layer with qk_fp8 (the bench's configuration): sampled
    rows of four heads against the oracle on the GPU's clustering and selection."""
    L = synth.make_layer("480p-5s")
    wl = L.workload
    BH, N, D = L.q.shape
    layer = svg.SvgLayer(BH, N, D, wl.cq, wl.ck)
    out, st = layer(dev_bf16(L.q), dev_bf16(L.k), dev_bf16(L.v), dev_f32(L.init_centroids("q")),
                    dev_f32(L.init_centroids("k")), wl.iters, wl.top_p[0], qk_fp8=True)
    torch.cuda.synchronize()
    assert svg.get_error() == 0
    sel = selection_lists(st.sel_count, st.sel_cols)
    perm_q, perm_k = st.perm_q.cpu().numpy(), st.perm_k.cpu().numpy()
    q_off, k_off = st.q_off.cpu().numpy(), st.k_off.cpu().numpy()
    got = out.float()
    for h in (0, 17, 29, 39):
        rows = synth.sample_rows(N, 192, 50 + h)
        inv = np.empty_like(perm_q[h])
        inv[perm_q[h]] = np.arange(N)
        prow = np.sort(inv[rows])
        op, _ = f8.sparse_attention_fp8(so.gather_rows(L.q[h], perm_q[h]), so.gather_rows(L.k[h], perm_k[h]),
                                        so.gather_rows(L.v[h], perm_k[h]), q_off[h], k_off[h], sel[h],
                                        1.0 / math.sqrt(D), rows=prow)
        have = got[h][torch.from_numpy(perm_q[h][prow]).to(got.device)].cpu().numpy()
        check_attention(have, op[prow], f"480p fp8 head {h}")


def test_fp8_degenerate_inputs(case_data):
    """Degenerate inputs against the oracle: a head whose K is all zero (scale 1, every
    logit 0: uniform weights over the selected keys), zero query rows, and Q and K scaled
    by 8 (logits up to ~10^3 in magnitude: the softmax's running max must hold)."""
    L, ref = case_data("small-d128")
    qp, kp, vp, q_off, k_off, cnt, cols = permuted_inputs(L, ref)
    qp, kp = qp.copy(), kp.copy()
    kp[0] = 0.0                                  # head 0: K all zero
    qp[1, ::7] = 0.0                             # head 1: every 7th query row zero
    qp[2] = synth.round_bf16(qp[2] * 8.0)        # head 2: logits x 64
    kp[2] = synth.round_bf16(kp[2] * 8.0)
    op, lse = run_fp8(qp, kp, vp, q_off, k_off, cnt, cols)
    got, got_lse = host_f32(op), lse.cpu().numpy()
    D = qp.shape[2]
    for h in range(qp.shape[0]):
        sel = [s.cols for s in ref[h].selection]
        want, want_lse = f8.sparse_attention_fp8(qp[h], kp[h], vp[h], q_off[h], k_off[h], sel, 1.0 / math.sqrt(D))
        check_attention(got[h], want, f"degenerate head {h}")
        assert np.max(np.abs(got_lse[h] - want_lse) / np.maximum(1.0, np.abs(want_lse))) < 1e-3


def rand_bf16(shape, seed):
    return synth.round_bf16(np.random.default_rng(seed).standard_normal(shape).astype(np.float32))


@pytest.mark.parametrize("case", ["max-clusters", "one-token-clusters", "empty-clusters"])
def test_fp8_layer_edge_cases(case):
    """The 8-bit layer on the edge cases of the bf16 path, every row against the oracle on the
    GPU's clustering and selection: 1024 clusters with a ragged N = 4100 (max k-clusters per row,
    a partial last tile), one token per cluster (C = N), duplicated seeds (empty clusters) with p = 0.01."""
    if case == "max-clusters":
        q, k, v = (rand_bf16((1, 4100, 128), s) for s in (20, 21, 22))
        mu_q0, mu_k0, iters, p = q[:, :1024], k[:, :1024], 1, 0.9
    elif case == "one-token-clusters":
        q, k, v = (rand_bf16((1, 96, 128), s) for s in (23, 24, 25))
        mu_q0, mu_k0, iters, p = q.copy(), k.copy(), 2, 0.7
    else:
        q, k, v = (rand_bf16((2, 1500, 128), s) for s in (26, 27, 28))
        mu_q0, mu_k0, iters, p = np.repeat(q[:, :5], 4, axis=1), np.repeat(k[:, :9], 3, axis=1), 3, 0.01
    H, N, D = q.shape
    layer = svg.SvgLayer(H, N, D, mu_q0.shape[1], mu_k0.shape[1])
    out, st = layer(dev_bf16(q), dev_bf16(k), dev_bf16(v), dev_f32(mu_q0), dev_f32(mu_k0), iters, p, qk_fp8=True)
    torch.cuda.synchronize()
    assert svg.get_error() == 0
    got = host_f32(out)
    sel = selection_lists(st.sel_count, st.sel_cols)
    for h in range(H):
        perm_q, perm_k = st.perm_q.cpu().numpy()[h], st.perm_k.cpu().numpy()[h]
        op, _ = f8.sparse_attention_fp8(so.gather_rows(q[h], perm_q), so.gather_rows(k[h], perm_k),
                                        so.gather_rows(v[h], perm_k), st.q_off.cpu().numpy()[h],
                                        st.k_off.cpu().numpy()[h], sel[h], 1.0 / math.sqrt(D))
        check_attention(got[h], so.scatter_rows(op, perm_q), f"fp8 {case} head {h}")
    if case == "empty-clusters":
        n_q, cnt = st.n_q.cpu().numpy(), st.sel_count.cpu().numpy()
        assert (n_q == 0).any() and np.all(cnt[n_q == 0] == 0) and np.all(cnt[n_q > 0] >= 1)
