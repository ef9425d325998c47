"""Benchmark of the semantic-aware top-p sparse attention layer on B200.

One step = one pass of the whole hot path over one layer of synthetic
input: k-means of Q and of K from the seeded token-sampled centroids,
permutation of Q and of K/V, centroid top-p selection, block-sparse
attention and un-permutation (the stages of the Sparse VideoGen2 page,
section 2).  Default workload: 480p, 5 s clip = 32,760 latent tokens
(21x30x52), 40 heads, head dim 128, 100/500 clusters, 5 k-means rounds,
top-p 0.9.

Prints ONE JSON line (rank 0).  value = whole-job throughput in effective
TFLOP/s: algorithmic attention FLOPs on the selected blocks
(4 * D * sum over selected (q-cluster, k-cluster) pairs of n_q * n_k) of all
layers processed by all ranks, divided by the max-over-ranks device time of
the timed steps; ms_per_step is ms per layer.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl svg|reference]
                  [--heads H] [--no-cpu-baseline]

Multi-GPU (one process per GPU, torchrun): every rank runs its own layer
(heads are independent problems), no collective on the data path; the only
collectives are the timing barrier and the max-over-ranks reduction.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import synth  # noqa: E402

METRIC = "ms/layer & effective TFLOPS (% bf16 peak) of top-p sparse attn, 32.7K tok"
UNIT = "TFLOP/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_BYTES = 126 * 2 ** 20


# ----------------------------------------------------------------------------- helpers

def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", str(rank)))
    return rank, world, local


def reduce_max(value: float, world: int, device=None) -> float:
    """Max over ranks (identity on one rank)."""
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def reduce_sum(value: float, world: int, device=None) -> float:
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


class ClockSampler:
    """nvidia-smi clock/throttle sampling during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = os.path.join("/tmp", f"svg_clocks_{os.getpid()}.csv")

    def __enter__(self):
        try:
            self.out = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "20"],
                                         stdout=self.out, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
            return self
        # the sampler must already be streaming when the timed region starts
        t0 = time.time()
        while time.time() - t0 < 5.0 and self.proc.poll() is None:
            if os.path.getsize(self.path) > 0:
                break
            time.sleep(0.02)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.out.close()

    def summary(self):
        if self.proc is None or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]), float(parts[3]), parts[4:]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        load = [r for r in rows if r[2] > 200.0] or rows
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in load for i, v in enumerate(r[3][1:5]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(r[0] for r in load), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(rows), "power_w_max": max(r[2] for r in rows)}


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        n = [d.get("num_threads", 0) for d in info if d.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


# ----------------------------------------------------------------------------- CPU oracle leg

# Heads of each workload the CPU oracle runs for its timed sample (about 10-30 s
# of host work at the box's core count); the value is scaled to the whole layer
# only through the metric (attention FLOPs per second), never extrapolated in time.
ORACLE_SAMPLE_HEADS = {"tiny": 1, "480p-5s": 8, "720p-5s": 2, "480p-10s": 2, "dense-d128": 1, "dense-d64": 1}


def oracle_sample(wl, heads: int):
    """Runs the oracle on the first `heads` heads; returns (seconds, attention FLOPs).

    For a warm-started workload the timed part is the second call, which starts
    from the oracle's own first-call centroids (the first call is not timed)."""
    from oracle import svg_oracle as so
    heads = min(heads, wl.heads)
    L = synth.make_layer(wl, heads=heads)
    D = L.q.shape[2]
    mu_q0, mu_k0 = L.init_centroids("q"), L.init_centroids("k")
    T = wl.iters
    if wl.warm_iters:
        first = [so.svg_head(L.q[h], L.k[h], L.v[h], mu_q0[h], mu_k0[h], wl.iters, wl.top_p[0], attention=False)
                 for h in range(heads)]
        mu_q0 = [r.mu_q for r in first]
        mu_k0 = [r.mu_k for r in first]
        L = synth.make_layer(wl, heads=heads, call=1)
        T = wl.warm_iters
    flops = 0.0
    t0 = time.perf_counter()
    for h in range(heads):
        r = so.svg_head(L.q[h], L.k[h], L.v[h], mu_q0[h], mu_k0[h], T, wl.top_p[0])
        pairs, _ = so.density(r.q_off, r.k_off, [s.cols for s in r.selection])
        flops += 4.0 * D * pairs
    return time.perf_counter() - t0, flops


def run_reference(args, wl):
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    heads = 1
    for _ in range(args.warmup):
        oracle_sample(wl, heads)
    secs, flops = 0.0, 0.0
    for _ in range(args.steps):
        s, f = oracle_sample(wl, heads)
        secs += s
        flops += f
    value = flops / secs / 1e12
    sample = f"{heads} of {wl.heads} heads of the {wl.name} layer per step, whole path (k-means, permute, select, attention)"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": secs / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(wl, args.gpus),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": blas_threads(), "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def workload_config(wl, n_gpus, heads=None, iters=None, top_p=None):
    heads = heads or wl.heads
    cfg = {"workload": wl.name, "heads": heads, "tokens": wl.tokens, "grid": list(wl.grid),
           "head_dim": wl.head_dim, "cq": wl.cq, "ck": wl.ck, "kmeans_iters": iters or wl.iters,
           "top_p": top_p if top_p is not None else wl.top_p[0],
            "layers_per_step_per_gpu": 1, "parallelism": f"dp{n_gpus} (independent layers per GPU)",
            "l2": "inputs larger than L2 (Q/K/V bf16 = %.0f MB > 126 MB); no flush" %
                  (3 * heads * wl.tokens * wl.head_dim * 2 / 1e6)}
    if wl.warm_iters:
        cfg["warm_start"] = ("timed call 1 starts from call 0's final centroids (the centroid cache) "
                             "and runs %d rounds" % wl.warm_iters)
    return cfg


# ----------------------------------------------------------------------------- GPU leg

def kernel_launches_per_step(iters: int, qk_fp8: bool = False, kv_gather: bool = False) -> int:
    """Our kernels per step (counted from the launch sequence in svg.cu)."""
    per_kmeans = 1 + 4 * iters               # split + T x (assign, refine, bucket, accumulate); ||x||^2 in the first assign
    per_permute = 3 + 1                      # hist, scan, scatter + row gather
    if qk_fp8:   # Q's permutation moves no rows; quantise Q per row, K per head (amax, quantise, scale)
        return 2 * per_kmeans + 2 * per_permute - 1 + 1 + 4 + 4
    if kv_gather:   # K's permutation moves no rows (attention gathers K/V through it)
        return 2 * per_kmeans + 2 * per_permute - 1 + 1 + 4
    return 2 * per_kmeans + 2 * per_permute + 1 + 4       # select; plan x3 + attention (un-permute fused)


def dynrad_launches_per_step(mode: str) -> int:
    """Kernels per DynamicRad step: the mask (offsets, [block means,] select) and the attention
    (plan merge, count, emit + the attention kernel)."""
    return (3 if mode == "dynamic" else 2) + 4


def attention_pairs(layer, wl):
    cnt = layer.sel_count.cpu().numpy()
    cols = layer.sel_cols.cpu().numpy()
    q_off = layer.q_off.cpu().numpy()
    k_off = layer.k_off.cpu().numpy()
    pairs = 0
    for h in range(cnt.shape[0]):
        nq = np.diff(q_off[h])
        nk = np.diff(k_off[h])
        for i in range(cnt.shape[1]):
            if cnt[h, i]:
                pairs += int(nq[i]) * int(nk[cols[h, i, :cnt[h, i]]].sum())
    return pairs


def pipelined_e2e(host_inputs, out_like, run_step, steps):
    """End-to-end timing with host buffers: every step copies its inputs from pinned host memory, runs
    `run_step(device_inputs, device_out, stream)` (which returns the tensor to copy back) and copies the
    result to pinned host memory, all inside the timed region.  Steps are pipelined over two device
    buffer sets and three streams: the H2D copies of step i + 1 and the D2H copy of step i - 1 run
    while step i computes (PCIe is full duplex).  Returns the elapsed milliseconds on this rank."""
    import torch
    device = out_like.device
    hout = [torch.empty(out_like.shape, dtype=out_like.dtype).pin_memory() for _ in range(2)]
    sets = [([torch.empty(h.shape, dtype=h.dtype, device=device) for h in host_inputs], torch.empty_like(out_like))
            for _ in range(2)]
    s_comp = torch.cuda.current_stream()
    s_h2d, s_d2h = torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(2)]      # inputs of set b have landed
    ev_comp = [torch.cuda.Event() for _ in range(2)]    # step on set b done (inputs free, output ready)
    ev_d2h = [torch.cuda.Event() for _ in range(2)]     # the output of set b has been copied back
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_comp)
    s_h2d.wait_event(e0)
    s_d2h.wait_event(e0)
    for i in range(steps):
        b = i % 2
        dins, dout = sets[b]
        with torch.cuda.stream(s_h2d):
            if i >= 2:
                s_h2d.wait_event(ev_comp[b])            # step i - 2 has consumed this set's inputs
            for d, h in zip(dins, host_inputs):
                d.copy_(h, non_blocking=True)
            ev_in[b].record(s_h2d)
        s_comp.wait_event(ev_in[b])
        if i >= 2:
            s_comp.wait_event(ev_d2h[b])                # step i - 2's output has left this set's buffer
        o = run_step(dins, dout, s_comp)
        ev_comp[b].record(s_comp)
        with torch.cuda.stream(s_d2h):
            s_d2h.wait_event(ev_comp[b])
            hout[b].copy_(o, non_blocking=True)
            ev_d2h[b].record(s_d2h)
    s_comp.wait_stream(s_h2d)
    s_comp.wait_stream(s_d2h)
    e1.record(s_comp)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1)


def run_svg(args, wl):
    import torch
    rank, world, local = dist_env()
    if world > 1:
        import torch.distributed as dist
        import datetime
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    else:
        torch.cuda.set_device(0)
    device = torch.device("cuda", torch.cuda.current_device())

    import sparse_attention_long_svg_b200 as svg
    svg.load_library()
    peaks, peak_kind = load_peaks()

    def to_dev(x):
        return torch.from_numpy(synth.bf16_bits(x).view(np.int16)).view(torch.bfloat16).to(device)

    p = args.top_p if args.top_p is not None else wl.top_p[0]
    T = wl.warm_iters or wl.iters            # k-means rounds of the timed call
    if wl.warm_iters:
        # centroid cache: call 0 (cold, wl.iters rounds) on this step's predecessor,
        # then the timed call 1 starts from its final centroids
        L0 = synth.make_layer(wl, heads=args.heads, call=0)
        BH, N, D = L0.q.shape
        layer0 = svg.SvgLayer(BH, N, D, wl.cq, wl.ck, device)
        cache_q = torch.from_numpy(L0.init_centroids("q")).to(device)
        cache_k = torch.from_numpy(L0.init_centroids("k")).to(device)
        layer0(to_dev(L0.q), to_dev(L0.k), to_dev(L0.v), cache_q, cache_k, wl.iters, p)
        torch.cuda.synchronize()
        del layer0, L0
        L = synth.make_layer(wl, heads=args.heads, call=1)
        mu_q0, mu_k0 = cache_q, cache_k
    else:
        L = synth.make_layer(wl, heads=args.heads)
        mu_q0 = torch.from_numpy(L.init_centroids("q")).to(device)
        mu_k0 = torch.from_numpy(L.init_centroids("k")).to(device)
    BH, N, D = L.q.shape
    q, k, v = to_dev(L.q), to_dev(L.k), to_dev(L.v)
    mu_q, mu_k = mu_q0.clone(), mu_k0.clone()
    layer = svg.SvgLayer(BH, N, D, wl.cq, wl.ck, device)
    out = torch.empty_like(q)
    stream = torch.cuda.current_stream()
    stage_names = ["kmeans_q", "kmeans_k", "permute", "select", "attn+unpermute"]
    if args.qk_fp8:
        if args.kv_gather:
            raise SystemExit("--qk-fp8 and --kv-gather cannot be combined")
        q8 = torch.empty((BH, N, D), dtype=torch.float8_e4m3fn, device=device)
        k8 = torch.empty_like(q8)
        sq = torch.empty((BH, N), dtype=torch.float32, device=device)
        sk = torch.empty((BH,), dtype=torch.float32, device=device)

    def step(ev=None):   # the un-permutation is fused into the attention kernel's store
        mu_q.copy_(mu_q0)
        mu_k.copy_(mu_k0)
        if ev:
            ev[0].record()
        svg.kmeans(q, mu_q, T, layer.assign_q, layer.n_q, layer.workspace)
        if ev:
            ev[1].record()
        svg.kmeans(k, mu_k, T, layer.assign_k, layer.n_k, layer.workspace)
        if ev:
            ev[2].record()
        if args.qk_fp8:          # Q and K are gathered by their quantisation; only V is moved
            svg.permute(layer.assign_q, wl.cq, [], [], layer.perm_q, layer.q_off, layer.workspace)
            svg.permute(layer.assign_k, wl.ck, [v], [layer.vp], layer.perm_k, layer.k_off, layer.workspace)
        else:
            svg.permute(layer.assign_q, wl.cq, [q], [layer.qp], layer.perm_q, layer.q_off, layer.workspace)
            if args.kv_gather:   # K permutation only: attention fetches K/V rows through it
                svg.permute(layer.assign_k, wl.ck, [], [], layer.perm_k, layer.k_off, layer.workspace)
            else:
                svg.permute(layer.assign_k, wl.ck, [k, v], [layer.kp, layer.vp], layer.perm_k, layer.k_off,
                            layer.workspace)
        if ev:
            ev[3].record()
        svg.select_topp(mu_q, layer.n_q, mu_k, layer.n_k, p, 0.0, layer.sel_count, layer.sel_cols)
        if ev:
            ev[4].record()
        if args.kv_gather:
            svg.sparse_attn_gather(layer.qp, k, v, layer.perm_k, layer.q_off, layer.k_off, layer.sel_count,
                                   layer.sel_cols, 0.0, out, workspace=layer.workspace, perm_q=layer.perm_q)
        elif args.qk_fp8:        # E4M3 Q (per row) and K (per head) gathered by the permutations, then attention
            svg.quantize_e4m3(q, True, q8, sq, perm=layer.perm_q)
            svg.quantize_e4m3(k, False, k8, sk, perm=layer.perm_k)
            svg.sparse_attn_fp8(q8, sq, k8, sk, layer.vp, layer.q_off, layer.k_off, layer.sel_count,
                                layer.sel_cols, 0.0, out, workspace=layer.workspace, perm_q=layer.perm_q)
        else:
            svg.sparse_attn(layer.qp, layer.kp, layer.vp, layer.q_off, layer.k_off, layer.sel_count,
                            layer.sel_cols, 0.0, out, workspace=layer.workspace, perm_q=layer.perm_q)
        if ev:
            ev[5].record()

    clocks = ClockSampler(device.index)
    clocks.__enter__()          # sampling starts with the warm-up so short runs still see load
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    err = svg.get_error_detail()
    if err[0] != 0:
        raise RuntimeError("device error word set during warm-up: status %d at %s, CTA %d" % err)

    events = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(args.steps)]
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    svg.profile_enable(True)             # live per-kernel CUDA-event timing of the two heavy kernels
    svg.profile_read("kmeans_assign")
    svg.profile_read("sparse_attn")
    svg.profile_attn_pairs()
    if True:
        t_start.record()
        for s in range(args.steps):
            step(events[s])
        t_end.record()
        torch.cuda.synchronize()
    assign_ms, assign_n, _ = svg.profile_read("kmeans_assign")
    attn_k_ms, attn_n, _ = svg.profile_read("sparse_attn")
    issued_pairs = svg.profile_attn_pairs()   # (128-row query tile, 128-key tile) pairs of the timed launches
    svg.profile_enable(False)
    if world > 1:
        torch.distributed.barrier()
    local_ms = t_start.elapsed_time(t_end)
    err = svg.get_error_detail()
    if err[0] != 0:
        raise RuntimeError("device error word set during the timed steps: status %d at %s, CTA %d" % err)
    stage_ms = {n: statistics.mean(events[s][i].elapsed_time(events[s][i + 1]) for s in range(args.steps))
                for i, n in enumerate(stage_names)}
    eager_ms = local_ms
    if args.graph:
        # the same layer step recorded once as a CUDA graph (centroid reset included) and replayed:
        # one host launch per step instead of ~55, so no launch gaps between the kernels
        graph = svg.LayerGraph(layer, q, k, v, mu_q0, mu_k0, T, p, 0.0, kv_gather=bool(args.kv_gather),
                               qk_fp8=bool(args.qk_fp8))
        for _ in range(args.warmup):
            graph.replay()
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize()
        g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        g0.record()
        for _ in range(args.steps):
            graph.replay()
        g1.record()
        torch.cuda.synchronize()
        if world > 1:
            torch.distributed.barrier()
        local_ms = g0.elapsed_time(g1)
        err = svg.get_error_detail()
        if err[0] != 0:
            raise RuntimeError("device error word set during the graph replays: status %d at %s, CTA %d" % err)
        del graph
    clocks.__exit__(None, None, None)   # the clock samples cover the eager and the graph-timed steps

    pairs = attention_pairs(layer, wl)
    flops_layer = 4.0 * D * pairs
    issued_flops = 4.0 * D * svg.ATTN_TILE * svg.ATTN_TILE * issued_pairs
    density = pairs / (BH * N * N)

    total_ms = reduce_max(local_ms, world, device)
    all_flops = reduce_sum(flops_layer * args.steps, world, device)
    value = all_flops / (total_ms * 1e-3) / 1e12

    # ---- end to end through the public API with host buffers (pinned), H2D + D2H inside the timed region
    e2e_steps = max(1, min(args.steps, 10))
    hq = torch.from_numpy(synth.bf16_bits(L.q).view(np.int16)).view(torch.bfloat16).pin_memory()
    hk = torch.from_numpy(synth.bf16_bits(L.k).view(np.int16)).view(torch.bfloat16).pin_memory()
    hv = torch.from_numpy(synth.bf16_bits(L.v).view(np.int16)).view(torch.bfloat16).pin_memory()
    hmq, hmk = mu_q0.cpu().pin_memory(), mu_k0.cpu().pin_memory()

    def e2e_step(d, o, stream):    # centroids d[3], d[4] are refilled from the host every step
        return layer(d[0], d[1], d[2], d[3], d[4], T, p, 0.0, o, stream=stream, kv_gather=bool(args.kv_gather),
                     qk_fp8=bool(args.qk_fp8))[0]
    if world > 1:
        torch.distributed.barrier()
    e2e_ms = reduce_max(pipelined_e2e([hq, hk, hv, hmq, hmk], q, e2e_step, e2e_steps), world, device)
    e2e_value = reduce_sum(flops_layer * e2e_steps, world, device) / (e2e_ms * 1e-3) / 1e12
    h2d = int(3 * hq.numel() * 2 + 2 * hmq.numel() * 4)
    d2h = int(q.numel() * 2)

    # ---- rooflines of the two heavy kernels, from the live event timings.  Each
    # launch is timed on its own (CUDA events around it, inside a timed region of
    # a fraction of a second), so the burst peak is the denominator; the
    # sustained (power-capped) peak is reported beside it.
    tc_peak = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    tc_sust = peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
    hbm_peak = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    attn_tflops = flops_layer / (stage_ms["attn+unpermute"] * 1e-3) / 1e12
    peak_note = (f"{peak_kind} bf16 burst (each launch timed on its own); "
                 f"{peak_kind} sustained {tc_sust:.0f} TFLOP/s reported as frac_of_sustained")
    attn_kernel_ms = attn_k_ms / max(attn_n, 1)
    attn_kernel_tflops = flops_layer / (attn_kernel_ms * 1e-3) / 1e12
    issued = issued_flops / max(attn_n, 1)
    attn_peak, attn_sust, attn_note, attn_name = tc_peak, tc_sust, peak_note, f"sparse_attn_kernel<{D}>"
    if args.qk_fp8:
        # half the FLOPs (S = Q K^T) at the E4M3 rate, half (P V) at the bf16 rate: with E4M3 at 2x bf16
        # (the nominal ratio, applied to the measured bf16 peak) the ideal time is 3/4 of all-bf16
        attn_peak, attn_sust = tc_peak * 4.0 / 3.0, tc_sust * 4.0 / 3.0
        attn_note = ("4/3 x the " + peak_note + " (Q K^T on E4M3 at 2x the bf16 rate, P V on bf16)")
        attn_name = f"sparse_attn_kernel<{D}, fp8 QK^T>"
    roof_attn = {"kernel": attn_name, "bound": "tensor", "achieved": attn_kernel_tflops,
                 "peak": attn_peak, "unit": "TFLOP/s", "frac": attn_kernel_tflops / attn_peak,
                 "frac_of_sustained": attn_kernel_tflops / attn_sust,
                 "frac_of_bf16_peak": attn_kernel_tflops / tc_peak,
                 "traffic": load_traffic("sparse_attn_kernel_fp8" if args.qk_fp8 else "sparse_attn_kernel", wl.name),
                 "peak_kind": attn_note,
                 "launch_ms": attn_kernel_ms, "launches": attn_n, "total_ms": attn_k_ms,
                 "algorithmic": "4*D*sum_selected(n_q*n_k) = %.4g FLOP per launch" % flops_layer,
                 "mma_issued_flop_per_launch": issued,
                 "mma_issued_tflops": issued / (attn_kernel_ms * 1e-3) / 1e12 if issued else None,
                 "padding_waste": 1.0 - flops_layer / issued if issued else None}
    # assign launches alternate: iters on Q (C = cq) then iters on K (C = ck) per step
    assign_flops = 2.0 * N * D * BH * T * (wl.cq + wl.ck) * args.steps
    assign_launch_ms = assign_ms / max(assign_n, 1)
    assign_tflops = assign_flops / (assign_ms * 1e-3) / 1e12 if assign_ms > 0 else 0.0
    roof_assign = {"kernel": f"kmeans_assign_tc_kernel<{D}>", "bound": "tensor", "achieved": assign_tflops,
                   "peak": tc_peak, "unit": "TFLOP/s", "frac": assign_tflops / tc_peak,
                   "frac_of_sustained": assign_tflops / tc_sust,
                   "traffic": load_traffic("kmeans_assign_tc_kernel", wl.name), "peak_kind": peak_note,
                   "launch_ms": assign_launch_ms, "launches": assign_n, "total_ms": assign_ms,
                   "algorithmic": "2*N*C*D*BH FLOP per launch (distance contraction; C = %d or %d)"
                                  % (wl.cq, wl.ck)}
    if assign_ms > attn_k_ms:
        roofline, roofline_other = roof_assign, roof_attn
    else:
        roofline, roofline_other = roof_attn, roof_assign
    tensor_bytes = BH * N * D * 2
    km_flops = {c: 2.0 * N * c * D * BH * T for c in (wl.cq, wl.ck)}
    km_bytes = 2.0 * tensor_bytes * T                 # assign read + update read per round
    stages = {
        "kmeans_q": {"ms": stage_ms["kmeans_q"], "tflops": km_flops[wl.cq] / stage_ms["kmeans_q"] / 1e9,
                     "gbs": km_bytes / stage_ms["kmeans_q"] / 1e6},
        "kmeans_k": {"ms": stage_ms["kmeans_k"], "tflops": km_flops[wl.ck] / stage_ms["kmeans_k"] / 1e9,
                     "gbs": km_bytes / stage_ms["kmeans_k"] / 1e6},
        "permute": {"ms": stage_ms["permute"], "gbs": 6.0 * tensor_bytes / stage_ms["permute"] / 1e6},
        "select": {"ms": stage_ms["select"]},
        "attn+unpermute": {"ms": stage_ms["attn+unpermute"], "tflops": attn_tflops,
                           "note": "un-permutation fused into the attention kernel's store"},
    }
    for sname in ("kmeans_q", "kmeans_k", "permute"):
        stages[sname]["hbm_frac"] = stages[sname]["gbs"] / hbm_peak
    for sname in ("kmeans_q", "kmeans_k", "attn+unpermute"):
        stages[sname]["tensor_frac"] = stages[sname]["tflops"] / tc_peak
    stages["hbm_peak_gbs"] = hbm_peak
    stages["tensor_peak_tflops"] = tc_peak

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        nh = min(ORACLE_SAMPLE_HEADS.get(wl.name, 1), wl.heads)
        secs, fl = oracle_sample(wl, nh)
        cpu = {"value": fl / secs / 1e12, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
               "sample": f"{nh} of {wl.heads} heads of the {wl.name} layer, whole path, {secs:.1f} s"}

    if world > 1:
        torch.distributed.barrier()
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "e4m3 QK^T, bf16 PV" if args.qk_fp8 else "bf16",
            "data": "synthetic",
            "config": dict(workload_config(wl, world, BH, T, p),
                           kv=("gathered by the attention kernel through the K permutation" if args.kv_gather
                               else "permuted copies written by svg_permute"),
                           **({"qk": "E4M3 Q (per-row scales) and K (per-head scales), quantised each step while "
                                     "gathered into permuted order"}
                              if args.qk_fp8 else {})),
            "attn_ms": stage_ms["attn+unpermute"], "attn_eff_tflops": attn_tflops,
            "attn_frac_of_bf16_peak": attn_tflops / tc_peak, "density": density, "stages": stages,
            "roofline": roofline, "roofline_other": roofline_other, "cpu_baseline": cpu,
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "ms_per_step": e2e_ms / e2e_steps, "steps": e2e_steps,
                    "pipelining": "H2D of step i+1 and D2H of step i-1 overlap the layer of step i "
                                  "(two device buffer sets, three streams)"},
            "gpu_launches": kernel_launches_per_step(T, bool(args.qk_fp8), bool(args.kv_gather)) * args.steps,
            "clocks": clocks.summary(),
            "timing": ("CUDA-graph replays of the whole step (stages and per-kernel rooflines from eager steps "
                       "with events; eager %.3f ms per step)" % (eager_ms / args.steps)) if args.graph else
                      "eager launches",
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()
    return 0


# DynamicRad settings of the --mask dynrad-* legs (block of 256 tokens: two query
# tiles per block; static density about 18 % and dynamic about 6 % on 480p-5s).
DYNRAD = {"block": 256, "w0": 3.0, "gamma": 0.5, "rho0": 0.5, "theta": 1.0}


def dynrad_oracle_sample(wl, heads: int, mode: str):
    """The DynamicRad oracle (mask + attention) on the first `heads` heads: (seconds, attention FLOPs)."""
    from oracle import dynrad_oracle as dr
    L = synth.make_layer(wl, heads=heads)
    H, N, D = L.q.shape
    frames = wl.grid[0]
    c = {k: float(np.float32(v)) for k, v in DYNRAD.items() if k != "block"}
    t0 = time.perf_counter()
    flops = 0.0
    for h in range(H):
        offs, nb = dr.block_layout(N, frames, DYNRAD["block"])
        if mode == "static":
            sel = dr.static_select(frames, nb, c["w0"], c["gamma"], c["rho0"])
        else:
            sel = [r.cols for r in dr.dynamic_select(L.q[h], L.k[h], offs, frames, nb, c["w0"], c["gamma"],
                                                    c["theta"], 1.0 / math.sqrt(D))]
        dr.attention(L.q[h], L.k[h], L.v[h], offs, sel, 1.0 / math.sqrt(D))
        flops += 4.0 * D * dr.density(offs, sel)[0]
    return time.perf_counter() - t0, flops


def run_dynrad(args, wl):
    """The DynamicRad workload on the same attention kernel: block masks (svg_dynrad_select) + attention
    on Q, K, V in token order.  Same metric and timing rules as the SVG2 leg."""
    import torch
    rank, world, local = dist_env()
    if world > 1:
        import torch.distributed as dist
        import datetime
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    else:
        torch.cuda.set_device(0)
    device = torch.device("cuda", torch.cuda.current_device())
    import sparse_attention_long_svg_b200 as svg
    svg.load_library()
    peaks, peak_kind = load_peaks()
    mode = args.mask.split("-", 1)[1]
    L = synth.make_layer(wl, heads=args.heads)
    BH, N, D = L.q.shape
    frames, B = wl.grid[0], DYNRAD["block"]

    def to_dev(x):
        return torch.from_numpy(synth.bf16_bits(x).view(np.int16)).view(torch.bfloat16).to(device)
    q, k, v = to_dev(L.q), to_dev(L.k), to_dev(L.v)
    lib = svg.load_library()
    Cb = lib.svg_dynrad_num_blocks(N, frames, B)
    i32 = dict(dtype=torch.int32, device=device)
    offs, cnt, cols = torch.empty((BH, Cb + 1), **i32), torch.empty((BH, Cb), **i32), torch.empty((BH, Cb, Cb), **i32)
    ws = torch.empty(max(lib.svg_dynrad_workspace_size(BH, N, D, frames, B),
                         lib.svg_sparse_attn_workspace_size(BH, N, Cb), 256), dtype=torch.uint8, device=device)
    out = torch.empty_like(q)
    prm = dict(w0=DYNRAD["w0"], gamma=DYNRAD["gamma"], rho0=DYNRAD["rho0"], theta=DYNRAD["theta"])

    def step(qq, kk, vv, ev=None):
        if ev:
            ev[0].record()
        svg.dynrad_select(qq, kk, frames, B, mode, offsets=offs, sel_count=cnt, sel_cols=cols, workspace=ws, **prm)
        if ev:
            ev[1].record()
        svg.sparse_attn(qq, kk, vv, offs, offs, cnt, cols, 0.0, out, workspace=ws)
        if ev:
            ev[2].record()

    clocks = ClockSampler(device.index)
    clocks.__enter__()
    for _ in range(args.warmup):
        step(q, k, v)
    torch.cuda.synchronize()
    err = svg.get_error_detail()
    if err[0] != 0:
        raise RuntimeError("device error word set during warm-up: status %d at %s, CTA %d" % err)
    events = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    svg.profile_enable(True)
    svg.profile_read("sparse_attn")
    svg.profile_attn_pairs()
    t_start.record()
    for s in range(args.steps):
        step(q, k, v, events[s])
    t_end.record()
    torch.cuda.synchronize()
    clocks.__exit__(None, None, None)
    attn_k_ms, attn_n, _ = svg.profile_read("sparse_attn")
    issued_pairs = svg.profile_attn_pairs()
    svg.profile_enable(False)
    if world > 1:
        torch.distributed.barrier()
    local_ms = t_start.elapsed_time(t_end)
    err = svg.get_error_detail()
    if err[0] != 0:
        raise RuntimeError("device error word set during the timed steps: status %d at %s, CTA %d" % err)
    mask_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in events)
    attn_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in events)
    o_h, c_h, s_h = offs.cpu().numpy(), cnt.cpu().numpy(), cols.cpu().numpy()
    pairs = 0
    for h in range(BH):
        nb_sizes = np.diff(o_h[h])
        for i in range(Cb):
            pairs += int(nb_sizes[i]) * int(nb_sizes[s_h[h, i, :c_h[h, i]]].sum())
    flops_layer = 4.0 * D * pairs
    total_ms = reduce_max(local_ms, world, device)
    value = reduce_sum(flops_layer * args.steps, world, device) / (total_ms * 1e-3) / 1e12

    e2e_steps = max(1, min(args.steps, 10))
    hq, hk, hv = (torch.from_numpy(synth.bf16_bits(x).view(np.int16)).view(torch.bfloat16).pin_memory()
                  for x in (L.q, L.k, L.v))

    def e2e_step(d, o, stream):
        with torch.cuda.stream(stream):
            svg.dynrad_select(d[0], d[1], frames, B, mode, offsets=offs, sel_count=cnt, sel_cols=cols, workspace=ws,
                              **prm)
            svg.sparse_attn(d[0], d[1], d[2], offs, offs, cnt, cols, 0.0, o, workspace=ws)
        return o
    e2e_ms = reduce_max(pipelined_e2e([hq, hk, hv], q, e2e_step, e2e_steps), world, device)
    e2e_value = reduce_sum(flops_layer * e2e_steps, world, device) / (e2e_ms * 1e-3) / 1e12

    tc_peak = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    tc_sust = peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
    attn_kernel_ms = attn_k_ms / max(attn_n, 1)
    attn_kernel_tflops = flops_layer / (attn_kernel_ms * 1e-3) / 1e12
    issued = 4.0 * D * svg.ATTN_TILE * svg.ATTN_TILE * issued_pairs / max(attn_n, 1)
    roofline = {"kernel": f"sparse_attn_kernel<{D}>", "bound": "tensor", "achieved": attn_kernel_tflops,
                "peak": tc_peak, "unit": "TFLOP/s", "frac": attn_kernel_tflops / tc_peak,
                "frac_of_sustained": attn_kernel_tflops / tc_sust, "traffic": None,
                "peak_kind": f"{peak_kind} bf16 burst (each launch timed on its own)",
                "launch_ms": attn_kernel_ms, "launches": attn_n,
                "algorithmic": "4*D*sum_selected(n_q*n_k) = %.4g FLOP per launch" % flops_layer,
                "mma_issued_flop_per_launch": issued,
                "padding_waste": 1.0 - flops_layer / issued if issued else None}
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        secs, fl = dynrad_oracle_sample(wl, 1, mode)
        cpu = {"value": fl / secs / 1e12, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
               "sample": f"1 of {wl.heads} heads of the {wl.name} layer, DynamicRad {mode} mask + attention, "
                         f"{secs:.1f} s"}
    if world > 1:
        torch.distributed.barrier()
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": dict({kk: vv for kk, vv in workload_config(wl, world, BH).items()
                            if kk not in ("kmeans_iters", "top_p", "cq", "ck")},
                           mask=f"DynamicRad {mode}", frames=frames, blocks=Cb, **DYNRAD),
            "attn_ms": attn_ms, "attn_eff_tflops": flops_layer / (attn_ms * 1e-3) / 1e12,
            "density": pairs / (BH * N * N),
            "stages": {"mask": {"ms": mask_ms}, "attn": {"ms": attn_ms}},
            "roofline": roofline, "cpu_baseline": cpu,
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": int(3 * hq.numel() * 2),
                    "d2h_bytes_per_step": int(q.numel() * 2), "ms_per_step": e2e_ms / e2e_steps,
                    "steps": e2e_steps, "pipelining": "H2D of step i+1 and D2H of step i-1 overlap step i "
                                                      "(two device buffer sets, three streams)"},
            "gpu_launches": dynrad_launches_per_step(mode) * args.steps,
            "clocks": clocks.summary(),
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()
    return 0


def load_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from a committed ncu capture, if it matches the current source."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    entry = d.get(kernel, {}).get(workload)
    if not entry:
        return None
    from sparse_attention_long_svg_b200 import build
    if entry.get("source_hash") != build.source_hash(kernel):
        return None
    return entry.get("dram_bytes_per_launch")


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="480p-5s", choices=sorted(synth.WORKLOADS))
    ap.add_argument("--impl", default="svg", choices=["svg", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--top-p", type=float, default=None, help="override the workload's (first) top-p")
    ap.add_argument("--graph", type=int, default=1, choices=[0, 1],
                    help="1: time CUDA-graph replays of the whole layer step (0: eager launches)")
    ap.add_argument("--kv-gather", type=int, default=0, choices=[0, 1],
                    help="1: no permuted K/V copies; the attention kernel gathers K/V rows through the K permutation")
    ap.add_argument("--qk-fp8", type=int, default=0, choices=[0, 1],
                    help="1: Q and K quantised to E4M3 after the permutation; S = Q K^T on 8-bit tensor cores")
    ap.add_argument("--mask", default="svg2", choices=["svg2", "dynrad-static", "dynrad-dynamic"],
                    help="block masks: SVG2 (k-means + top-p, the headline) or DynamicRad's two modes")
    ap.add_argument("--heads", type=int, default=None,
                    help="first H heads of the workload only (smaller case for profiler captures)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    wl = synth.WORKLOADS[args.workload]
    if args.impl == "reference":
        return run_reference(args, wl)
    if args.mask != "svg2":
        return run_dynrad(args, wl)
    return run_svg(args, wl)


if __name__ == "__main__":
    sys.exit(main())
