"""Benchmark of the SSA sparse stream on B200 (one JSON line on rank 0).

A step is one pass of the sparse-stream forward over one batch of the
workload: ssa_block_pool -> ssa_block_select -> ssa_sparse_attn_fwd, with the
inputs already resident in HBM.  The metric is TFLOP/s over the selected
blocks: 4 * D FLOPs per unmasked (query, key) pair of the selected blocks
(QK^T and PV), summed over batch and query heads, per second.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
    python bench.py --impl reference ...     # the fp64 CPU oracle on host cores

Under torchrun (N > 1) every rank runs its own replica of the workload (the
path has no exchange step; units are independent), the timed region is
bracketed by barriers, and the time is the max over ranks.
"""
from __future__ import annotations

import argparse
import dataclasses
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import gen  # noqa: E402

METRIC = "sparse attn fwd TFLOP/s (selected blocks) and % of B200 BF16 peak at 8k/32k"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_FLUSH_BYTES = 256 << 20


def selected_pairs(workload) -> int:
    """Unmasked (query, key) pairs of the selected blocks for one (b, query head)
    summed over query blocks; selection always holds min(k, i + 1) blocks, the
    diagonal one causally masked (64 * 65 / 2 pairs), the others full (64 * 64)."""
    n, k = workload.n_blocks, workload.top_k
    total = 0
    for i in range(n):
        m = min(k, i + 1)
        total += (m - 1) * 64 * 64 + 64 * 65 // 2
    return total


def algorithmic_flops(workload) -> float:
    w = workload
    return 4.0 * w.head_dim * selected_pairs(w) * w.batch * w.n_q_heads


def causal_flops(workload) -> float:
    """FLOPs of dense causal attention (the alignment pass's full stream):
    4 D per unmasked (query, key) pair over all causal blocks."""
    w = workload
    n = w.n_blocks
    pairs = n * (n - 1) // 2 * 64 * 64 + n * (64 * 65 // 2)
    return 4.0 * w.head_dim * pairs * w.batch * w.n_q_heads


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled while the timed loop runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap,"
              "utilization.gpu")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.out = ""
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.out, _ = self.proc.communicate()
        return False

    def summary(self):
        """Median SM clock over the samples taken under load (GPU utilisation
        of at least 50% in the sample period; all samples if none is), the
        throttle reasons seen in those samples, and the sample counts."""
        rows = []
        for line in (self.out or "").strip().splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 10:
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]), parts[5:9], float(parts[9])))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        loaded = [r for r in rows if r[3] >= 50.0] or rows
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, _, flags, _ in loaded for i, f in enumerate(flags)
                          if f.lower() == "active"})
        return {"sm_mhz": statistics.median(r[0] for r in loaded), "sm_max_mhz": rows[0][1],
                "reasons": reasons, "samples": len(rows), "samples_under_load": len(loaded),
                "window": "warm-up, timed steps, kernel-alone timings and the other workloads"}


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def dist_max(value: float, world: int) -> float:
    if world == 1:
        return value
    import torch.distributed as dist
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def dist_barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def check_device(where: str) -> None:
    """Raise if a kernel reported a device-side error (a bounded wait that
    expired), naming the wait site the library recorded."""
    import block_sparse_attention_21_b200 as ssa
    err = ssa.ssa_get_device_error()
    if err != 0:
        raise RuntimeError(f"device error {err} after the {where}, wait site "
                           f"{hex(ssa.ssa_get_device_error_site())}")


def config_of(w, l2: str):
    return {"workload": w.name, "batch": w.batch, "seq_len": w.seq_len, "n_q_heads": w.n_q_heads,
            "n_kv_heads": w.n_kv_heads, "head_dim": w.head_dim, "block_size": 64,
            "top_k": w.top_k, "causal": True, "between_steps": l2}


# ------------------------------------------------------------------ our arm

def run_ours(args, world, rank, local):
    import block_sparse_attention_21_b200 as ssa
    from block_sparse_attention_21_b200 import build as ssa_build
    ssa_build.build()
    dev = torch.device("cuda", torch.cuda.current_device())
    x = gen.make_inputs(args.workload)
    w = x.workload
    p = ssa.problem(w.batch, w.seq_len, w.n_q_heads, w.n_kv_heads, w.head_dim, w.top_k)
    q, k, v = (t.to(dev) for t in (x.q, x.k, x.v))
    st = ssa.SparseStream(p, dev)
    stream = torch.cuda.current_stream()
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    flush_sink = torch.empty((), dtype=torch.int64, device=dev)

    def flush_l2(s):
        # write a buffer twice the L2 size, then read it back: L2 is left
        # holding clean lines, so no write-back of the flush is charged to the
        # timed kernels
        flush.fill_(s & 0xFF)
        torch.sum(flush.view(torch.int64), dim=0, out=flush_sink)
    flops = algorithmic_flops(w)

    # the step as one CUDA graph (pool, select, sparse attention), and the
    # sparse-attention kernel alone for its roofline
    n0 = ssa.ssa_launch_count()
    g_step = st.capture_forward(q, k, v)
    launches_per_step = (ssa.ssa_launch_count() - n0) // 2   # warm call + captured call
    g_fwd = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_fwd):
        ssa.ssa_sparse_attn_fwd(p, q, k, v, st.block_idx, st.o, st.lse)
    g_pool = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_pool):
        ssa.ssa_block_pool(p, k, q, st.k_pooled, st.q_pooled)
    g_sel = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_sel):
        ssa.ssa_block_select(p, st.q_pooled, st.k_pooled, st.block_idx)

    def timed(graph, n):
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(n)]
        for s in range(n):
            flush_l2(s)                    # L2 flushed between steps, outside the timed span
            evs[s][0].record(stream)
            graph.replay()
            evs[s][1].record(stream)
        torch.cuda.synchronize()
        return sum(a.elapsed_time(b) for a, b in evs)

    def reps_for(graph, seconds):
        """Repetitions of graph (with its L2 flush) that take about `seconds`."""
        t0 = time.perf_counter()
        timed(graph, 10)
        per = (time.perf_counter() - t0) / 10
        return int(min(max(seconds / max(per, 1e-6), 20), 20000))

    # the clock sampler spans the warm-up, the timed steps, the kernel-alone
    # timings and the other workloads, so that it holds samples under load
    # even when the timed steps alone last milliseconds
    clk = ClockSampler(local)
    clk.__enter__()
    try:
        for _ in range(args.warmup):
            flush_l2(1)
            g_step.replay()
        torch.cuda.synchronize()
        dist_barrier(world)
        torch.cuda.synchronize()
        step_ms = timed(g_step, args.steps)
        dist_barrier(world)
        launches = launches_per_step * args.steps
        n_k = max(args.steps // 4, 20)
        n_fwd = reps_for(g_fwd, 1.0)       # about one second of kernel-alone launches
        fwd_ms = timed(g_fwd, n_fwd) / n_fwd
        pool_ms = timed(g_pool, n_k) / n_k
        sel_ms = timed(g_sel, n_k) / n_k
        total_ms = dist_max(step_ms, world)
        ms_per_step = total_ms / args.steps
        value = flops * world / (ms_per_step * 1e-3) / 1e12

        # end to end through the public API on host buffers: ssa_sparse_attn_fwd_host
        # copies the pinned Q, K, V in, pools, selects and attends, and copies O
        # and LSE back, pipelined by (batch, KV head) so both copy directions and
        # the kernels overlap
        hq, hk, hv = (t.contiguous().pin_memory() for t in (x.q, x.k, x.v))
        ho = torch.empty(st.o.shape, dtype=st.o.dtype).pin_memory()
        hl = torch.empty(st.lse.shape, dtype=st.lse.dtype).pin_memory()
        e2e_steps = max(1, min(args.steps, 200))

        def e2e_step():
            st.forward_host(hq, hk, hv, ho, hl)

        for _ in range(2):
            e2e_step()
        torch.cuda.synchronize()
        dist_barrier(world)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(e2e_steps):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize()
        e2e_ms = dist_max(e0.elapsed_time(e1), world) / e2e_steps
        h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv))
        d2h = ho.numel() * ho.element_size() + hl.numel() * hl.element_size()

        # the other rows of the path on the same workload, outside the step: the
        # alignment pass (dense causal attention, counterpart sparse output and
        # dropped mass in one launch) and the sparse backward with a seeded dO
        of, lsef, dmass = torch.empty_like(st.o), torch.empty_like(st.lse), torch.empty_like(st.lse)
        ssa.ssa_full_attn_fwd_with_mass(p, q, k, v, st.block_idx, st.o, st.lse, of, lsef, dmass)
        g_mass = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_mass):
            ssa.ssa_full_attn_fwd_with_mass(p, q, k, v, st.block_idx, st.o, st.lse, of, lsef, dmass)
        g_step.replay()
        gen_do = torch.Generator().manual_seed(7)
        d_o = torch.randn(st.o.shape, generator=gen_do).to(torch.bfloat16).to(dev)
        st.backward(q, k, v, d_o)
        g_bwd = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_bwd):
            st.backward(q, k, v, d_o)
        # the alignment objective's backward (mode 0: d_o belongs to the sparse output)
        st.alignment(q, k, v)
        st.alignment_backward(q, k, v, d_o, 0, 1.0)
        g_abwd = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_abwd):
            st.alignment_backward(q, k, v, d_o, 0, 1.0)
        mass_ms = timed(g_mass, n_k) / n_k
        bwd_ms = timed(g_bwd, n_k) / n_k
        abwd_ms = timed(g_abwd, n_k) / n_k
        torch.cuda.synchronize()
        check_device("timed rows")

        decode = decode_rows(dev, timed)
        dash = dash_rows(p, w, q, k, v, timed, n_k)
        early = early_rows(p, w, st, q, k, v, timed, n_k, fwd_ms)
        del of, lsef, dmass, d_o, g_mass, g_bwd, g_abwd
        st._grad = st._agrad = st._full = None
        torch.cuda.empty_cache()

        # the other workloads on their own shapes: 32k with the top-k sweep
        # against dense causal attention, the batch-2 alignment pass and the
        # batch-4 forward + backward
        others = {} if args.no_other_workloads else workload_rows(dev, timed, reps_for)
    finally:
        clk.__exit__(None, None, None)
    clocks = clk.summary()

    peaks, peak_src = load_peaks()
    peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    achieved = flops / (fwd_ms * 1e-3) / 1e12
    traffic = load_traffic(w.name)
    rec = {
        "metric": METRIC, "value": round(value, 3), "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic", "config": config_of(w, "l2_flushed"),
        "e2e": {"value": round(flops * world / (e2e_ms * 1e-3) / 1e12, 3), "unit": "TFLOP/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": round(e2e_ms, 4)},
        "roofline": {"bound": "tensor", "achieved": round(achieved, 2), "peak": peak,
                     "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                     "traffic": traffic, "kernel": "attn_fwd_kernel (ssa_sparse_attn_fwd)",
                     "peak_source": f"{peak_src} bf16_tflops (burst)",
                     "kernel_ms": round(fwd_ms, 5), "kernel_reps": n_fwd,
                     "kernel_kcycles_at_median_clock": (round(fwd_ms * clocks["sm_mhz"], 2)
                                                        if clocks.get("sm_mhz") else None)},
        "kernels_ms": {"block_pool": round(pool_ms, 5), "block_select": round(sel_ms, 5),
                       "sparse_attn_fwd": round(fwd_ms, 5)},
        "other_rows": {
            "full_attn_fwd_with_mass": {
                "ms": round(mass_ms, 5), "flops": "4 D per causal (query, key) pair",
                "tflops": round(causal_flops(w) / (mass_ms * 1e-3) / 1e12, 2)},
            "sparse_attn_bwd": {
                "ms": round(bwd_ms, 5), "flops": "10 D per selected (query, key) pair",
                "tflops": round(2.5 * flops / (bwd_ms * 1e-3) / 1e12, 2)},
            "alignment_bwd": {
                "ms": round(abwd_ms, 5),
                "flops": "10 D per selected pair (sparse stream) + 10 D per causal pair (full stream)",
                "tflops": round(2.5 * (flops + causal_flops(w)) / (abwd_ms * 1e-3) / 1e12, 2)},
            "decode": decode,
            "sparse_attn_fwd_early_stop": early,
            "dash_attention": dash},
        "workloads": others,
        "gpu_launches": int(launches),
        "clocks": clocks,
        "pct_of_peak_step": round(100.0 * value / world / peak, 2),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rec["cpu_baseline"] = cpu_baseline(x)
    return rec


def early_rows(p, w, st, q, k, v, timed_fn, n_k, fwd_ms):
    """The early-stop variant of the sparse forward on the bench inputs and
    table at tau = 0, 0.1, 0.2, 0.5: time, and blocks visited per query head
    and query block against the blocks selected."""
    import block_sparse_attention_21_b200 as ssa
    dev = q.device
    early = {}
    vis = torch.empty(w.batch, w.n_q_heads, w.n_blocks, dtype=torch.int32, device=dev)
    st.forward(q, k, v)
    nsel_mean = float((st.block_idx >= 0).sum(dim=-1).float().mean())
    for tau in (0.0, 0.1, 0.2, 0.5):
        ssa.ssa_sparse_attn_fwd_early_stop(p, q, k, v, st.q_pooled, st.k_pooled, st.block_idx, tau,
                                           st.o, st.lse, vis)
        g_es = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_es):
            ssa.ssa_sparse_attn_fwd_early_stop(p, q, k, v, st.q_pooled, st.k_pooled, st.block_idx, tau,
                                               st.o, st.lse, vis)
        es_ms = timed_fn(g_es, n_k) / n_k
        torch.cuda.synchronize()
        check_device("early-stop rows")
        early[f"tau_{tau:g}"] = {"ms": round(es_ms, 5), "blocks_visited_mean": round(float(vis.float().mean()), 3),
                                 "blocks_selected_mean": round(nsel_mean, 3),
                                 "speedup_vs_sparse_fwd": round(fwd_ms / es_ms, 3)}
    st.forward(q, k, v)
    return early


def workload_rows(dev, timed_fn, reps_for):
    """The sparse forward and the other rows on the other workloads' own shapes.

    long_32k (B 1, S 32768, Hq 16, Hkv 2, D 128): the step (pool, select,
    forward) and the forward alone with its own roofline, then the forward
    alone at top-k 8, 16, 32, 64, 128 and at top-k = every block (dense causal
    attention through the same kernel), each on its own selection; the
    crossover is the smallest budget whose time reaches the dense one, or, when
    none does, the budget where the line through the two largest budgets'
    times meets it.  torch's scaled_dot_product_attention (causal, the K/V
    heads repeated per group) is timed beside it as an outside reference.
    align_8k (B 2): the alignment pass, dense causal FLOPs.  train_8k (B 4):
    the forward step and the sparse backward, and their sum."""
    import block_sparse_attention_21_b200 as ssa
    peaks, peak_src = load_peaks()
    peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    out = {}

    # ---------------------------------------------------------------- 32k
    x = gen.make_inputs("long_32k")
    w = x.workload
    q, k, v = (t.to(dev) for t in (x.q, x.k, x.v))
    p = ssa.problem(w.batch, w.seq_len, w.n_q_heads, w.n_kv_heads, w.head_dim, w.top_k)
    st = ssa.SparseStream(p, dev)
    g_step = st.capture_forward(q, k, v)
    g_fwd = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_fwd):
        ssa.ssa_sparse_attn_fwd(p, q, k, v, st.block_idx, st.o, st.lse)
    n_step = 40
    step_ms = timed_fn(g_step, n_step) / n_step
    n_fwd = reps_for(g_fwd, 1.0)
    fwd_ms = timed_fn(g_fwd, n_fwd) / n_fwd
    check_device("32k forward")
    flops = algorithmic_flops(w)
    achieved = flops / (fwd_ms * 1e-3) / 1e12
    row = {"config": config_of(w, "l2_flushed"), "ms_per_step": round(step_ms, 5),
           "step_tflops": round(flops / (step_ms * 1e-3) / 1e12, 2),
           "roofline": {"bound": "tensor", "achieved": round(achieved, 2), "peak": peak,
                        "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                        "traffic": load_traffic(w.name),
                        "kernel": "attn_fwd_psmem_kernel (ssa_sparse_attn_fwd)",
                        "peak_source": f"{peak_src} bf16_tflops (burst)",
                        "kernel_ms": round(fwd_ms, 5), "kernel_reps": n_fwd}}
    del g_step, g_fwd
    # the budget sweep, each budget on its own selection, into shared outputs
    sweep = {}
    n = w.n_blocks
    for kk in (8, 16, 32, 64, 128, n):
        pk = ssa.problem(w.batch, w.seq_len, w.n_q_heads, w.n_kv_heads, w.head_dim, kk)
        idx = torch.empty(w.batch, w.n_kv_heads, n, kk, dtype=torch.int32, device=dev)
        ssa.ssa_block_select(pk, st.q_pooled, st.k_pooled, idx)
        ssa.ssa_sparse_attn_fwd(pk, q, k, v, idx, st.o, st.lse)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            ssa.ssa_sparse_attn_fwd(pk, q, k, v, idx, st.o, st.lse)
        reps = 30 if kk >= 64 else 60
        ms = timed_fn(g, reps) / reps
        check_device(f"32k sweep top-k {kk}")
        wk = dataclasses.replace(w, top_k=kk)
        fk = algorithmic_flops(wk)
        sweep["dense_causal" if kk == n else f"top_k_{kk}"] = {
            "top_k": kk, "ms": round(ms, 5), "flops": fk, "tflops": round(fk / (ms * 1e-3) / 1e12, 2),
            "frac": round(fk / (ms * 1e-3) / 1e12 / peak, 4)}
        del g, idx
    dense_ms = sweep["dense_causal"]["ms"]
    ks = [8, 16, 32, 64, 128]
    for kk in ks:
        sweep[f"top_k_{kk}"]["speedup_vs_dense"] = round(dense_ms / sweep[f"top_k_{kk}"]["ms"], 3)
    reached = [kk for kk in ks if sweep[f"top_k_{kk}"]["ms"] >= dense_ms]
    if reached:
        cross = {"top_k": reached[0], "how": "measured: the smallest budget at least as slow as dense"}
    else:
        t1, t2 = sweep["top_k_64"]["ms"], sweep["top_k_128"]["ms"]
        slope = (t2 - t1) / 64.0
        est = 128 + (dense_ms - t2) / slope if slope > 0 else None
        cross = {"top_k": (round(est, 1) if est is not None else None), "blocks": n,
                 "how": "extrapolated: the line through top-k 64 and 128 meets the dense time"}
    sweep["crossover"] = cross
    # torch SDPA, dense causal, as an outside reference point only
    try:
        G = w.n_q_heads // w.n_kv_heads
        qt = q.transpose(1, 2).contiguous()
        kt = k.transpose(1, 2).repeat_interleave(G, dim=1).contiguous()
        vt = v.transpose(1, 2).repeat_interleave(G, dim=1).contiguous()
        F = torch.nn.functional
        F.scaled_dot_product_attention(qt, kt, vt, is_causal=True)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            F.scaled_dot_product_attention(qt, kt, vt, is_causal=True)
        ms = timed_fn(g, 20) / 20
        fc = causal_flops(w)
        sweep["torch_sdpa_dense_causal"] = {"ms": round(ms, 5), "tflops": round(fc / (ms * 1e-3) / 1e12, 2),
                                            "note": "library kernel, outside reference only"}
        del qt, kt, vt, g
    except Exception as e:  # a comparison point only; the sweep stands without it
        sweep["torch_sdpa_dense_causal"] = {"unavailable": str(e)[:200]}
    row["top_k_sweep"] = sweep
    out["long_32k"] = row
    del q, k, v, st
    torch.cuda.empty_cache()

    # ---------------------------------------------------------------- align_8k
    x = gen.make_inputs("align_8k")
    w = x.workload
    q, k, v = (t.to(dev) for t in (x.q, x.k, x.v))
    p = ssa.problem(w.batch, w.seq_len, w.n_q_heads, w.n_kv_heads, w.head_dim, w.top_k)
    st = ssa.SparseStream(p, dev)
    st.alignment(q, k, v)
    o_full, lse_full, dropped = st._full
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        ssa.ssa_full_attn_fwd_with_mass(p, q, k, v, st.block_idx, st.o, st.lse, o_full, lse_full, dropped)
    reps = 40
    ms = timed_fn(g, reps) / reps
    check_device("align_8k alignment pass")
    fc = causal_flops(w)
    out["align_8k"] = {"config": config_of(w, "l2_flushed"), "full_attn_fwd_with_mass_ms": round(ms, 5),
                       "tflops": round(fc / (ms * 1e-3) / 1e12, 2), "frac": round(fc / (ms * 1e-3) / 1e12 / peak, 4),
                       "flops": "4 D per causal (query, key) pair"}
    del q, k, v, st, g, o_full, lse_full, dropped
    torch.cuda.empty_cache()

    # ---------------------------------------------------------------- train_8k
    x = gen.make_inputs("train_8k")
    w = x.workload
    q, k, v, d_o = (t.to(dev) for t in (x.q, x.k, x.v, x.do))
    p = ssa.problem(w.batch, w.seq_len, w.n_q_heads, w.n_kv_heads, w.head_dim, w.top_k)
    st = ssa.SparseStream(p, dev)
    g_step = st.capture_forward(q, k, v)
    g_step.replay()
    st.backward(q, k, v, d_o)
    g_bwd = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_bwd):
        st.backward(q, k, v, d_o)
    reps = 40
    fwd_ms = timed_fn(g_step, reps) / reps
    bwd_ms = timed_fn(g_bwd, reps) / reps
    check_device("train_8k forward and backward")
    flops = algorithmic_flops(w)
    tot = 3.5 * flops / ((fwd_ms + bwd_ms) * 1e-3) / 1e12
    out["train_8k"] = {"config": config_of(w, "l2_flushed"),
                       "forward_step_ms": round(fwd_ms, 5), "backward_ms": round(bwd_ms, 5),
                       "forward_tflops": round(flops / (fwd_ms * 1e-3) / 1e12, 2),
                       "backward_tflops": round(2.5 * flops / (bwd_ms * 1e-3) / 1e12, 2),
                       "fwd_plus_bwd_tflops": round(tot, 2), "frac_fwd_plus_bwd": round(tot / peak, 4),
                       "flops": "forward 4 D, backward 10 D per selected (query, key) pair"}
    del q, k, v, d_o, st, g_step, g_bwd
    torch.cuda.empty_cache()
    return out


def load_traffic(name):
    """DRAM bytes per launch of the sparse forward (dram__bytes_read.sum +
    dram__bytes_write.sum from one ncu capture) from the committed summary of
    this workload, or None."""
    path = os.path.join(ROOT, "profiles", f"attn_fwd_{name}.md")
    if not os.path.exists(path):
        return None
    import re
    with open(path) as f:
        m = re.search(r"^dram_bytes_per_launch:\s*(\d+)", f.read(), re.M)
    return int(m.group(1)) if m else None


# ------------------------------------------------------------------ decode

def dash_rows(p, w, q, k, v, timed_fn, n_k, alpha=1.5, gamma=8.0, sigma=1.0):
    """DashAttention on the bench workload: the routing (keys-only pooling then
    ssa_dash_route) and the prior-induced softmax (ssa_dash_attn_fwd), each
    timed alone.  gamma = 8 routes about as many chunks as the sparse stream's
    top-k = 16 on these inputs.  FLOPs: 4 D per unmasked (query, key) pair of
    the routed chunks and the diagonal, counted from the mask and weights the
    routing wrote."""
    import block_sparse_attention_21_b200 as ssa
    da = ssa.DashAttention(p, alpha=alpha, gamma=gamma, sigma=sigma)
    da.forward(q, k, v)
    g_route, g_attn = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_route):
        da.route(q, k)
    with torch.cuda.graph(g_attn):
        ssa.ssa_dash_attn_fwd(p, q, k, v, da.weights, da.mask, sigma, da.o, da.lse)
    route_ms = timed_fn(g_route, n_k) / n_k
    attn_ms = timed_fn(g_attn, n_k) / n_k
    torch.cuda.synchronize()
    check_device("decode and routing rows")
    n = w.n_blocks
    bits = np.unpackbits(da.mask.cpu().numpy().view(np.uint8), axis=-1, bitorder="little")[..., :n].astype(bool)
    earlier = np.tril(np.ones((n, n), dtype=bool), -1)
    routed = (bits & earlier & (da.weights.cpu().numpy() > 0)).sum(axis=-1)     # [B, Hkv, n]
    pairs = float((routed * 64 * 64 + 64 * 65 // 2).sum()) * (w.n_q_heads // w.n_kv_heads)
    flops = 4.0 * w.head_dim * pairs
    return {"alpha": alpha, "gamma": gamma, "sigma": sigma,
            "chunks_routed_mean": round(float(routed.mean()) + 1.0, 3),
            "route_ms": round(route_ms, 5), "attn_ms": round(attn_ms, 5),
            "attn_tflops": round(flops / (attn_ms * 1e-3) / 1e12, 2),
            "flops": "4 D per unmasked (query, key) pair of the routed chunks and the diagonal"}


def decode_rows(dev, timed_fn):
    """One decoding step of the sparse stream (ssa_decode_attn) on two batch
    shapes of the Llama-3.2-1B-like layer (Hq 32, Hkv 4, D 64, top-k 16):
    64 sequences with 8k caches, and 8 sequences with 128k caches, the latter
    also with top-k = every block (dense decode by the same kernels).  The
    caches are seeded normal draws made on the device.  Algorithmic bytes: the
    mean keys scored, the kept blocks' K and V, q and o."""
    import block_sparse_attention_21_b200 as ssa
    out = {}
    for name, B, S, dense in (("decode_8k_b64", 64, 8192, False), ("decode_128k_b8", 8, 131072, False),
                              ("decode_128k_b8_dense", 8, 131072, True)):
        Hq, Hkv, D = 32, 4, 64
        n = S // 64
        topk = n if dense else 16
        g = torch.Generator(device=dev).manual_seed(11 + S)
        k = torch.randn(B, S, Hkv, D, generator=g, device=dev).to(torch.bfloat16)
        v = torch.randn(B, S, Hkv, D, generator=g, device=dev).to(torch.bfloat16)
        q = torch.randn(B, Hq, D, generator=g, device=dev).to(torch.bfloat16)
        lengths = torch.full((B,), S, dtype=torch.int32, device=dev)
        p = ssa.problem(B, S, Hq, Hkv, D, topk)
        kb = torch.empty(B, Hkv, n, D, device=dev)
        ssa.ssa_block_pool(p, k, None, kb, None)
        o = torch.empty(B, Hq, D, dtype=torch.bfloat16, device=dev)
        lse = torch.empty(B, Hq, device=dev)
        ws = torch.empty(max(ssa.ssa_decode_attn_workspace(p), 256), dtype=torch.uint8, device=dev)
        ssa.ssa_decode_attn(p, q, k, v, kb, lengths, o, lse, None, ws, ws.numel())
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            ssa.ssa_decode_attn(p, q, k, v, kb, lengths, o, lse, None, ws, ws.numel())
        reps = 50
        ms = timed_fn(graph, reps) / reps
        c = n - 1                                  # full caches: block n - 1 holds the query
        kept = min(topk, c + 1)
        nbytes = B * Hkv * ((c if kept < c + 1 else 0) * D * 4 + kept * 64 * D * 2 * 2) + 2 * B * Hq * D * 2
        out[name] = {"ms": round(ms, 5), "batch": B, "cache_tokens": S, "top_k": topk,
                     "gb_s": round(nbytes / (ms * 1e-3) / 1e9, 1), "bytes_per_step": int(nbytes)}
        del k, v, kb, ws
    out["decode_128k_sparse_vs_dense"] = round(out["decode_128k_b8_dense"]["ms"] / out["decode_128k_b8"]["ms"], 2)
    return out


# ----------------------------------------------------------- CPU baseline

def _row_flops(workload, idx, rows):
    """Selected-pair FLOPs (4 * D per unmasked pair) of each (b, hq, t) row."""
    nsel = np.minimum(workload.top_k, rows[:, 2] // 64 + 1)
    return 4.0 * workload.head_dim * ((nsel - 1) * 64 + rows[:, 2] % 64 + 1)


def cpu_baseline(x):
    """The fp64 oracle as it stands on the host cores, on the whole workload:
    pooling, selection and sparse attention of every row, reported as TFLOP/s
    of the selected-pair FLOPs."""
    import oracle
    w = x.workload
    threads = oracle.default_threads()
    q64, k64, v64 = oracle.widen(x.q), oracle.widen(x.k), oracle.widen(x.v)
    rows = oracle.all_rows(w.batch, w.n_q_heads, w.seq_len)
    t0 = time.perf_counter()
    kbar, qbar = oracle.block_pool(k64, q64, nthreads=threads)
    idx, _ = oracle.block_select(qbar, kbar, w.top_k, nthreads=threads)
    oracle.attn_rows(q64, k64, v64, idx, rows, want_full=False, nthreads=threads)
    dt = time.perf_counter() - t0
    flops = algorithmic_flops(w)
    return {"value": round(flops / dt / 1e12, 6), "unit": "TFLOP/s", "cores": threads,
            "kind": "oracle", "seconds": round(dt, 2),
            "sample": (f"the whole workload: pooling, selection and sparse attention of all "
                       f"{len(rows)} rows, fp64, {threads} threads")}


def run_reference(args, world, rank):
    """The reference arm: the fp64 oracle on the host cores, on this arm's
    workload.  Pooling and selection of the whole workload run once (timed and
    reported); each step then computes the sparse attention of a random sample
    of query rows, sized so that the whole run takes about two minutes."""
    if rank != 0:
        return None
    import oracle
    x = gen.make_inputs(args.workload)
    w = x.workload
    threads = oracle.default_threads()
    q64, k64, v64 = oracle.widen(x.q), oracle.widen(x.k), oracle.widen(x.v)
    t0 = time.perf_counter()
    kbar, qbar = oracle.block_pool(k64, q64, nthreads=threads)
    idx, _ = oracle.block_select(qbar, kbar, w.top_k, nthreads=threads)
    select_s = time.perf_counter() - t0
    rng = np.random.Generator(np.random.PCG64(4242))

    def sample(nrows):
        return np.stack([rng.integers(0, w.batch, nrows), rng.integers(0, w.n_q_heads, nrows),
                         rng.integers(0, w.seq_len, nrows)], axis=1).astype(np.int64)

    def run(rows):
        t = time.perf_counter()
        oracle.attn_rows(q64, k64, v64, idx, rows, want_full=False, nthreads=threads)
        return time.perf_counter() - t

    cal = sample(4 * threads)
    rate = _row_flops(w, idx, cal).sum() / max(run(cal), 1e-6)
    mean_row = algorithmic_flops(w) / (w.batch * w.n_q_heads * w.seq_len)
    budget = 120.0 / (args.steps + args.warmup)
    nrows = int(np.clip(budget * rate / mean_row, 8, 1 << 16))
    for _ in range(args.warmup):
        run(sample(nrows))
    flops = secs = 0.0
    for _ in range(args.steps):
        rows = sample(nrows)
        secs += run(rows)
        flops += _row_flops(w, idx, rows).sum()
    value = flops / secs / 1e12
    cb = {"value": round(value, 6), "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
          "sample": (f"per step the sparse attention of {nrows} random query rows "
                     f"(fp64, {threads} threads); pooling and selection of the whole workload "
                     f"once beforehand ({select_s:.2f} s)")}
    return {"impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(1000.0 * secs / max(1, args.steps), 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": config_of(w, "host_cpu"), "cpu_baseline": cb,
            "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def decode_only():
    """The decode rows alone, timed as in run_ours (L2 flushed by a write and a
    read-back of 256 MiB before each step, CUDA events around each replay)."""
    import torch
    import block_sparse_attention_21_b200 as ssa
    dev = torch.device("cuda", 0)
    check_device("decode rows")
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    sink = torch.empty((), dtype=torch.int64, device=dev)
    stream = torch.cuda.current_stream()

    def timed(graph, n):
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(n)]
        for s in range(n):
            flush.fill_(s & 0xFF)
            torch.sum(flush.view(torch.int64), dim=0, out=sink)
            evs[s][0].record(stream)
            graph.replay()
            evs[s][1].record(stream)
        torch.cuda.synchronize()
        return sum(a.elapsed_time(b) for a, b in evs)

    n0 = ssa.ssa_launch_count()
    rows = decode_rows(dev, timed)
    rows["gpu_launches_total"] = int(ssa.ssa_launch_count() - n0)
    return {"decode": rows}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default="llama1b_8k", choices=sorted(gen.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-other-workloads", action="store_true",
                    help="skip the 32k, batch-2 alignment and batch-4 training workloads")
    ap.add_argument("--decode-only", action="store_true",
                    help="time only the decode rows (one GPU) and print them; for profiling")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.decode_only:
        print(json.dumps(decode_only()), flush=True)
        return
    world, rank, local = dist_setup(args)
    try:
        if args.impl == "reference":
            rec = run_reference(args, world, rank)
        else:
            rec = run_ours(args, world, rank, local)
        if rank == 0 and rec is not None:
            print(json.dumps(rec), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
