#!/usr/bin/env python
"""HCA benchmark: prefill TFLOP/s and decode tokens/s at head_dim 512 on B200.

Main line (the step): compress + prefill of one batch of the bf16 prefill workload
(batch 1, T = 32768, 64 query heads sharing 1 KV head, head_dim 512, block 128,
window 128, scale 1/sqrt(512), N(0,1) inputs rounded to bf16, gate off). The value is
algorithmic TFLOP/s (visible query-key pairs only) over all ranks. Inputs (Q alone is
2.1 GB) are larger than the 126 MB L2, so no flush runs between steps.

Extra results in the same JSON line:
  decode_batched  128 sequences, context lengths uniform in [8192, 131072]: tokens/s
  decode_1m       16 sequences at 1,048,576 context, 4 decode steps each, gate on, with
                  the compress call of the block the first step completes: tokens/s
  prefill_128k    batch 2 x 131072, heterogeneous blocks, fused gate: TFLOP/s
  backward_32k    the prefill backward of the 32K workload (dQ, dK, dV): TFLOP/s
  gate_from_latent  G = sigmoid(q_lat . W_g) for 32768 tokens: TFLOP/s
  compress_2x128k hca_compress of the K and V of 2 x 131072 tokens alone: GB/s vs HBM
  e2e             the main metric with host-resident inputs and output (pinned host
                  memory, H2D + D2H inside the timed region)
  roofline        prefill kernel vs the measured bf16 dense peak (and HBM)
  cpu_baseline    the float64 oracle on a bounded sample of the same workload

Multi-GPU (torchrun): the same workloads cut over the ranks (compressed_long_context_hca_b200.
parallel): prefill by query rows (entry all-gather + window-1 halo), batched decode by
sequences, 1M decode by compressed-entry ranges (all-gather of (m, l, O) partials + merge).
Total work is fixed as N grows ("scaling": "strong"); the time is the max over ranks.
``--impl reference`` times the float64 oracle (rank 0 only) on bounded samples.
"""

from __future__ import annotations

import argparse
import json
import math
import os
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# DRAM bytes (read + write) of one prefill launch, from ncu captures of 8K cases scaled by
# query positions (Q, O and the gate dominate and scale with them; K/V stay in L2): the
# 32K workload is x4 of the 8K case; the gated 2 x 128K workload is x32 of the gated 8K
# case with every 4th block x4. Keyed by the SHA-1 prefix of the kernel source the
# captures were made on: any change to the kernel makes the figures null.
PREFILL_KERNEL_SRC = "prefill_pair.cu"
PREFILL_TRAFFIC = {"569d220a1c08": 4 * 1.037858e9}         # 1.0379 GB at 8K
PREFILL_128K_TRAFFIC = {"569d220a1c08": 32 * 1.584315e9}   # 1.5843 GB at 8K, gated
D, HQ, BLOCK, WIN = 512, 64, 128, 128


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(PEAKS_FALLBACK), "fallback"


def visible_pairs(T: int, block: int = BLOCK, W: int = WIN):
    """Closed-form count of visible (query, key) pairs per head of one sequence."""
    c = 0
    # sum_t max(0, floor((t + 1 - W) / block)) for t in [0, T)
    for x in range(1, T - W + 1):
        c += x // block
    w = sum(min(W, t + 1) for t in range(min(T, W))) + max(0, T - W) * W
    return c, w


def prefill_flops(T: int, batch: int = 1) -> float:
    c, w = visible_pairs(T)
    return 4.0 * D * HQ * (c + w) * batch


def prefill_flops_rows(T: int, t0: int, t1: int, batch: int = 1) -> float:
    """Algorithmic FLOPs of query positions [t0, t1) of a T-token sequence."""
    c1, w1 = visible_pairs(t1)
    c0, w0 = visible_pairs(t0)
    return 4.0 * D * HQ * ((c1 - c0) + (w1 - w0)) * batch


# ------------------------------------------------------------------ clocks sampler
class Clocks:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        time.sleep(0.12)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out = ""
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for n, v in zip(names, parts[3:7]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        sm.sort()
        med = sm[len(sm) // 2] if sm else None
        return {"sm_mhz": med, "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------ oracle timing
def oracle_sample_prefill(seconds: float, T: int = 32768, seed: int = 0):
    """Time the float64 oracle on random query positions of the 32K workload.

    Returns (tflops, positions_done, wall_s, threads). Inputs are regenerated on the CPU
    with the same recipe (values differ from the GPU's generator; the cost does not)."""
    import numpy as np
    from compressed_long_context_hca_b200 import inputs
    from oracle import hca_oracle as orc
    x = inputs.prefill_inputs(1, T, HQ, 1, D, "bf16", seed=seed)
    Q = x.Q[0].float().numpy().astype(np.float64)
    K = x.K[0].float().numpy().astype(np.float64)
    V = x.V[0].float().numpy().astype(np.float64)
    s = 1.0 / math.sqrt(D)
    Kc, Vc = orc.compress_blocks(K, BLOCK), orc.compress_blocks(V, BLOCK)
    rng = np.random.default_rng(seed)
    done, flops = 0, 0.0
    t0 = time.perf_counter()
    while time.perf_counter() - t0 < seconds:
        t = int(rng.integers(0, T))
        orc.attend_position(Q[t], Kc, Vc, K, V, t, BLOCK, WIN, s)
        n = orc.visible_compressed_count(t, BLOCK, WIN) + (t - max(0, t - WIN + 1) + 1)
        flops += 4.0 * D * HQ * n
        done += 1
    wall = time.perf_counter() - t0
    threads = blas_threads()
    return flops / wall / 1e12, done, wall, threads


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        n = max([i.get("num_threads", 1) for i in info] or [1])
        return int(n)
    except Exception:
        return os.cpu_count() or 1


# ------------------------------------------------------------------ GPU workloads
def rank_tools(world, device):
    """The two collectives of a timed region: a barrier on both sides, and the max over
    ranks of the measured time (NCCL tensors on the GPU; CPU tensors under gloo)."""
    import torch
    import torch.distributed as dist

    def barrier():
        if world > 1:
            dist.barrier()

    def max_over_ranks(x: float) -> float:
        if world == 1:
            return x
        t = torch.tensor([x], dtype=torch.float64, device=device)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())

    return barrier, max_over_ranks


def gpu_main(args, rank, world, local_rank):
    import torch
    from compressed_long_context_hca_b200 import binding as B
    from compressed_long_context_hca_b200 import build as build_mod
    from compressed_long_context_hca_b200 import ops

    if not torch.cuda.is_available():
        raise SystemExit("bench.py: no CUDA device (the product has no CPU path)")
    build_mod.build()
    B.lib()
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    peaks, peak_kind = load_peaks()

    barrier, max_over_ranks = rank_tools(world, dev)

    # ---------------------------------------------------------------- main: 32K prefill
    # One sequence; with N ranks its query rows are cut into N ranges of whole blocks
    # (parallel.prefill_rows: own-block compress, entry all-gather, halo, range prefill).
    # Every rank draws the whole sequence from the same seed and keeps its rows.
    from compressed_long_context_hca_b200 import parallel as P
    T = args.seqlen
    t0, t1 = P.row_range(T, world, rank, BLOCK)
    g = torch.Generator(device=dev)
    g.manual_seed(1000)
    Qf = torch.randn((1, T, HQ, D), generator=g, device=dev).to(torch.bfloat16)
    Q = Qf[:, t0:t1].contiguous()
    del Qf
    Kf = torch.randn((1, T, 1, D), generator=g, device=dev).to(torch.bfloat16)
    Vf = torch.randn((1, T, 1, D), generator=g, device=dev).to(torch.bfloat16)
    K, V = Kf[:, t0:t1].contiguous(), Vf[:, t0:t1].contiguous()
    del Kf, Vf
    group = None
    be = P.GpuBackend()

    def step():
        return P.prefill_rows(be, group, Q, K, V, T, BLOCK, WIN)

    for _ in range(args.warmup):
        O = step()
    torch.cuda.synchronize()
    flops = prefill_flops(T)
    be.kernel_events = []
    clocks = Clocks(local_rank)
    clocks.start()
    time.sleep(0.1)
    barrier()
    torch.cuda.synchronize()
    e_start = torch.cuda.Event(enable_timing=True)
    e_end = torch.cuda.Event(enable_timing=True)
    e_start.record(stream)
    for i in range(args.steps):
        O = step()
    e_end.record(stream)
    torch.cuda.synchronize()
    barrier()
    clk = clocks.stop()
    total_ms = max_over_ranks(e_start.elapsed_time(e_end))
    ms_step = total_ms / args.steps
    ev = be.kernel_events
    be.kernel_events = None
    prefill_ms = sum(a.elapsed_time(b) for a, b in ev) / len(ev)
    # ours per step: compress and prefill (the entry copies into the range call's cache are
    # torch copies; at N > 1 the entry and halo gathers are NCCL kernels)
    launches = 2 * args.steps
    for c in be._caches.values():
        assert int(c.err.item()) == 0, "kernel raised an error bit"

    value = flops / (ms_step * 1e-3) / 1e12
    # this rank's share of the algorithmic work, over its kernel's time
    my_flops = prefill_flops_rows(T, t0, t1)
    achieved = my_flops / (prefill_ms * 1e-3) / 1e12
    bytes_prefill = (2 * Q.numel() + 2 * K.numel() + 2 * V.numel()) * 2  # Q,O + K,V
    # the burst peak for a short timed loop; the sustained one (measured over a seconds-long
    # loop under the power cap) once the timed loop itself runs for a sizeable fraction of
    # a second
    sustained = total_ms > 300.0
    peak_tf = peaks["bf16_tflops_sustained"] if sustained else peaks["bf16_tflops"]
    peak_note = (f"{peak_kind} bf16 dense sustained (timed loop of {total_ms:.0f} ms)"
                 if sustained else
                 f"{peak_kind} bf16 dense burst (timed loop of {total_ms:.0f} ms)")
    traffic = args.traffic
    if traffic is None and T == 32768 and world == 1:
        traffic = PREFILL_TRAFFIC.get(_prefill_kernel_sha())
    hbm_achieved = bytes_prefill / (prefill_ms * 1e-3) / 1e9
    result = {
        "metric": "HCA prefill TFLOP/s at d=512 (32K bf16, compress+prefill step); "
                  "decode tokens/s in decode_batched / decode_1m",
        "value": round(value, 2),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_step, 4),
        "higher_is_better": True,
        "scaling": "strong",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic N(0,1) rounded to bf16, seeded",
        "config": {"workload": "HCA prefill bf16: batch 1, T=32768, 64 query heads, 1 KV head, "
                               "head_dim 512, block 128, window 128, gate off",
                   "global_batch": 1, "seq_len": T,
                   "parallelism": f"query rows x{world} (whole blocks; entry all-gather + "
                                  f"window-1 halo)" if world > 1 else "single GPU",
                   "l2": "inputs larger than L2 (Q 2.1 GB), no flush"},
        "gpu_launches": launches,
        "roofline": {"bound": "tensor", "achieved": round(achieved, 1),
                     "peak": peak_tf, "unit": "TFLOP/s",
                     "frac": round(achieved / peak_tf, 4),
                     "traffic": traffic, "kernel": "prefill_pair_kernel",
                     "peak_source": peak_note,
                     "hbm": {"achieved": round(hbm_achieved, 1), "peak": peaks["hbm_gbs"],
                             "unit": "GB/s", "frac": round(hbm_achieved / peaks["hbm_gbs"], 4),
                             "bytes_per_launch": bytes_prefill}},
        "clocks": clk,
    }

    # ---------------------------------------------------------------- e2e (host buffers)
    # Every step copies this rank's input rows from pinned host memory, runs the same
    # partitioned compress + prefill and copies its output rows back. Steps are pipelined
    # over three streams with two device buffer sets: the upload of step i + 1 and the
    # download of step i - 1 run while step i computes (PCIe is full duplex). The timed
    # region runs from the first upload to the last download, so the first upload and the
    # last download (one step's worth of each) are spread over the timed steps.
    if not args.no_e2e:
        hQ = Q.cpu().pin_memory()
        hK = K.cpu().pin_memory()
        hV = V.cpu().pin_memory()
        hO = torch.empty(O.shape, dtype=O.dtype).pin_memory()
        e2e_steps = max(2, min(args.steps, args.e2e_steps))
        bufs = [(Q, K, V, torch.empty_like(Q)),
                (torch.empty_like(Q), torch.empty_like(K), torch.empty_like(V),
                 torch.empty_like(Q))]
        up, comp, down = torch.cuda.Stream(), stream, torch.cuda.Stream()
        ev = lambda: torch.cuda.Event()  # noqa: E731
        inputs_free = [ev(), ev()]   # compute of the buffer set's last step is done
        out_free = [ev(), ev()]      # download of the buffer set's last output is done
        uploaded = [ev(), ev()]
        computed = [ev(), ev()]

        def run(n):
            for i in range(n):
                x = i % 2
                q_, k_, v_, o_ = bufs[x]
                with torch.cuda.stream(up):
                    if i >= 2:
                        up.wait_event(inputs_free[x])
                    q_.copy_(hQ, non_blocking=True)
                    k_.copy_(hK, non_blocking=True)
                    v_.copy_(hV, non_blocking=True)
                    uploaded[x].record(up)
                comp.wait_event(uploaded[x])
                if i >= 2:
                    comp.wait_event(out_free[x])
                with torch.cuda.stream(comp):
                    P.prefill_rows(be, group, q_, k_, v_, T, BLOCK, WIN, out=o_)
                computed[x].record(comp)
                inputs_free[x].record(comp)
                with torch.cuda.stream(down):
                    down.wait_event(computed[x])
                    hO.copy_(o_, non_blocking=True)
                    out_free[x].record(down)

        run(2)
        torch.cuda.synchronize()
        barrier()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(up)
        comp.wait_stream(up)
        down.wait_stream(up)
        run(e2e_steps)
        comp.wait_stream(down)
        b.record(comp)
        torch.cuda.synchronize()
        e2e_ms = max_over_ranks(a.elapsed_time(b)) / e2e_steps
        result["e2e"] = {"value": round(flops / (e2e_ms * 1e-3) / 1e12, 3),
                         "unit": "TFLOP/s", "ms_per_step": round(e2e_ms, 3),
                         "h2d_bytes_per_step": (hQ.numel() + hK.numel() + hV.numel()) * 2,
                         "d2h_bytes_per_step": hO.numel() * 2,
                         "overlap": "uploads / compute / downloads of consecutive steps on "
                                    "three streams, two device buffer sets"}
        del hQ, hK, hV, hO, bufs

    del Q, K, V, O, be
    torch.cuda.empty_cache()

    # ---------------------------------------------------------------- decode workloads
    if not args.no_decode:
        result["decode_batched"] = bench_decode_batched(args, dev, rank, world, barrier,
                                                        max_over_ranks, peaks)
        result["decode_1m"] = bench_decode_1m(args, dev, rank, world, barrier, max_over_ranks,
                                              peaks)
        if not args.no_e4m3:
            result["decode_batched_e4m3"] = bench_decode_batched(
                args, dev, rank, world, barrier, max_over_ranks, peaks, e4m3=True)
            result["decode_1m_e4m3"] = bench_decode_1m(args, dev, rank, world, barrier,
                                                       max_over_ranks, peaks, e4m3=True)
    if args.with_128k:
        result["compress_2x128k"] = bench_compress_2x128k(args, dev, rank, world, barrier,
                                                          max_over_ranks, peaks)
        result["prefill_128k"] = bench_prefill_128k(args, dev, rank, world, barrier,
                                                    max_over_ranks, peaks)

    if not args.no_backward and world == 1:
        result["backward_32k"] = bench_backward_32k(args, dev, rank, world, barrier,
                                                    max_over_ranks, peaks)
        result["gate_from_latent"] = bench_gate_from_latent(args, dev, rank, world, barrier,
                                                            max_over_ranks, peaks)

    # ---------------------------------------------------------------- CPU baseline
    if rank == 0 and world == 1 and not args.no_cpu:
        tf, n, wall, threads = oracle_sample_prefill(args.cpu_seconds, T)
        result["cpu_baseline"] = {"value": tf, "unit": "TFLOP/s", "cores": threads,
                                  "kind": "oracle",
                                  "sample": f"{n} random query positions x 64 heads of the 32K "
                                            f"workload, {wall:.1f} s float64 NumPy"}
    return result


def _time_graph(fn, steps, warmup, barrier, max_over_ranks, stream):
    """Capture one call of `fn` (every launch of a decode step) in a CUDA graph and time
    `steps` replays back to back, as a serving loop replays its decode step: the host's
    per-launch work is left out, the device work is the same."""
    import torch
    side = torch.cuda.Stream()
    side.wait_stream(stream)
    with torch.cuda.stream(side):
        for _ in range(warmup):
            fn()
    stream.wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    torch.cuda.synchronize()
    ms = _time_loop(g.replay, steps, warmup, barrier, max_over_ranks, stream)
    del g
    return ms


def _time_loop(fn, steps, warmup, barrier, max_over_ranks, stream):
    import torch
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    barrier()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(steps):
        fn()
    b.record(stream)
    torch.cuda.synchronize()
    barrier()
    return max_over_ranks(a.elapsed_time(b)) / steps


E4M3_SCALES = (1.0 / 16, 1.0 / 16)


def _fill_e4m3(t, g):
    """Random e4m3 codes in place: a random sign over a magnitude code uniform in
    0..0x5F (the recipe of inputs.e4m3_codes, drawn on the device)."""
    import torch
    t.random_(0, 0x60, generator=g)
    sign = torch.randint(0, 2, t.shape, generator=g, device=t.device, dtype=torch.uint8)
    t.bitwise_or_(sign << 7)


def bench_decode_batched(args, dev, rank, world, barrier, max_over_ranks, peaks, e4m3=False):
    """128 sequences, context lengths U[8192, 131072]; with N ranks each serves a
    contiguous range of the sequences (no exchange). e4m3: the compressed cache holds
    8-bit codes (per-pool scales 1/16); the window ring stays bf16."""
    import torch
    from compressed_long_context_hca_b200 import binding as B
    from compressed_long_context_hca_b200 import ops
    from compressed_long_context_hca_b200 import parallel as P
    nseq_all, lo, hi = 128, 8192, 131072
    g = torch.Generator(device=dev)
    g.manual_seed(2000)
    ctx_all = torch.randint(lo, hi + 1, (nseq_all,), generator=g, device=dev,
                            dtype=torch.int64).to(torch.int32)
    s0, s1 = P.seq_range(nseq_all, world, rank)
    nseq = s1 - s0
    ctx = ctx_all[s0:s1].contiguous()
    g.manual_seed(2001 + rank)
    max_ent = (hi - WIN) // BLOCK + 1
    cache = B.PagedCache(nseq, max_ent, 1, D, torch.bfloat16, 128, device=dev,
                         e4m3_scales=E4M3_SCALES if e4m3 else None)
    if e4m3:
        _fill_e4m3(cache.kc, g)
        _fill_e4m3(cache.vc, g)
    else:
        cache.kc.normal_(generator=g)
        cache.vc.normal_(generator=g)
    cache.n_entries.fill_(max_ent)
    q = torch.randn((nseq, HQ, D), generator=g, device=dev).to(torch.bfloat16)
    rk = torch.randn((nseq, WIN, 1, D), generator=g, device=dev).to(torch.bfloat16)
    rv = torch.randn((nseq, WIN, 1, D), generator=g, device=dev).to(torch.bfloat16)
    desc = B.make_desc(nseq, hi, HQ, 1, D)
    ws = ops.decode_workspace(desc, dev)
    O = torch.empty_like(q)
    stream = torch.cuda.current_stream()
    clocks = Clocks(dev.index)
    fn = lambda: ops.decode(desc, q, ctx, cache, rk, rv, O=O, workspace=ws)  # noqa: E731
    clocks.start()
    ms = _time_graph(fn, args.decode_steps, 3, barrier, max_over_ranks, stream)
    clk = clocks.stop()
    ctx_h = ctx_all.cpu().tolist()
    entries = sum(max(0, c - WIN) // BLOCK for c in ctx_h)
    raw = sum(min(WIN, c) for c in ctx_h)
    # K and V of every visible key (1 byte per element for e4m3 entries), Q in, O out
    byts = (entries * D * 2 * (1 if e4m3 else 2) + raw * D * 2 * 2 +
            nseq_all * HQ * D * 2 * 2)
    nsplit = B.hca_decode_workspace_bytes(desc) // (nseq * HQ * (D + 2) * 4)
    gbs = byts / (ms * 1e-3) / 1e9 / world  # per GPU
    cache_txt = ("e4m3 compressed cache (scales 1/16) + bf16 128-token ring" if e4m3 else
                 "paged cache + 128-token ring, N(0,1) bf16")
    return {"value": round(nseq_all / (ms * 1e-3), 1), "unit": "tokens/s",
            "ms_per_step": round(ms, 4),
            "workload": "128 sequences, context U[8192,131072], 1 query each, 64 heads, "
                        "head_dim 512, " + cache_txt,
            "parallelism": f"sequences x{world}" if world > 1 else "single GPU",
            "timing": "CUDA graph replay of one step",
            "gpu_launches_per_step": 2, "splits": int(nsplit),
            "roofline": {"bound": "hbm", "achieved": round(gbs, 1),
                         "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": round(gbs / peaks["hbm_gbs"], 4),
                         "bytes_per_step": byts},
            "clocks": clk}


def _shard_cache(nseq, e0, e1, n_total, dev, g, e4m3=False):
    """A paged cache holding only entries [e0, min(e1, n_total)) of every sequence, at
    their absolute entry indices (pages outside the shard map to page 0 and are never
    read), filled with N(0,1) values (or random e4m3 codes)."""
    import torch
    from compressed_long_context_hca_b200 import binding as B
    p0 = e0 // 128
    p1 = -(-min(e1, n_total) // 128)
    shard_pages = max(1, p1 - p0)
    cache = B.PagedCache(nseq, shard_pages * 128, 1, D, torch.bfloat16, 128, device=dev,
                         e4m3_scales=E4M3_SCALES if e4m3 else None)
    if e4m3:
        _fill_e4m3(cache.kc, g)
        _fill_e4m3(cache.vc, g)
    else:
        cache.kc.normal_(generator=g)
        cache.vc.normal_(generator=g)
    total_pages = -(-n_total // 128)
    pt = torch.zeros((nseq, total_pages), dtype=torch.int32)
    for b in range(nseq):
        for p in range(p0, min(p1, total_pages)):
            pt[b, p] = b * shard_pages + (p - p0)
    cache.page_table = pt.to(dev)
    cache.c.page_table = cache.page_table.data_ptr()
    cache.c.max_pages = total_pages
    return cache


def bench_decode_1m(args, dev, rank, world, barrier, max_over_ranks, peaks, e4m3=False):
    """16 sequences at 1,048,576 context, 4 decode steps each with the compress of the block
    the first step completes. With N ranks the compressed entries of every sequence are cut
    into N ranges of whole 128-entry tiles (rank r holds only its range), the last rank also
    holds the ring; every step all-gathers the (m, l, O) partials and merges them."""
    import torch
    from compressed_long_context_hca_b200 import binding as B
    from compressed_long_context_hca_b200 import ops
    from compressed_long_context_hca_b200 import parallel as P
    nseq, ctx0, steps_per = 16, 1048576, 4
    n_ent = (ctx0 - WIN) // BLOCK  # 8191 visible entries at the first step
    g = torch.Generator(device=dev)
    g.manual_seed(3000)
    q = torch.randn((steps_per, nseq, HQ, D), generator=g, device=dev).to(torch.bfloat16)
    G = torch.sigmoid(torch.randn((steps_per, nseq, HQ, D), generator=g, device=dev))
    G = G.to(torch.bfloat16)
    new_k = torch.randn((steps_per, nseq, 1, 1, D), generator=g, device=dev).to(torch.bfloat16)
    new_v = torch.randn((steps_per, nseq, 1, 1, D), generator=g, device=dev).to(torch.bfloat16)
    rk = torch.randn((nseq, WIN, 1, D), generator=g, device=dev).to(torch.bfloat16)
    rv = torch.randn((nseq, WIN, 1, D), generator=g, device=dev).to(torch.bfloat16)
    g.manual_seed(3001 + rank)
    e0, e1 = P.entry_range(n_ent, world, rank) if world > 1 else (0, 1 << 30)
    last = rank == world - 1
    cache = _shard_cache(nseq, e0, e1, n_ent + 2, dev, g, e4m3)
    cache.n_entries.fill_(n_ent)
    ctx = [torch.full((nseq,), ctx0 + s, dtype=torch.int32, device=dev) for s in range(steps_per)]
    descs = []
    for s in range(steps_per):
        d = B.make_desc(nseq, ctx0 + steps_per, HQ, 1, D)
        ops.attach_gate(d, G[s])
        descs.append(d)
    cdesc = B.make_desc(nseq, ctx0, HQ, 1, D)  # compress of the block ending at ctx0 - 1
    O1 = torch.empty((nseq, HQ, D), dtype=torch.bfloat16, device=dev)
    ws1 = ops.decode_workspace(descs[0], dev) if world == 1 else None
    stream = torch.cuda.current_stream()
    be = P.GpuBackend()
    group = None

    def four_steps():
        for s in range(steps_per):
            p = ctx0 - 1 + s                 # position of the new token
            if world == 1:
                # the new token into ring slot p % WIN inside the decode call
                ops.decode_append(descs[s], q[s], ctx[s], cache, new_k[s], new_v[s], rk, rv,
                                  O=O1, workspace=ws1)
            else:
                if last:  # the rank holding the ring: the new token into its slot
                    ops.ring_append(descs[s], new_k[s], new_v[s], ctx[s], rk, rv)
                P.decode_split_entries(be, group, q[s], ctx[s], cache, rk, rv, n_ent, descs[s])
            if last and (p + 1) % BLOCK == 0:
                # the token completes block p // BLOCK: its entry (invisible to the token's
                # own query) is compressed after the step
                B.check(B.hca_compress(cdesc, rk.data_ptr(), rv.data_ptr(), WIN, p // BLOCK, 1,
                                       cache.c, torch.cuda.current_stream().cuda_stream),
                        "hca_compress")

    clocks = Clocks(dev.index)
    clocks.start()
    if world == 1:
        ms = _time_graph(four_steps, args.decode_steps, 3, barrier, max_over_ranks, stream)
        timing = "CUDA graph replay of the 4 steps"
    else:
        ms = _time_loop(four_steps, args.decode_steps, 3, barrier, max_over_ranks, stream)
        timing = "launch loop (the steps hold NCCL all-gathers)"
    clk = clocks.stop()
    assert int(cache.err.item()) == 0, "kernel raised an error bit"
    eb = 1 if e4m3 else 2  # bytes per compressed element
    byts_step = nseq * (n_ent * D * 2 * eb + WIN * D * 2 * 2 + 3 * HQ * D * 2)
    # the compress reads the ring's K and V once and writes one entry each
    byts = steps_per * byts_step + nseq * (BLOCK * D * 2 * 2 + D * 2 * eb)
    gbs = byts / (ms * 1e-3) / 1e9 / world  # per GPU
    nsplit = B.hca_decode_workspace_bytes(descs[0]) // (nseq * HQ * (D + 2) * 4)
    # per step: decode (with the ring update inside), merge; one compress. N > 1: per step
    # the ring update (the rank holding the ring), the partial decode and its merge, the
    # merge of the gathered parts
    launches = (4 * 2 + 1) if world == 1 else (4 * 3 + (4 + 1 if last else 0))
    return {"value": round(nseq * steps_per / (ms * 1e-3), 1), "unit": "tokens/s",
            "ms_per_step": round(ms, 4), "ms_per_decode_step": round(ms / steps_per, 4),
            "workload": "16 sequences at context 1,048,576 (8191 entries + 128 raw), 64 heads, "
                        "head_dim 512, 4 decode steps each incl. one hca_compress, gate on" +
                        (", e4m3 compressed cache (scales 1/16), bf16 ring" if e4m3 else ""),
            "parallelism": (f"compressed entries x{world} (128-entry tiles; all-gather of "
                            f"(m, l, O) partials + merge)") if world > 1 else "single GPU",
            "timing": timing,
            "gpu_launches_per_step": launches, "splits": int(nsplit),
            "roofline": {"bound": "hbm", "achieved": round(gbs, 1),
                         "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": round(gbs / peaks["hbm_gbs"], 4),
                         "bytes_per_step": byts},
            "clocks": clk}


def bench_compress_2x128k(args, dev, rank, world, barrier, max_over_ranks, peaks):
    """hca_compress alone on the K and V of the training-context prefill workload
    (2 x 131072 tokens, 2048 entries per sequence): read K + V once, write the entries.
    With N ranks each compresses the blocks of its query-row range."""
    import torch
    from compressed_long_context_hca_b200 import binding as B
    from compressed_long_context_hca_b200 import ops
    from compressed_long_context_hca_b200 import parallel as P
    b, T = 2, 131072
    t0, t1 = P.row_range(T, world, rank, BLOCK)
    n = t1 - t0
    g = torch.Generator(device=dev)
    g.manual_seed(5000 + rank)
    K = torch.randn((b, n, 1, D), generator=g, device=dev).to(torch.bfloat16)
    V = torch.randn((b, n, 1, D), generator=g, device=dev).to(torch.bfloat16)
    desc = ops.desc_for_prefill(K, K)
    cache = B.PagedCache(b, -(-n // BLOCK), 1, D, torch.bfloat16, 128, device=dev)
    stream = torch.cuda.current_stream()
    clocks = Clocks(dev.index)
    clocks.start()
    ms = _time_loop(lambda: ops.compress(desc, K, V, cache), args.decode_steps, 3, barrier,
                    max_over_ranks, stream)
    clk = clocks.stop()
    assert int(cache.err.item()) == 0, "kernel raised an error bit"
    byts = 2 * b * T * D * 2 + 2 * b * (T // BLOCK) * D * 2
    gbs = byts / (ms * 1e-3) / 1e9
    return {"value": round(gbs, 1), "unit": "GB/s", "ms_per_step": round(ms, 4),
            "workload": "hca_compress of K and V, batch 2 x 131072 tokens, head_dim 512, bf16 "
                        "(536 MB read, larger than L2)",
            "parallelism": f"query rows x{world}" if world > 1 else "single GPU",
            "gpu_launches_per_step": 1,
            "roofline": {"bound": "hbm", "achieved": round(gbs / world, 1),
                         "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": round(gbs / world / peaks["hbm_gbs"], 4),
                         "bytes_per_step": byts},
            "clocks": clk}


def bench_prefill_128k(args, dev, rank, world, barrier, max_over_ranks, peaks):
    """2 x 131072 tokens, every 4th block x4, fused gate; with N ranks the query rows of
    both sequences are cut into N ranges of whole blocks (parallel.prefill_rows)."""
    import torch
    from compressed_long_context_hca_b200 import parallel as P
    b, T = 2, 131072
    t0, t1 = P.row_range(T, world, rank, BLOCK)
    n = t1 - t0
    g = torch.Generator(device=dev)
    g.manual_seed(4000 + rank)
    blk = ((torch.arange(t0, t1, device=dev) // BLOCK) % 4 == 3)

    def draw(h):
        x = torch.randn((b, n, h, D), generator=g, device=dev)
        x[:, blk] *= 4.0
        return x.to(torch.bfloat16)

    Q, K, V = draw(HQ), draw(1), draw(1)
    G = torch.sigmoid(torch.randn((b, n, HQ, D), generator=g, device=dev)).to(torch.bfloat16)
    be = P.GpuBackend()
    stream = torch.cuda.current_stream()

    def step():
        P.prefill_rows(be, None, Q, K, V, T, BLOCK, WIN, G=G)

    clocks = Clocks(dev.index)
    clocks.start()
    ms = _time_loop(step, args.steps_128k, 3, barrier, max_over_ranks, stream)
    clk = clocks.stop()
    for c in be._caches.values():
        assert int(c.err.item()) == 0, "kernel raised an error bit"
    flops = prefill_flops(T, b)
    tf = flops / (ms * 1e-3) / 1e12
    per_gpu = tf / world
    e2e = None
    if not args.no_e2e and world == 1:
        e2e = _e2e_prefill_128k(args, dev, Q, K, V, G, flops, barrier, max_over_ranks)
    del Q, K, V, G, be
    torch.cuda.empty_cache()
    out = _prefill_128k_result(tf, ms, per_gpu, world, peaks, clk)
    if e2e is not None:
        out["e2e"] = e2e
    return out


def _e2e_prefill_128k(args, dev, Q, K, V, G, flops, barrier, max_over_ranks):
    """The 2 x 128K gated prefill end to end through the C ABI from pinned host memory:
    per step, K and V of both sequences are uploaded and compressed, then every chunk of
    8192 query positions uploads its Q and G rows, runs hca_attn_prefill_range (K/V rows from
    127 positions before the chunk) and downloads its O rows. Uploads, compute and downloads
    of consecutive chunks overlap on three streams with two device buffer sets."""
    import torch
    from compressed_long_context_hca_b200 import binding as B
    from compressed_long_context_hca_b200 import ops
    b, T = Q.shape[0], Q.shape[1]
    C = 8192
    hQ = torch.empty(Q.shape, dtype=Q.dtype, pin_memory=True)
    hG = torch.empty(G.shape, dtype=G.dtype, pin_memory=True)
    hO = torch.empty(Q.shape, dtype=Q.dtype, pin_memory=True)
    hQ.copy_(Q)
    hG.copy_(G)
    hK = K.cpu().pin_memory()
    hV = V.cpu().pin_memory()
    dK, dV = torch.empty_like(K), torch.empty_like(V)
    desc_all = B.make_desc(b, T, HQ, 1, D)
    cache = B.PagedCache(b, T // BLOCK, 1, D, torch.bfloat16, 128, device=dev)
    bufs = [(torch.empty((1, C, HQ, D), dtype=Q.dtype, device=dev),
             torch.empty((1, C, HQ, D), dtype=Q.dtype, device=dev),
             torch.empty((1, C, HQ, D), dtype=Q.dtype, device=dev)) for _ in range(2)]
    up, comp, down = torch.cuda.Stream(), torch.cuda.current_stream(), torch.cuda.Stream()
    ev = lambda: torch.cuda.Event()  # noqa: E731
    in_free, out_free, uploaded, computed = [ev(), ev()], [ev(), ev()], [ev(), ev()], [ev(), ev()]
    kv_up = ev()
    chunks = [(bi, q0) for bi in range(b) for q0 in range(0, T, C)]
    # one descriptor per chunk position: the gate rows of the chunk buffer, K/V rows of the
    # sequence from kv0 = q0 - 127 (the cache holds every block's entry)
    descs = {}
    for bi, q0 in chunks:
        d = B.make_desc(1, C, HQ, 1, D)
        descs[(bi, q0)] = d

    def run():
        up.wait_stream(comp)  # the previous step's range calls have read dK, dV and buffers
        with torch.cuda.stream(up):
            dK.copy_(hK, non_blocking=True)
            dV.copy_(hV, non_blocking=True)
            kv_up.record(up)
        comp.wait_event(kv_up)
        with torch.cuda.stream(comp):
            ops.compress(desc_all, dK, dV, cache)
        for i, (bi, q0) in enumerate(chunks):
            x = i % 2
            q_, g_, o_ = bufs[x]
            with torch.cuda.stream(up):
                if i >= 2:
                    up.wait_event(in_free[x])
                q_.copy_(hQ[bi:bi + 1, q0:q0 + C], non_blocking=True)
                g_.copy_(hG[bi:bi + 1, q0:q0 + C], non_blocking=True)
                uploaded[x].record(up)
            comp.wait_event(uploaded[x])
            if i >= 2:
                comp.wait_event(out_free[x])
            with torch.cuda.stream(comp):
                d = descs[(bi, q0)]
                ops.attach_gate(d, g_)
                kv0 = max(0, q0 - WIN + 1)
                ops.prefill_range(d, q0, kv0, q_, dK[bi:bi + 1, kv0:q0 + C],
                                  dV[bi:bi + 1, kv0:q0 + C], _SeqCache(cache, bi), O=o_)
                computed[x].record(comp)
                in_free[x].record(comp)
            with torch.cuda.stream(down):
                down.wait_event(computed[x])
                hO[bi:bi + 1, q0:q0 + C].copy_(o_, non_blocking=True)
                out_free[x].record(down)
        comp.wait_stream(down)

    run()
    torch.cuda.synchronize()
    steps = max(1, min(2, args.e2e_steps))
    barrier()
    a, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(comp)
    up.wait_stream(comp)
    down.wait_stream(comp)
    for _ in range(steps):
        run()
    e.record(comp)
    torch.cuda.synchronize()
    ms = max_over_ranks(a.elapsed_time(e)) / steps
    assert int(cache.err.item()) == 0, "kernel raised an error bit"
    out = {"value": round(flops / (ms * 1e-3) / 1e12, 3), "unit": "TFLOP/s",
           "ms_per_step": round(ms, 2),
           "h2d_bytes_per_step": (hQ.numel() + hG.numel() + hK.numel() + hV.numel()) * 2,
           "d2h_bytes_per_step": hO.numel() * 2,
           "overlap": "8192-position chunks through hca_attn_prefill_range; uploads / compute / "
                      "downloads of consecutive chunks on three streams"}
    del hQ, hG, hO, hK, hV, bufs, dK, dV
    return out


class _SeqCache:
    """The cache of one sequence of a batch, as a one-sequence cache (its page-table row and
    entry count), so a per-sequence range call reads that sequence's entries."""

    def __init__(self, cache, b):
        from compressed_long_context_hca_b200 import binding as B
        c = B.HcaCache()
        c.kc_pool, c.vc_pool = cache.c.kc_pool, cache.c.vc_pool
        c.page_table = cache.page_table[b].data_ptr()
        c.n_entries = cache.n_entries[b:b + 1].data_ptr()
        c.page_entries, c.max_pages, c.num_pages = (cache.c.page_entries, cache.c.max_pages,
                                                    cache.c.num_pages)
        c.err_word = cache.c.err_word
        self.c = c


def _prefill_kernel_sha():
    import hashlib
    src = os.path.join(ROOT, "compressed_long_context_hca_b200", "csrc", PREFILL_KERNEL_SRC)
    with open(src, "rb") as f:
        return hashlib.sha1(f.read()).hexdigest()[:12]


def _prefill_128k_result(tf, ms, per_gpu, world, peaks, clk):
    traffic = PREFILL_128K_TRAFFIC.get(_prefill_kernel_sha()) if world == 1 else None
    return {"value": round(tf, 2), "unit": "TFLOP/s", "ms_per_step": round(ms, 3),
            "workload": "batch 2 x 131072, 64 heads, 1 KV head, head_dim 512, every 4th block "
                        "x4, fused gate",
            "parallelism": f"query rows x{world}" if world > 1 else "single GPU",
            "gpu_launches_per_step": 2,
            "roofline": {"bound": "tensor", "achieved": round(per_gpu, 1),
                         "peak": peaks["bf16_tflops_sustained"], "unit": "TFLOP/s",
                         "frac": round(per_gpu / peaks["bf16_tflops_sustained"], 4),
                         "traffic": traffic, "kernel": "prefill_pair_kernel",
                         "peak_source": "measured bf16 dense sustained (a 53 ms step under "
                                        "the power cap)"},
            "clocks": clk}


def bench_backward_32k(args, dev, rank, world, barrier, max_over_ranks, peaks):
    """The prefill backward (hca_attn_prefill_backward) of the 32K workload (1 x 32768,
    64 heads, head_dim 512, N(0,1) bf16, gate off) for an N(0,1) output gradient. The
    forward (compress + prefill with lse) runs once, untimed; every step is one backward
    call. Algorithmic work: 5 products per visible query-key pair (S, dP, dQ, dK, dV),
    10 * head_dim * heads FLOPs per pair. Single GPU (the backward is not partitioned)."""
    import torch
    from compressed_long_context_hca_b200 import binding as B
    from compressed_long_context_hca_b200 import ops
    T = 32768
    g = torch.Generator(device=dev)
    g.manual_seed(6000 + rank)
    Q = torch.randn((1, T, HQ, D), generator=g, device=dev).to(torch.bfloat16)
    K = torch.randn((1, T, 1, D), generator=g, device=dev).to(torch.bfloat16)
    V = torch.randn((1, T, 1, D), generator=g, device=dev).to(torch.bfloat16)
    dO = torch.randn((1, T, HQ, D), generator=g, device=dev).to(torch.bfloat16)
    desc = ops.desc_for_prefill(Q, K)
    cache = B.PagedCache(1, T // BLOCK, 1, D, torch.bfloat16, 128, device=dev)
    ops.compress(desc, K, V, cache)
    _, lse, _ = ops.prefill(desc, Q, K, V, cache, want_lse=True)
    n = B.hca_prefill_backward_workspace_bytes(desc)
    ws = torch.empty(n, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    fn = lambda: ops.prefill_backward(desc, Q, K, V, cache, lse, dO, workspace=ws)  # noqa: E731
    clocks = Clocks(dev.index)
    clocks.start()
    ms = _time_loop(fn, args.steps_bwd, 1, barrier, max_over_ranks, stream)
    clk = clocks.stop()
    assert int(cache.err.item()) == 0, "kernel raised an error bit"
    c, w = visible_pairs(T)
    flops = 10.0 * D * HQ * (c + w)
    tf = flops / (ms * 1e-3) / 1e12
    return {"value": round(tf, 2), "unit": "TFLOP/s", "ms_per_step": round(ms, 3),
            "workload": "prefill backward, batch 1 x 32768, 64 heads, 1 KV head, head_dim 512, "
                        "N(0,1) bf16, gate off; dQ, dK, dV",
            "workspace_bytes": n,
            "roofline": {"bound": "tensor", "achieved": round(tf, 1),
                         "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                         "frac": round(tf / peaks["bf16_tflops"], 4),
                         "peak_source": "measured bf16 dense burst",
                         "note": "algorithmic FLOPs (5 products per visible pair); the "
                                 "kernels run the window as 256-key bands and every P / dS "
                                 "product twice (bf16 hi + lo)"},
            "clocks": clk}


def bench_gate_from_latent(args, dev, rank, world, barrier, max_over_ranks, peaks):
    """The gate from the query latent for the 32K workload: G [32768, 64, 512] =
    sigmoid(q_lat [32768, 1024] . W_g [1024, 32768]) (hca_gate_from_latent, one GEMM)."""
    import torch
    from compressed_long_context_hca_b200 import ops
    rows, L = 32768, 1024
    g = torch.Generator(device=dev)
    g.manual_seed(7000 + rank)
    q = torch.randn((rows, L), generator=g, device=dev).to(torch.bfloat16)
    W = (torch.randn((L, HQ * D), generator=g, device=dev) / 32).to(torch.bfloat16)
    G = torch.empty((rows, HQ, D), dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream()
    clocks = Clocks(dev.index)
    clocks.start()
    ms = _time_loop(lambda: ops.gate_from_latent(q, W, HQ, D, G=G), args.decode_steps, 3,
                    barrier, max_over_ranks, stream)
    clk = clocks.stop()
    tf = 2.0 * rows * L * HQ * D / (ms * 1e-3) / 1e12
    return {"value": round(tf, 1), "unit": "TFLOP/s", "ms_per_step": round(ms, 4),
            "workload": "G = sigmoid(q_lat . W_g): 32768 x 1024 latent, 1024 x 32768 weights, "
                        "bf16 gate [32768, 64, 512] out",
            "roofline": {"bound": "tensor", "achieved": round(tf, 1),
                         "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                         "frac": round(tf / peaks["bf16_tflops"], 4),
                         "peak_source": "measured bf16 dense burst"},
            "clocks": clk}


# ------------------------------------------------------------------ reference arm
def reference_main(args, rank, world):
    if rank != 0:
        return None
    per_step = max(1.0, args.ref_seconds)
    vals = []
    threads = blas_threads()
    for _ in range(args.warmup):
        oracle_sample_prefill(min(1.0, per_step), args.seqlen)
    n_tot, wall_tot = 0, 0.0
    for _ in range(args.steps):
        tf, n, wall, threads = oracle_sample_prefill(per_step, args.seqlen)
        vals.append(tf)
        n_tot += n
        wall_tot += wall
    v = sum(vals) / len(vals)
    return {"metric": "HCA prefill TFLOP/s at d=512 (32K bf16, compress+prefill step); "
                      "decode tokens/s in decode_batched / decode_1m",
            "value": v, "unit": "TFLOP/s", "impl": "reference", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(1e3 * wall_tot / args.steps, 1), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": "HCA prefill bf16: batch 1, T=32768, 64 query heads, 1 KV "
                                   "head, head_dim 512, block 128, window 128, gate off",
                       "global_batch": 1, "seq_len": args.seqlen, "parallelism": "host cores"},
            "cpu_baseline": {"value": v, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                             "sample": f"{n_tot} random query positions x 64 heads in "
                                       f"{args.steps} steps of {per_step:.0f} s"},
            "e2e": {"value": v, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def profile_case(args):
    """Small fixed case for ncu captures: compress + 2 prefill launches (or 2 decode
    launches, or 2 compress launches over 2 sequences); no timing. ``--profile prefill
    --seqlen T``, ``--profile decode --nseq N --ctx C`` or ``--profile compress --seqlen T``."""
    import torch
    from compressed_long_context_hca_b200 import binding as B
    from compressed_long_context_hca_b200 import build as build_mod
    from compressed_long_context_hca_b200 import ops
    build_mod.build()
    dev = torch.device("cuda")
    g = torch.Generator(device=dev)
    g.manual_seed(0)
    if args.profile == "compress":
        T = args.seqlen
        K = torch.randn((2, T, 1, D), generator=g, device=dev).to(torch.bfloat16)
        V = torch.randn((2, T, 1, D), generator=g, device=dev).to(torch.bfloat16)
        desc = ops.desc_for_prefill(K, K)
        cache = B.PagedCache(2, -(-T // BLOCK), 1, D, torch.bfloat16, 128, device=dev)
        for _ in range(2):
            ops.compress(desc, K, V, cache)
    elif args.profile in ("prefill", "prefill_gate"):
        # prefill_gate: the 2 x 128K leg's features (every 4th block x4, fused gate)
        T = args.seqlen
        blk = ((torch.arange(T, device=dev) // BLOCK) % 4 == 3)

        def draw(h):
            x = torch.randn((1, T, h, D), generator=g, device=dev)
            if args.profile == "prefill_gate":
                x[:, blk] *= 4.0
            return x.to(torch.bfloat16)

        Q, K, V = draw(HQ), draw(1), draw(1)
        desc = ops.desc_for_prefill(Q, K)
        if args.profile == "prefill_gate":
            G = torch.sigmoid(torch.randn((1, T, HQ, D), generator=g, device=dev))
            ops.attach_gate(desc, G.to(torch.bfloat16))
        cache = B.PagedCache(1, -(-T // BLOCK), 1, D, torch.bfloat16, 128, device=dev)
        O = torch.empty_like(Q)
        ops.compress(desc, K, V, cache)
        for _ in range(2):
            ops.prefill(desc, Q, K, V, cache, O=O)
    elif args.profile == "backward":
        T = args.seqlen
        Q = torch.randn((1, T, HQ, D), generator=g, device=dev).to(torch.bfloat16)
        K = torch.randn((1, T, 1, D), generator=g, device=dev).to(torch.bfloat16)
        V = torch.randn((1, T, 1, D), generator=g, device=dev).to(torch.bfloat16)
        dO = torch.randn((1, T, HQ, D), generator=g, device=dev).to(torch.bfloat16)
        desc = ops.desc_for_prefill(Q, K)
        cache = B.PagedCache(1, -(-T // BLOCK), 1, D, torch.bfloat16, 128, device=dev)
        ops.compress(desc, K, V, cache)
        _, lse, _ = ops.prefill(desc, Q, K, V, cache, want_lse=True)
        for _ in range(2):
            ops.prefill_backward(desc, Q, K, V, cache, lse, dO)
    else:
        nseq, ctx = args.nseq, args.ctx
        nent = (ctx - WIN) // BLOCK + 1
        e4m3 = args.profile == "decode_e4m3"
        cache = B.PagedCache(nseq, nent, 1, D, torch.bfloat16, 128, device=dev,
                             e4m3_scales=E4M3_SCALES if e4m3 else None)
        if e4m3:
            _fill_e4m3(cache.kc, g)
            _fill_e4m3(cache.vc, g)
        else:
            cache.kc.normal_(generator=g)
            cache.vc.normal_(generator=g)
        cache.n_entries.fill_(nent)
        q = torch.randn((nseq, HQ, D), generator=g, device=dev).to(torch.bfloat16)
        rk = torch.randn((nseq, WIN, 1, D), generator=g, device=dev).to(torch.bfloat16)
        rv = torch.randn((nseq, WIN, 1, D), generator=g, device=dev).to(torch.bfloat16)
        ctx_t = torch.full((nseq,), ctx, dtype=torch.int32, device=dev)
        desc = B.make_desc(nseq, ctx, HQ, 1, D)
        ws = ops.decode_workspace(desc, dev)
        for _ in range(2):
            ops.decode(desc, q, ctx_t, cache, rk, rv, workspace=ws)
    torch.cuda.synchronize()
    assert int(cache.err.item()) == 0
    print(f"profile case {args.profile} done")


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--seqlen", type=int, default=32768)
    ap.add_argument("--decode-steps", type=int, default=50)
    ap.add_argument("--steps-128k", type=int, default=10)
    ap.add_argument("--e2e-steps", type=int, default=12,
                    help="steps of the 32K e2e pipeline (fill and drain amortised over them)")
    ap.add_argument("--steps-bwd", type=int, default=5)
    ap.add_argument("--no-backward", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--ref-seconds", type=float, default=10.0)
    ap.add_argument("--traffic", type=float, default=None,
                    help="dram bytes per prefill launch from an ncu capture of this build")
    ap.add_argument("--with-128k", action="store_true", default=True)
    ap.add_argument("--no-128k", dest="with_128k", action="store_false")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-e4m3", action="store_true", help="skip the 8-bit cache decode legs")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--profile", choices=["prefill", "prefill_gate", "decode", "decode_e4m3",
                                          "compress", "backward"], default=None,
                    help="run a small fixed case for ncu and exit")
    ap.add_argument("--nseq", type=int, default=16)
    ap.add_argument("--ctx", type=int, default=1048576)
    args = ap.parse_args()
    if args.profile:
        profile_case(args)
        return
    if args.warmup < 3:
        args.warmup = 3

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        res = reference_main(args, rank, world)
        if rank == 0 and res is not None:
            print(json.dumps(res), flush=True)
        return
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    try:
        res = gpu_main(args, rank, world, local_rank)
        if rank == 0 and res is not None:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.barrier()
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
