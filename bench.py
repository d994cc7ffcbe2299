#!/usr/bin/env python
"""Benchmark of the VSA forward path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

A step is one pass of the whole path over one batch: tile q, k, v into
cubes and pool them per cube (one pass over the inputs); coarse attention and
top-k; fine block-sparse attention, whose epilogue applies the gated combine
and writes the token-order output (the untile step).  Inputs are drawn once on the host from the
seeded synthetic recipe and are resident in HBM before the timed region; each
input tensor (774 MB at the default workload) is larger than the 126 MB L2,
so no flush is needed between steps.

Metric: effective TFLOP/s of the whole call, counting only the FLOPs the
chosen sparsity needs: 4*d*sum_i n_i*sum_{j in sel(i)} n_j for the fine stage
(valid tokens of the actual selection) plus 4*d*C^2 per head for the coarse
attention.  ms/call is ``ms_per_step``.

Prints ONE JSON line on rank 0.  With ``--impl reference`` the same metric is
measured for the CPU oracle (float64 NumPy) on a bounded sample of the
workload on the host cores.
"""

from __future__ import annotations

import argparse
import csv
import dataclasses
import io
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from video_dit_block_vsa_b200 import workloads as wl  # noqa: E402

DEFAULT_WORKLOAD = "wan14b_720p_21x45x80_k180"
METRIC = "block-sparse attention ms/call & effective TFLOP/s (% bf16 peak), 1 B200"


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return dict(hbm=p["hbm_gbs"], bf16=p["bf16_tflops"], bf16_sustained=p["bf16_tflops_sustained"],
                    source="measured")
    except (OSError, KeyError, ValueError):
        return dict(hbm=6650.0, bf16=1590.0, bf16_sustained=1400.0, source="fallback")


def cube_counts(grid):
    """Valid tokens per cube for a 4x4x4 tiling (bench accounting only)."""
    T, Y, X = grid
    ct = np.minimum(4, T - 4 * np.arange(-(-T // 4)))
    cy = np.minimum(4, Y - 4 * np.arange(-(-Y // 4)))
    cx = np.minimum(4, X - 4 * np.arange(-(-X // 4)))
    return (ct[:, None, None] * cy[None, :, None] * cx[None, None, :]).reshape(-1).astype(np.int64)


def key_chunks(counts, sel):
    """16-row key chunks the fine kernel loads and multiplies per query cube:
    4 for a selected cube with more than 16 valid tokens, 1 otherwise."""
    per_cube = np.where(counts > 16, 4, 1)
    return per_cube[sel].sum(axis=-1)          # [B, H, C]


def flop_counts(w, counts, sel):
    """(fine effective FLOPs, fine issued FLOPs, coarse FLOPs) of one call.
    Issued: every query cube's 64 rows against its packed key chunks."""
    d, C = w.head_dim, counts.shape[0]
    nsel = counts[sel]                         # [B, H, C, k]
    fine_eff = 4.0 * d * float(np.sum(counts[None, None, :] * nsel.sum(axis=-1)))
    fine_issued = 4.0 * d * 64 * 16 * float(key_chunks(counts, sel).sum())
    coarse = 4.0 * d * w.batch * w.heads * C * C
    return fine_eff, fine_issued, coarse


class ClockSampler:
    """nvidia-smi clock/throttle sampling during the timed region."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=10)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        rows = [r for r in csv.reader(io.StringIO(out)) if len(r) >= 9]
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].strip().replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].strip().replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v.strip() == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons, "samples": len(rows)}


# ------------------------------------------------------------------ oracle (CPU)

def oracle_sample(w, x, time_budget_s, cubes_cap=None):
    """Runs the oracle head by head (batch 0, heads 0, 1, ...) until the time
    budget: a head that fits runs the whole path (tile q, k, v; pool, coarse
    attention, top-k; fine attention over every query cube; combine; untile),
    the head that meets the budget runs its fine stage cube by cube until it
    runs out.  ``cubes_cap`` limits the first head to that many query cubes.
    Returns (seconds, effective FLOPs processed, description, per-stage
    seconds summed over whole heads, whole heads)."""
    from oracle import vsa_oracle as vo
    t0 = time.perf_counter()
    C, d = w.cubes, w.head_dim
    flops = 0.0
    stages = dict(tile_permute=0.0, coarse_select=0.0, block_sparse_fwd=0.0, combine=0.0, untile=0.0)
    full_heads, partial = 0, None

    def clock(name, fn, *a, **kw):
        s0 = time.perf_counter()
        r = fn(*a, **kw)
        stages_head[name] += time.perf_counter() - s0
        return r

    for h in range(w.heads):
        stages_head = dict.fromkeys(stages, 0.0)
        one = lambda n: vo.bf16_bits_to_f64(x[n][0:1, h:h + 1])
        q_t, counts = clock("tile_permute", vo.tile_permute, one("q"), w.grid)
        k_t, _ = clock("tile_permute", vo.tile_permute, one("k"), w.grid)
        v_t, _ = clock("tile_permute", vo.tile_permute, one("v"), w.grid)
        s0 = time.perf_counter()
        S, O_c = vo.coarse_attention(vo.pool(q_t, counts), vo.pool(k_t, counts), vo.pool(v_t, counts))
        sel = vo.topk_select(S, w.topk)
        stages_head["coarse_select"] += time.perf_counter() - s0
        flops += 4.0 * d * C * C
        O_f = np.zeros_like(q_t)
        done = 0
        while done < C and (cubes_cap is None or done < cubes_cap):
            s0 = time.perf_counter()
            o, _ = vo.block_sparse_attention(q_t, k_t, v_t, counts, sel, query_cubes=[done])
            stages_head["block_sparse_fwd"] += time.perf_counter() - s0
            O_f[:, :, 64 * done:64 * done + 64] = o[:, :, 64 * done:64 * done + 64]
            flops += 4.0 * d * counts[done] * counts[sel[0, 0, done]].sum()
            done += 1
            if time.perf_counter() - t0 > time_budget_s:
                break
        if done < C:
            partial = (h, done)
            break
        gf = x["g_f"][0:1, h:h + 1].astype(np.float64) if w.gated else None
        gc = x["g_c"][0:1, h:h + 1].astype(np.float64) if w.gated else None
        out_t = clock("combine", vo.combine, O_f, O_c, counts, w.grid, gf, gc)
        clock("untile", vo.untile, out_t, w.grid)
        for k_ in stages:
            stages[k_] += stages_head[k_]
        full_heads += 1
        if time.perf_counter() - t0 > time_budget_s:
            break
    dt = time.perf_counter() - t0
    desc = (f"batch 0: the whole path for {full_heads} of {w.batch * w.heads} head(s)"
            + (f", plus tile/coarse/top-k and query cubes 0..{partial[1] - 1} of head {partial[0]}"
               if partial else ""))
    return dt, flops, desc, stages, full_heads


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads") for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else os.cpu_count()
    except Exception:  # pragma: no cover
        return os.cpu_count()


def run_reference(args, w):
    from video_dit_block_vsa_b200 import dist as vdist
    if vdist.rank_info().rank != 0:  # rank 0 alone times the CPU oracle
        return 0
    x = wl.make_inputs(w)
    per_step_budget = 8.0
    for _ in range(args.warmup):
        oracle_sample(w, x, per_step_budget, cubes_cap=4)
    tot_t = tot_f = 0.0
    desc = ""
    for _ in range(args.steps):
        dt, fl, desc, _, _ = oracle_sample(w, x, per_step_budget)
        tot_t += dt
        tot_f += fl
    value = tot_f / tot_t / 1e12
    cores = blas_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * tot_t / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_dict(w),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": desc + f"; {args.steps} steps"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def config_dict(w):
    C = w.cubes
    return {"workload": w.name, "batch": w.batch, "heads": w.heads, "head_dim": w.head_dim,
            "grid": list(w.grid), "tokens": w.tokens, "cubes": C, "topk": w.topk,
            "sparsity": round(1.0 - w.topk / C, 4), "gated": w.gated,
            "l2": "inputs larger than L2 (no flush)"}


# ------------------------------------------------------------------ GPU arm

def run_gpu(args, w):
    import torch

    from video_dit_block_vsa_b200 import dist as vdist
    ri = vdist.rank_info()
    world, rank, local = ri.world, ri.rank, ri.local_rank
    torch.cuda.set_device(local)
    vdist.init("nccl")

    from video_dit_block_vsa_b200 import vsa

    peaks = load_peaks()
    x = wl.make_inputs(w)
    shape = vsa.make_shape(w.batch, w.heads, w.head_dim, w.grid)
    dev = torch.device("cuda", local)
    to_dev = lambda b: torch.from_numpy(b.view(np.int16)).to(dev).view(torch.bfloat16)
    q, k, v = to_dev(x["q"]), to_dev(x["k"]), to_dev(x["v"])
    g_f = torch.from_numpy(x["g_f"]).to(dev) if w.gated else None
    g_c = torch.from_numpy(x["g_c"]).to(dev) if w.gated else None
    out = torch.empty_like(q)
    bufs = vsa.VsaBuffers(shape, w.topk, device=dev, want_coarse=w.gated)
    stream = torch.cuda.current_stream()

    def step(ev=None):
        def mark(i):
            if ev is not None:
                ev[i].record(stream)
        mark(0)
        # one pass over q, k, v: tiled copies plus the cube means of the coarse stage
        vsa.vsa_tile_permute_pool(shape, q, k, v, bufs.q_t, bufs.k_t, bufs.v_t, bufs.workspace,
                                  bufs.counts)
        mark(1)
        vsa.vsa_coarse_select_pooled(shape, w.topk, bufs.sel, bufs.workspace, o_coarse=bufs.o_c)
        mark(2)
        # fine attention whose epilogue applies the gated combine (if gated) and
        # writes the token-order output: the combine and untile steps, fused
        vsa.vsa_block_sparse_fwd_out(shape, bufs.q_t, bufs.k_t, bufs.v_t, bufs.counts, bufs.sel,
                                     w.topk, out, bufs.o_c if w.gated else None, g_f, g_c)
        mark(3)

    launches_per_step = 3

    for _ in range(max(args.warmup, 1)):
        step()
    torch.cuda.synchronize()
    status = vsa.vsa_get_status()
    if status != 0:
        raise RuntimeError(f"device status after warm-up: {vsa.vsa_strerror(status)}")
    counts = cube_counts(w.grid)
    fine_eff, fine_issued, coarse_fl = flop_counts(w, counts, bufs.sel.cpu().numpy().astype(np.int64))
    step_flops = fine_eff + coarse_fl

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    clocks = ClockSampler(local)
    vdist.barrier(ri)
    torch.cuda.synchronize()
    clocks.start()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for s in range(args.steps):
        step(evs[s])
    t_end.record(stream)
    torch.cuda.synchronize()
    vdist.barrier(ri)
    clk = clocks.stop()
    elapsed_ms = vdist.max_over_ranks(t_start.elapsed_time(t_end), ri, dev)
    status = vsa.vsa_get_status()
    if status != 0:
        raise RuntimeError(f"device status after timed steps: {vsa.vsa_strerror(status)}")
    # stage "tile_permute" is the one pass that tiles q, k, v and pools them;
    # "coarse_select" is the coarse attention, top-k and O_c from those means;
    # "block_sparse_fwd" is the fine kernel with the combine and untile steps
    # in its epilogue
    pairs = {"tile_permute": (0, 1), "coarse_select": (1, 2), "block_sparse_fwd": (2, 3)}
    stage_all = {name: [evs[s][a_].elapsed_time(evs[s][b_]) for s in range(args.steps)]
                 for name, (a_, b_) in pairs.items()}
    stage_ms = {name: statistics.mean(v_) for name, v_ in stage_all.items()}
    step_all = [evs[s][0].elapsed_time(evs[s][3]) for s in range(args.steps)]
    spread = lambda v_: {"mean": statistics.mean(v_), "median": statistics.median(v_), "min": min(v_)}
    ms_per_step = elapsed_ms / args.steps
    value = vdist.job_throughput(step_flops, args.steps, elapsed_ms, world) / 1e12

    # ---- end to end through the host-buffer entry point (pinned host memory):
    # every step copies q, k, v (and gates) in and the output out, in chunks of
    # heads that overlap the copies with the kernels.
    hq, hk, hv = (t.cpu().pin_memory() for t in (q, k, v))
    hgf = g_f.cpu().pin_memory() if w.gated else None
    hgc = g_c.cpu().pin_memory() if w.gated else None
    hout = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
    chunk = args.host_chunk_heads
    hws = torch.empty(vsa.vsa_forward_host_workspace_bytes(shape, w.topk, chunk, w.gated),
                      dtype=torch.uint8, device=dev)

    def e2e_step():
        vsa.vsa_forward_host(shape, w.topk, hq, hk, hv, hout, hws, hgf, hgc, chunk)

    e2e_step()
    torch.cuda.synchronize()
    vdist.barrier(ri)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = vdist.max_over_ranks(e0.elapsed_time(e1), ri, dev)
    status = vsa.vsa_get_status()
    if status != 0:
        raise RuntimeError(f"device status after end-to-end steps: {vsa.vsa_strerror(status)}")
    h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv))
    if w.gated:
        h2d += hgf.numel() * 4 + hgc.numel() * 4
    d2h = hout.numel() * hout.element_size()

    # ---- roofline of the dominant kernel (fine block-sparse attention)
    fine_ms = stage_ms["block_sparse_fwd"]
    achieved = fine_eff / (fine_ms * 1e-3) / 1e12
    traffic_path = os.path.join(ROOT, "profiles", "fine_traffic.json")
    traffic = None
    try:
        with open(traffic_path) as f:
            tj = json.load(f)
        if tj.get("workload") == w.name and tj.get("kernel_rev") == KERNEL_REV:
            traffic = tj.get("bytes_per_launch")
    except (OSError, ValueError):
        pass
    # The fine kernel's other roofline: every packed K/V chunk and every Q tile
    # is moved from L2 into shared memory by TMA, and one SM sustains
    # TMA_INGEST_GBS_PER_SM.
    chunks = float(key_chunks(counts, bufs.sel.cpu().numpy().astype(np.int64)).sum())
    kv_bytes = (chunks * 2 * 16 + float(w.batch * w.heads * w.cubes) * 64) * w.head_dim * 2
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    feed_peak = TMA_INGEST_GBS_PER_SM * sms / 1e3
    feed = {"path": "L2 -> shared memory (TMA)", "bytes": kv_bytes,
            "achieved": kv_bytes / (fine_ms * 1e-3) / 1e12, "peak": feed_peak, "unit": "TB/s",
            "frac": kv_bytes / (fine_ms * 1e-3) / 1e12 / feed_peak,
            "peak_kind": f"{TMA_INGEST_GBS_PER_SM} GB/s per SM (measured) x {sms} SMs"}
    # The fine kernel runs for tens of milliseconds inside a step of the same
    # length, so its denominator is the burst bf16 figure; the sustained
    # (seconds-long, power-capped) figure is reported beside it.
    roofline = {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16"],
                "unit": "TFLOP/s", "frac": achieved / peaks["bf16"], "traffic": traffic,
                "kernel": "vsa_block_sparse_fwd_out (fine attention; combine and untile in its epilogue)",
                "peak_kind": f"bf16 burst ({peaks['source']})",
                "peak_sustained": peaks["bf16_sustained"],
                "frac_of_sustained": achieved / peaks["bf16_sustained"],
                "kernel_ms": spread(stage_all["block_sparse_fwd"]),
                "issued_tflops": fine_issued / (fine_ms * 1e-3) / 1e12, "feed": feed}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        dt, fl, desc, st, nh = oracle_sample(w, x, args.cpu_seconds)
        cpu = {"value": fl / dt / 1e12, "unit": "TFLOP/s", "cores": blas_threads(),
               "kind": "oracle", "sample": desc + f", {dt:.1f} s"}
        if nh:
            per_head = {k_: v_ / nh for k_, v_ in st.items()}
            cpu["stages_s_per_head"] = per_head
            cpu["s_per_call_extrapolated"] = sum(per_head.values()) * w.batch * w.heads

    if rank == 0:
        hbm_bytes = {
            # read q, k, v once; write the tiled copies and the float32 cube means
            "tile_permute": (3 * w.batch * w.heads * (w.tokens + 64 * w.cubes) * w.head_dim * 2
                             + 3 * w.batch * w.heads * w.cubes * w.head_dim * 4),
        }
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded N(0,1) + per-cube mean N(0,0.5^2), bf16)",
            "config": config_dict(w),
            "roofline": roofline,
            "cpu_baseline": cpu,
            "e2e": {"value": vdist.job_throughput(step_flops, args.steps, e2e_ms, world) / 1e12,
                    "unit": "TFLOP/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "ms_per_step": e2e_ms / args.steps, "api": "vsa_forward_host",
                    "heads_per_chunk": chunk},
            "gpu_launches": launches_per_step * args.steps,
            "clocks": clk,
            "stages_ms": stage_ms,
            "step_ms": spread(step_all),
            "stages_note": ("tile_permute is one pass that tiles q, k, v and writes their cube "
                            "means (the coarse stage's pooling); coarse_select starts from those; "
                            "block_sparse_fwd writes the final token-order output, applying the "
                            "gated combine in its epilogue (the combine and untile steps)"),
            "stages_gbs": {k: v / (stage_ms[k] * 1e-3) / 1e9 for k, v in hbm_bytes.items()},
            "flops": {"fine_effective": fine_eff, "fine_issued": fine_issued, "coarse": coarse_fl},
            "kernel_rev": KERNEL_REV,
        }
        print(json.dumps(line), flush=True)
    vdist.shutdown(ri)
    return 0


# Sustained TMA ingest of one SM for random 64-row x 128-byte swizzled boxes
# from L2, measured on B200 with one issuing thread filling a ring of 32 KB
# slots (148 SMs loading at once): the best of the probe layouts, 99.3 GB/s.
TMA_INGEST_GBS_PER_SM = 99.3

# (b, h) planes per chunk of the host-buffer path in the end-to-end leg.
HOST_CHUNK_HEADS = 2

def run_backward_pieces(args, w):
    """Times the backward pieces built so far on the workload (one GPU, not the
    default bench line): the combine-gradient prep pass, the selection
    transpose and the coarse attention backward, each after a forward that
    leaves O_f tiled, the selection and O_c resident.  Prints one JSON line."""
    import torch

    from video_dit_block_vsa_b200 import vsa

    x = wl.make_inputs(w)
    shape = vsa.make_shape(w.batch, w.heads, w.head_dim, w.grid)
    dev = torch.device("cuda", 0)
    to_dev = lambda b: torch.from_numpy(b.view(np.int16)).to(dev).view(torch.bfloat16)
    q, k, v = to_dev(x["q"]), to_dev(x["k"]), to_dev(x["v"])
    B, H, N, d, C = w.batch, w.heads, w.tokens, w.head_dim, w.cubes
    bufs = vsa.VsaBuffers(shape, w.topk, device=dev, want_lse=True)
    vsa.vsa_tile_permute_pool(shape, q, k, v, bufs.q_t, bufs.k_t, bufs.v_t, bufs.workspace,
                              bufs.counts)
    vsa.vsa_coarse_select_pooled(shape, w.topk, bufs.sel, bufs.workspace, o_coarse=bufs.o_c)
    vsa.vsa_block_sparse_fwd(shape, bufs.q_t, bufs.k_t, bufs.v_t, bufs.counts, bufs.sel, w.topk,
                             bufs.o_f, bufs.lse)
    rng = np.random.default_rng(w.seed + 1)
    dout = to_dev(wl.f32_to_bf16_bits(rng.standard_normal((B, H, N, d), dtype=np.float32)))
    g_f = torch.full((B, H, N), 0.5, dtype=torch.float32, device=dev)
    g_c = torch.full((B, H, N), 0.5, dtype=torch.float32, device=dev)
    dof = torch.empty_like(bufs.o_f)
    delta = torch.empty(B, H, 64 * C, dtype=torch.float32, device=dev)
    doc = torch.empty(B, H, C, d, dtype=torch.float32, device=dev)
    dgf = torch.empty(B, H, N, dtype=torch.float32, device=dev)
    dgc = torch.empty_like(dgf)
    offs = torch.empty(B, H, C + 1, dtype=torch.int32, device=dev)
    lists = torch.empty(B, H, C * w.topk, dtype=torch.int32, device=dev)
    t_ws = torch.empty(B * H * C * w.topk * 4, dtype=torch.uint8, device=dev)
    d_pooled = torch.empty(3, B, H, C, d, dtype=torch.float32, device=dev)
    c_ws = torch.empty(vsa.vsa_coarse_backward_workspace_bytes(shape), dtype=torch.uint8, device=dev)
    pooled = vsa.pooled_view(shape, bufs.workspace)
    stream = torch.cuda.current_stream()
    dq, dk, dv = (torch.empty_like(q) for _ in range(3))
    pieces = {
        "backward_prep": lambda: vsa.vsa_backward_prep(shape, dout, bufs.o_f, dof, delta, bufs.o_c,
                                                       g_f, g_c, doc, dgf, dgc),
        "select_transpose": lambda: vsa.vsa_select_transpose(shape, bufs.sel, w.topk, offs, lists,
                                                             t_ws),
        "coarse_backward": lambda: vsa.vsa_coarse_backward(shape, pooled, bufs.o_c, doc, d_pooled,
                                                           c_ws),
        "fine_backward": lambda: vsa.vsa_block_sparse_bwd(shape, bufs.q_t, bufs.k_t, bufs.v_t,
                                                          bufs.sel, w.topk, offs, lists, bufs.lse,
                                                          dof, delta, dq, dk, dv, d_pooled),
    }
    ms = {}
    for name, fn in pieces.items():
        for _ in range(max(args.warmup, 1)):
            fn()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        a.record(stream)
        for _ in range(args.steps):
            fn()
        b.record(stream)
        torch.cuda.synchronize()
        ms[name] = a.elapsed_time(b) / args.steps
    status = vsa.vsa_get_status()
    if status != 0:
        raise RuntimeError(f"device status: {vsa.vsa_strerror(status)}")
    peaks = load_peaks()
    valid = N * B * H  # valid rows over all (b, h)
    # prep: dout, O_f (valid rows), gates read; dO_f, delta (all 64*C rows),
    # dO_c, dg_f, dg_c written
    prep_bytes = (valid * d * 2 * 2 + valid * 4 * 2 + B * H * 64 * C * (d * 2 + 4)
                  + B * H * C * d * 4 + valid * 4 * 2 + B * H * C * d * 4)
    # coarse backward: the 5 C x C x d products (S, dP, dQ, dK, dV) of a
    # backward, 2 flops each multiply-add
    coarse_flops = 10.0 * B * H * C * C * d
    # fine backward: per (query cube, selected key cube) the products S, dP, dQ
    # (query side) and S^T, dP^T, dK, dV (key side) over valid tokens only
    counts = cube_counts(w.grid)
    sel_np = bufs.sel.cpu().numpy().astype(np.int64)
    pair_tokens = float(np.sum(counts[None, None, :] * counts[sel_np].sum(axis=-1)))
    fine_bwd_flops = 14.0 * d * pair_tokens
    # issued: the 7 products run on whole 64 x 64 blocks
    fine_bwd_issued = 14.0 * d * 64 * 64 * float(sel_np.size)
    line = {"mode": "backward_pieces", "workload": w.name, "steps": args.steps,
            "warmup": args.warmup, "ms": {k_: round(v_, 4) for k_, v_ in ms.items()},
            "backward_prep": {"algorithmic_bytes": prep_bytes,
                              "achieved_gbs": round(prep_bytes / ms["backward_prep"] / 1e6, 1),
                              "peak_gbs": peaks["hbm"], "peak_source": peaks["source"],
                              "gated": True},
            "coarse_backward": {"algorithmic_flops": coarse_flops,
                                "achieved_tflops": round(coarse_flops / ms["coarse_backward"] / 1e9, 2),
                                "dtype": "f32", "note": "SIMT float32 register-tiled products"},
            "fine_backward": {"algorithmic_flops": fine_bwd_flops,
                              "achieved_tflops": round(fine_bwd_flops / ms["fine_backward"] / 1e9, 2),
                              "issued_flops": fine_bwd_issued,
                              "issued_tflops": round(fine_bwd_issued / ms["fine_backward"] / 1e9, 2),
                              "peak_tflops": peaks["bf16"], "peak_source": peaks["source"],
                              "frac": round(fine_bwd_flops / ms["fine_backward"] / 1e9 / peaks["bf16"], 4),
                              "dtype": "bf16",
                              "note": "tcgen05 (M = 64) products, float32 accumulation; 7 products "
                                      "per block pair (S and dP in both the dq and the dk/dv kernel)"}}
    print(json.dumps(line))
    return 0


def run_sparse_linear(args, w):
    """Times the sparse + linear forward on the workload (one GPU, not the
    default bench line): the three-launch block-sparse forward, then the
    low-rank linear compensation branch added to its output in place.  The
    branch moves little data per flop (two d x d products per token), so its
    roofline is HBM: q, k, v read once and the output read and written.
    Prints one JSON line."""
    import torch

    from video_dit_block_vsa_b200 import vsa

    x = wl.make_inputs(w)
    shape = vsa.make_shape(w.batch, w.heads, w.head_dim, w.grid)
    dev = torch.device("cuda", 0)
    to_dev = lambda b: torch.from_numpy(b.view(np.int16)).to(dev).view(torch.bfloat16)
    q, k, v = to_dev(x["q"]), to_dev(x["k"]), to_dev(x["v"])
    B, H, N, d = w.batch, w.heads, w.tokens, w.head_dim
    g_f = torch.from_numpy(x["g_f"]).to(dev) if w.gated else None
    g_c = torch.from_numpy(x["g_c"]).to(dev) if w.gated else None
    out = torch.empty_like(q)
    bufs = vsa.VsaBuffers(shape, w.topk, device=dev, want_coarse=w.gated)
    ws = torch.empty(vsa.vsa_linear_workspace_bytes(shape), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def forward():
        vsa.vsa_forward_fused(shape, q, k, v, w.topk, out, g_f, g_c, bufs=bufs)

    def branch():
        vsa.vsa_linear_branch_add(shape, q, k, v, out, ws)

    def both():
        forward()
        branch()

    sampler = ClockSampler(0)
    clocks = None
    ms = {}
    for name, fn in (("sparse_forward", forward), ("linear_branch", branch), ("sparse_plus_linear", both)):
        for _ in range(max(args.warmup, 3)):
            fn()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        if name == "linear_branch":
            sampler.start()
        a.record(stream)
        for _ in range(args.steps):
            fn()
        b.record(stream)
        torch.cuda.synchronize()
        if name == "linear_branch":
            clocks = sampler.stop() or {}
        ms[name] = a.elapsed_time(b) / args.steps
    status = vsa.vsa_get_status()
    if status != 0:
        raise RuntimeError(f"device status: {vsa.vsa_strerror(status)}")
    # KV = phi(K)^T V and phi(Q) KV: 2 N d^2 flops each; z and phi(Q) z: 2 N d each
    flops = float(B * H) * (4.0 * N * d * d + 4.0 * N * d)
    # compulsory HBM bytes: q, k, v read once, the output read and written
    bytes_ = float(B * H * N * d * 2) * 5
    achieved_gbs = bytes_ / ms["linear_branch"] / 1e6
    peaks = load_peaks()
    line = {"mode": "sparse_linear", "workload": w.name, "steps": args.steps,
            "warmup": max(args.warmup, 3), "ms": {k_: round(v_, 4) for k_, v_ in ms.items()},
            "linear_branch": {"bound": "hbm", "algorithmic_bytes": bytes_,
                              "achieved_gbs": round(achieved_gbs, 1), "peak_gbs": peaks["hbm"],
                              "peak_source": peaks["source"],
                              "frac": round(achieved_gbs / peaks["hbm"], 4),
                              "algorithmic_flops": flops,
                              "achieved_tflops": round(flops / ms["linear_branch"] / 1e9, 2),
                              "dtype": "bf16",
                              "note": "phi(q), phi(k) written to and read back from the "
                                      "workspace (bf16) by a separate pass; tcgen05 products "
                                      "with float32 accumulation"},
            "clocks": clocks}
    print(json.dumps(line))
    return 0


# Model width of the DiT block around the 720p workload (Wan-14B: 40 heads x 128).
DIT_HIDDEN = {"wan14b_720p_21x45x80_k180": 5120, "wan14b_720p_21x45x80_k43": 5120,
              "wan1.3b_ft_16x28x52": 1536, "wan1.3b_480p_21x30x52": 1536,
              "scaling_16x32x32": 1536}


def run_dit_block(args, w):
    """Times a DiT attention block around VSA with the layout changes fused
    into the projections (one GPU, not the default bench line): the QKV
    projection writing q, k, v tiled, the coarse stage, the fine stage
    (tiled output), and the output projection reading it tiled.  Random
    weights of the model's width; prints one JSON line."""
    import torch

    from video_dit_block_vsa_b200 import vsa

    hidden = DIT_HIDDEN.get(w.name, w.heads * w.head_dim)
    B, H, N, d = w.batch, w.heads, w.tokens, w.head_dim
    shape = vsa.make_shape(B, H, d, w.grid)
    dev = torch.device("cuda", 0)
    gen = torch.Generator(device=dev).manual_seed(w.seed)
    x = torch.randn(B, N, hidden, device=dev, generator=gen).to(torch.bfloat16)
    w_qkv = (torch.randn(3 * H * d, hidden, device=dev, generator=gen) * hidden ** -0.5).to(torch.bfloat16)
    w_o = (torch.randn(hidden, H * d, device=dev, generator=gen) * (H * d) ** -0.5).to(torch.bfloat16)
    y = torch.empty(B, N, hidden, dtype=torch.bfloat16, device=dev)
    bufs = vsa.VsaBuffers(shape, w.topk, device=dev, want_coarse=False)
    stream = torch.cuda.current_stream()
    pieces = {
        "qkv_projection_tiled": lambda: vsa.vsa_qkv_projection_tiled(
            shape, hidden, x, w_qkv, bufs.q_t, bufs.k_t, bufs.v_t, bufs.counts),
        "coarse_select": lambda: vsa.vsa_coarse_select(
            shape, bufs.q_t, bufs.k_t, bufs.v_t, bufs.counts, w.topk, bufs.sel, bufs.workspace),
        "block_sparse_fwd": lambda: vsa.vsa_block_sparse_fwd(
            shape, bufs.q_t, bufs.k_t, bufs.v_t, bufs.counts, bufs.sel, w.topk, bufs.o_f),
        "out_projection_tiled": lambda: vsa.vsa_out_projection_tiled(shape, hidden, bufs.o_f, w_o, y),
    }
    sampler = ClockSampler(0)
    ms = {}
    for name, fn in list(pieces.items()) + [("block", lambda: [f() for f in pieces.values()])]:
        for _ in range(max(args.warmup, 3)):
            fn()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        if name == "block":
            sampler.start()
        a.record(stream)
        for _ in range(args.steps):
            fn()
        b.record(stream)
        torch.cuda.synchronize()
        if name == "block":
            clocks = sampler.stop() or {}
        ms[name] = a.elapsed_time(b) / args.steps
    status = vsa.vsa_get_status()
    if status != 0:
        raise RuntimeError(f"device status: {vsa.vsa_strerror(status)}")
    peaks = load_peaks()
    qkv_flops = 2.0 * B * N * hidden * 3 * H * d
    out_flops = 2.0 * B * N * hidden * H * d
    proj = {}
    for name, fl in (("qkv_projection_tiled", qkv_flops), ("out_projection_tiled", out_flops)):
        t = fl / ms[name] / 1e9
        proj[name] = {"flops": fl, "achieved_tflops": round(t, 1), "peak_tflops": peaks["bf16"],
                      "peak_source": peaks["source"], "frac": round(t / peaks["bf16"], 4)}
    line = {"mode": "dit_block", "workload": w.name, "hidden": hidden, "steps": args.steps,
            "warmup": max(args.warmup, 3), "ms": {k_: round(v_, 4) for k_, v_ in ms.items()},
            "projections": proj, "clocks": clocks,
            "note": "tcgen05 GEMMs (128 x 256 tiles, bf16, float32 accumulation); the QKV "
                    "projection writes q, k, v in the tiled layout and the output projection "
                    "reads the tiled attention output and writes token order"}
    print(json.dumps(line))
    return 0


# Revision tag of the fine kernel; ncu traffic figures are only reported for
# the revision they were captured on.
KERNEL_REV = "fine-v7-q-in-tmem-out"


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(wl.WORKLOADS))
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=20.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--backward-pieces", action="store_true",
                    help="time the backward pieces built so far instead (one GPU)")
    ap.add_argument("--sparse-linear", action="store_true",
                    help="time the sparse + linear forward (block-sparse forward plus the low-rank "
                         "linear branch) instead (one GPU)")
    ap.add_argument("--dit-block", action="store_true",
                    help="time a DiT attention block with the projections fused around VSA instead "
                         "(one GPU)")
    ap.add_argument("--host-chunk-heads", type=int, default=HOST_CHUNK_HEADS,
                    help="(b, h) planes per chunk of the host-buffer path in the end-to-end leg")
    ap.add_argument("--heads", type=int, default=None,
                    help="run the workload with fewer heads (small cases for profiler captures; "
                         "the bench line's config names the heads)")
    args = ap.parse_args()
    w = wl.WORKLOADS[args.workload]
    if args.heads is not None:
        w = dataclasses.replace(w, heads=args.heads)
    if args.backward_pieces:
        return run_backward_pieces(args, w)
    if args.sparse_linear:
        return run_sparse_linear(args, w)
    if args.dit_block:
        return run_dit_block(args, w)
    if args.impl == "reference":
        return run_reference(args, w)
    return run_gpu(args, w)


if __name__ == "__main__":
    sys.exit(main())
