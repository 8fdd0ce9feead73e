"""Benchmark: one content-adaptive block-sparse attention layer at the Wan-14B
720p shape (40 heads, d=128, 21x48x80 tokens, thr=0.1 unioned with the +-1
STA window), seeded synthetic inputs.

A step is one pass of the whole path on one layer's inputs: fractal flatten of
Q, K, V -> block mean pooling -> reduced softmax + CDF selection + STA union +
CSR -> block-sparse attention (O, LSE) -> unflatten of O.  `value` is ms per
layer (lower is better); with N GPUs every rank runs its own layer (weak
scaling, no collective on the data path) and value = max-over-ranks time / N.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

`--impl reference` times the CPU oracle (the plain fp64 restatement under
oracle/) on a bounded sample of the same workload, extrapolated to one layer.
"""
from __future__ import annotations

import argparse
import functools
import hashlib
import json
import math
import os
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WORKLOAD = "wan14b-720p"
METRIC = "ms/attention layer and kept-tile TFLOP/s at Wan-14B 720p shape, thr=0.1"
UNIT = "ms/layer"
L2_FLUSH_BYTES = 256 << 20
# DRAM bytes per launch of each benchmarked kernel, from ncu captures, with a
# hash of the kernel's source files at capture time
TRAFFIC_RECORD = os.path.join(ROOT, "profiles", "dram_traffic.json")
# files whose contents make up the attention kernel (hashed against the record)
ATTN_SOURCES = [os.path.join(ROOT, "content_adaptive_block_fractal_b200", "csrc", f)
                for f in ("k_attn.cu", "vsa_device.cuh")]


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="vsa", choices=["vsa", "reference"])
    ap.add_argument("--workload", default=WORKLOAD)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--layout", default="flat", choices=["flat", "raster"],
                    help="raster: the kernels gather the fractal blocks from raster q, k, v "
                         "and write raster o; flat: explicit flatten / unflatten passes")
    ap.add_argument("--cluster", action="store_true",
                    help="only the semantic-aware permutation path at the Wan-14B 720p shape")
    ap.add_argument("--heads", type=int, default=0,
                    help="run only the first N heads of the workload (small profiling captures; "
                         "0: all)")
    ap.add_argument("--shard", default="replicas", choices=["replicas", "heads"],
                    help="N > 1: every rank runs its own layer (replicas, weak scaling), or the "
                         "ranks split one layer's heads (heads, strong scaling)")
    ap.add_argument("--sweep", action="store_true",
                    help="thr x STA sweep at the Wan-14B 720p shape: one JSON line per point "
                         "(mask + attention; inputs generated once)")
    return ap.parse_args()


def measured_peaks():
    """(bf16 burst TFLOP/s, bf16 sustained TFLOP/s, HBM GB/s, source)."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return p["bf16_tflops"], p["bf16_tflops_sustained"], p["hbm_gbs"], "measured"
    except Exception:
        return 1590.0, 1400.0, 6650.0, "fallback"


def kernel_source_hash(paths) -> str:
    h = hashlib.sha256()
    for p in paths:
        with open(p, "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def profile_traffic(kernel, kernel_srcs, record=TRAFFIC_RECORD):
    """DRAM bytes per launch of `kernel` from the traffic record, if they were
    captured on the current kernel source (same hash of the kernel's files);
    else None."""
    try:
        with open(record) as f:
            entry = json.load(f)["kernels"][kernel]
    except (OSError, KeyError, ValueError, TypeError):
        return None
    if kernel_source_hash(kernel_srcs) != entry.get("source_sha256"):
        return None
    return float(entry["dram_bytes_per_launch"])


class ClockSampler:
    """nvidia-smi clock / throttle samples during the timed region."""
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        self.out = ""
        if self.proc is not None:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.out, _ = self.proc.communicate()

    def summary(self):
        rows = [r.split(",") for r in self.out.strip().splitlines() if r.count(",") >= 8]
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        sm = np.array([float(r[1]) for r in rows])
        mx = float(rows[0][2])
        power = np.array([float(r[3]) for r in rows if r[3].strip() not in ("", "[N/A]")] or [0.0])
        loaded = sm[power >= np.percentile(power, 50)] if power.size == sm.size else sm
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].strip() == "Active"})
        return {"sm_mhz": float(np.median(loaded)), "sm_max_mhz": mx, "reasons": reasons,
                "samples": len(rows)}


# --------------------------------------------------------------------------- ranks
def reduce_over_ranks(values, device):
    """Max over ranks of each device-timed value: the slowest rank sets the
    job's time.  Every rank calls it, in the same order."""
    import torch
    import torch.distributed as dist
    t = torch.tensor(values, device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t]


def sum_over_ranks(values, device):
    """Sum over ranks (work counts of a layer split across ranks)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor(values, device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return [float(x) for x in t]


def head_slice(heads: int, rank: int, world: int):
    """Heads [h0, h1) of one layer that `rank` computes when `world` ranks
    split the layer by heads: contiguous, disjoint, sizes differing by at most
    one.  Every step of the path is independent per head, so no data crosses
    ranks."""
    return heads * rank // world, heads * (rank + 1) // world


def job_ms_per_layer(ms_max: float, world: int, shard: str = "replicas") -> float:
    """Replicas (weak scaling): each of `world` ranks runs one layer in at most
    ms_max, so the job turns out a layer every ms_max / world.  Heads (strong
    scaling): the ranks share one layer, which is done when the slowest rank
    is, after ms_max."""
    return ms_max / world if shard == "replicas" else ms_max


# --------------------------------------------------------------------------- GPU arm
def run_gpu(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    import content_adaptive_block_fractal_b200 as vsa
    from content_adaptive_block_fractal_b200 import workloads

    torch.cuda.set_device(local_rank)
    wl = workloads.get(args.workload)
    if args.heads:
        wl = wl.replace(heads=min(args.heads, wl.heads))
    params = vsa.MaskParams(wl.thr, wl.use_sta, wl.sta)
    shard = args.shard if world > 1 else "replicas"
    h0, h1 = head_slice(wl.heads, rank, world) if shard == "heads" else (0, wl.heads)
    shape = vsa.Shape(wl.B, h1 - h0, wl.T, wl.H, wl.W, wl.d)

    q, k, v = workloads.make_qkv(wl, heads=range(h0, h1))   # host bf16, raster order
    qh, kh, vh = (x.pin_memory() for x in (q, k, v))
    qd, kd, vd = (x.cuda() for x in (qh, kh, vh))
    stream = torch.cuda.current_stream()
    raster = args.layout == "raster"
    layer = vsa.Layer(shape, params, qd.device, layout=args.layout)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=qd.device)
    csr, o, lse = layer.csr, layer.o, layer.lse
    if raster:
        # pool straight from raster; the attention gathers each fractal block
        # with one patch-shaped TMA box and writes O and LSE in raster order
        o_raster = o
        stages = [
            ("pool_qk", lambda x: vsa.pool_qk_raster(x[0], x[1], shape, out=(layer.qp, layer.kp))),
            ("mask", lambda x: vsa.block_mask(layer.qp, layer.kp, shape, params, out=csr,
                                              workspace=layer.ws_mask)),
            ("sparse_attn", lambda x: vsa.sparse_attn_fwd_raster(
                x[0], x[1], x[2], csr.row_ptr, csr.col_idx, shape, 0.0, out=(o, lse),
                workspace=layer.ws_attn)),
        ]
        # pool; mask (digits, select, recheck, chunk sums, chunk scan, expand); plan + attention
        launches_per_step = 1 + 6 + 2
    else:
        qf, kf, vf = (torch.empty_like(qd) for _ in range(3))
        o_raster = o            # the layer's output buffer, written in raster order
        stages = [
            ("flatten_pool_qk", lambda x: vsa.flatten_pool_qk(x[0], x[1], shape,
                                                              out=(qf, kf, layer.qp, layer.kp))),
            ("flatten_v", lambda x: vsa.fractal_flatten(x[2], shape, out=vf)),
            ("mask", lambda x: vsa.block_mask(layer.qp, layer.kp, shape, params, out=csr,
                                              workspace=layer.ws_mask)),
            # the attention stores O and LSE at raster positions: no unflatten pass
            ("sparse_attn", lambda x: vsa.sparse_attn_fwd_to_raster(
                qf, kf, vf, csr.row_ptr, csr.col_idx, shape, 0.0, out=(o_raster, lse),
                workspace=layer.ws_attn)),
        ]
        # flatten+pool of Q,K; flatten of V; mask (6); plan + attention
        launches_per_step = 1 + 1 + 6 + 2
    n_st = len(stages)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(n_st + 1)]
    inputs = (qd, kd, vd)

    def step(record=False):
        if record: ev[0].record(stream)
        for i, (_, fn) in enumerate(stages):
            fn(inputs)
            if record: ev[i + 1].record(stream)

    for _ in range(args.warmup):
        step()
    vsa.device_status()
    kept = int(csr.row_ptr[-1].item())
    rows = shape.B * shape.heads * shape.Nb
    kept_frac = kept / (rows * shape.Nb)
    flop_per_tile = 4 * 64 * 64 * shape.d
    tensor_bytes = shape.B * shape.heads * shape.N * shape.d * 2   # one bf16 [B,h,N,d]
    kept_flop = kept * flop_per_tile

    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    parts = np.zeros(n_st)
    total = 0.0
    with ClockSampler(local_rank) as clk:
        for _ in range(args.steps):
            flush.zero_()
            step(record=True)
            ev[n_st].synchronize()
            parts += [ev[i].elapsed_time(ev[i + 1]) for i in range(n_st)]
            total += ev[0].elapsed_time(ev[n_st])
    torch.cuda.synchronize()
    vsa.device_status()
    ms = total / args.steps
    parts = {name: t / args.steps for (name, _), t in zip(stages, parts)}

    # end to end through the public API with host buffers: every step copies
    # its raster Q, K, V in from pinned memory and its O and LSE back out.
    # Two sets of device inputs and outputs let the copies of one step run on
    # their own streams (the copy engines are full duplex) while its
    # neighbours compute.
    e2e = None
    if not args.no_e2e:
        n_e2e = max(3, min(args.steps, 10))
        ins = [(qd, kd, vd), tuple(torch.empty_like(qd) for _ in range(3))]
        outs_o = [o_raster, torch.empty_like(o_raster)]
        outs_l = [torch.empty_like(lse) for _ in range(2)]
        o_host = [torch.empty(qh.shape, dtype=torch.bfloat16, pin_memory=True) for _ in range(2)]
        l_host = [torch.empty(lse.shape, dtype=torch.float32, pin_memory=True)
                  for _ in range(2)]
        s_h2d, s_d2h = torch.cuda.Stream(), torch.cuda.Stream()
        ev_in = [torch.cuda.Event() for _ in range(2)]     # inputs landed
        ev_used = [torch.cuda.Event() for _ in range(2)]   # inputs consumed (buffer free)
        ev_out = [torch.cuda.Event() for _ in range(2)]    # outputs written
        ev_read = [torch.cuda.Event() for _ in range(2)]   # outputs copied out (buffer free)

        def e2e_steps(n):
            for i in range(n):
                b = i % 2
                s_h2d.wait_event(ev_used[b])
                with torch.cuda.stream(s_h2d):
                    for dst, src in zip(ins[b], (qh, kh, vh)):
                        dst.copy_(src, non_blocking=True)
                ev_in[b].record(s_h2d)
                stream.wait_event(ev_in[b])
                qx, kx, vx = ins[b]
                if raster:
                    vsa.pool_qk_raster(qx, kx, shape, out=(layer.qp, layer.kp))
                    vsa.block_mask(layer.qp, layer.kp, shape, params, out=csr,
                                   workspace=layer.ws_mask)
                    stream.wait_event(ev_read[b])
                    vsa.sparse_attn_fwd_raster(qx, kx, vx, csr.row_ptr, csr.col_idx, shape, 0.0,
                                               out=(outs_o[b], outs_l[b]),
                                               workspace=layer.ws_attn)
                    ev_used[b].record(stream)
                else:
                    vsa.flatten_pool_qk(qx, kx, shape, out=(qf, kf, layer.qp, layer.kp))
                    vsa.fractal_flatten(vx, shape, out=vf)
                    ev_used[b].record(stream)
                    vsa.block_mask(layer.qp, layer.kp, shape, params, out=csr,
                                   workspace=layer.ws_mask)
                    stream.wait_event(ev_read[b])
                    vsa.sparse_attn_fwd_to_raster(qf, kf, vf, csr.row_ptr, csr.col_idx, shape,
                                                  0.0, out=(outs_o[b], outs_l[b]),
                                                  workspace=layer.ws_attn)
                ev_out[b].record(stream)
                s_d2h.wait_event(ev_out[b])
                with torch.cuda.stream(s_d2h):
                    o_host[b].copy_(outs_o[b], non_blocking=True)
                    l_host[b].copy_(outs_l[b], non_blocking=True)
                ev_read[b].record(s_d2h)

        e2e_steps(2)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(s_h2d)
        stream.wait_event(e0)
        s_d2h.wait_event(e0)
        e2e_steps(n_e2e)
        stream.wait_event(ev_read[(n_e2e - 1) % 2])
        e1.record(stream)
        torch.cuda.synchronize()
        e2e_ms = e0.elapsed_time(e1) / n_e2e
        vsa.device_status()
        e2e = {"value": e2e_ms, "unit": UNIT,
               "h2d_bytes_per_step": 3 * qh.numel() * 2,
               "d2h_bytes_per_step": o_host[0].numel() * 2 + l_host[0].numel() * 4,
               "overlap": "H2D, compute and D2H on separate streams, two buffer sets"}

    if world > 1:
        names = list(parts)
        maxed = reduce_over_ranks([ms, e2e["value"] if e2e else 0.0] + [parts[n] for n in names],
                                  qd.device)
        ms, e2e_max = maxed[0], maxed[1]
        parts = dict(zip(names, maxed[2:]))
        if e2e:
            e2e["value"] = job_ms_per_layer(e2e_max, world, shard)
        if shard == "heads":
            # the layer's kept tiles are the sum of the ranks' slices
            kept = int(sum_over_ranks([kept], qd.device)[0])
            kept_flop = kept * flop_per_tile
            rows = wl.B * wl.heads * shape.Nb
            kept_frac = kept / (rows * shape.Nb)
    value = job_ms_per_layer(ms, world, shard)
    # The attention kernel is one launch of ~10 ms per step, timed alone by
    # CUDA events between L2 flushes; its clocks stay near the maximum, so the
    # burst GEMM figure is its denominator (the sustained one is printed too).
    burst_tf, sus_tf, peak_gbs, peak_src = measured_peaks()
    attn_ms = parts["sparse_attn"]
    achieved_tf = kept_flop / (attn_ms * 1e-3) / 1e12
    attn_kernel = f"sparse_attn_kernel<{shape.d}, 0, {1 if raster else 2}>"
    traffic = profile_traffic(attn_kernel, ATTN_SOURCES)
    pooled_bytes = 2 * rows * shape.d * 8
    if raster:
        # pooling reads Q and K and writes the means; nothing else moves
        hbm = {"pool_qk": (2 * tensor_bytes + pooled_bytes) / (parts["pool_qk"] * 1e-3) / 1e9}
        step_desc = ("pool q,k + mask + sparse attention on raster q,k,v -> raster o,lse "
                     "(the fractal order is applied by the kernels' addressing)")
    else:
        hbm = {"flatten_pool_qk": (4 * tensor_bytes + pooled_bytes)
               / (parts["flatten_pool_qk"] * 1e-3) / 1e9,
               "flatten_v": 2 * tensor_bytes / (parts["flatten_v"] * 1e-3) / 1e9}
        step_desc = ("flatten q,k,v + pool + mask + sparse attention storing o,lse in raster "
                     "order (the unflatten folded into the attention's stores)")
    hbm["peak"] = peak_gbs
    result = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": False,
        "scaling": "strong" if shard == "heads" else "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {**wl.describe(),
                   "parallelism": (f"{shard}{world}" if world > 1 else "single"),
                   **({"heads_per_rank": [wl.heads * r // world for r in range(world + 1)]}
                      if shard == "heads" else {}),
                   "l2": "256 MiB flush written between timed steps; Q/K/V 2.5 GB > L2",
                   "layout": args.layout, "step": step_desc},
        "kept_tile_tflops": achieved_tf,
        "kept_tile_tflops_layer": kept_flop / (ms * 1e-3) / 1e12,
        "kept_fraction": kept_frac,
        "kept_tiles": kept,
        "breakdown_ms": parts,
        "roofline": {"bound": "tensor", "kernel": attn_kernel,
                     "achieved": achieved_tf, "peak": burst_tf, "unit": "TFLOP/s",
                     "frac": achieved_tf / burst_tf, "traffic": traffic,
                     "peak_source": f"{peak_src} bf16 burst (one launch timed by CUDA events)",
                     "frac_of_sustained": achieved_tf / sus_tf,
                     "algorithmic_bytes": 4 * tensor_bytes + rows * 4 * 64,
                     "flop_per_kept_tile": flop_per_tile},
        # HBM kernels: algorithmic bytes / time (read + write, each byte once)
        "hbm_gbs": hbm,
        "gpu_launches": launches_per_step * args.steps * world,   # all ranks
        "clocks": clk.summary(),
    }
    if e2e:
        result["e2e"] = e2e
    return result, (q, k, v, wl)


# --------------------------------------------------------------------------- sweep
def run_sweep(args):
    """Mask + attention at every (thr, STA) point of the Wan-14B sweep, on one
    set of inputs (the points differ only in the mask parameters)."""
    import torch
    import content_adaptive_block_fractal_b200 as vsa
    from content_adaptive_block_fractal_b200 import workloads

    torch.cuda.set_device(0)
    points = workloads.sweep_workloads()
    wl0 = points[0]
    shape = vsa.Shape.of(wl0)
    q, k, v = workloads.make_qkv(wl0)
    qd, kd, vd = (x.cuda() for x in (q, k, v))
    layer = vsa.Layer(shape, vsa.MaskParams(wl0.thr, wl0.use_sta, wl0.sta), qd.device)
    qf, kf = torch.empty_like(qd), torch.empty_like(kd)
    vsa.flatten_pool_qk(qd, kd, shape, out=(qf, kf, layer.qp, layer.kp))
    vf = vsa.fractal_flatten(vd, shape)
    del q, k, v
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=qd.device)
    stream = torch.cuda.current_stream()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    peak_tf, _, _, peak_src = measured_peaks()       # burst: single timed launches
    flop_per_tile = 4 * 64 * 64 * shape.d
    steps = max(args.steps, 1)
    k10 = shape.Nb // 10
    sta_csr = vsa.Csr(layer.csr.row_ptr, layer.csr.col_idx, layer.csr.kept_count)
    cases = [(f"top-p thr={wl.thr}" + (" + STA" if wl.use_sta else ""), wl,
              functools.partial(vsa.block_mask, layer.qp, layer.kp, shape,
                                vsa.MaskParams(wl.thr, wl.use_sta, wl.sta),
                                out=layer.csr, workspace=layer.ws_mask))
             for wl in points]
    for sta in (True, False):
        cases.append((f"static-ratio k={k10} (Nb/10)" + (" + STA" if sta else ""), wl0,
                      functools.partial(vsa.block_mask_topk, layer.qp, layer.kp, shape, k10,
                                        vsa.MaskParams(0.0, sta, wl0.sta), out=layer.csr,
                                        workspace=layer.ws_mask)))
    cases = [c + (None,) for c in cases]
    cases.append(("STA window alone (+-1)", wl0,
                  functools.partial(vsa.sta_mask, shape, wl0.sta, out=sta_csr), None))
    # query subsets (HSA-style active blocks): a seeded 25% of the query blocks
    rows_all = shape.B * shape.heads * shape.Nb
    active = torch.as_tensor(np.sort(np.random.default_rng(7).choice(
        rows_all, rows_all // 4, replace=False)), dtype=torch.int32, device=qd.device)
    cases.append(("query subset 25% of blocks, every key block (full context)", points[0],
                  functools.partial(vsa.block_mask, layer.qp, layer.kp, shape,
                                    vsa.MaskParams(0.0, False), out=layer.csr,
                                    workspace=layer.ws_mask), active))
    cases.append(("query subset 25% of blocks, top-p thr=0.1 + STA", wl0,
                  functools.partial(vsa.block_mask, layer.qp, layer.kp, shape,
                                    vsa.MaskParams(0.1, True, wl0.sta), out=layer.csr,
                                    workspace=layer.ws_mask), active))
    for label, wl, make_mask, qblocks in cases:

        def step(record=False):
            if record: ev[0].record(stream)
            make_mask()
            if record: ev[1].record(stream)
            if qblocks is None:
                vsa.sparse_attn_fwd(qf, kf, vf, layer.csr.row_ptr, layer.csr.col_idx, shape,
                                    0.0, out=(layer.o, layer.lse), workspace=layer.ws_attn)
            else:
                vsa.sparse_attn_fwd_rows(qf, kf, vf, layer.csr.row_ptr, layer.csr.col_idx,
                                         shape, qblocks, 0.0, out=(layer.o, layer.lse),
                                         workspace=layer.ws_attn)
            if record: ev[2].record(stream)

        for _ in range(max(args.warmup, 3)):
            step()
        vsa.device_status()
        if qblocks is None:
            kept = int(layer.csr.row_ptr[-1].item())
        else:   # tiles of the listed query blocks only
            kept = int(layer.csr.kept_count[qblocks.long()].sum().item())
        t_mask = t_attn = 0.0
        with ClockSampler(0) as clk:
            for _ in range(steps):
                flush.zero_()
                step(record=True)
                ev[2].synchronize()
                t_mask += ev[0].elapsed_time(ev[1])
                t_attn += ev[1].elapsed_time(ev[2])
        vsa.device_status()
        t_mask /= steps
        t_attn /= steps
        tf = kept * flop_per_tile / (t_attn * 1e-3) / 1e12
        print(json.dumps({
            "metric": "mask + sparse attention ms at Wan-14B 720p shape, sweep point",
            "value": t_mask + t_attn, "unit": "ms", "steps": steps, "mask": label,
            "config": {"workload": "wan14b-720p", "B": shape.B, "heads": shape.heads,
                       "d": shape.d, "grid": [shape.T, shape.H, shape.W], "seed": wl.seed,
                       "data": "synthetic"},
            "kept_tiles": kept, "kept_fraction": kept / (shape.B * shape.heads * shape.Nb ** 2),
            "query_blocks": int(qblocks.numel()) if qblocks is not None else rows_all,
            "mask_ms": t_mask, "sparse_attn_ms": t_attn, "kept_tile_tflops": tf,
            "roofline": {"bound": "tensor", "achieved": tf, "peak": peak_tf, "frac": tf / peak_tf,
                         "peak_source": f"{peak_src} bf16 burst"},
            "clocks": clk.summary()}), flush=True)
    # the semantic-aware permutation path, on the raster inputs
    print(json.dumps(run_cluster_point(args, qd, kd, vd, shape, peak_tf, peak_src,
                                       vsa.ClusterParams(256, 512, 2, 0.9))), flush=True)


def run_cluster_point(args, q, k, v, shape, peak_tf, peak_src, params):
    """The semantic-aware permutation path as one call, timed whole (k-means,
    permutation, centroid top-p, attention, inverse permutation)."""
    import torch
    import content_adaptive_block_fractal_b200 as vsa
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=q.device)
    ws = vsa._workspace(vsa.cluster_attn_workspace_size(shape, params), q.device)
    o = torch.empty_like(q)
    lse = torch.empty((shape.B, shape.heads, shape.N), dtype=torch.float32, device=q.device)
    _, _, st = vsa.cluster_attention(q, k, v, shape, params, want_state=True, out=(o, lse),
                                     workspace=ws)
    for _ in range(max(args.warmup, 3) - 1):
        vsa.cluster_attention(q, k, v, shape, params, out=(o, lse), workspace=ws)
    vsa.device_status()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    steps = max(args.steps, 1)
    total = 0.0
    with ClockSampler(0) as clk:
        for _ in range(steps):
            flush.zero_()
            e0.record()
            vsa.cluster_attention(q, k, v, shape, params, out=(o, lse), workspace=ws)
            e1.record()
            e1.synchronize()
            total += e0.elapsed_time(e1)
    vsa.device_status()
    ms = total / steps
    # work: padded 64x64 tiles the attention kernel runs, and the useful
    # query-key token pairs (each kept cluster pair counted at its true sizes)
    nq = st["q_counts"].double()
    nk = st["k_counts"].double()
    keep = st["keep"].double()
    tiles = float(((nq / 64).ceil() * (keep @ (nk / 64).ceil().unsqueeze(-1)).squeeze(-1)).sum())
    pairs = float((nq * (keep @ nk.unsqueeze(-1)).squeeze(-1)).sum())
    flop_tile = 4 * 64 * 64 * shape.d
    return {
        "metric": "semantic-aware permutation attention ms at Wan-14B 720p shape",
        "value": ms, "unit": "ms", "steps": steps,
        "mask": f"semantic permutation Cq={params.Cq} Ck={params.Ck} iters={params.iters} "
                f"p={params.p}",
        "config": {"workload": "wan14b-720p", "B": shape.B, "heads": shape.heads, "d": shape.d,
                   "grid": [shape.T, shape.H, shape.W], "data": "synthetic"},
        "kept_pair_fraction": pairs / (shape.B * shape.heads * shape.N ** 2),
        "padded_tiles": tiles,
        "tflops_useful_pairs_whole_call": pairs * 4 * shape.d / (ms * 1e-3) / 1e12,
        "tflops_padded_tiles_whole_call": tiles * flop_tile / (ms * 1e-3) / 1e12,
        "peak": peak_tf, "peak_source": f"{peak_src} bf16 burst",
        "clocks": clk.summary()}


# --------------------------------------------------------------------------- CPU oracle
def oracle_sample(wl, heads, n_qblocks, seed=0):
    """Time the oracle on `heads` (flatten, pool, mask in full; attention on
    n_qblocks sampled query blocks per head) and extrapolate to one layer."""
    import oracle
    from content_adaptive_block_fractal_b200 import workloads
    oracle.lib()
    heads = [h for h in heads if h < wl.heads]          # small workloads have fewer
    n_qblocks = min(n_qblocks, wl.Nb)
    t_perm = t_pool = t_mask = t_attn = 0.0
    kept_total = kept_sampled = 0
    for h in heads:
        q, k, v = workloads.make_qkv(wl, heads=[h])
        t0 = time.perf_counter()
        qf, kf, vf = (oracle.flatten(x, wl.T, wl.H, wl.W) for x in (q, k, v))
        t1 = time.perf_counter()
        qp, kp = oracle.pool(qf), oracle.pool(kf)
        t2 = time.perf_counter()
        keep, _ = oracle.block_mask(qp, kp, wl.Hb, wl.Wb, float(np.float32(wl.thr)), wl.use_sta, wl.sta)
        rp, ci = oracle.mask_to_csr(keep)
        t3 = time.perf_counter()
        rng = np.random.default_rng(seed + h)
        qb = rng.choice(wl.Nb, n_qblocks, replace=False)
        oracle.sparse_attention(qf, kf, vf, rp, ci, qblocks=qb)
        t4 = time.perf_counter()
        cnt = np.diff(rp)
        t_perm += (t1 - t0) * 4.0 / 3.0            # unflatten of O costs one more permute
        t_pool += t2 - t1
        t_mask += t3 - t2
        t_attn += t4 - t3
        kept_total += int(cnt.sum())
        kept_sampled += int(cnt[qb].sum())
    nh = len(heads)
    scale_heads = wl.B * wl.heads / nh
    ms = 1e3 * ((t_perm + t_pool + t_mask) * scale_heads
                + t_attn * (kept_total / max(kept_sampled, 1)) * scale_heads)
    work_s = t_perm + t_pool + t_mask + t_attn
    sample = (f"{nh} of {wl.B * wl.heads} heads: flatten/pool/mask in full, attention on "
              f"{n_qblocks} query blocks per head; extrapolated by heads and by kept tiles")
    return ms, work_s, sample


def run_reference(args):
    import oracle
    from content_adaptive_block_fractal_b200 import workloads
    wl = workloads.get(args.workload)
    cores = oracle.num_threads()
    vals = []
    for i in range(args.warmup + args.steps):
        ms, _, sample = oracle_sample(wl, [i % wl.heads], 16, seed=i)
        if i >= args.warmup:
            vals.append(ms)
    value = float(np.mean(vals))
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": value,
        "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": wl.describe(),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)


def main():
    args = parse_args()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        if rank == 0:
            run_reference(args)
        return
    if args.sweep or args.cluster:
        if rank == 0:
            if args.sweep:
                run_sweep(args)
            else:
                import torch
                import content_adaptive_block_fractal_b200 as vsa
                from content_adaptive_block_fractal_b200 import workloads
                wl = workloads.get(WORKLOAD)
                shape = vsa.Shape.of(wl)
                q, k, v = (x.cuda() for x in workloads.make_qkv(wl))
                peak_tf, _, _, peak_src = measured_peaks()
                print(json.dumps(run_cluster_point(args, q, k, v, shape, peak_tf, peak_src,
                                                   vsa.ClusterParams(256, 512, 2, 0.9))),
                      flush=True)
        return
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local_rank))
    try:
        result, _ = run_gpu(args, rank, world, local_rank)
        if rank == 0:
            # the oracle's CPU baseline is taken at N = 1 only
            if not args.no_cpu_baseline and world == 1:
                import oracle
                wl = __import__("content_adaptive_block_fractal_b200.workloads",
                                fromlist=["get"]).get(args.workload)
                ms, work_s, sample = oracle_sample(wl, [0, 1, 2, 3, 4, 5], 480)
                result["cpu_baseline"] = {"value": ms, "unit": UNIT, "cores": oracle.num_threads(),
                                          "kind": "oracle", "sample": sample,
                                          "cpu_seconds_measured": work_s}
            print(json.dumps(result), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.barrier()
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
