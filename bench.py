#!/usr/bin/env python
"""Benchmark of the NSA forward hot path on B200 (one JSON line on rank 0).

Workload (default): causal prefill of one 65536-token sequence, 64 query /
4 KV heads, head dim 128, blocks l = d = l' = 64, top-16, window 512, bf16
Q/K/V ~ N(0, 1), fp32 gates ~ U(0, 1), compressor weights ~ N(0, 1/(l D))
(the 64k configuration of the NSA config page's knobs; synthetic data).
A step is one nsa_prefill call: compression, compressed attention and block
scores, top-n, fused selected + window attention with the gate combine.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

With N > 1 (torchrun) every rank runs its own sequence (independent problems,
no collective on the data path: weak scaling); the time is the max over ranks.
`--impl reference` times the fp64 CPU oracle on a bounded sample of the same
workload on the host cores (rank 0 only).
"""
from __future__ import annotations

import argparse
import dataclasses
import hashlib
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

from sparse_attention_long_06_b200 import workloads as wl  # noqa: E402

METRIC = "NSA prefill tokens/s"
KERNEL_NAMES = ["nsa_meta_kernel", "nsa_weight_split_kernel", "nsa_compress_tc_kernel",
                "nsa_cmp_attn_kernel", "nsa_topn_kernel", "nsa_win_kernel", "nsa_slc_kernel"]
# tensor-core kernels: (stage index, source file, algorithmic FLOP key)
TENSOR_KERNELS = {"nsa_compress_tc_kernel": (2, "k_compress.cu", "compress"),
                  "nsa_cmp_attn_kernel": (3, "k_cmp.cu", "cmp"),
                  "nsa_win_kernel": (5, "k_win.cu", "win"),
                  "nsa_slc_kernel": (6, "k_slc.cu", "slc")}


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return p["hbm_gbs"], p["bf16_tflops"], p["bf16_tflops_sustained"], "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


# ---------------------------------------------------------------- config
def prefill_config(cfg, T, world):
    """The workload description both arms print."""
    return {"workload": cfg.name, "batch": len(wl.seqlens_of(cfg)), "seq_len": T,
            "q_heads": cfg.num_q_heads, "kv_heads": cfg.num_kv_heads, "head_dim": cfg.head_dim,
            "cmp_block": cfg.cmp_block, "cmp_stride": cfg.cmp_stride, "sel_block": cfg.sel_block,
            "top_n": cfg.top_n,
            "window": cfg.window, "out": "bf16",
            "l2": "flushed (256 MB write) before every timed step",
            "parallelism": f"replicas x{world} (independent sequences)"}


# ---------------------------------------------------------------- ranks
def max_over_ranks(x, world, device):
    """The largest of every rank's `x` (device time of the slowest replica);
    every rank must call it at the same point."""
    if world <= 1:
        return float(x)
    import torch
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_rate(units_per_rank, world, ms):
    """Whole-job throughput: the units all ranks processed over the max time."""
    return world * units_per_rank / (ms / 1e3)


# ---------------------------------------------------------------- algorithmic work
def algorithmic_flops_packed(cfg, lens, sel):
    """algorithmic_flops summed over the sequences of a packed batch."""
    tot = {"cmp": 0, "slc": 0, "win": 0, "compress": 0, "total": 0}
    s = 0
    for T in lens:
        f = algorithmic_flops(cfg, T, sel[s:s + T])
        for k in tot:
            tot[k] += f[k]
        s += T
    return tot


def algorithmic_flops(cfg, T, sel):
    """Exact FLOPs of the method on one sequence (the work it does, not the
    dense work it avoids): per (t, head) 4 D (|cmp(t)| + |slc(t)| + |win(t)|),
    plus compression 4 l D^2 per complete block per KV head."""
    D, G, l, d, ls, w = (cfg.head_dim, cfg.group, cfg.cmp_block, cfg.cmp_stride, cfg.sel_block,
                         cfg.window)
    t = np.arange(T, dtype=np.int64)
    ncmp = np.where(t + 1 >= l, (t + 1 - l) // d + 1, 0)  # complete compressed blocks
    nwin = np.minimum(w, t + 1)
    blk = sel.astype(np.int64)                            # [T, Hkv, n]
    keys = np.where(blk >= 0, np.minimum(ls, t[:, None, None] - blk * ls + 1), 0)
    nslc = keys.clip(min=0).sum(axis=2)                   # [T, Hkv]
    per_head = 4 * D
    f_cmp = per_head * G * cfg.num_kv_heads * int(ncmp.sum())
    f_win = per_head * G * cfg.num_kv_heads * int(nwin.sum())
    f_slc = per_head * G * int(nslc.sum())
    n_blocks = (T - l) // d + 1 if T >= l else 0
    f_compress = 4 * n_blocks * cfg.num_kv_heads * l * D * D
    return {"cmp": f_cmp, "slc": f_slc, "win": f_win, "compress": f_compress,
            "total": f_cmp + f_slc + f_win + f_compress}


# ---------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid):
        self.uuid = uuid
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        time.sleep(0.15)
        self.lines = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()
                out = ""
            self.lines = [ln for ln in out.splitlines() if ln.strip()]

    def summary(self):
        sm, smax, reasons = [], None, set()
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9 or (self.uuid and self.uuid not in parts[0]):
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
            for nm, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": smax, "reasons": [], "samples": 0}
        busy = [x for x in sm if x > 0.5 * (smax or max(sm))] or sm
        return {"sm_mhz": statistics.median(busy), "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------- oracle baseline
def oracle_sample(cfg, inputs, nrows=512):
    """Times the fp64 oracle on a bounded sample: compression of the whole
    sequence plus `nrows` evenly spaced query rows (the latest rows, with the
    full causal history, included).  Returns tokens/s with the compression
    amortised over the sequence length, and a description."""
    import oracle
    from oracle import OracleParams
    p = OracleParams.of(cfg)
    T = int(inputs["cu_seqlens"][-1])
    t0 = time.perf_counter()
    _, kc = oracle.compress(p, inputs["k"], inputs["w_k"])
    _, vc = oracle.compress(p, inputs["v"], inputs["w_v"])
    t_cmp = time.perf_counter() - t0
    rows = np.linspace(T - 1, 0, num=nrows).astype(np.int32)[::-1].copy()
    t0 = time.perf_counter()
    oracle.nsa_rows(p, inputs["q"], inputs["k"], inputs["v"], kc, vc, inputs["gates"], rows,
                    cmax=max(1, T // cfg.cmp_block, T // cfg.sel_block + 1))
    t_rows = time.perf_counter() - t0
    sec_per_token = t_rows / nrows + t_cmp / T
    cores = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    return {"value": 1.0 / sec_per_token, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": (f"fp64 oracle on the {cfg.name} input: compression of all {oracle.num_cmp_blocks(p, T)} "
                       f"blocks ({t_cmp:.2f} s, amortised over {T} tokens) + {nrows} evenly spaced "
                       f"query rows ({t_rows:.2f} s)")}


# ---------------------------------------------------------------- traffic record
def traffic_record(kernel, src_file):
    """DRAM bytes per 64k launch of `kernel` from the committed ncu summary
    profiles/traffic_<kernel>.json, or None when the kernel's source changed
    since the counters were taken."""
    path = os.path.join(ROOT, "profiles", f"traffic_{kernel}.json")
    src = os.path.join(ROOT, "sparse_attention_long_06_b200", "csrc", src_file)
    try:
        rec = json.load(open(path))
        digest = hashlib.sha256(open(src, "rb").read()).hexdigest()
        if rec.get("source_sha256") != digest:
            return None
        return rec.get("dram_bytes_per_launch_64k")
    except Exception:
        return None


# ---------------------------------------------------------------- end to end
def e2e_pipelined(plan, host, d, out, kc, vc, sel, ws, out_host, steps):
    """Mean ms per step of `steps` prefill calls through the public API, each
    uploading its inputs from pinned host memory and downloading its output,
    with upload / kernels / download on three streams and two device buffer
    sets so that consecutive steps overlap."""
    import torch
    dsets = [d, {k: torch.empty_like(v) for k, v in d.items()}]
    outs = [out, torch.empty_like(out)]
    hosts_out = [out_host, torch.empty_like(out_host).pin_memory()]
    s_in, s_c, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    in_done = [torch.cuda.Event() for _ in range(steps)]
    c_done = [torch.cuda.Event() for _ in range(steps)]
    out_done = [torch.cuda.Event() for _ in range(steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    t0.record(s_in)
    for i in range(steps):
        b = i % 2
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(c_done[i - 2])  # kernels of step i-2 are done with set b
            for k in dsets[b]:
                dsets[b][k].copy_(host[k], non_blocking=True)
            in_done[i].record(s_in)
        s_c.wait_event(in_done[i])
        if i >= 2:
            s_c.wait_event(out_done[i - 2])  # download of step i-2 is done with outs[b]
        ds = dsets[b]
        plan.prefill(ds["q"], ds["k"], ds["v"], ds["gates"], ds["w_k"], ds["w_v"], ds["cu_seqlens"],
                     outs[b], kc, vc, ws, sel_idx=sel, stream=s_c)
        c_done[i].record(s_c)
        with torch.cuda.stream(s_out):
            s_out.wait_event(c_done[i])
            hosts_out[b].copy_(outs[b], non_blocking=True)
            out_done[i].record(s_out)
    t1.record(s_out)
    torch.cuda.synchronize()
    return t0.elapsed_time(t1) / steps


# ---------------------------------------------------------------- our arm
def run_ours(args, rank, world):
    import torch
    from sparse_attention_long_06_b200 import nsa

    cfg = wl.CONFIGS[args.workload]
    inputs = wl.prefill_inputs(cfg)
    T = int(inputs["cu_seqlens"][-1])
    D, Hq, Hkv = cfg.head_dim, cfg.num_q_heads, cfg.num_kv_heads
    dev = torch.device("cuda", torch.cuda.current_device())

    def pinned(a):
        t = torch.from_numpy(a.view(np.int16) if a.dtype == np.uint16 else a)
        return t.pin_memory()

    host = {k: pinned(np.ascontiguousarray(inputs[k])) for k in
            ("q", "k", "v", "gates", "w_k", "w_v", "cu_seqlens")}
    d = {k: torch.empty_like(v, device=dev) for k, v in host.items()}
    for k in d:
        d[k].copy_(host[k])
    plan = nsa.Plan.for_config(cfg, max_batch=1, max_seqlen=T, max_total_tokens=T,
                               out_dtype=nsa.OUT_BF16)
    out = torch.empty((T, Hq, D), dtype=torch.int16, device=dev)
    kc = torch.empty((plan.cmp_rows(T), Hkv, D), dtype=torch.int16, device=dev)
    vc = torch.empty_like(kc)
    sel = torch.empty((T, Hkv, cfg.top_n), dtype=torch.int32, device=dev)
    ws = plan.alloc_workspace(device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)  # 2x the 126 MB L2
    out_host = torch.empty((T, Hq, D), dtype=torch.int16).pin_memory()

    def step():
        plan.prefill(d["q"], d["k"], d["v"], d["gates"], d["w_k"], d["w_v"], d["cu_seqlens"],
                     out, kc, vc, ws, sel_idx=sel)

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    status = nsa.read_device_status(ws)
    if status != nsa.NSA_OK:
        raise RuntimeError(f"device status {nsa.strerror(status)} after warm-up")
    launches_per_step = nsa.last_launch_count()

    uuid = str(torch.cuda.get_device_properties(dev).uuid)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    with ClockSampler(uuid) as clocks:
        for i in range(args.steps):
            flush.zero_()  # L2 flushed between timed steps (outside the events)
            ev[i][0].record()
            step()
            ev[i][1].record()
        torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    step_ms = [a.elapsed_time(b) for a, b in ev]
    total_ms = max_over_ranks(sum(step_ms), world, dev)
    status = nsa.read_device_status(ws)
    if status != nsa.NSA_OK:
        raise RuntimeError(f"device status {nsa.strerror(status)} in the timed region")
    ms_per_step = total_ms / args.steps
    value = job_rate(T, world, ms_per_step)

    # per-launch times (same stream, events recorded by the library)
    nsa.profile_enable(True)
    stage = []
    for _ in range(3):
        flush.zero_()
        step()
        stage.append(nsa.profile_stage_ms())
    nsa.profile_enable(False)
    stage_ms = [statistics.median(s[i] for s in stage) for i in range(len(stage[0]))]

    sel_h = sel.cpu().numpy()
    flops = algorithmic_flops(cfg, T, sel_h)
    hbm, tc_burst, tc_sust, peak_src = _peaks()
    rooflines = {}
    for name, (idx, src_file, key) in TENSOR_KERNELS.items():
        ach = flops[key] / (stage_ms[idx] / 1e3) / 1e12
        rooflines[name] = {"bound": "tensor", "kernel": name, "achieved": round(ach, 2),
                           "peak": tc_sust, "unit": "TFLOP/s", "frac": round(ach / tc_sust, 4),
                           "traffic": traffic_record(name, src_file),
                           "peak_source": f"{peak_src} bf16 sustained (kernel timed inside a repeated step)"}
    dominant = max(TENSOR_KERNELS, key=lambda k: stage_ms[TENSOR_KERNELS[k][0]])
    roofline = rooflines[dominant]
    # the selected kernel's other bound: every (token, group) gathers its
    # selected blocks' K and V (l' keys x D x 2 B each) from L2 into shared memory
    nblk = int((sel_h >= 0).sum())
    gather_bytes = nblk * cfg.sel_block * cfg.head_dim * 2 * 2
    slc_ms = stage_ms[TENSOR_KERNELS["nsa_slc_kernel"][0]]
    l2_gather = {"kernel": "nsa_slc_kernel", "bound": "l2", "bytes_per_call": gather_bytes,
                 "achieved": round(gather_bytes / (slc_ms / 1e3) / 1e12, 2), "unit": "TB/s",
                 "peak": None,
                 "note": "selected K/V blocks moved L2 -> shared memory per call; no measured "
                         "L2 peak on this pool"}

    # end to end through the public API with host buffers: every step uploads
    # its inputs from pinned host memory and downloads its output; steps are
    # pipelined as a server would run them (upload of step i+1 and download of
    # step i-1 overlap the kernels of step i, on two device buffer sets)
    e2e_steps = max(4, min(8, args.steps))
    h2d = sum(host[k].numel() * host[k].element_size() for k in host)
    d2h = out_host.numel() * out_host.element_size()
    e2e_step_ms = e2e_pipelined(plan, host, d, out, kc, vc, sel, ws, out_host, e2e_steps)
    e2e_ms_max = max_over_ranks(e2e_step_ms, world, dev)
    e2e_value = job_rate(T, world, e2e_ms_max)

    result = {
        "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) bf16 Q/K/V, U(0,1) gates, N(0,1/(l*D)) compressor)",
        "config": prefill_config(cfg, T, world),
        "sparse_tflops": round(flops["total"] / (ms_per_step / 1e3) / 1e12, 2),
        "algorithmic_flop_per_step": flops,
        "stage_ms": dict(zip(KERNEL_NAMES, [round(x, 4) for x in stage_ms])),
        "roofline": roofline,
        "rooflines": rooflines,
        "e2e": {"value": round(e2e_value, 1), "unit": "tokens/s", "h2d_bytes_per_step": int(h2d),
                "d2h_bytes_per_step": int(d2h), "ms_per_step": round(e2e_ms_max, 3),
                "steps": e2e_steps, "schedule": "pipelined: upload, kernels, download on 3 streams, "
                                                "2 device buffer sets"},
        "l2_gather": l2_gather,
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks.summary(),
    }
    if not args.no_decode:
        del d, host
        torch.cuda.empty_cache()
        result["decode"] = run_decode_leg(args, dev, world)
    if not args.no_legs:
        torch.cuda.empty_cache()
        result["legs"] = {name: run_prefill_leg(name, dev, world)
                          for name in ("prefill_8k", "varlen", "prefill_8k_overlap")
                          if name != args.workload}
        torch.cuda.empty_cache()
        result["legs"]["block_select_64k"] = run_block_select_leg(dev, world)
        torch.cuda.empty_cache()
        result["legs"]["block_select_decode_64k"] = run_block_select_decode_leg(dev, world)
        torch.cuda.empty_cache()
        result["legs"]["token_select_8k"] = run_token_select_leg(dev, world)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = oracle_sample(cfg, inputs)
        result["cpu_baseline_1core"] = oracle_single_core()
    return result


# ---------------------------------------------------------------- other prefill workloads
def run_prefill_leg(name, dev, world, steps=10, warmup=3):
    """Device-timed prefill of another configuration (8k, varlen): tokens/s,
    sparse TFLOP/s and the tensor roofline of every tensor-core kernel."""
    import torch
    from sparse_attention_long_06_b200 import nsa
    cfg = wl.CONFIGS[name]
    inputs = wl.prefill_inputs(cfg)
    lens = list(inputs["seqlens"])
    T = int(inputs["cu_seqlens"][-1])
    D, Hq, Hkv = cfg.head_dim, cfg.num_q_heads, cfg.num_kv_heads
    d = {}
    for k in ("q", "k", "v", "gates", "w_k", "w_v", "cu_seqlens"):
        a = np.ascontiguousarray(inputs[k])
        d[k] = torch.from_numpy(a.view(np.int16) if a.dtype == np.uint16 else a).to(dev)
    plan = nsa.Plan.for_config(cfg, max_batch=len(lens), max_seqlen=max(lens), max_total_tokens=T,
                               out_dtype=nsa.OUT_BF16)
    out = torch.empty((T, Hq, D), dtype=torch.int16, device=dev)
    kc = torch.empty((max(plan.cmp_rows(T), 1), Hkv, D), dtype=torch.int16, device=dev)
    vc = torch.empty_like(kc)
    sel = torch.empty((T, Hkv, cfg.top_n), dtype=torch.int32, device=dev)
    ws = plan.alloc_workspace(device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def step():
        plan.prefill(d["q"], d["k"], d["v"], d["gates"], d["w_k"], d["w_v"], d["cu_seqlens"],
                     out, kc, vc, ws, sel_idx=sel)

    for _ in range(warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    if nsa.read_device_status(ws) != nsa.NSA_OK:
        raise RuntimeError(f"{name}: device status after warm-up")
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    for i in range(steps):
        flush.zero_()
        ev[i][0].record()
        step()
        ev[i][1].record()
    torch.cuda.synchronize()
    ms = max_over_ranks(statistics.median(a.elapsed_time(b) for a, b in ev), world, dev)
    nsa.profile_enable(True)
    stage = []
    for _ in range(3):
        flush.zero_()
        step()
        stage.append(nsa.profile_stage_ms())
    nsa.profile_enable(False)
    stage_ms = [statistics.median(x[i] for x in stage) for i in range(len(stage[0]))]
    flops = algorithmic_flops_packed(cfg, lens, sel.cpu().numpy())
    _, _, tc_sust, src = _peaks()
    roof = {}
    for kname, (idx, _, key) in TENSOR_KERNELS.items():
        ach = flops[key] / (stage_ms[idx] / 1e3) / 1e12
        roof[kname] = {"achieved": round(ach, 2), "frac": round(ach / tc_sust, 4)}
    tflops = flops["total"] / (ms / 1e3) / 1e12
    return {"metric": "NSA prefill tokens/s", "value": round(job_rate(T, world, ms), 1),
            "unit": "tokens/s", "ms_per_step_median": round(ms, 4), "steps": steps,
            "sparse_tflops": round(tflops, 2), "frac_of_peak": round(tflops / tc_sust, 4),
            "peak": tc_sust, "peak_source": f"{src} bf16 sustained",
            "config": prefill_config(cfg, T, world) | {"seqlens": lens},
            "algorithmic_flop_per_step": flops,
            "stage_ms": dict(zip(KERNEL_NAMES, [round(x, 4) for x in stage_ms])),
            "rooflines": roof}


BLOCK_SELECT_KERNELS = ["nsa_meta_kernel", "nsa_block_mean_kernel", "nsa_block_score_kernel",
                        "nsa_topn_kernel", "nsa_slc_kernel"]


def block_select_flops(cfg, lens, sel):
    """Exact FLOPs of select-only block attention on a packed batch: routing
    2 D per (token, head, candidate block) over the t // l' blocks before the
    own block, plus attention 4 D per (token, head, attended key)."""
    D, G, ls, Hkv = cfg.head_dim, cfg.group, cfg.sel_block, cfg.num_kv_heads
    f_route = f_attn = 0
    s = 0
    for T in lens:
        t = np.arange(T, dtype=np.int64)
        f_route += 2 * D * G * Hkv * int((t // ls).sum())
        blk = sel[s:s + T].astype(np.int64)
        keys = np.where(blk >= 0, np.minimum(ls, t[:, None, None] - blk * ls + 1), 0)
        f_attn += 4 * D * G * int(keys.clip(min=0).sum())
        s += T
    return {"route": f_route, "attn": f_attn, "total": f_route + f_attn}


def run_block_select_leg(dev, world, steps=10, warmup=3, name="prefill_64k"):
    """Select-only block attention (own block + n - 1 routed blocks of l'
    tokens, mean-pooled routing keys) on the geometry and length of `name`:
    tokens/s and the tensor roofline of the routing and attention kernels."""
    import torch
    from sparse_attention_long_06_b200 import nsa
    cfg = wl.CONFIGS[name]
    inputs = wl.prefill_inputs(cfg)
    lens = list(inputs["seqlens"])
    T = int(inputs["cu_seqlens"][-1])
    D, Hq, Hkv = cfg.head_dim, cfg.num_q_heads, cfg.num_kv_heads
    d = {}
    for k in ("q", "k", "v", "cu_seqlens"):
        a = np.ascontiguousarray(inputs[k])
        d[k] = torch.from_numpy(a.view(np.int16) if a.dtype == np.uint16 else a).to(dev)
    plan = nsa.Plan.for_config(cfg, max_batch=len(lens), max_seqlen=max(lens), max_total_tokens=T,
                               out_dtype=nsa.OUT_BF16)
    out = torch.empty((T, Hq, D), dtype=torch.int16, device=dev)
    km = torch.empty((max(plan.block_rows(T), 1), Hkv, D), dtype=torch.int16, device=dev)
    sel = torch.empty((T, Hkv, cfg.top_n), dtype=torch.int32, device=dev)
    ws = plan.alloc_workspace(nsa.MODE_BLOCK_SELECT, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def step():
        plan.block_select_prefill(d["q"], d["k"], d["v"], d["cu_seqlens"], out, km, ws, sel_idx=sel)

    for _ in range(warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    if nsa.read_device_status(ws) != nsa.NSA_OK:
        raise RuntimeError("block select: device status after warm-up")
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    for i in range(steps):
        flush.zero_()
        ev[i][0].record()
        step()
        ev[i][1].record()
    torch.cuda.synchronize()
    ms = max_over_ranks(statistics.median(a.elapsed_time(b) for a, b in ev), world, dev)
    nsa.profile_enable(True)
    stage = []
    for _ in range(3):
        flush.zero_()
        step()
        stage.append(nsa.profile_stage_ms())
    nsa.profile_enable(False)
    stage_ms = [statistics.median(x[i] for x in stage) for i in range(len(stage[0]))]
    flops = block_select_flops(cfg, lens, sel.cpu().numpy())
    _, _, tc_sust, src = _peaks()
    roof = {}
    for kname, key in (("nsa_block_score_kernel", "route"), ("nsa_slc_kernel", "attn")):
        idx = BLOCK_SELECT_KERNELS.index(kname)
        ach = flops[key] / (stage_ms[idx] / 1e3) / 1e12
        roof[kname] = {"achieved": round(ach, 2), "frac": round(ach / tc_sust, 4)}
    tflops = flops["total"] / (ms / 1e3) / 1e12
    return {"metric": "select-only block attention tokens/s", "value": round(job_rate(T, world, ms), 1),
            "unit": "tokens/s", "ms_per_step_median": round(ms, 4), "steps": steps,
            "sparse_tflops": round(tflops, 2), "frac_of_peak": round(tflops / tc_sust, 4),
            "peak": tc_sust, "peak_source": f"{src} bf16 sustained",
            "config": prefill_config(cfg, T, world) | {"mode": "block_select (own block + n - 1 routed)"},
            "algorithmic_flop_per_step": flops,
            "stage_ms": dict(zip(BLOCK_SELECT_KERNELS, [round(x, 4) for x in stage_ms])),
            "rooflines": roof}


def run_block_select_decode_leg(dev, world=1, steps=20, warmup=3):
    """Select-only decode step (own block + n - 1 routed blocks) on the decode
    workload (32 sequences x 65 537 cached tokens): tokens/s and the time of
    each launch.  The routing-key cache holds the generator's synthetic cache
    state (the amount of work does not depend on its values)."""
    import torch
    from sparse_attention_long_06_b200 import nsa
    cfg = wl.CONFIGS["decode_64k"]
    inp = wl.decode_inputs(cfg)
    B, cap = cfg.decode_batch, int(inp["capacity"])
    d = {}
    for k in ("q", "k", "v", "seqlens"):
        a = np.ascontiguousarray(inp[k])
        d[k] = torch.from_numpy(a.view(np.int16) if a.dtype == np.uint16 else a).to(dev)
    km = np.ascontiguousarray(inp["kc"][:, :cap // cfg.sel_block])
    d["km"] = torch.from_numpy(km.view(np.int16)).to(dev)
    del inp
    plan = nsa.Plan.for_config(cfg, max_batch=B, max_seqlen=cap, out_dtype=nsa.OUT_BF16)
    out = torch.empty((B, cfg.num_q_heads, cfg.head_dim), dtype=torch.int16, device=dev)
    sel = torch.empty((B, cfg.num_kv_heads, cfg.top_n), dtype=torch.int32, device=dev)
    ws = plan.alloc_workspace(nsa.MODE_BLOCK_SELECT_DECODE, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def step():
        plan.block_select_decode(d["q"], d["k"], d["v"], d["km"], d["seqlens"], out, ws,
                                 sel_idx=sel)

    for _ in range(max(3, warmup)):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    if nsa.read_device_status(ws) != nsa.NSA_OK:
        raise RuntimeError("select-only decode: device status after warm-up")
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    for i in range(steps):
        flush.zero_()
        ev[i][0].record()
        step()
        ev[i][1].record()
    torch.cuda.synchronize()
    ms = max_over_ranks(statistics.median(a.elapsed_time(b) for a, b in ev), world, dev)
    nsa.profile_enable(True)
    flush.zero_()
    step()
    stage = nsa.profile_stage_ms()
    nsa.profile_enable(False)
    return {"metric": "select-only block attention decode tokens/s",
            "value": round(job_rate(B, world, ms), 1), "unit": "tokens/s",
            "ms_per_step_median": round(ms, 5), "steps": steps,
            "config": {"workload": cfg.name, "batch": B, "context": int(cfg.decode_len),
                       "l_sel": cfg.sel_block, "top_n": cfg.top_n,
                       "mode": "block_select (own block + n - 1 routed)",
                       "routing_key_cache": "synthetic random state",
                       "l2": "flushed before every timed step"},
            "stage_ms": {"nsa_decode_block_mean_kernel": round(stage[0], 5),
                         "nsa_decode_a_kernel": round(stage[1], 5),
                         "nsa_decode_b_kernel": round(stage[2], 5)}}


TOKEN_SELECT_KERNELS = ["nsa_meta_kernel", "nsa_block_score_kernel", "nsa_token_topk_kernel",
                        "nsa_token_attn_kernel"]


def token_select_work(lens, D, Hq, Hkv, index_heads, index_dim, top_k):
    """Algorithmic work of token-level top-k attention on a packed batch:
    index scores 2 Di per (query, indexer head, visible token), attention
    4 D per (query, head, chosen token), and the bytes of the chosen tokens'
    key and value rows gathered per (query, KV group)."""
    f_index = chosen = 0
    for Tb in lens:
        t = np.arange(Tb, dtype=np.int64)
        f_index += 2 * index_dim * index_heads * int((t + 1).sum())
        chosen += int(np.minimum(t + 1, top_k).sum())
    return {"index": f_index, "attn": 4 * D * Hq * chosen, "gather_bytes": chosen * Hkv * D * 2 * 2}


def run_token_select_leg(dev, world, steps=5, warmup=3, name="prefill_8k", index_heads=16,
                         index_dim=128, top_k=2048):
    """Token-level top-k attention (DSA style: indexer of `index_heads` x
    `index_dim`, top_k tokens per query) on the geometry and length of
    `name`: tokens/s, the index scores and the attention over the chosen
    tokens against the tensor peak, and the attention's L2 gather rate."""
    import torch
    from sparse_attention_long_06_b200 import nsa
    cfg = wl.CONFIGS[name]
    inputs = wl.prefill_inputs(cfg)
    lens = list(inputs["seqlens"])
    T = int(inputs["cu_seqlens"][-1])
    idx = wl.indexer_inputs(lens, index_heads, index_dim, seed=cfg.seed)
    D, Hq = cfg.head_dim, cfg.num_q_heads
    d = {}
    for k in ("q", "k", "v", "cu_seqlens"):
        a = np.ascontiguousarray(inputs[k])
        d[k] = torch.from_numpy(a.view(np.int16) if a.dtype == np.uint16 else a).to(dev)
    for k in ("q_index", "w_index", "k_index"):
        a = np.ascontiguousarray(idx[k])
        d[k] = torch.from_numpy(a.view(np.int16) if a.dtype == np.uint16 else a).to(dev)
    plan = nsa.Plan.for_config(cfg, max_batch=len(lens), max_seqlen=max(lens), max_total_tokens=T,
                               out_dtype=nsa.OUT_BF16)
    out = torch.empty((T, Hq, D), dtype=torch.int16, device=dev)
    sel = torch.empty((T, top_k), dtype=torch.int32, device=dev)
    ws = torch.empty(plan.token_select_workspace_size(top_k), dtype=torch.uint8, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def step():
        plan.token_select_prefill(d["q"], d["k"], d["v"], d["q_index"], d["w_index"], d["k_index"],
                                  top_k, d["cu_seqlens"], out, ws, sel_idx=sel)

    for _ in range(warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    if nsa.read_device_status(ws) != nsa.NSA_OK:
        raise RuntimeError("token select: device status after warm-up")
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    for i in range(steps):
        flush.zero_()
        ev[i][0].record()
        step()
        ev[i][1].record()
    torch.cuda.synchronize()
    ms = max_over_ranks(statistics.median(a.elapsed_time(b) for a, b in ev), world, dev)
    nsa.profile_enable(True)
    flush.zero_()
    step()
    stage = nsa.profile_stage_ms()
    nsa.profile_enable(False)
    work = token_select_work(lens, D, Hq, cfg.num_kv_heads, index_heads, index_dim, top_k)
    f_index, f_attn, gather_bytes = work["index"], work["attn"], work["gather_bytes"]
    _, _, tc_sust, src = _peaks()
    ach_i = f_index / (stage[1] / 1e3) / 1e12
    ach_a = f_attn / (stage[3] / 1e3) / 1e12
    return {"metric": "token-level top-k attention tokens/s", "value": round(job_rate(T, world, ms), 1),
            "unit": "tokens/s", "ms_per_step_median": round(ms, 4), "steps": steps,
            "config": prefill_config(cfg, T, world) | {
                "mode": f"token select (indexer {index_heads} x {index_dim}, top_k {top_k})"},
            "algorithmic_flop_per_step": {"index": f_index, "attn": f_attn},
            "stage_ms": dict(zip(TOKEN_SELECT_KERNELS, [round(x, 4) for x in stage])),
            "rooflines": {
                "nsa_block_score_kernel": {"bound": "tensor", "achieved": round(ach_i, 2),
                                           "peak": tc_sust, "unit": "TFLOP/s",
                                           "frac": round(ach_i / tc_sust, 4),
                                           "peak_source": f"{src} bf16 sustained"},
                "nsa_token_attn_kernel": {"bound": "tensor", "achieved": round(ach_a, 2),
                                          "peak": tc_sust, "unit": "TFLOP/s",
                                          "frac": round(ach_a / tc_sust, 4),
                                          "peak_source": f"{src} bf16 sustained",
                                          "l2_gather_bytes": gather_bytes,
                                          "l2_gather_tbs": round(gather_bytes / (stage[3] / 1e3) / 1e12, 2)}}}


def oracle_single_core(names=("tiny", "prefill_8k"), nrows=64):
    """The oracle's tokens/s on one host core for small configurations, in a
    child process with OMP_NUM_THREADS=1 (bounded: `nrows` sampled rows)."""
    env = dict(os.environ, OMP_NUM_THREADS="1")
    out = {}
    for name in names:
        r = subprocess.run([sys.executable, os.path.abspath(__file__), "--oracle-sample", name,
                            "--oracle-rows", str(nrows)], env=env, capture_output=True, text=True,
                           timeout=600)
        if r.returncode != 0:
            out[name] = {"error": r.stderr.strip().splitlines()[-1:]}
            continue
        out[name] = json.loads(r.stdout.strip().splitlines()[-1])
    return out


# ---------------------------------------------------------------- decode leg
def decode_bytes(cfg, lens, sel):
    """Unique HBM bytes one decode step must read/write: per (sequence, group)
    the compressed keys and values of the complete blocks, the selected blocks'
    keys and values and the window's (their union counted once), plus q,
    gates and out."""
    D, Hq, Hkv, w = cfg.head_dim, cfg.num_q_heads, cfg.num_kv_heads, cfg.window
    l, d, ls = cfg.cmp_block, cfg.cmp_stride, cfg.sel_block
    total = 0
    for b, L in enumerate(lens):
        t = L - 1
        C = (L - l) // d + 1 if L >= l else 0
        win = set(range(max(0, t - w + 1), t + 1))
        for g in range(Hkv):
            keys = set(win)
            for blk in sel[b, g]:
                if blk >= 0:
                    keys.update(range(blk * ls, min(blk * ls + ls, t + 1)))
            total += C * D * 2 * 2 + len(keys) * D * 2 * 2
        total += Hq * D * 2 + Hq * 3 * 4 + Hq * D * 2
    return total


def run_decode_leg(args, dev, world=1):
    import torch
    from sparse_attention_long_06_b200 import nsa
    cfg = wl.CONFIGS["decode_64k"]
    if args.decode_batch:
        cfg = dataclasses.replace(cfg, decode_batch=args.decode_batch)
    inp = wl.decode_inputs(cfg)
    B, cap = cfg.decode_batch, int(inp["capacity"])
    d = {}
    for k in ("q", "k", "v", "kc", "vc", "gates", "w_k", "w_v", "seqlens"):
        a = np.ascontiguousarray(inp[k])
        d[k] = torch.from_numpy(a.view(np.int16) if a.dtype == np.uint16 else a).to(dev)
    del inp["k"], inp["v"]
    plan = nsa.Plan.for_config(cfg, max_batch=B, max_seqlen=cap, out_dtype=nsa.OUT_BF16)
    out = torch.empty((B, cfg.num_q_heads, cfg.head_dim), dtype=torch.int16, device=dev)
    sel = torch.empty((B, cfg.num_kv_heads, cfg.top_n), dtype=torch.int32, device=dev)
    ws = plan.alloc_workspace(nsa.MODE_DECODE, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def step():
        plan.decode(d["q"], d["k"], d["v"], d["kc"], d["vc"], d["seqlens"], d["gates"], d["w_k"],
                    d["w_v"], out, ws, sel_idx=sel)

    for _ in range(max(3, args.warmup)):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    if nsa.read_device_status(ws) != nsa.NSA_OK:
        raise RuntimeError("decode device status after warm-up")
    steps = max(args.steps, 20)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for i in range(steps):
        flush.zero_()
        ev[i][0].record()
        step()
        ev[i][1].record()
    torch.cuda.synchronize()
    ms = [a.elapsed_time(b) for a, b in ev]
    med = max_over_ranks(statistics.median(ms), world, dev)
    nsa.profile_enable(True)
    flush.zero_()
    step()
    stage = nsa.profile_stage_ms()
    nsa.profile_enable(False)
    nbytes = decode_bytes(cfg, [int(x) for x in d["seqlens"].cpu()], sel.cpu().numpy())
    hbm, _, _, src = _peaks()
    gbs = nbytes / (med / 1e3) / 1e9
    kern_ms = stage[1] + stage[2]  # the two decode kernels (after the block compression)
    kgbs = nbytes / (kern_ms / 1e3) / 1e9
    return {"metric": "NSA decode tokens/s", "value": round(job_rate(B, world, med), 1), "unit": "tokens/s",
            "ms_per_step_median": round(med, 5), "steps": steps,
            "config": {"workload": cfg.name, "batch": B, "context": int(cfg.decode_len),
                       "q_heads": cfg.num_q_heads, "kv_heads": cfg.num_kv_heads, "head_dim": cfg.head_dim,
                       "l": cfg.cmp_block, "d": cfg.cmp_stride, "l_sel": cfg.sel_block,
                       "top_n": cfg.top_n, "window": cfg.window,
                       "l2": "flushed before every timed step"},
            "stage_ms": {"nsa_decode_compress_kernel": round(stage[0], 5),
                         "nsa_decode_a_kernel": round(stage[1], 5),
                         "nsa_decode_b_kernel": round(stage[2], 5)},
            "roofline": {"bound": "hbm", "kernel": "nsa_decode_a_kernel + nsa_decode_b_kernel",
                         "achieved": round(kgbs, 1),
                         "peak": hbm, "unit": "GB/s", "frac": round(kgbs / hbm, 4),
                         "algorithmic_bytes": int(nbytes), "step_gbs": round(gbs, 1),
                         "peak_source": f"{src} copy bandwidth"}}


# ---------------------------------------------------------------- reference arm
def run_reference(args):
    cfg = wl.CONFIGS[args.workload]
    inputs = wl.prefill_inputs(cfg)
    for _ in range(args.warmup):
        oracle_sample(cfg, inputs, nrows=4)
    vals, descs = [], []
    t0 = time.perf_counter()
    for _ in range(args.steps):
        r = oracle_sample(cfg, inputs, nrows=8)
        vals.append(r["value"])
        descs.append(r["sample"])
    wall = time.perf_counter() - t0
    v = statistics.median(vals)
    cb = {"value": round(v, 3), "unit": "tokens/s", "cores": r["cores"], "kind": "oracle",
          "sample": "per step: " + descs[-1]}
    return {"impl": "reference", "metric": METRIC, "value": round(v, 3), "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(1e3 * wall / args.steps, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": prefill_config(cfg, int(inputs["cu_seqlens"][-1]), args.gpus),
            "cpu_baseline": cb,
            "e2e": {"value": round(v, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=60)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="prefill_64k",
                    choices=["prefill_64k", "prefill_8k", "varlen", "prefill_8k_overlap"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--decode-only", action="store_true",
                    help="run only the decode leg and print its object (profiling)")
    ap.add_argument("--decode-batch", type=int, default=0,
                    help="sequences in the decode leg (default: the workload's 32)")
    ap.add_argument("--token-select-only", action="store_true",
                    help="time only the token-level top-k leg (on --workload)")
    ap.add_argument("--block-select-decode-only", action="store_true",
                    help="time only the select-only decode leg")
    ap.add_argument("--block-select-only", action="store_true",
                    help="time only the select-only block attention leg")
    ap.add_argument("--no-legs", action="store_true",
                    help="skip the 8k / varlen prefill lines")
    ap.add_argument("--oracle-sample", default="",
                    help=argparse.SUPPRESS)  # child process of oracle_single_core
    ap.add_argument("--oracle-rows", type=int, default=64, help=argparse.SUPPRESS)
    args = ap.parse_args()
    if args.oracle_sample:
        cfg = wl.CONFIGS[args.oracle_sample]
        print(json.dumps(oracle_sample(cfg, wl.prefill_inputs(cfg), nrows=args.oracle_rows)))
        return
    if args.warmup < 3 and args.impl == "ours":
        args.warmup = 3
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference":
        if rank != 0:
            return
        print(json.dumps(run_reference(args)), flush=True)
        return
    import torch
    if world > 1:
        import datetime
        local = int(os.environ.get("LOCAL_RANK", "0"))
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    from sparse_attention_long_06_b200 import build
    if rank == 0 or world == 1:
        build.build()
    if world > 1:
        torch.distributed.barrier()
    if args.decode_only:
        res = run_decode_leg(args, torch.device("cuda", torch.cuda.current_device()), world)
    elif args.token_select_only:
        res = run_token_select_leg(torch.device("cuda", torch.cuda.current_device()), world,
                                   steps=max(args.steps, 3), warmup=args.warmup, name=args.workload)
    elif args.block_select_decode_only:
        res = run_block_select_decode_leg(torch.device("cuda", torch.cuda.current_device()), world,
                                          steps=max(args.steps, 20), warmup=args.warmup)
    elif args.block_select_only:
        res = run_block_select_leg(torch.device("cuda", torch.cuda.current_device()), world,
                                   steps=max(args.steps, 3), warmup=args.warmup,
                                   name=args.workload)
    else:
        res = run_ours(args, rank, world)
    if world > 1:
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
