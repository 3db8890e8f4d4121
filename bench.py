#!/usr/bin/env python
"""Benchmark of the fused-attention hot path on B200.

One step = one pass of the whole hot path over one batch of synthetic input:
  * fused causal prefill, B=4, Hq=Hkv=16, N=4096, d=128 (attn_fwd), and
  * split-KV paged decode, 64 sequences x 1 token, Hq=32, Hkv=8, d=128,
    16-token pages, lengths uniform on [512, 32768] (attn_paged_decode + combine).
The headline metric is the prefill's TFLOP/s (visible (q, k) pairs, both
contractions, 2 flop per multiply-add); the decode's KV GB/s is reported in
the same line under "decode".  Timed on their own after the step: the other
two prefill workloads (long: N=16384 non-causal with sharp key peaks; gqa:
Hq=32 over Hkv=8, N=8192 causal) under "long" and "gqa", the backward pass
(attn_bwd on the prefill workload) under "backward", a varlen chunked prefill
over the paged cache (attn_paged_prefill) under "paged_prefill" and the FP8
prefill under "fp8_prefill".  The CPU-baseline leg also compares the step's
prefill output with the oracle on every row ("parity").  Inputs are
resident in HBM when timing starts;
L2 (126 MB) is flushed by writing a 256 MB buffer before every step, outside
the kernels' event brackets.  Kernel times are CUDA events on the launching
stream; multi-GPU runs take the max over ranks.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

With N > 1 (torchrun, one process per GPU, NCCL for the barrier and the
max-over-ranks reduction only) every rank runs its own replica of the
workload with its own seed: weak scaling, no data-path collective.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from tiled_attention_17_b200 import accounting, inputs  # noqa: E402

PREFILL = inputs.PREFILL_CONFIGS["causal"]
DECODE = inputs.DECODE_CONFIG
METRIC = "prefill attention TFLOP/s & % BF16 peak; paged decode KV GB/s & % HBM BW"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_FLUSH_BYTES = 256 << 20


# ---------------------------------------------------------------------------
# ranks
# ---------------------------------------------------------------------------

def rank_info():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def init_dist(world: int, backend: str = "nccl", timeout_s: int = 120):
    if world <= 1:
        return None
    import torch.distributed as dist
    if not dist.is_initialized():
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s))
    return dist


def barrier(dist, device=None):
    if dist is not None:
        if device is not None:
            dist.barrier(device_ids=[device])
        else:
            dist.barrier()


def max_over_ranks(values, dist, device="cpu"):
    """Element-wise max of a list of floats over all ranks (identity on 1 rank)."""
    if dist is None:
        return list(values)
    import torch
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.cpu().tolist()


def rank_seed(base: int, rank: int) -> int:
    """Each rank's replica draws its own inputs (distinct units per rank)."""
    return base + 1000 * rank


# ---------------------------------------------------------------------------
# peaks, clocks, profiles
# ---------------------------------------------------------------------------

def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def kernel_source_hash(fname: str) -> str:
    with open(os.path.join(ROOT, "tiled_attention_17_b200", "csrc", fname), "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def recorded_traffic(kernel: str, fname: str, units: float):
    """DRAM bytes per launch from a committed ncu capture, scaled to `units`
    (the capture records bytes per unit); None if absent or the kernel source
    changed since it was taken."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(p) as f:
            rec = json.load(f).get(kernel)
    except (OSError, ValueError):
        return None
    if not rec or rec.get("source_sha256_16") != kernel_source_hash(fname):
        return None
    return rec["dram_bytes_per_unit"] * units


class ClockSampler:
    """Samples nvidia-smi clocks/throttle reasons while the timed region runs."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.t = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "100",
                 "-i", str(self.gpu)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.t = threading.Thread(target=self._read, daemon=True)
        self.t.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self.t:
            self.t.join(timeout=2)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------
# CPU oracle baseline (rank 0, N=1, bounded sample)
# ---------------------------------------------------------------------------

def prefill_sample_rows(stride: int, shift: int = 0):
    """Every `stride`-th query row (starting at `shift`) of every (b, head): a
    bounded, representative sample of the causal workload (rows at all depths
    of the mask)."""
    c = PREFILL
    i = np.arange(shift, c.Nq, stride, dtype=np.int64)
    bh = np.arange(c.B * c.Hq, dtype=np.int64)
    rows = (bh[:, None] * c.Nq + i[None, :]).reshape(-1)
    flops = 4.0 * c.d * float((np.minimum(i + 1, c.Nkv)).sum()) * c.B * c.Hq
    return rows, flops


def host_cpu_model() -> str:
    """The host CPU's model name (first 'model name' line of /proc/cpuinfo)."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def parity_metrics(o_gpu, o_ref, lse_gpu, lse_ref) -> dict:
    """Max-abs and relative L2 error of O and max absolute lse error over the
    rows given (the parity bar: 2e-2, 5e-3, 1e-3)."""
    o_gpu = np.asarray(o_gpu, dtype=np.float64)
    o_ref = np.asarray(o_ref, dtype=np.float64)
    lg = np.asarray(lse_gpu, dtype=np.float64)
    lr = np.asarray(lse_ref, dtype=np.float64)
    both = np.isneginf(lg) & np.isneginf(lr)
    with np.errstate(invalid="ignore"):
        lse_err = float(np.abs(np.where(both, 0.0, lg - lr)).max())
    max_abs = float(np.abs(o_gpu - o_ref).max())
    rel = float(np.linalg.norm(o_gpu - o_ref) / np.linalg.norm(o_ref))
    return {"max_abs": max_abs, "rel_l2": rel, "lse_abs": lse_err,
            "pass": bool(max_abs <= 2e-2 and rel <= 5e-3 and lse_err <= 1e-3)}


def cpu_oracle_sample(q, k, v, stride: int, o_gpu=None, lse_gpu=None):
    """The oracle on every `stride`-th row of the causal workload, timed on the
    host cores; with the GPU's output of the same rows given, also the parity
    of that output against the oracle's (over all rows when stride is 1)."""
    import oracle
    rows, flops = prefill_sample_rows(stride)
    t0 = time.perf_counter()
    o_ref, lse_ref = oracle.attn(q, k, v, True, scale=PREFILL.scale, rows=rows)
    dt = time.perf_counter() - t0
    out = {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": oracle.num_threads(), "kind": "oracle",
           "cpu_model": host_cpu_model(), "hardware_threads": os.cpu_count(),
           "sample": f"fp64 oracle on every {stride}th query row of all {PREFILL.B}x{PREFILL.Hq} heads of the "
                     f"causal prefill workload ({rows.size} rows, {flops / 1e9:.1f} GFLOP, {dt:.1f} s)"}
    if o_gpu is not None:
        par = parity_metrics(o_gpu.reshape(-1, PREFILL.d)[rows], o_ref, lse_gpu.reshape(-1)[rows], lse_ref)
        par["rows"] = f"{rows.size} of {PREFILL.B * PREFILL.Hq * PREFILL.Nq}"
        out["parity"] = par
    return out


# ---------------------------------------------------------------------------
# reference arm: the oracle, timed on host cores
# ---------------------------------------------------------------------------

def run_reference(args):
    rank, world, _ = rank_info()
    if rank != 0:
        return 0
    import oracle
    q, k, v = inputs.prefill_inputs(PREFILL)
    stride = 256      # one step ~ 1/256 of the rows: a fraction of a second on 8 cores
    times, work = [], []
    for s in range(args.warmup + args.steps):
        rows, flops = prefill_sample_rows(stride, s % stride)   # a different slice of rows every step
        t0 = time.perf_counter()
        oracle.attn(q, k, v, True, scale=PREFILL.scale, rows=rows)
        if s >= args.warmup:
            times.append(time.perf_counter() - t0)
            work.append(flops)
    dt = sum(times) / len(times)
    val = sum(work) / sum(times) / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": val, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": "causal prefill B=4 Hq=Hkv=16 N=4096 d=128 bf16 (bounded row sample per step)",
                   "parallelism": "host cores"},
        "cpu_baseline": {"value": val, "unit": "TFLOP/s", "cores": oracle.num_threads(), "kind": "oracle",
                         "cpu_model": host_cpu_model(), "hardware_threads": os.cpu_count(),
                         "sample": f"every {stride}th query row per step ({len(rows)} rows)"},
        "e2e": {"value": val, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------

def run_ours(args):
    import torch
    from tiled_attention_17_b200 import binding

    rank, world, local = rank_info()
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    dist = init_dist(world)
    dev = torch.device("cuda", local)
    binding.load()
    stream = torch.cuda.current_stream()

    # ---- inputs (host, seeded per rank) -> HBM
    c = PREFILL
    q_h, k_h, v_h = inputs.prefill_inputs(c, seed=rank_seed(inputs.CONFIG_SEEDS["causal"], rank))
    dinp = inputs.paged_inputs(DECODE, seed=rank_seed(inputs.CONFIG_SEEDS["decode"], rank))

    def dev_bf16(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)

    q, k, v = dev_bf16(q_h), dev_bf16(k_h), dev_bf16(v_h)
    o = torch.empty_like(q)
    lse = torch.empty((c.B, c.Hq, c.Nq), dtype=torch.float32, device=dev)
    dq, dkc, dvc = dev_bf16(dinp.q), dev_bf16(dinp.k_cache), dev_bf16(dinp.v_cache)
    dbt = torch.from_numpy(dinp.block_table).to(dev)
    dsl = torch.from_numpy(dinp.seq_lens).to(dev)
    D = DECODE
    ws_bytes = binding.attn_paged_decode_workspace_size(D.num_seqs, D.Hq, D.Hkv, D.d, D.max_pages, D.page_size)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    do = torch.empty_like(dq)
    dlse = torch.empty((D.num_seqs, D.Hq), dtype=torch.float32, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def prefill():
        binding.attn_fwd(q, k, v, o, lse, c.B, c.Hq, c.Hkv, c.Nq, c.Nkv, c.d, c.scale, 1, stream)

    def decode():
        binding.attn_paged_decode(dq, dkc, dvc, dbt, dsl, D.page_size, D.num_seqs, D.Hq, D.Hkv, D.d, D.max_pages,
                                  dinp.num_pages_total, D.scale, do, dlse, ws, ws_bytes, stream)

    launches_per_step = 1 + 2   # prefill kernel; decode split kernel + combine kernel

    for _ in range(args.warmup):
        flush.zero_()
        prefill()
        decode()
    torch.cuda.synchronize()

    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    sampler = ClockSampler(local) if not args.no_clocks else None
    barrier(dist, local)
    torch.cuda.synchronize()
    if sampler:
        sampler.start()
        time.sleep(0.3)
    r0 = torch.cuda.Event(enable_timing=True)
    r1 = torch.cuda.Event(enable_timing=True)
    r0.record(stream)
    for s in range(args.steps):
        flush.zero_()
        ev[s][0].record(stream)
        prefill()
        ev[s][1].record(stream)
        decode()
        ev[s][2].record(stream)
    r1.record(stream)
    torch.cuda.synchronize()
    barrier(dist, local)
    clocks = sampler.stop() if sampler else None
    t_pre = sum(ev[s][0].elapsed_time(ev[s][1]) for s in range(args.steps)) / args.steps   # ms
    t_dec = sum(ev[s][1].elapsed_time(ev[s][2]) for s in range(args.steps)) / args.steps
    t_region = r0.elapsed_time(r1) / args.steps
    t_pre, t_dec, t_region = max_over_ranks([t_pre, t_dec, t_region], dist, device=dev)

    pre_flops = accounting.prefill_flops(c.B, c.Hq, c.Nq, c.Nkv, c.d, True)
    dec_bytes = accounting.decode_bytes(dinp.seq_lens, D.Hq, D.Hkv, D.d, D.page_size)
    tflops = pre_flops * world / (t_pre * 1e-3) / 1e12
    gbs = dec_bytes * world / (t_dec * 1e-3) / 1e9
    peaks, peak_kind = load_peaks()

    # ---- end to end through the public API with host buffers
    e2e = None
    dec_e2e = None
    if not args.no_e2e:
        e2e, dec_e2e = run_e2e(args, torch, binding, dev, stream, q_h, k_h, v_h, dinp, dist)

    # ---- varlen prefill over the paged cache (timed on its own, after the step)
    paged = None
    if not args.no_paged_prefill:
        paged = run_paged_prefill(args, torch, binding, dev, stream, flush, dist, rank, world, peaks)

    # ---- backward pass on the prefill workload (timed on its own, after the step)
    bwd = None
    if not args.no_backward:
        bwd = run_backward(args, torch, binding, dev, stream, q, k, v, o, lse, flush, dist, rank, world, peaks)

    # ---- FP8 (E4M3) prefill on the same shape (timed on its own, after the step)
    fp8 = None
    if not args.no_fp8:
        fp8 = run_fp8_prefill(args, torch, binding, dev, stream, flush, dist, rank, world, peaks)

    # ---- the other two prefill workloads (timed on their own, after the step)
    legs = {}
    if not args.no_prefill_legs:
        for name in ("long", "gqa"):
            legs[name] = run_prefill_leg(args, torch, binding, dev, stream, flush, dist, rank, world, peaks, name)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        # the step's output (every step writes the same o and lse) against the
        # oracle on the same rows
        o_step = o.float().cpu().numpy()
        lse_step = lse.cpu().numpy()
        cpu = cpu_oracle_sample(q_h, k_h, v_h, args.cpu_stride, o_step, lse_step)

    if rank == 0:
        pre_per_gpu = pre_flops / (t_pre * 1e-3) / 1e12
        dec_per_gpu = dec_bytes / (t_dec * 1e-3) / 1e9
        line = {
            "metric": METRIC, "value": tflops, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": t_pre + t_dec, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": f"causal prefill B={c.B} Hq=Hkv={c.Hq} N={c.Nq} d={c.d} bf16 + paged decode "
                                   f"{D.num_seqs} seqs x 1 token Hq={D.Hq} Hkv={D.Hkv} d={D.d} page {D.page_size} "
                                   f"len U[{D.len_lo},{D.len_hi}] (sum {int(dinp.seq_lens.sum())})",
                       "per_rank": "one replica per GPU, seed offset per rank",
                       "l2": "256 MB buffer written before every step (outside kernel events); decode KV 4.4 GB > L2",
                       "parallelism": f"replicas x{world}"},
            "prefill": {"ms": t_pre, "tflops": tflops, "flops_per_step_per_gpu": pre_flops},
            "decode": {"value": gbs, "unit": "GB/s", "ms": t_dec, "bytes_per_step_per_gpu": dec_bytes,
                       "roofline": roofline("hbm", dec_per_gpu, peaks["hbm_gbs"], "GB/s",
                                            recorded_traffic("decode_split_g4_kernel", "decode_paged.cu",
                                                             float(dinp.seq_lens.sum()))),
                       "e2e": dec_e2e},
            "long": legs.get("long"),
            "gqa": legs.get("gqa"),
            "backward": bwd,
            "paged_prefill": paged,
            "fp8_prefill": fp8,
            "roofline": roofline("tensor", pre_per_gpu, peaks["bf16_tflops"], "TFLOP/s",
                                 recorded_traffic("prefill_fwd_kernel", "prefill_sm100.cu", float(c.B * c.Hq))),
            "peaks": {"source": peak_kind, "bf16_tflops": peaks["bf16_tflops"], "hbm_gbs": peaks["hbm_gbs"],
                      "note": "prefill against the burst bf16 GEMM peak; decode against the copy bandwidth"},
            "region_ms_per_step": t_region,
            "gpu_launches": launches_per_step * args.steps,
            "e2e": e2e,
            "cpu_baseline": cpu,
            "parity": cpu.get("parity") if cpu else None,
            "clocks": clocks,
        }
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.destroy_process_group()
    return 0


def run_prefill_leg(args, torch, binding, dev, stream, flush, dist, rank, world, peaks, name):
    """attn_fwd on another prefill workload (long: B=1, H=8, N=16384,
    non-causal, every 64th key row x4; gqa: B=2, Hq=32, Hkv=8, N=8192,
    causal): CUDA events around each call, L2 flushed before every call, max
    over ranks."""
    c = inputs.PREFILL_CONFIGS[name]
    q_h, k_h, v_h = inputs.prefill_inputs(c, seed=rank_seed(inputs.CONFIG_SEEDS[name], rank))

    def bf(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)

    q, k, v = bf(q_h), bf(k_h), bf(v_h)
    del q_h, k_h, v_h
    o = torch.empty_like(q)
    lse = torch.empty((c.B, c.Hq, c.Nq), dtype=torch.float32, device=dev)

    def call():
        binding.attn_fwd(q, k, v, o, lse, c.B, c.Hq, c.Hkv, c.Nq, c.Nkv, c.d, c.scale, int(c.causal), stream)

    for _ in range(3):
        flush.zero_()
        call()
    torch.cuda.synchronize()
    steps = max(3, min(args.steps, 10))
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    barrier(dist, dev.index)
    for e0, e1 in ev:
        flush.zero_()
        e0.record(stream)
        call()
        e1.record(stream)
    torch.cuda.synchronize()
    t = sum(e0.elapsed_time(e1) for e0, e1 in ev) / steps
    (t,) = max_over_ranks([t], dist, device=dev)
    flops = accounting.prefill_flops(c.B, c.Hq, c.Nq, c.Nkv, c.d, c.causal)
    per_gpu = flops / (t * 1e-3) / 1e12
    workload = (f"B={c.B} Hq={c.Hq} Hkv={c.Hkv} N={c.Nq} d={c.d} {'causal' if c.causal else 'non-causal'}"
                + (f", key rows j%{c.peak_rows_every}==0 x{c.peak_factor:g}" if c.peak_rows_every else ""))
    return {"value": per_gpu * world, "unit": "TFLOP/s", "ms": t, "steps": steps, "workload": workload,
            "flops_per_call_per_gpu": flops, "gpu_launches_per_call": 1,
            "roofline": roofline("tensor", per_gpu, peaks["bf16_tflops"], "TFLOP/s",
                                 recorded_traffic(f"prefill_fwd_kernel_{name}", "prefill_sm100.cu",
                                                  float(c.B * c.Hq)))}


PAGED_MIX = dict(num_seqs=32, q_lo=1, q_hi=2048, prefix_lo=0, prefix_hi=8192, Hq=32, Hkv=8, d=128, page_size=16)


def run_paged_prefill(args, torch, binding, dev, stream, flush, dist, rank, world, peaks):
    """attn_paged_prefill on a serving-like chunked-prefill batch: 32 sequences,
    1-2048 new tokens each after a 0-8192-token prefix already in the pool
    (Hq=32, Hkv=8, d=128, 16-token pages at a seeded permutation), causal.
    CUDA events around each call, L2 flushed before every call."""
    m = PAGED_MIX
    rng = np.random.Generator(np.random.PCG64(rank_seed(4321, rank)))
    q_lens = rng.integers(m["q_lo"], m["q_hi"], size=m["num_seqs"], endpoint=True)
    kv_lens = q_lens + rng.integers(m["prefix_lo"], m["prefix_hi"], size=m["num_seqs"], endpoint=True)
    inp = inputs.paged_prefill_inputs(q_lens, kv_lens, m["Hq"], m["Hkv"], m["d"], m["page_size"],
                                      seed=rank_seed(4322, rank))

    def bf(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)

    def i32(a):
        return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(dev)

    q, kc, vc = bf(inp.q), bf(inp.k_cache), bf(inp.v_cache)
    bt, cu, sl = i32(inp.block_table), i32(inp.cu_seqlens), i32(inp.seq_lens)
    o = torch.empty_like(q)
    lse = torch.empty((q.shape[0], m["Hq"]), dtype=torch.float32, device=dev)

    def call():
        binding.attn_paged_prefill(q, kc, vc, bt, cu, sl, m["page_size"], m["num_seqs"], q.shape[0], inp.max_q_len,
                                   m["Hq"], m["Hkv"], m["d"], bt.shape[1], kc.shape[0], m["d"] ** -0.5, 1, o, lse,
                                   stream)

    for _ in range(3):
        flush.zero_()
        call()
    torch.cuda.synchronize()
    steps = max(3, min(args.steps, 10))
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    barrier(dist, dev.index)
    for e0, e1 in ev:
        flush.zero_()
        e0.record(stream)
        call()
        e1.record(stream)
    torch.cuda.synchronize()
    t = sum(e0.elapsed_time(e1) for e0, e1 in ev) / steps
    (t,) = max_over_ranks([t], dist, device=dev)
    flops = accounting.varlen_prefill_flops(q_lens, kv_lens, m["Hq"], m["d"], True)
    per_gpu = flops / (t * 1e-3) / 1e12
    return {"value": per_gpu * world, "unit": "TFLOP/s", "ms": t, "steps": steps,
            "workload": (f"{m['num_seqs']} seqs, new tokens U[{m['q_lo']},{m['q_hi']}] after prefix "
                         f"U[{m['prefix_lo']},{m['prefix_hi']}], Hq={m['Hq']} Hkv={m['Hkv']} d={m['d']}, "
                         f"{m['page_size']}-token pages, causal; total_q {int(q_lens.sum())}, "
                         f"keys {int(kv_lens.sum())}"),
            "flops_per_call_per_gpu": flops, "gpu_launches_per_call": 1,
            "roofline": roofline("tensor", per_gpu, peaks["bf16_tflops"], "TFLOP/s",
                                 recorded_traffic("paged_prefill", "prefill_sm100.cu", 1.0))}


def run_backward(args, torch, binding, dev, stream, q, k, v, o, lse, flush, dist, rank, world, peaks):
    """attn_bwd on the causal prefill workload (o and lse from the step's
    forward call, seeded dO): CUDA events around each call, L2 flushed before
    every call, max over ranks.  FLOPs are the method's five products
    (2.5x the forward count); the kernels compute seven."""
    c = PREFILL
    do_h = inputs.grad_output((c.B, c.Hq, c.Nq, c.d), seed=rank_seed(inputs.CONFIG_SEEDS["causal"] + 100, rank))
    dout = torch.from_numpy(np.ascontiguousarray(do_h).view(np.int16)).view(torch.bfloat16).to(dev)
    ws_bytes = binding.attn_bwd_workspace_size(c.B, c.Hq, c.Nq)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    gq, gk, gv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)

    def call():
        binding.attn_bwd(q, k, v, o, dout, lse, gq, gk, gv, ws, ws_bytes, c.B, c.Hq, c.Hkv, c.Nq, c.Nkv, c.d,
                         c.scale, 1, stream)

    for _ in range(3):
        flush.zero_()
        call()
    torch.cuda.synchronize()
    steps = max(3, min(args.steps, 10))
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    barrier(dist, dev.index)
    for e0, e1 in ev:
        flush.zero_()
        e0.record(stream)
        call()
        e1.record(stream)
    torch.cuda.synchronize()
    t = sum(e0.elapsed_time(e1) for e0, e1 in ev) / steps
    (t,) = max_over_ranks([t], dist, device=dev)
    flops = 2.5 * accounting.prefill_flops(c.B, c.Hq, c.Nq, c.Nkv, c.d, True)
    per_gpu = flops / (t * 1e-3) / 1e12
    return {"value": per_gpu * world, "unit": "TFLOP/s", "ms": t, "steps": steps,
            "flops_per_call_per_gpu": flops, "flops_note": "5 products of the method (2.5x forward); 7 computed",
            "gpu_launches_per_call": 3,
            "roofline": roofline("tensor", per_gpu, peaks["bf16_tflops"], "TFLOP/s",
                                 recorded_traffic("attn_bwd", "backward_sm100.cu", float(c.B * c.Hkv)))}


def run_fp8_prefill(args, torch, binding, dev, stream, flush, dist, rank, world, peaks):
    """attn_fwd_fp8 on the causal prefill workload's shape (the same N(0, 1)
    draws quantised per tensor to E4M3): CUDA events around each call, L2
    flushed before every call, max over ranks.  The roofline peak is the
    measured bf16 GEMM peak times the nominal fp8/bf16 ratio (4.5 / 2.25)."""
    c = PREFILL
    q8, k8, v8, desc = inputs.random_prefill_fp8(c.B, c.Hq, c.Hkv, c.Nq, c.Nkv, c.d,
                                                 seed=rank_seed(inputs.CONFIG_SEEDS["causal"], rank))
    q, k, v = (torch.from_numpy(x).to(dev) for x in (q8, k8, v8))
    o = torch.empty((c.B, c.Hq, c.Nq, c.d), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((c.B, c.Hq, c.Nq), dtype=torch.float32, device=dev)

    def call():
        binding.attn_fwd_fp8(q, k, v, *desc, o, lse, c.B, c.Hq, c.Hkv, c.Nq, c.Nkv, c.d, c.scale, 1, stream)

    for _ in range(3):
        flush.zero_()
        call()
    torch.cuda.synchronize()
    steps = max(3, min(args.steps, 10))
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    barrier(dist, dev.index)
    for e0, e1 in ev:
        flush.zero_()
        e0.record(stream)
        call()
        e1.record(stream)
    torch.cuda.synchronize()
    t = sum(e0.elapsed_time(e1) for e0, e1 in ev) / steps
    (t,) = max_over_ranks([t], dist, device=dev)
    flops = accounting.prefill_flops(c.B, c.Hq, c.Nq, c.Nkv, c.d, True)
    per_gpu = flops / (t * 1e-3) / 1e12
    fp8_peak = 2.0 * peaks["bf16_tflops"]
    return {"value": per_gpu * world, "unit": "TFLOP/s", "ms": t, "steps": steps, "dtype": "e4m3 in, f32 accumulate",
            "flops_per_call_per_gpu": flops, "gpu_launches_per_call": 1,
            "vs_bf16_peak": per_gpu / peaks["bf16_tflops"],
            "roofline": roofline("tensor", per_gpu, fp8_peak, "TFLOP/s",
                                 recorded_traffic("prefill_fwd_kernel_fp8", "prefill_sm100.cu", float(c.B * c.Hq)))}


def roofline(bound, achieved, peak, unit, traffic):
    return {"bound": bound, "achieved": achieved, "peak": peak, "unit": unit, "frac": achieved / peak,
            "traffic": traffic}


def run_e2e(args, torch, binding, dev, stream, q_h, k_h, v_h, dinp, dist):
    """Same metrics through the public API with pinned host buffers: every step
    copies its inputs host->device and its outputs device->host."""
    c, D = PREFILL, DECODE
    steps = max(1, min(args.steps, args.e2e_steps))

    def pinned(a):
        t = torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)
        return t.pin_memory()

    hq, hk, hv = pinned(q_h), pinned(k_h), pinned(v_h)
    ho = torch.empty(hq.shape, dtype=torch.bfloat16).pin_memory()
    hl = torch.empty((c.B, c.Hq, c.Nq), dtype=torch.float32).pin_memory()
    q = torch.empty(hq.shape, dtype=torch.bfloat16, device=dev)
    k = torch.empty(hk.shape, dtype=torch.bfloat16, device=dev)
    v = torch.empty(hv.shape, dtype=torch.bfloat16, device=dev)
    o = torch.empty_like(q)
    lse = torch.empty((c.B, c.Hq, c.Nq), dtype=torch.float32, device=dev)
    h2d = (hq.numel() + hk.numel() + hv.numel()) * 2
    d2h = ho.numel() * 2 + hl.numel() * 4

    def pre_step():
        q.copy_(hq, non_blocking=True)
        k.copy_(hk, non_blocking=True)
        v.copy_(hv, non_blocking=True)
        binding.attn_fwd(q, k, v, o, lse, c.B, c.Hq, c.Hkv, c.Nq, c.Nkv, c.d, c.scale, 1, stream)
        ho.copy_(o, non_blocking=True)
        hl.copy_(lse, non_blocking=True)

    t_pre = timed(torch, stream, pre_step, steps)

    dq_h, dk_h, dv_h = pinned(dinp.q), pinned(dinp.k_cache), pinned(dinp.v_cache)
    dbt_h = torch.from_numpy(dinp.block_table).pin_memory()
    dsl_h = torch.from_numpy(dinp.seq_lens).pin_memory()
    dq = torch.empty(dq_h.shape, dtype=torch.bfloat16, device=dev)
    dk = torch.empty(dk_h.shape, dtype=torch.bfloat16, device=dev)
    dv = torch.empty(dv_h.shape, dtype=torch.bfloat16, device=dev)
    dbt = torch.empty(dbt_h.shape, dtype=torch.int32, device=dev)
    dsl = torch.empty(dsl_h.shape, dtype=torch.int32, device=dev)
    ws_bytes = binding.attn_paged_decode_workspace_size(D.num_seqs, D.Hq, D.Hkv, D.d, D.max_pages, D.page_size)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    do = torch.empty_like(dq)
    dl = torch.empty((D.num_seqs, D.Hq), dtype=torch.float32, device=dev)
    ho2 = torch.empty(dq_h.shape, dtype=torch.bfloat16).pin_memory()
    hl2 = torch.empty((D.num_seqs, D.Hq), dtype=torch.float32).pin_memory()
    dh2d = (dq_h.numel() + dk_h.numel() + dv_h.numel()) * 2 + (dbt_h.numel() + dsl_h.numel()) * 4
    dd2h = ho2.numel() * 2 + hl2.numel() * 4

    def dec_step():
        dq.copy_(dq_h, non_blocking=True)
        dk.copy_(dk_h, non_blocking=True)
        dv.copy_(dv_h, non_blocking=True)
        dbt.copy_(dbt_h, non_blocking=True)
        dsl.copy_(dsl_h, non_blocking=True)
        binding.attn_paged_decode(dq, dk, dv, dbt, dsl, D.page_size, D.num_seqs, D.Hq, D.Hkv, D.d, D.max_pages,
                                  dinp.num_pages_total, D.scale, do, dl, ws, ws_bytes, stream)
        ho2.copy_(do, non_blocking=True)
        hl2.copy_(dl, non_blocking=True)

    t_dec = timed(torch, stream, dec_step, steps)
    t_pre, t_dec = max_over_ranks([t_pre, t_dec], dist, device=dev)
    world = rank_info()[1]
    pre_flops = accounting.prefill_flops(c.B, c.Hq, c.Nq, c.Nkv, c.d, True)
    dec_bytes = accounting.decode_bytes(dinp.seq_lens, D.Hq, D.Hkv, D.d, D.page_size)
    e2e = {"value": pre_flops * world / (t_pre * 1e-3) / 1e12, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
           "d2h_bytes_per_step": d2h, "ms_per_step": t_pre, "steps": steps}
    dec = {"value": dec_bytes * world / (t_dec * 1e-3) / 1e9, "unit": "GB/s", "h2d_bytes_per_step": dh2d,
           "d2h_bytes_per_step": dd2h, "ms_per_step": t_dec, "steps": steps}
    return e2e, dec


def timed(torch, stream, fn, steps):
    fn()                      # warm-up
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        fn()
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / steps


def run_ncu_case(args):
    """A small, self-contained case for a profiler capture of one kernel:
    prefill = the causal workload (about 270 MB on the device); long and gqa =
    those prefill workloads (about 135 and 340 MB); decode = 16
    sequences with the benchmark's length distribution (about 1.1 GB, larger
    than L2).  Runs `--reps` launches and exits."""
    import torch
    from tiled_attention_17_b200 import binding
    binding.load()
    dev = torch.device("cuda", 0)

    def dev_bf16(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)

    if args.ncu_case == "fp8":
        c = PREFILL
        q8, k8, v8, desc = inputs.random_prefill_fp8(c.B, c.Hq, c.Hkv, c.Nq, c.Nkv, c.d,
                                                     seed=inputs.CONFIG_SEEDS["causal"])
        q, k, v = (torch.from_numpy(x).to(dev) for x in (q8, k8, v8))
        o = torch.empty((c.B, c.Hq, c.Nq, c.d), dtype=torch.bfloat16, device=dev)
        lse = torch.empty((c.B, c.Hq, c.Nq), dtype=torch.float32, device=dev)
        for _ in range(args.reps):
            binding.attn_fwd_fp8(q, k, v, *desc, o, lse, c.B, c.Hq, c.Hkv, c.Nq, c.Nkv, c.d, c.scale, 1)
    elif args.ncu_case == "paged":
        m = PAGED_MIX
        rng = np.random.Generator(np.random.PCG64(4321))
        q_lens = rng.integers(m["q_lo"], m["q_hi"], size=m["num_seqs"], endpoint=True)
        kv_lens = q_lens + rng.integers(m["prefix_lo"], m["prefix_hi"], size=m["num_seqs"], endpoint=True)
        inp = inputs.paged_prefill_inputs(q_lens, kv_lens, m["Hq"], m["Hkv"], m["d"], m["page_size"], seed=4322)
        i32 = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(dev)
        q, kc, vc = dev_bf16(inp.q), dev_bf16(inp.k_cache), dev_bf16(inp.v_cache)
        bt, cu, sl = i32(inp.block_table), i32(inp.cu_seqlens), i32(inp.seq_lens)
        for _ in range(args.reps):
            binding.paged_prefill(q, kc, vc, bt, cu, sl, inp.max_q_len, True)
    elif args.ncu_case == "backward":
        c = PREFILL
        q_h, k_h, v_h = inputs.prefill_inputs(c)
        q, k, v = dev_bf16(q_h), dev_bf16(k_h), dev_bf16(v_h)
        dout = dev_bf16(inputs.grad_output(q_h.shape, seed=inputs.CONFIG_SEEDS["causal"] + 100))
        o, lse = binding.attention(q, k, v, True, c.scale)
        for _ in range(args.reps):
            binding.attention_backward(q, k, v, o, lse, dout, True, c.scale)
    elif args.ncu_case in ("prefill", "long", "gqa"):
        c = PREFILL if args.ncu_case == "prefill" else inputs.PREFILL_CONFIGS[args.ncu_case]
        q_h, k_h, v_h = inputs.prefill_inputs(c)
        q, k, v = dev_bf16(q_h), dev_bf16(k_h), dev_bf16(v_h)
        o = torch.empty_like(q)
        lse = torch.empty((c.B, c.Hq, c.Nq), dtype=torch.float32, device=dev)
        for _ in range(args.reps):
            binding.attn_fwd(q, k, v, o, lse, c.B, c.Hq, c.Hkv, c.Nq, c.Nkv, c.d, c.scale, int(c.causal))
    else:
        import dataclasses
        D = dataclasses.replace(DECODE, num_seqs=16)
        dinp = inputs.paged_inputs(D)
        dq, dkc, dvc = dev_bf16(dinp.q), dev_bf16(dinp.k_cache), dev_bf16(dinp.v_cache)
        dbt = torch.from_numpy(dinp.block_table).to(dev)
        dsl = torch.from_numpy(dinp.seq_lens).to(dev)
        ws = None
        for _ in range(args.reps):
            _o, _l, ws = binding.paged_decode(dq, dkc, dvc, dbt, dsl, workspace=ws)
    torch.cuda.synchronize()
    print(json.dumps({"ncu_case": args.ncu_case, "reps": args.reps, "ok": True}))
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-stride", type=int, default=1, help="oracle baseline: every n-th query row")
    ap.add_argument("--no-clocks", action="store_true")
    ap.add_argument("--no-backward", action="store_true")
    ap.add_argument("--no-paged-prefill", action="store_true")
    ap.add_argument("--no-fp8", action="store_true")
    ap.add_argument("--no-prefill-legs", action="store_true", help="skip the long and gqa prefill legs")
    ap.add_argument("--ncu-case", choices=["prefill", "long", "gqa", "decode", "backward", "paged", "fp8"],
                    default=None,
                    help="run a small single-kernel case for a profiler capture and exit")
    ap.add_argument("--reps", type=int, default=4)
    args = ap.parse_args(argv)
    if args.ncu_case:
        return run_ncu_case(args)
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
