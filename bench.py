#!/usr/bin/env python
"""Paged decode attention benchmark (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config 2..8] [--impl ours|reference]

A step is one pass of the hot path over one batch: the host slot bookkeeping
(page allocation at block boundaries), kv_append of the new token's K/V and
paged_decode_attention (split-KV + combine where chosen).
Workloads (synthetic, seeded; no dataset is involved):
  --config 2  Llama-3.1-8B-shaped decode layer, bf16 K/V: B=64, H_q=32, H_kv=8,
              Dh=128, page 16, cached lengths U[512, 4096] (the default). On
              one GPU the line also carries, under "configs", the 32K-context
              and mixed-sweep records measured in the same process.
  --config 3  one 32K-token sequence, 32 layers, fp16 K/V (4 GiB cache); the
              32 per-layer calls of a step are replayed as one CUDA graph.
  --config 4..8  shared prefix, mixed sweep, RoPE append, E4M3 cache, prefill.
`value` is device-timed over exactly K steps with all step inputs resident in
HBM; `sustained` replays the timed window for >= 1 s, five times, and gives
the median; `e2e` repeats the loop through the same calls with the step's
inputs copied from pinned host memory and the output read back every step.
Multi-GPU runs are replicas (each rank its own batch, no data-path
collective): weak scaling.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "paged decode attention seq-steps/s; achieved HBM GB/s and % of B200 peak"
PROFILE_DECODE = os.path.join(ROOT, "profiles", "paged_decode_mma_kernel__llama8b_layer_bf16_B64.md")
UNIT = "seq-steps/s"
FALLBACK_HBM_GBS = 6650.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=None)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", type=int, choices=[2, 3, 4, 5, 6, 7, 8], default=2,
                    help="2: 8B-shaped layer (default); 3: 32K context x 32 layers; 4: shared-prefix batch; "
                         "5: mixed continuous-batching sweep; 6: rotary embedding + append of a prefill chunk; "
                         "7: the 8B-shaped layer with an E4M3 K/V cache; 8: chunked prefill (8 x 512 new tokens "
                         "over 4096 cached)")
    ap.add_argument("--chunk", type=int, default=512, help="config 8: chunk tokens per sequence")
    ap.add_argument("--splits", type=int, default=0, help="num_splits passed to paged_decode_attention (0 = auto)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--e2e-parts", type=int, default=1,
                    help="end-to-end steps: the batch goes through in this many contiguous parts, the copies of one "
                         "part overlapping the decode of another (1: copy in, decode, copy out, one after another)")
    ap.add_argument("--no-sustained", action="store_true",
                    help="skip the >= 1 s repeats (median of 5) that follow the timed steps")
    ap.add_argument("--no-extra", action="store_true",
                    help="default run: do not add the 32K-context and mixed-sweep records to the config-2 line")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-clocks", action="store_true")
    ap.add_argument("--no-graph", action="store_true",
                    help="launch without CUDA graphs (config 3's 32 layers; config 2's end-to-end steps)")
    ap.add_argument("--mixed-point", type=str, default=None,
                    help="config 5: run one point only, 'H_kv,page_size' (e.g. 1,16)")
    ap.add_argument("--page-size", type=int, choices=[16, 32], default=None,
                    help="override the workload's page size (the 8B-shaped workload uses 16)")
    ap.add_argument("--page-order", choices=["shuffled", "sequential"], default="shuffled",
                    help="physical page order of the pool's free list (the workloads use shuffled pages)")
    ap.add_argument("--append", choices=["fused", "separate"], default="fused",
                    help="append the new token inside the decode launch (paged_decode_attention_append) "
                         "or with kv_append before paged_decode_attention")
    ap.add_argument("--tokens", type=int, default=8192, help="config 6: tokens in the prefill chunk")
    ap.add_argument("--kernel", choices=["auto", "simt", "mma", "tc"], default="auto",
                    help="decode kernel: automatic choice, CUDA cores (simt), warp MMA (mma) or the tcgen05 kernel "
                         "wherever it applies (tc)")
    return ap.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def decode_kernel_digest():
    """Digest of the tensor-core decode kernel's sources (a profile is valid only for these)."""
    import hashlib

    h = hashlib.sha256()
    for name in ("decode_mma.cuh", "decode_kernel.cuh", "ptx.cuh"):
        with open(os.path.join(ROOT, "paged_kv_cache_433_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def measured_traffic_ratio():
    """DRAM bytes / algorithmic bytes of the decode kernel from the committed ncu summary, or None
    when that capture was not taken from the current kernel sources."""
    import re

    try:
        with open(PROFILE_DECODE, encoding="utf-8") as f:
            text = f.read()
    except OSError:
        return None
    dg = re.search(r"source digest:\s*`?([0-9a-f]{16})", text)
    ratio = re.search(r"traffic / algorithmic bytes:\s*([0-9.]+)", text)
    if not dg or not ratio or dg.group(1) != decode_kernel_digest():
        return None
    return float(ratio.group(1))


# ---------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 200 ms while running."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int, enabled: bool = True):
        self.proc = None
        self.gpu = gpu_index
        if enabled:
            try:
                self.proc = subprocess.Popen(["nvidia-smi", f"--id={gpu_index}", f"--query-gpu={self.FIELDS}",
                                              "--format=csv,noheader,nounits", "-lms", "200"],
                                             stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            except Exception:
                self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in out.strip().splitlines():
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        if not sm:
            return None
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": float(max(mx)), "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------- workload setup
class Workload:
    """Device-resident inputs of every step, built through the library's own calls."""

    def __init__(self, cfg, lens, n_steps, rank, splits, layers=1, sequential=False, fp8=False):
        import torch

        from paged_kv_cache_433_b200 import kvpaged as K
        from paged_kv_cache_433_b200 import workloads as W

        self.K, self.W, self.torch = K, W, torch
        self.cfg = cfg
        self.layers = layers
        P = cfg.page_size
        B = len(lens)
        self.B = B
        dt = {"bf16": torch.bfloat16, "fp16": torch.float16, "fp32": torch.float32}[cfg.dtype]
        self.dt = dt
        self.max_blocks = max(-(-(int(L) + n_steps) // P) for L in lens) + 1
        self.num_pages = int(sum(-(-(int(L) + n_steps) // P) for L in lens)) + 8
        order = (np.arange(self.num_pages, dtype=np.int32) if sequential
                 else W.page_order(self.num_pages, cfg.seed + 1000 * rank))
        self.pool = K.KvPool(self.num_pages, P, order)
        self.tab = np.full((B, self.max_blocks), -1, np.int32)
        for b in range(B):
            k = -(-int(lens[b]) // P)
            self.tab[b, :k] = self.pool.alloc(k)
        self.lens0 = np.asarray(lens, np.int32).copy()
        self.lens = self.lens0.copy()
        dev = torch.device("cuda")
        gen = torch.Generator(device=dev)
        gen.manual_seed(cfg.seed * 7919 + rank)
        shape = (self.num_pages, cfg.H_kv, P, cfg.Dh)
        self.fp8 = fp8
        # E4M3 pools: per-head scales that map N(0,1) values up to 4.5 onto the E4M3 range
        self.k_scale = torch.full((cfg.H_kv,), 4.5 / 448, dtype=torch.float32, device=dev)
        self.v_scale = self.k_scale.clone()
        self.k_pages, self.v_pages = [], []
        slots = np.concatenate([K.kv_slots_for_range(self.tab[b], P, 0, int(lens[b])) for b in range(B)])
        slots_dev = torch.from_numpy(slots).to(dev)
        for _ in range(layers):
            kp = torch.zeros(shape, dtype=torch.uint8 if fp8 else dt, device=dev)
            vp = torch.zeros_like(kp)
            chunk = 1 << 20
            for s0 in range(0, slots.size, chunk):
                n = min(chunk, slots.size - s0)
                kr = torch.randn((n, cfg.H_kv, cfg.Dh), generator=gen, device=dev).to(dt)
                vr = torch.randn((n, cfg.H_kv, cfg.Dh), generator=gen, device=dev).to(dt)
                if fp8:
                    K.kv_append_fp8(kp, vp, kr, vr, self.k_scale, self.v_scale, slots_dev[s0:s0 + n], P)
                else:
                    K.kv_append(kp, vp, kr, vr, slots_dev[s0:s0 + n], P)
            self.k_pages.append(kp)
            self.v_pages.append(vp)
        self.splits = splits
        self.gen = gen
        torch.cuda.synchronize()

    def bookkeeping(self):
        """Host step a1: slot of each new token, allocating pages at block boundaries."""
        slots = self.pool.append_slots(self.tab, self.lens)
        return slots, self.lens.copy()

    def workspace(self):
        cfg = self.cfg
        nb = self.K.paged_decode_workspace_bytes(self.B, cfg.H_q, cfg.H_kv, cfg.Dh, self.max_blocks, cfg.page_size,
                                                 self.splits)
        return self.torch.zeros(max(nb, 16), dtype=self.torch.uint8, device="cuda")

    def step_bytes(self, lens_after):
        """Algorithmic bytes of one decode launch (one layer): K/V rows actually attended,
        q, fp32 out, block-table entries and seq_lens."""
        cfg = self.cfg
        kv = int(np.sum(lens_after)) * cfg.H_kv * cfg.Dh * 2 * (1 if getattr(self, "fp8", False) else cfg.elem_bytes)
        q = self.B * cfg.H_q * cfg.Dh * cfg.elem_bytes
        out = self.B * cfg.H_q * cfg.Dh * 4
        tables = int(np.sum(-(-lens_after // cfg.page_size))) * 4 + self.B * 4
        return kv + q + out + tables


def launches_per_call(S, args):
    """Library kernels per append+decode call: plan + decode + combine for a device-planned launch (S == 0),
    decode (+ combine when split) otherwise, plus kv_append when it is not fused."""
    return (3 if S == 0 else (2 if S > 1 else 1)) + (args.append == "separate")


def hot_path(K, args, cfg, kp, vp, kn, vn, slots, q, tab, lens, out, ws, err, stream, ev=None):
    """One layer's step on the device: append the new token, then decode (fused into one launch by default).
    `ev` = (start, end) events recorded around the timed kernel call."""
    P = cfg.page_size
    if args.append == "fused":
        if ev is not None:
            ev[0].record(stream)
        K.paged_decode_attention_append(out, q, kn, vn, kp, vp, tab, lens, cfg.scale, num_splits=args.splits,
                                        workspace=ws, err_flag=err, stream=stream)
    else:
        K.kv_append(kp, vp, kn, vn, slots, P, err_flag=err, stream=stream)
        if ev is not None:
            ev[0].record(stream)
        K.paged_decode_attention(out, q, kp, vp, tab, lens, cfg.scale, num_splits=args.splits, workspace=ws,
                                 err_flag=err, stream=stream)
    if ev is not None:
        ev[1].record(stream)


def setup_dist(args):
    import torch

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist

        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


def max_over_ranks(x, world):
    """Max of a per-rank float over the process group (device tensor for NCCL, host tensor for gloo)."""
    import torch

    if world == 1:
        return x
    import torch.distributed as dist

    dev = "cpu" if dist.get_backend() == "gloo" else "cuda"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_value(seqs_per_rank, steps, world, elapsed_ms_max):
    """Whole-job seq-steps/s: every rank decodes its own batch (weak scaling); time = slowest rank."""
    return seqs_per_rank * steps * world / (elapsed_ms_max / 1e3)


KERNEL_NAMES = {1: "cuda cores", 2: "warp mma (mma.sync)", 3: "tcgen05 (tensor memory)"}
DATASHEET_HBM_GBS = 8000.0  # B200 HBM3e datasheet figure (~8 TB/s), shown beside the measured-copy fraction


def kv_byte_variants(cfg, lens_after, B, kv_elem_bytes, S, C, plan_C=None, layers=1):
    """Per-launch byte figures beside the algorithmic bytes (one layer unless `layers`):
    K/V bytes when whole pages are read (page-rounded), and the split partials' fp32 (m, l, u) bytes written by
    the decode kernel and read back by the combine (grid split: every non-empty split of a row; planned launch:
    every chunk of a row that has more than one, with the device's chunk size plan_C)."""
    P = cfg.page_size
    lens_after = np.asarray(lens_after, np.int64)
    pages = -(-lens_after // P)
    rounded = int(pages.sum()) * P * cfg.H_kv * cfg.Dh * 2 * kv_elem_bytes
    row_partial = cfg.g * (cfg.Dh + 2) * 4  # one (m, l, u) per query head of a (row, chunk)
    if plan_C:
        n_chunks = -(-pages // plan_C)
        parts = int(np.sum(np.where(n_chunks > 1, n_chunks, 0))) * cfg.H_kv
    elif S > 1:
        parts = int(np.sum(-(-pages // C))) * cfg.H_kv  # splits that hold pages of the row
    else:
        parts = 0
    return {"kv_bytes_page_rounded": layers * rounded, "partials_bytes_write_read": layers * 2 * parts * row_partial}


def roofline_fracs(achieved_gbs, peak):
    return {"frac": achieved_gbs / peak, "frac_datasheet": achieved_gbs / DATASHEET_HBM_GBS,
            "datasheet_gbs": DATASHEET_HBM_GBS}


def sustained_repeats(launch, n_window, stream, est_ms_per_call, local, args, repeats=5, min_s=1.0):
    """Median of `repeats` device-timed runs, each at least `min_s` long: the recorded window of n_window
    calls is replayed in order (launch(i), i cycling over the window), CUDA events on the launching stream;
    nvidia-smi clocks sampled over all repeats."""
    import torch

    iters = max(n_window, int(math.ceil(min_s * 1e3 / max(est_ms_per_call, 1e-3))))
    iters = -(-iters // n_window) * n_window
    clk = ClockSampler(local, enabled=not args.no_clocks)
    per_call = []
    for _ in range(repeats):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        e0.record(stream)
        for i in range(iters):
            launch(i % n_window)
        e1.record(stream)
        torch.cuda.synchronize()
        per_call.append(e0.elapsed_time(e1) / iters)
    clocks = clk.stop()
    return {"ms_per_step_median": float(np.median(per_call)), "ms_per_step_repeats": per_call, "repeats": repeats,
            "steps_per_repeat": iters, "repeat_s_median": float(np.median(per_call)) * iters / 1e3,
            "clocks": clocks}


# ---------------------------------------------------------------------------- our arm: config 2
def run_layer_bench(args, world, rank, local):
    import torch

    from paged_kv_cache_433_b200 import kvpaged as K
    from paged_kv_cache_433_b200 import workloads as W

    cfg = W.LLAMA8B
    if args.page_size is not None and args.page_size != cfg.page_size:
        import dataclasses

        cfg = dataclasses.replace(cfg, page_size=args.page_size, name=cfg.name.replace("-P16", f"-P{args.page_size}"))
    steps = args.steps if args.steps is not None else cfg.timed_steps
    warm = args.warmup if args.warmup is not None else cfg.warmup_steps
    lens = W.cached_lengths(cfg)
    e2e_steps = 0 if args.no_e2e else steps
    # room for the timed pass and the e2e pass (which books one step ahead)
    n_steps = warm + steps + (warm + e2e_steps + 1 if e2e_steps else 0)
    wl = Workload(cfg, lens, n_steps, rank, args.splits, sequential=args.page_order == "sequential")
    B, P = wl.B, cfg.page_size
    dev = torch.device("cuda")

    # ---- host bookkeeping for the device-timed steps (inputs resident before timing)
    T1 = warm + steps
    slot_list, lens_list = [], []
    for _ in range(T1):
        s, l = wl.bookkeeping()
        slot_list.append(s)
        lens_list.append(l)
    slots_dev = torch.from_numpy(np.stack(slot_list)).to(dev)
    lens_dev = torch.from_numpy(np.stack(lens_list)).to(dev)
    tab_dev = torch.from_numpy(wl.tab).to(dev)
    q_dev = torch.randn((T1, B, cfg.H_q, cfg.Dh), generator=wl.gen, device=dev).to(wl.dt)
    kn_dev = torch.randn((T1, B, cfg.H_kv, cfg.Dh), generator=wl.gen, device=dev).to(wl.dt)
    vn_dev = torch.randn((T1, B, cfg.H_kv, cfg.Dh), generator=wl.gen, device=dev).to(wl.dt)
    out = torch.empty((B, cfg.H_q, cfg.Dh), dtype=torch.float32, device=dev)
    ws = wl.workspace()
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    S, kernel_kind = K.paged_decode_launch_info(B, cfg.H_q, cfg.H_kv, cfg.Dh, wl.max_blocks, P, cfg.dtype, args.splits)
    stream = torch.cuda.current_stream()
    kp, vp = wl.k_pages[0], wl.v_pages[0]

    def step(i, ev=None):
        hot_path(K, args, cfg, kp, vp, kn_dev[i], vn_dev[i], slots_dev[i], q_dev[i], tab_dev, lens_dev[i], out, ws, err,
                 stream, ev)

    for i in range(warm):
        step(i)
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clk = ClockSampler(local, enabled=not args.no_clocks)
    barrier(world)
    torch.cuda.synchronize()
    start.record(stream)
    for i in range(warm, T1):
        step(i)
    end.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    clocks = clk.stop()
    elapsed_ms = max_over_ranks(start.elapsed_time(end), world)
    # the steps run back to back (each one launch of the fused append + decode, and the combine): the average
    # launch duration is the timed window over the steps (no events between steps to break their overlap)
    dec_ms = [elapsed_ms / steps]
    append_bytes = 2 * 2 * B * cfg.H_kv * cfg.Dh * cfg.elem_bytes if args.append == "fused" else 0
    bytes_per_launch = [wl.step_bytes(lens_list[i]) + append_bytes for i in range(warm, T1)]
    if int(err.item()) != 0:
        raise RuntimeError(f"device error flag {int(err.item())}")
    plan_C = int(ws[:4].view(torch.int32).item()) if S == 0 else None
    C = -(-wl.max_blocks // S) if S > 0 else 0

    # ---- sustained: the timed window replayed for >= 1 s, median of 5 repeats (replaying step i rewrites
    # step i's token at its own slot, so the cache stays that of the window)
    sus = None
    if not args.no_sustained:
        sus = sustained_repeats(lambda i: step(warm + i), steps, stream, elapsed_ms / steps, local, args)

    # ---- end-to-end: same calls, inputs from pinned host memory, output read back each step
    e2e = None
    if e2e_steps:
        e2e = run_e2e(wl, cfg, warm, e2e_steps, args, world)

    value = replica_value(B, steps, world, elapsed_ms)
    peak, peak_kind = peaks()
    mean_bytes = float(np.mean(bytes_per_launch))
    mean_dec_s = float(np.mean(dec_ms)) / 1e3
    achieved = mean_bytes / mean_dec_s / 1e9
    ratio = measured_traffic_ratio() if args.kernel != "simt" and P == 16 else None
    traffic = ratio * mean_bytes if ratio is not None else None
    variants = kv_byte_variants(cfg, np.mean(np.stack(lens_list[warm:T1]), axis=0), B, cfg.elem_bytes, S, C, plan_C)
    roof = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", **roofline_fracs(achieved, peak),
            "peak_source": f"{peak_kind} copy bandwidth (MEASURED_PEAKS hbm_gbs)" if peak_kind == "measured" else "fallback",
            "traffic": traffic,
            "traffic_source": ("ncu dram bytes of the decode kernel (profiles/" + os.path.basename(PROFILE_DECODE)
                               + "), scaled to this run's algorithmic bytes") if traffic else None,
            "kernel": "paged_decode_attention" + (" (split + combine)" if S != 1 else " (single pass)"),
            "bytes_per_launch": mean_bytes, "launch_us": mean_dec_s * 1e6, **variants}
    if sus is not None:
        sus["frac_median"] = mean_bytes / (sus["ms_per_step_median"] / 1e3) / 1e9 / peak
        sus["value_median"] = replica_value(B, 1, world, sus["ms_per_step_median"])
    res = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": steps, "warmup": warm,
        "ms_per_step": elapsed_ms / steps, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": cfg.dtype, "data": "synthetic (seeded N(0,1) K/V, q; lengths U[512,4096])",
        "config": {"workload": cfg.name, "B": B, "H_q": cfg.H_q, "H_kv": cfg.H_kv, "Dh": cfg.Dh, "page_size": P,
                   "layers": 1, "num_splits": S, "page_order": args.page_order, "parallelism": f"replicas x{world}" if world > 1 else "1 GPU",
                   "l2": "inputs larger than L2 (K/V working set %.0f MB > 126 MB L2); no flush" % (mean_bytes / 1e6)},
        "roofline": roof,
        "gpu_launches": steps * launches_per_call(S, args),
        "e2e": e2e,
        "clocks": clocks,
        "sustained": sus,
    }
    return res


def run_fp8_bench(args, world, rank, local):
    """The 8B-shaped layer with an E4M3 K/V cache (per-head scales) and bf16 q: each step appends the new
    token (kv_append_fp8, quantising) and decodes (paged_decode_attention_fp8). The roofline is the decode call."""
    import torch

    from paged_kv_cache_433_b200 import kvpaged as K
    from paged_kv_cache_433_b200 import workloads as W

    cfg = W.LLAMA8B
    steps = args.steps if args.steps is not None else cfg.timed_steps
    warm = args.warmup if args.warmup is not None else cfg.warmup_steps
    lens = W.cached_lengths(cfg)
    wl = Workload(cfg, lens, warm + steps, rank, args.splits, fp8=True)
    B, P = wl.B, cfg.page_size
    dev = torch.device("cuda")
    T1 = warm + steps
    slot_list, lens_list = [], []
    for _ in range(T1):
        sl, ln = wl.bookkeeping()
        slot_list.append(sl)
        lens_list.append(ln)
    slots_dev = torch.from_numpy(np.stack(slot_list)).to(dev)
    lens_dev = torch.from_numpy(np.stack(lens_list)).to(dev)
    tab_dev = torch.from_numpy(wl.tab).to(dev)
    q_dev = torch.randn((T1, B, cfg.H_q, cfg.Dh), generator=wl.gen, device=dev).to(wl.dt)
    kn_dev = torch.randn((T1, B, cfg.H_kv, cfg.Dh), generator=wl.gen, device=dev).to(wl.dt)
    vn_dev = torch.randn((T1, B, cfg.H_kv, cfg.Dh), generator=wl.gen, device=dev).to(wl.dt)
    out = torch.empty((B, cfg.H_q, cfg.Dh), dtype=torch.float32, device=dev)
    ws = wl.workspace()
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    S, kernel_kind = K.paged_decode_launch_info(B, cfg.H_q, cfg.H_kv, cfg.Dh, wl.max_blocks, P, cfg.dtype, args.splits)
    stream = torch.cuda.current_stream()
    kp, vp = wl.k_pages[0], wl.v_pages[0]

    def step(i, ev=None):
        K.kv_append_fp8(kp, vp, kn_dev[i], vn_dev[i], wl.k_scale, wl.v_scale, slots_dev[i], P, err_flag=err,
                        stream=stream)
        if ev is not None:
            ev[0].record(stream)
        K.paged_decode_attention_fp8(out, q_dev[i], kp, vp, wl.k_scale, wl.v_scale, tab_dev, lens_dev[i], cfg.scale,
                                     num_splits=args.splits, workspace=ws, err_flag=err, stream=stream)
        if ev is not None:
            ev[1].record(stream)

    for i in range(warm):
        step(i)
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clk = ClockSampler(local, enabled=not args.no_clocks)
    barrier(world)
    torch.cuda.synchronize()
    start.record(stream)
    for n, i in enumerate(range(warm, T1)):
        step(i, ev[n])
    end.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    clocks = clk.stop()
    if int(err.item()) != 0:
        raise RuntimeError(f"device error flag {int(err.item())}")
    elapsed_ms = max_over_ranks(start.elapsed_time(end), world)
    dec_ms = [a.elapsed_time(b) for a, b in ev]
    mean_bytes = float(np.mean([wl.step_bytes(lens_list[i]) for i in range(warm, T1)]))
    peak, peak_kind = peaks()
    mean_dec_s = float(np.mean(dec_ms)) / 1e3
    achieved = mean_bytes / mean_dec_s / 1e9
    return {
        "metric": METRIC, "value": replica_value(B, steps, world, elapsed_ms), "unit": UNIT, "n_gpus": world,
        "steps": steps, "warmup": warm, "ms_per_step": elapsed_ms / steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "e4m3 K/V, bf16 q, f16 MMA",
        "data": "synthetic (N(0,1) K/V quantised with scale 4.5/448 per head; bf16 q; lengths U[512,4096])",
        "config": {"workload": cfg.name.replace("-bf16-", "-fp8kv-"), "B": B, "H_q": cfg.H_q, "H_kv": cfg.H_kv,
                   "Dh": cfg.Dh, "page_size": P, "kv_dtype": "e4m3",
                   "num_splits": args.splits if args.splits else "auto (E4M3 rule: half the 16-bit CTAs per SM)",
                   "l2": "inputs larger than L2 (K/V working set %.0f MB > 126 MB L2); no flush" % (mean_bytes / 1e6)},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "peak_source": peak_kind, "traffic": None,
                     "kernel": "paged_decode_attention_fp8" + (" (split + combine)" if S > 1 else ""),
                     "bytes_per_launch": mean_bytes, "launch_us": mean_dec_s * 1e6},
        "gpu_launches": steps * (1 + (3 if S == 0 else (2 if S > 1 else 1))),
        "e2e": None, "clocks": clocks,
    }


def run_prefill_bench(args, world, rank, local):
    """Chunked prefill on the 8B-shaped layer: 8 sequences each extend a 4096-token cached context by a
    512-token chunk (its K/V already appended); one step = paged_prefill_attention over the 4096 chunk rows.
    Tensor-bound: roofline against the measured bf16 dense peak, causal flops only."""
    import torch

    from paged_kv_cache_433_b200 import kvpaged as K
    from paged_kv_cache_433_b200 import workloads as W

    cfg = W.LLAMA8B
    B, ctx, n = 8, 4096, args.chunk
    steps = args.steps if args.steps is not None else 20
    warm = args.warmup if args.warmup is not None else 3
    P = cfg.page_size
    total = ctx + n
    lens = np.full(B, total, np.int64)
    wl = Workload(dataclasses_replace(cfg, B=B), lens, 0, rank, 1)
    dev = torch.device("cuda")
    q = torch.randn((B * n, cfg.H_q, cfg.Dh), generator=wl.gen, device=dev).to(wl.dt)
    out = torch.empty((B * n, cfg.H_q, cfg.Dh), dtype=torch.float32, device=dev)
    q_start = torch.arange(0, B * n + 1, n, dtype=torch.int32, device=dev)
    seq = torch.from_numpy(lens.astype(np.int32)).to(dev)
    tab = torch.from_numpy(wl.tab).to(dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream()

    def call():
        K.paged_prefill_attention(out, q, q_start, n, wl.k_pages[0], wl.v_pages[0], tab, seq, cfg.scale, err_flag=err,
                                  stream=stream)

    for _ in range(warm):
        call()
    torch.cuda.synchronize()
    clk = ClockSampler(local, enabled=not args.no_clocks)
    barrier(world)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        call()
    e1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    clocks = clk.stop()
    if int(err.item()) != 0:
        raise RuntimeError(f"device error flag {int(err.item())}")
    ms = max_over_ranks(e0.elapsed_time(e1), world)
    per_s = ms / steps / 1e3
    keys = B * (n * ctx + n * (n + 1) // 2)                    # sum over chunk rows of the keys each one sees
    flops = 4.0 * cfg.Dh * cfg.H_q * keys                      # QK^T and PV, 2 flops per multiply-add
    peak, peak_src = peaks_tensor()
    achieved = flops / per_s / 1e12
    g = cfg.H_q // cfg.H_kv
    # the library's choice for a chunk (automatic kernel kind): tcgen05 for Dh 128 when the group divides 128
    prefill_kernel = ("paged_prefill_tc_kernel (tcgen05, 128-row tiles)" if cfg.Dh == 128 and 128 % g == 0
                      else "paged_decode_mma_kernel (multi-token query)")
    return {
        "metric": "chunked prefill tokens/s; achieved TFLOP/s", "value": B * n * steps * world / (ms / 1e3),
        "unit": "tokens/s", "n_gpus": world, "steps": steps, "warmup": warm, "ms_per_step": ms / steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (N(0,1) K/V, q)",
        "config": {"workload": f"chunked-prefill-{cfg.name}-B{B}-ctx{ctx}-chunk{n}", "B": B, "context": ctx, "chunk": n,
                   "H_q": cfg.H_q, "H_kv": cfg.H_kv, "Dh": cfg.Dh, "page_size": P,
                   "l2": "K/V %.0f MB, re-read per query tile mostly from L2; no flush" % (
                       B * total * cfg.H_kv * cfg.Dh * 4 / 1e6)},
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak, "peak_source": peak_src,
                     "traffic": None, "kernel": prefill_kernel,
                     "flops_per_launch": flops, "launch_us": per_s * 1e6},
        "gpu_launches": steps, "e2e": None, "clocks": clocks,
    }


def dataclasses_replace(cfg, **kw):
    import dataclasses

    return dataclasses.replace(cfg, **kw)


def peaks_tensor():
    """(dense bf16 TFLOP/s, source): the measured cuBLAS burst figure when the peaks file is present, else the
    earlier B200 measurement (1590 TFLOP/s burst)."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops"]), "measured cuBLAS bf16 dense (burst)"
    except Exception:
        return 1590.0, "fallback (1590 TFLOP/s cuBLAS bf16 burst)"


def run_e2e(wl, cfg, warm, steps, args, world):
    """Each step: the step's inputs (q, k_new, v_new, slots, lengths and the block table, packed in a pinned
    staging buffer) copied to the device, kv_append + paged_decode_attention (fused by default), the fp32
    output copied back, then a wait for it. Steps are serial, as in a decode loop whose next input depends on
    this step's output; only the host slot bookkeeping of the next step (which does not depend on the output)
    is done while the device runs this one. With --e2e-parts > 1 the batch goes through in that many
    contiguous parts, each one call of the public entry point on its rows, on three streams: the copy of part
    k + 1's inputs runs while part k is decoded, and the copy of part k's output while part k + 1 is (8B-shaped
    layer, B = 64: 182.7 us a step with two parts, 183.9 with one, 217.8 with four -- the smaller decodes cost
    what the overlapped copies save, so one part is the default). Unless
    --no-graph, each step's copies and launches are captured once as a CUDA graph (as a serving loop captures
    its decode step) and replayed."""
    import torch

    K = wl.K
    B = wl.B
    dev = torch.device("cuda")
    n = warm + steps
    eb = cfg.elem_bytes
    nparts = max(1, min(args.e2e_parts, B))
    bounds = [B * k // nparts for k in range(nparts + 1)]
    mb = wl.tab.shape[1]

    def a16(x):
        return (x + 15) // 16 * 16

    # staging layout: part k's rows [b0, b1) as q, k_new, v_new, slots, lengths, block table, one contiguous
    # range per part
    parts = []
    off = 0
    for k in range(nparts):
        b0, b1 = bounds[k], bounds[k + 1]
        nb = b1 - b0
        o = {"b0": b0, "b1": b1, "nb": nb, "start": off, "nq": nb * cfg.H_q * cfg.Dh * eb,
             "nkv": nb * cfg.H_kv * cfg.Dh * eb}
        for name, size in (("q", o["nq"]), ("kn", o["nkv"]), ("vn", o["nkv"]), ("slots", 8 * nb), ("lens", 4 * nb),
                           ("tab", 4 * nb * mb)):
            o[name] = off
            off = a16(off + size)
        o["end"] = off
        parts.append(o)
    total = off
    host_in = [torch.empty(total, dtype=torch.uint8).pin_memory() for _ in range(n + 1)]
    gen = torch.Generator().manual_seed(cfg.seed + 77)
    for i in range(n):  # step inputs prepared before timing (q, k_new, v_new as the model would produce them)
        h = host_in[i]
        for o in parts:
            for name, size in (("q", o["nq"]), ("kn", o["nkv"]), ("vn", o["nkv"])):
                h[o[name]:o[name] + size].view(wl.dt).copy_(torch.randn(size // eb, generator=gen).to(wl.dt))
    host_out = torch.empty((B, cfg.H_q, cfg.Dh), dtype=torch.float32).pin_memory()
    d_in = torch.empty(total, dtype=torch.uint8, device=dev)
    views = []
    for o in parts:
        nb = o["nb"]
        v = {"q": d_in[o["q"]:o["q"] + o["nq"]].view(wl.dt).view(nb, cfg.H_q, cfg.Dh),
             "kn": d_in[o["kn"]:o["kn"] + o["nkv"]].view(wl.dt).view(nb, cfg.H_kv, cfg.Dh),
             "vn": d_in[o["vn"]:o["vn"] + o["nkv"]].view(wl.dt).view(nb, cfg.H_kv, cfg.Dh),
             "slots": d_in[o["slots"]:o["slots"] + 8 * nb].view(torch.int64),
             "lens": d_in[o["lens"]:o["lens"] + 4 * nb].view(torch.int32),
             "tab": d_in[o["tab"]:o["tab"] + 4 * nb * mb].view(torch.int32).view(nb, mb)}
        v["tab"].copy_(torch.from_numpy(wl.tab[o["b0"]:o["b1"]]))
        views.append(v)
    d_out = torch.empty((B, cfg.H_q, cfg.Dh), dtype=torch.float32, device=dev)
    # one workspace serves every part: their launches are ordered on one stream
    nws = max(K.paged_decode_workspace_bytes(o["nb"], cfg.H_q, cfg.H_kv, cfg.Dh, mb, cfg.page_size, wl.splits)
              for o in parts)
    ws = torch.zeros(max(nws, 16), dtype=torch.uint8, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream()
    copy_in, copy_out = torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in parts]
    ev_done = [torch.cuda.Event() for _ in parts]

    def prep(i):
        """Host step a1 for step i (slots, lengths, block table), packed into its staging buffer."""
        s, l = wl.bookkeeping()
        h = host_in[i].numpy()
        for o in parts:
            b0, b1, nb = o["b0"], o["b1"], o["nb"]
            h[o["slots"]:o["slots"] + 8 * nb] = s[b0:b1].view(np.uint8)
            h[o["lens"]:o["lens"] + 4 * nb] = l[b0:b1].astype(np.int32).view(np.uint8)
            h[o["tab"]:o["tab"] + 4 * nb * mb] = np.ascontiguousarray(wl.tab[b0:b1]).view(np.uint8).reshape(-1)

    def body(i, st):
        """Step i's copies and launches: forked from st onto the copy streams and joined back into it."""
        copy_in.wait_stream(st)
        copy_out.wait_stream(st)
        with torch.cuda.stream(copy_in):
            for k, o in enumerate(parts):
                d_in[o["start"]:o["end"]].copy_(host_in[i][o["start"]:o["end"]], non_blocking=True)
                ev_in[k].record(copy_in)
        for k, (o, v) in enumerate(zip(parts, views)):
            st.wait_event(ev_in[k])
            hot_path(K, args, cfg, wl.k_pages[0], wl.v_pages[0], v["kn"], v["vn"], v["slots"], v["q"], v["tab"],
                     v["lens"], d_out[o["b0"]:o["b1"]], ws, err, st)
            ev_done[k].record(st)
            copy_out.wait_event(ev_done[k])
            with torch.cuda.stream(copy_out):
                host_out[o["b0"]:o["b1"]].copy_(d_out[o["b0"]:o["b1"]], non_blocking=True)
        st.wait_stream(copy_in)
        st.wait_stream(copy_out)

    graphs = None
    if not args.no_graph:
        # one graph per step (each reads its own staging buffer); the host bookkeeping is not in them
        side = torch.cuda.Stream()
        side.wait_stream(stream)
        graphs = []
        for i in range(n):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=side):
                body(i, torch.cuda.current_stream())
            graphs.append(g)
        stream.wait_stream(side)
        torch.cuda.synchronize()

    def one(i):
        if graphs is not None:
            graphs[i].replay()
        else:
            body(i, stream)
        prep(i + 1)  # overlaps the device work of step i
        stream.synchronize()

    prep(0)
    for i in range(warm):
        one(i)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    start.record(stream)
    for i in range(warm, n):
        one(i)
    end.record(stream)
    torch.cuda.synchronize()
    if int(err.item()) != 0:
        raise RuntimeError(f"device error flag {int(err.item())}")
    ms = max_over_ranks(start.elapsed_time(end), world)
    del graphs
    return {"value": replica_value(B, steps, world, ms), "unit": UNIT, "h2d_bytes_per_step": float(total),
            "d2h_bytes_per_step": host_out.numel() * 4, "ms_per_step": ms / steps,
            "copies_declared": True, "cuda_graph": not args.no_graph, "parts": nparts,
            "path": f"pinned staging -> device in {nparts} part(s), one public call per part, output back per part "
                    f"(copies of one part overlap the other part's decode), wait every step"}


def run_long_bench(args, world, rank, local):
    """One 32K-token sequence, 32 layers (fp16, 4 GiB cache): a step is 32 x (append + decode + combine),
    captured once as a CUDA graph that reads its inputs from one staging buffer and replayed every step."""
    import torch

    from paged_kv_cache_433_b200 import kvpaged as K
    from paged_kv_cache_433_b200 import workloads as W

    cfg = W.LONG32K
    steps = args.steps if args.steps is not None else cfg.timed_steps
    warm = args.warmup if args.warmup is not None else cfg.warmup_steps
    L = cfg.layers
    lens = W.cached_lengths(cfg)
    T1 = warm + steps
    e2e_steps = 0 if args.no_e2e else steps
    wl = Workload(cfg, lens, T1 + 1 + (warm + e2e_steps + 1 if e2e_steps else 0), rank, args.splits, layers=L,
                  sequential=args.page_order == "sequential")
    B, P = wl.B, cfg.page_size
    dev = torch.device("cuda")
    slot_list, lens_list = [], []
    for _ in range(T1):
        s, l = wl.bookkeeping()
        slot_list.append(s)
        lens_list.append(l)
    eb = cfg.elem_bytes
    # staging layout of one step's inputs: q, k_new, v_new of every layer, slots, lengths, block table
    nq, nkv = L * B * cfg.H_q * cfg.Dh * eb, L * B * cfg.H_kv * cfg.Dh * eb
    off_kn, off_vn, off_slots = nq, nq + nkv, nq + 2 * nkv
    off_lens = off_slots + 8 * B
    off_tab = (off_lens + 4 * B + 15) // 16 * 16
    tab_bytes = wl.tab.nbytes
    total = off_tab + tab_bytes
    d_stage = torch.empty(total, dtype=torch.uint8, device=dev)
    cur = {"q": d_stage[:nq].view(wl.dt).view(L, B, cfg.H_q, cfg.Dh),
           "kn": d_stage[off_kn:off_kn + nkv].view(wl.dt).view(L, B, cfg.H_kv, cfg.Dh),
           "vn": d_stage[off_vn:off_vn + nkv].view(wl.dt).view(L, B, cfg.H_kv, cfg.Dh),
           "slots": d_stage[off_slots:off_slots + 8 * B].view(torch.int64),
           "lens": d_stage[off_lens:off_lens + 4 * B].view(torch.int32)}
    tab_dev = d_stage[off_tab:].view(torch.int32).view(wl.tab.shape)
    tab_dev.copy_(torch.from_numpy(wl.tab))
    slots_dev = torch.from_numpy(np.stack(slot_list)).to(dev)
    lens_dev = torch.from_numpy(np.stack(lens_list)).to(dev)
    q_dev = torch.randn((T1, L, B, cfg.H_q, cfg.Dh), generator=wl.gen, device=dev).to(wl.dt)
    kn_dev = torch.randn((T1, L, B, cfg.H_kv, cfg.Dh), generator=wl.gen, device=dev).to(wl.dt)
    vn_dev = torch.randn((T1, L, B, cfg.H_kv, cfg.Dh), generator=wl.gen, device=dev).to(wl.dt)
    out = torch.empty((L, B, cfg.H_q, cfg.Dh), dtype=torch.float32, device=dev)
    ws = wl.workspace()
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    S, kernel_kind = K.paged_decode_launch_info(B, cfg.H_q, cfg.H_kv, cfg.Dh, wl.max_blocks, P, cfg.dtype, args.splits)
    side = torch.cuda.Stream()

    def layers_pass(stream):
        for layer in range(L):
            hot_path(K, args, cfg, wl.k_pages[layer], wl.v_pages[layer], cur["kn"][layer], cur["vn"][layer], cur["slots"],
                     cur["q"][layer], tab_dev, cur["lens"], out[layer], ws, err, stream)

    def stage(i, stream):
        with torch.cuda.stream(stream):
            cur["slots"].copy_(slots_dev[i], non_blocking=True)
            cur["lens"].copy_(lens_dev[i], non_blocking=True)
            cur["q"].copy_(q_dev[i], non_blocking=True)
            cur["kn"].copy_(kn_dev[i], non_blocking=True)
            cur["vn"].copy_(vn_dev[i], non_blocking=True)

    graph = None
    stream = torch.cuda.current_stream()
    stage(0, stream)
    layers_pass(stream)  # first launch configures kernels outside any capture
    torch.cuda.synchronize()
    if not args.no_graph:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=side):
            layers_pass(side)
        torch.cuda.synchronize()

    def run_step(i):
        stage(i, stream)
        graph.replay() if graph is not None else layers_pass(stream)

    # the warm-up pass above consumed step 0's slots: rebuild state by replaying from step 0
    for i in range(warm):
        run_step(i)
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    stage_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    clk = ClockSampler(local, enabled=not args.no_clocks)
    barrier(world)
    torch.cuda.synchronize()
    start.record(stream)
    for n, i in enumerate(range(warm, T1)):
        stage(i, stream)
        stage_ev[n][0].record(stream)
        graph.replay() if graph is not None else layers_pass(stream)
        stage_ev[n][1].record(stream)
    end.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    clocks = clk.stop()
    elapsed_ms = max_over_ranks(start.elapsed_time(end), world)
    pass_ms = [a.elapsed_time(b) for a, b in stage_ev]
    if int(err.item()) != 0:
        raise RuntimeError(f"device error flag {int(err.item())}")
    sus = None
    if not args.no_sustained:
        sus = sustained_repeats(lambda i: run_step(warm + i), steps, stream, elapsed_ms / steps, local, args)
    C = -(-wl.max_blocks // S) if S > 0 else 0

    # ---- end-to-end: each step's inputs (all 32 layers) from one pinned buffer, outputs read back
    e2e = None
    if e2e_steps and graph is not None:
        n = warm + e2e_steps
        host_in = [torch.empty(total, dtype=torch.uint8).pin_memory() for _ in range(n + 1)]
        gen = torch.Generator().manual_seed(cfg.seed + 77)
        for i in range(n):
            host_in[i][:off_slots].view(wl.dt).copy_(torch.randn(off_slots // eb, generator=gen).to(wl.dt))
        host_out = torch.empty(tuple(out.shape), dtype=torch.float32).pin_memory()

        def prep(i):
            before = wl.lens.copy()
            s_, l_ = wl.bookkeeping()
            h = host_in[i].numpy()
            h[off_slots:off_slots + 8 * B] = s_.view(np.uint8)
            h[off_lens:off_lens + 4 * B] = l_.astype(np.int32).view(np.uint8)
            if np.any(before % P == 0):
                h[off_tab:off_tab + tab_bytes] = wl.tab.view(np.uint8).reshape(-1)
                return total
            return off_tab

        def one(i, nb):
            d_stage[:nb].copy_(host_in[i][:nb], non_blocking=True)
            graph.replay()
            host_out.copy_(out, non_blocking=True)
            nxt = prep(i + 1)
            stream.synchronize()
            return nxt

        nb = prep(0)
        for i in range(warm):
            nb = one(i, nb)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier(world)
        torch.cuda.synchronize()
        h2d = 0
        e0.record(stream)
        for i in range(warm, n):
            h2d += nb
            nb = one(i, nb)
        e1.record(stream)
        torch.cuda.synchronize()
        if int(err.item()) != 0:
            raise RuntimeError(f"device error flag {int(err.item())}")
        ms = max_over_ranks(e0.elapsed_time(e1), world)
        e2e = {"value": replica_value(B, e2e_steps, world, ms), "unit": UNIT, "h2d_bytes_per_step": h2d / e2e_steps,
               "d2h_bytes_per_step": host_out.numel() * 4, "ms_per_step": ms / e2e_steps, "copies_declared": True,
               "path": "one H2D of the step's packed inputs, the captured 32-layer graph, D2H of all outputs"}
    bytes_step = [L * wl.step_bytes(lens_list[i]) for i in range(warm, T1)]
    value = replica_value(B, steps, world, elapsed_ms)
    peak, peak_kind = peaks()
    mean_bytes = float(np.mean(bytes_step))
    achieved = mean_bytes / (float(np.mean(pass_ms)) / 1e3) / 1e9
    variants = kv_byte_variants(cfg, np.mean(np.stack(lens_list[warm:T1]), axis=0), B, cfg.elem_bytes, S, C,
                                layers=L)
    if sus is not None:
        sus["frac_median"] = mean_bytes / (sus["ms_per_step_median"] / 1e3) / 1e9 / peak
        sus["value_median"] = replica_value(B, 1, world, sus["ms_per_step_median"])
        sus["note"] = "each repeat: staging copies + graph replay per step, back to back"
    return {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": steps, "warmup": warm,
        "ms_per_step": elapsed_ms / steps, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": cfg.dtype, "data": "synthetic (seeded N(0,1) K/V, q)",
        "config": {"workload": cfg.name, "B": B, "T": int(lens[0]), "layers": L, "H_q": cfg.H_q, "H_kv": cfg.H_kv,
                   "Dh": cfg.Dh, "page_size": P, "num_splits": S, "cuda_graph": graph is not None,
                   "l2": "inputs larger than L2 (4 GiB cache); no flush"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     **roofline_fracs(achieved, peak),
                     "peak_source": f"{peak_kind} copy bandwidth", "traffic": None,
                     "kernel": ("32 x (paged_decode_attention_append + combine) per step" if args.append == "fused"
                                else "32 x (kv_append + paged_decode_attention + combine) per step"),
                     "bytes_per_step": mean_bytes, "pass_us": float(np.mean(pass_ms)) * 1e3, **variants},
        "gpu_launches": steps * L * launches_per_call(S, args),
        "e2e": e2e,
        "clocks": clocks,
        "sustained": sus,
    }


# ---------------------------------------------------------------------------- our arm: configs 4 and 5
class PagedState:
    """A batch on the device built through the library: pool, block table, pools filled by kv_append."""

    def __init__(self, cfg, lens, max_blocks, num_pages, seed, dev="cuda"):
        import torch

        from paged_kv_cache_433_b200 import kvpaged as K
        from paged_kv_cache_433_b200 import workloads as W

        self.K, self.torch, self.cfg = K, torch, cfg
        self.P = cfg.page_size
        self.B = len(lens)
        self.max_blocks = max_blocks
        self.num_pages = num_pages
        self.dt = {"bf16": torch.bfloat16, "fp16": torch.float16, "fp32": torch.float32}[cfg.dtype]
        self.pool = K.KvPool(num_pages, self.P, W.page_order(num_pages, seed))
        self.tab = np.full((self.B, max_blocks), -1, np.int32)
        self.lens = np.asarray(lens, np.int32).copy()
        shape = (num_pages, cfg.H_kv, self.P, cfg.Dh)
        self.k_pages = torch.zeros(shape, dtype=self.dt, device=dev)
        self.v_pages = torch.zeros(shape, dtype=self.dt, device=dev)
        self.gen = torch.Generator(device=dev)
        self.gen.manual_seed(seed)

    def fill(self, b, start, n):
        """Write n synthetic tokens at positions start.. of row b (the row's pages must exist)."""
        if n <= 0:
            return
        cfg, torch = self.cfg, self.torch
        slots = self.torch.from_numpy(self.K.kv_slots_for_range(self.tab[b], self.P, start, n)).cuda()
        kr = torch.randn((n, cfg.H_kv, cfg.Dh), generator=self.gen, device="cuda").to(self.dt)
        vr = torch.randn((n, cfg.H_kv, cfg.Dh), generator=self.gen, device="cuda").to(self.dt)
        self.K.kv_append(self.k_pages, self.v_pages, kr, vr, slots, self.P)

    def admit(self, b, n_tokens):
        k = -(-int(n_tokens) // self.P)
        self.tab[b, :] = -1
        self.tab[b, :k] = self.pool.alloc(k)
        self.lens[b] = n_tokens
        self.fill(b, 0, int(n_tokens))

    def release(self, b):
        held = self.tab[b][self.tab[b] >= 0]
        self.pool.free(held)
        self.tab[b, :] = -1
        self.lens[b] = 0

    def step_bytes(self, lens_after, fused=True):
        cfg = self.cfg
        kv = int(np.sum(lens_after)) * cfg.H_kv * cfg.Dh * 2 * (1 if getattr(self, "fp8", False) else cfg.elem_bytes)
        q = self.B * cfg.H_q * cfg.Dh * cfg.elem_bytes
        out = self.B * cfg.H_q * cfg.Dh * 4
        tables = int(np.sum(-(-np.asarray(lens_after) // self.P))) * 4 + self.B * 4
        app = 2 * 2 * self.B * cfg.H_kv * cfg.Dh * cfg.elem_bytes if fused else 0
        return kv + q + out + tables + app


LEAD_CYCLES = 250_000  # device spin ahead of a timed step (~0.13 ms at 1.965 GHz)


def time_steps(args, st, steps, warm, before_step=None):
    """Run warm + steps decode steps on `st`; each step: optional untimed host work (before_step),
    bookkeeping + uploads (untimed), then the timed append + decode call, its launches queued behind a short
    device spin so that the events time the device's work only. Returns per-step (ms, bytes) and a
    closure that re-issues the last step's call (same inputs), for the sustained repeats."""
    import torch

    K, cfg = st.K, st.cfg
    dev = torch.device("cuda")
    stream = torch.cuda.current_stream()
    out = torch.empty((st.B, cfg.H_q, cfg.Dh), dtype=torch.float32, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    nb = K.paged_decode_workspace_bytes(st.B, cfg.H_q, cfg.H_kv, cfg.Dh, st.max_blocks, st.P, args.splits)
    ws = torch.zeros(max(nb, 16), dtype=torch.uint8, device=dev)
    res = []
    S, st.kernel_kind = K.paged_decode_launch_info(st.B, cfg.H_q, cfg.H_kv, cfg.Dh, st.max_blocks, st.P, cfg.dtype,
                                                    args.splits)
    st.launches_per_step = launches_per_call(S, args)
    st.splits_used = S
    last = None
    for i in range(warm + steps):
        if before_step is not None:
            before_step(i)
        slots = st.pool.append_slots(st.tab, st.lens)
        d_slots = torch.from_numpy(slots).to(dev)
        d_lens = torch.from_numpy(st.lens.copy()).to(dev)
        d_tab = torch.from_numpy(st.tab).to(dev)
        q = torch.randn((st.B, cfg.H_q, cfg.Dh), generator=st.gen, device=dev).to(st.dt)
        kn = torch.randn((st.B, cfg.H_kv, cfg.Dh), generator=st.gen, device=dev).to(st.dt)
        vn = torch.randn((st.B, cfg.H_kv, cfg.Dh), generator=st.gen, device=dev).to(st.dt)
        ev = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
        torch.cuda.synchronize()
        # the device spins (~0.13 ms) while the host enqueues the step's launches, so the timed window holds the
        # step's kernels back to back, as in a decode loop that runs ahead of the device: the host's launch
        # latency (a few ctypes calls) is not device time
        torch.cuda._sleep(LEAD_CYCLES)
        hot_path(K, args, cfg, st.k_pages, st.v_pages, kn, vn, d_slots, q, d_tab, d_lens, out, ws, err, stream, ev)
        torch.cuda.synchronize()
        if i >= warm:
            res.append((ev[0].elapsed_time(ev[1]), st.step_bytes(st.lens, args.append == "fused")))
        last = (kn, vn, d_slots, q, d_tab, d_lens)
    if int(err.item()) != 0:
        raise RuntimeError(f"device error flag {int(err.item())}")
    st.plan_C = int(ws[:4].view(torch.int32).item()) if S == 0 else None

    def again(_i, last=last):
        kn, vn, d_slots, q, d_tab, d_lens = last
        hot_path(K, args, cfg, st.k_pages, st.v_pages, kn, vn, d_slots, q, d_tab, d_lens, out, ws, err, stream)

    return res, again


def run_prefix_bench(args, world, rank, local):
    """Shared-prefix batch: 32 sequences reuse one 4096-token prefix (256 refcounted pages) through the
    chained-hash prefix index, then append + decode. Logical bytes count the prefix once per sequence."""
    from paged_kv_cache_433_b200 import kvpaged as K
    from paged_kv_cache_433_b200 import workloads as W

    cfg = W.SHARED_PREFIX
    steps = args.steps if args.steps is not None else cfg.timed_steps
    warm = args.warmup if args.warmup is not None else cfg.warmup_steps
    P = cfg.page_size
    wl = W.prefix_workload(cfg)
    lens = W.cached_lengths(cfg)
    n_steps = steps + warm
    max_blocks = max(-(-(int(L) + n_steps) // P) for L in lens) + 1
    num_pages = W.PREFIX_LEN // P + int(sum(-(-(int(L) + n_steps - W.PREFIX_LEN) // P) + 1 for L in lens)) + 8
    st = PagedState(cfg, np.zeros(cfg.B, np.int32), max_blocks, num_pages, cfg.seed + 1000 * rank)
    ix = K.KvPrefixIndex(P, salt=0x5EED)
    hits = 0
    for b in range(cfg.B):
        toks = wl.tokens(b)
        hit = ix.match(toks)
        st.pool.incref(hit)
        own = st.pool.alloc(-(-len(toks) // P) - len(hit))
        row = np.concatenate([hit, own]).astype(np.int32)
        st.tab[b, :row.size] = row
        st.lens[b] = len(toks)
        ix.register(st.pool, toks, row)
        st.fill(b, len(hit) * P, len(toks) - len(hit) * P)
        hits += len(hit)
    res, _ = time_steps(args, st, steps, warm)
    ms = float(np.sum([r[0] for r in res]))
    logical = float(np.mean([r[1] for r in res]))
    unique = (W.PREFIX_LEN + float(np.sum(st.lens - W.PREFIX_LEN))) * cfg.H_kv * cfg.Dh * 2 * cfg.elem_bytes
    peak, _ = peaks()
    per_ms = ms / steps
    achieved = logical / (per_ms / 1e3) / 1e9
    return {
        "metric": METRIC, "value": replica_value(cfg.B, steps, world, max_over_ranks(ms, world)), "unit": UNIT,
        "n_gpus": world, "steps": steps, "warmup": warm, "ms_per_step": per_ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": cfg.dtype, "data": "synthetic (seeded token ids; N(0,1) K/V, q)",
        "config": {"workload": cfg.name, "B": cfg.B, "prefix_tokens": W.PREFIX_LEN, "prefix_pages_shared": hits // max(cfg.B - 1, 1),
                   "H_q": cfg.H_q, "H_kv": cfg.H_kv, "Dh": cfg.Dh, "page_size": P,
                   "l2": "prefix pages (~17 MB) stay L2-resident; logical bytes count them per sequence; no flush",
                   "timing": "per step, events around the device's work (launches queued behind a short spin)"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "traffic": None, "bytes": "logical (prefix read per sequence)", "logical_bytes_per_launch": logical,
                     "unique_kv_bytes": unique, "launch_us": per_ms * 1e3},
        "gpu_launches": steps * st.launches_per_step, "e2e": None, "clocks": None,
    }


def run_mixed_bench(args, world, rank, local):
    """Mixed continuous-batching sweep: B=256, log-normal lengths, H_kv in {1, 8, 32}, P in {16, 32}; before
    every step each sequence exits with probability 1/32 and a new one is admitted in its row (pages freed /
    allocated on the host, its K/V written outside the timed region); the timed part is append + decode.
    Per point: the device-timed steps with their clocks, and (sustained) the last step's call repeated
    back to back for >= 1 s, median of 5 repeats."""
    import torch

    from paged_kv_cache_433_b200 import workloads as W

    steps = args.steps if args.steps is not None else 20
    warm = args.warmup if args.warmup is not None else 3
    points = []
    tot_ms = tot_seq = tot_bytes = 0.0
    launches = 0
    pts = W.MIXED_POINTS
    if args.mixed_point:
        h, p = (int(x) for x in args.mixed_point.split(","))
        pts = [(h, p)]
    peak, _ = peaks()
    stream = torch.cuda.current_stream()
    for H_kv, P in pts:
        cfg = W.mixed_config(H_kv, P)
        lens = W.cached_lengths(cfg)
        events = W.churn_events(cfg, warm + steps)
        max_blocks = -(-(16384 + warm + steps + 1) // P) + 1
        num_pages = int(sum(-(-(int(L) + warm + steps) // P) for L in lens)) * 3 // 2 + 4 * max_blocks
        st = PagedState(cfg, lens, max_blocks, num_pages, cfg.seed * 100 + H_kv + P + 1000 * rank)
        for b in range(cfg.B):
            st.admit(b, int(lens[b]))

        def churn(i, st=st, events=events):
            ev = events[i]
            for b, L in zip(ev.exits, ev.new_lengths):
                st.release(int(b))
                st.admit(int(b), int(L))

        clk = ClockSampler(local, enabled=not args.no_clocks)
        res, again = time_steps(args, st, steps, warm, before_step=churn)
        clocks = clk.stop()
        ms = float(np.sum([r[0] for r in res]))
        byts = float(np.sum([r[1] for r in res]))
        S = st.splits_used
        C = -(-max_blocks // S) if S > 0 else 0
        variants = kv_byte_variants(cfg, st.lens, cfg.B, cfg.elem_bytes, S, C, st.plan_C)
        pt = {"H_kv": H_kv, "page_size": P, "seq_steps_per_s": cfg.B * steps / (ms / 1e3),
              "GBps": byts / (ms / 1e3) / 1e9, "frac": byts / (ms / 1e3) / 1e9 / peak,
              "us_per_step": ms / steps * 1e3, "mean_len": float(np.mean(st.lens)),
              "launch": "planned" if S == 0 else f"grid split S={S}", "plan_chunk_pages": st.plan_C,
              "kernel": KERNEL_NAMES.get(st.kernel_kind, str(st.kernel_kind)),
              "bytes_per_step": byts / steps, **variants, "clocks": clocks}
        if not args.no_sustained:
            sus = sustained_repeats(again, 1, stream, ms / steps, local, args)
            last_bytes = res[-1][1]
            sus["frac_median"] = last_bytes / (sus["ms_per_step_median"] / 1e3) / 1e9 / peak
            sus["note"] = "the last step's append + decode call repeated back to back"
            pt["sustained"] = sus
        points.append(pt)
        tot_ms += ms
        tot_seq += cfg.B * steps
        launches += steps * st.launches_per_step
        tot_bytes += byts
        del st
        torch.cuda.empty_cache()
    achieved = tot_bytes / (tot_ms / 1e3) / 1e9
    return {
        "metric": METRIC, "value": tot_seq * world / (max_over_ranks(tot_ms, world) / 1e3), "unit": UNIT,
        "n_gpus": world, "steps": steps, "warmup": warm, "ms_per_step": tot_ms / (steps * len(points)),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded log-normal lengths, churn 1/32 per step; N(0,1) K/V, q)",
        "config": {"workload": "mixed-bf16-B256-lognormal1024-sweep", "B": 256, "H_q": 32, "Dh": 128,
                   "points": "H_kv x page_size = {1,8,32} x {16,32}", "l2": "inputs larger than L2; no flush",
                   "timing": "per step, events around the device's work (launches queued behind a short spin)"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     **roofline_fracs(achieved, peak), "traffic": None},
        "sweep": points, "gpu_launches": launches, "e2e": None,
        "clocks": {"per_point": "see sweep[i].clocks"},
    }


# ---------------------------------------------------------------------------- CPU oracle (baseline / reference arm)
class OracleSample:
    """Host copy of the 8B-shaped decode workload for the fp64 oracle (seeded synthetic inputs)."""

    def __init__(self):
        from oracle import reference as R
        from paged_kv_cache_433_b200 import workloads as W

        self.R, self.W = R, W
        cfg = W.LLAMA8B
        self.cfg = cfg
        lens = W.cached_lengths(cfg) + 1  # lengths after the append
        P = cfg.page_size
        self.lens = lens.astype(np.int32)
        nblk = [-(-int(L) // P) for L in lens]
        self.max_blocks = max(nblk)
        n_pages = int(sum(nblk))
        order = W.page_order(n_pages, cfg.seed)
        self.tab = np.zeros((cfg.B, self.max_blocks), np.int32)
        shape = (n_pages, cfg.H_kv, P, cfg.Dh)
        self.kp = np.zeros(shape, np.uint16)
        self.vp = np.zeros(shape, np.uint16)
        k = 0
        for b in range(cfg.B):
            self.tab[b, :nblk[b]] = order[k:k + nblk[b]]
            k += nblk[b]
            kr, vr = W.kv_rows(cfg, 0, b, int(lens[b]))
            R.scatter_to_pages(self.kp, self.tab[b], kr)
            R.scatter_to_pages(self.vp, self.tab[b], vr)
        self.q = W.queries(cfg, 0, 0)

    def run(self, seqs):
        seqs = np.asarray(seqs)
        return self.R.paged_decode(self.q[seqs], self.kp, self.vp, self.tab[seqs], self.lens[seqs], self.cfg.scale,
                                   self.cfg.dtype)

    def cores(self):
        return self.R.max_threads()


def cpu_baseline(budget_s=10.0):
    """The oracle as it stands on this host's cores: whole 64-sequence decode steps, repeated for ~budget_s."""
    o = OracleSample()
    B = o.cfg.B
    t0 = time.perf_counter()
    runs = 0
    while True:
        o.run(np.arange(B))
        runs += 1
        if time.perf_counter() - t0 >= budget_s:
            break
    dt = time.perf_counter() - t0
    return {"value": B * runs / dt, "unit": UNIT, "cores": o.cores(), "kind": "oracle",
            "sample": f"{runs} full decode steps of the 64-sequence Llama-3.1-8B-shaped layer (bf16 K/V, fp64 math), "
                      f"{dt:.1f} s"}


def oracle_rows_baseline(cfg, rows, row_lens, budget_s=10.0, layers_per_step=1, what=""):
    """The fp64 oracle as it stands, timed on the host cores over a bounded sample: the K/V of the given rows
    (one layer) drawn from the seeded host generators into a compact pool, one decode of those rows repeated
    for ~budget_s. value = sequences decoded per second / layers_per_step (a step covers every layer)."""
    from oracle import reference as R
    from paged_kv_cache_433_b200 import workloads as W

    P = cfg.page_size
    npg = [-(-int(n) // P) for n in row_lens]
    kp = np.zeros((sum(npg), cfg.H_kv, P, cfg.Dh), np.uint16 if cfg.dtype != "fp32" else np.float32)
    vp = np.zeros_like(kp)
    tab = np.full((len(rows), max(npg)), -1, np.int32)
    first = 0
    for i, (b, n) in enumerate(zip(rows, row_lens)):
        tab[i, :npg[i]] = np.arange(first, first + npg[i], dtype=np.int32)
        first += npg[i]
        kr, vr = W.kv_rows(cfg, 0, int(b), int(n))
        R.scatter_to_pages(kp, tab[i], kr)
        R.scatter_to_pages(vp, tab[i], vr)
    q = W.queries(cfg, 0, 0)[np.asarray(rows)]
    lens = np.asarray(row_lens, np.int32)
    t0 = time.perf_counter()
    runs = 0
    while True:
        R.paged_decode(q, kp, vp, tab, lens, cfg.scale, cfg.dtype)
        runs += 1
        if time.perf_counter() - t0 >= budget_s:
            break
    dt = time.perf_counter() - t0
    return {"value": len(rows) * runs / dt / layers_per_step, "unit": UNIT, "cores": R.max_threads(),
            "kind": "oracle",
            "sample": f"{runs} decodes of {len(rows)} row(s) of {what or cfg.name} (one layer"
                      f"{f' of {layers_per_step}, scaled by 1/{layers_per_step}' if layers_per_step > 1 else ''}; "
                      f"fp64 over {cfg.dtype} K/V), {dt:.1f} s"}


def run_reference(args):
    """--impl reference: the fp64 oracle on the host cores, a bounded sample of the workload per step."""
    o = OracleSample()
    steps = args.steps if args.steps is not None else o.cfg.timed_steps
    warm = args.warmup if args.warmup is not None else o.cfg.warmup_steps
    per_step = 4  # sequences per step: keeps K=100 steps within about a minute on 8 cores
    B = o.cfg.B

    def step(i):
        o.run((np.arange(per_step) + per_step * i) % B)

    for i in range(warm):
        step(i)
    t0 = time.perf_counter()
    for i in range(steps):
        step(warm + i)
    dt = time.perf_counter() - t0
    value = per_step * steps / dt
    sample = (f"{per_step} of the 64 sequences per step (rotating), one layer, fp64 oracle over bf16 K/V; "
              f"{steps} steps in {dt:.1f} s")
    return {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus, "steps": steps, "warmup": warm,
        "ms_per_step": dt / steps * 1e3, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic (seeded N(0,1) K/V, q; lengths U[512,4096])",
        "config": {"workload": o.cfg.name, "B": B, "H_q": o.cfg.H_q, "H_kv": o.cfg.H_kv, "Dh": o.cfg.Dh,
                   "page_size": o.cfg.page_size, "layers": 1},
        "impl": "reference",
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": o.cores(), "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }


def run_rope_bench(args, world, rank, local):
    """kv_rope_append on a prefill chunk of the 8B-shaped layer: 8192 tokens rotate q (into a separate
    buffer) and k by their positions and append k, v into shuffled pages. HBM-bound streaming kernel."""
    import torch

    from paged_kv_cache_433_b200 import kvpaged as K
    from paged_kv_cache_433_b200 import workloads as W

    cfg = W.LLAMA8B
    T, max_pos, P = args.tokens, 65536, cfg.page_size
    steps = args.steps if args.steps is not None else 50
    warm = args.warmup if args.warmup is not None else 5
    dev = torch.device("cuda", local)
    dt = torch.bfloat16
    num_pages = T // P + 8
    gen = torch.Generator(device=dev)
    gen.manual_seed(cfg.seed + 6000 + rank)
    k_pages = torch.zeros((num_pages, cfg.H_kv, P, cfg.Dh), dtype=dt, device=dev)
    v_pages = torch.zeros_like(k_pages)
    q = torch.randn((T, cfg.H_q, cfg.Dh), generator=gen, device=dev).to(dt)
    q_out = torch.empty_like(q)
    kn = torch.randn((T, cfg.H_kv, cfg.Dh), generator=gen, device=dev).to(dt)
    vn = torch.randn((T, cfg.H_kv, cfg.Dh), generator=gen, device=dev).to(dt)
    order = torch.from_numpy(W.page_order(num_pages, cfg.seed + 6000)).to(dev).long()
    assert T + 4096 <= max_pos
    pos = torch.arange(T, dtype=torch.int32, device=dev) + 4096  # a chunk after a 4096-token prefix
    slots = (order[(pos.long() - 4096) // P] * P + (pos.long() - 4096) % P).contiguous()
    # cos / sin table of the usual rotary embedding (base 500000), fp32 [max_pos, Dh]
    k = torch.arange(cfg.Dh // 2, dtype=torch.float64, device=dev)
    ang = torch.arange(max_pos, dtype=torch.float64, device=dev)[:, None] * (500000.0 ** (-2.0 * k / cfg.Dh))[None, :]
    table = torch.cat([torch.cos(ang), torch.sin(ang)], dim=1).float().contiguous()
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream()

    def call():
        K.kv_rope_append(k_pages, v_pages, kn, vn, slots, pos, table, P, style="half", q=q, q_out=q_out, err_flag=err,
                         stream=stream)

    for _ in range(warm):
        call()
    torch.cuda.synchronize()
    sampler = ClockSampler(local, enabled=not args.no_clocks)
    barrier(world)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        call()
    e1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    clocks = sampler.stop()
    ms = max_over_ranks(e0.elapsed_time(e1), world)
    if int(err.item()) != 0:
        raise RuntimeError(f"device error flag {int(err.item())}")
    eb = 2
    bytes_per = (2 * T * cfg.H_q * cfg.Dh * eb            # q read, q_out written
                 + 2 * 2 * T * cfg.H_kv * cfg.Dh * eb     # k, v read and written
                 + T * (8 + 4) + T * cfg.Dh * 4)          # slots, positions, one cos/sin row per token
    peak, src = peaks()
    per_ms = ms / steps
    achieved = bytes_per / (per_ms / 1e3) / 1e9
    return {
        "metric": "kv_rope_append tokens/s; achieved HBM GB/s", "value": T * steps * world / (ms / 1e3),
        "unit": "tokens/s", "n_gpus": world, "steps": steps, "warmup": warm, "ms_per_step": per_ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": f"synthetic (N(0,1) q, k, v; positions 4096..{4095 + T}; shuffled pages)",
        "config": {"workload": f"rope-append-prefill-chunk-T{T}-{cfg.name}", "tokens": T, "H_q": cfg.H_q,
                   "H_kv": cfg.H_kv, "Dh": cfg.Dh, "page_size": P, "style": "half", "max_pos": max_pos,
                   "l2": f"{bytes_per / 1e6:.0f} MB moved per launch > 126 MB L2; no flush"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "peak_source": src, "traffic": None, "kernel": "kv_rope_append_kernel<bf16>",
                     "bytes_per_launch": bytes_per, "launch_us": per_ms * 1e3},
        "gpu_launches": steps, "e2e": None, "clocks": clocks,
    }


def W_mod():
    from paged_kv_cache_433_b200 import workloads as W

    return W


def args_for(args, **kw):
    """A copy of the parsed arguments with some fields replaced (the sub-records use their own step counts)."""
    import copy

    a = copy.copy(args)
    for k, v in kw.items():
        setattr(a, k, v)
    return a


def long_context_baseline(W):
    """Oracle baseline of the 32K-context step: one layer (of 32) of one step, scaled by 1/32."""
    cfg = W.LONG32K
    return oracle_rows_baseline(cfg, [0], [W.LONG_T + 1], budget_s=10.0, layers_per_step=cfg.layers)


def mixed_baseline(W):
    """Oracle baseline of the mixed sweep: 16 rows of the GQA point (H_kv = 8, P = 16) at their log-normal lengths."""
    cfg = W.mixed_config(8, 16)
    lens = W.cached_lengths(cfg) + 1
    rows = list(range(16))
    return oracle_rows_baseline(cfg, rows, lens[rows], budget_s=10.0, what=cfg.name + " (16 rows)")


def main():
    args = parse()
    if args.impl == "reference":
        if int(os.environ.get("RANK", "0")) != 0:
            return 0
        print(json.dumps(run_reference(args)), flush=True)
        return 0
    world, rank, local = setup_dist(args)
    from paged_kv_cache_433_b200 import kvpaged as K

    K.paged_decode_set_kernel({"auto": K.KV_DECODE_KERNEL_AUTO, "simt": K.KV_DECODE_KERNEL_SIMT,
                               "mma": K.KV_DECODE_KERNEL_MMA, "tc": K.KV_DECODE_KERNEL_TCGEN05}[args.kernel])
    run = {2: run_layer_bench, 3: run_long_bench, 4: run_prefix_bench, 5: run_mixed_bench, 6: run_rope_bench,
           7: run_fp8_bench, 8: run_prefill_bench}[args.config]
    res = run(args, world, rank, local)
    base = rank == 0 and world == 1 and not args.no_cpu_baseline
    if base and args.config == 2:
        res["cpu_baseline"] = cpu_baseline()
    if base:
        from paged_kv_cache_433_b200 import workloads as W

        if args.config == 3:
            res["cpu_baseline"] = long_context_baseline(W)
        elif args.config == 4:
            lens = W.cached_lengths(W.SHARED_PREFIX) + 1
            res["cpu_baseline"] = oracle_rows_baseline(W.SHARED_PREFIX, [0, 1, 2, 3], lens[:4], budget_s=10.0)
        elif args.config == 5:
            res["cpu_baseline"] = mixed_baseline(W)
    if args.config == 2 and world == 1 and not args.no_extra:
        # the other gated workload and the sweep, measured in the same process (sub-records)
        import torch

        torch.cuda.empty_cache()
        long = run_long_bench(args_for(args, steps=None, warmup=None), world, rank, local)
        if base:
            long["cpu_baseline"] = long_context_baseline(W_mod())
        torch.cuda.empty_cache()
        mixed = run_mixed_bench(args_for(args, steps=20, warmup=3), world, rank, local)
        if base:
            mixed["cpu_baseline"] = mixed_baseline(W_mod())
        res["configs"] = {long["config"]["workload"]: long, mixed["config"]["workload"]: mixed}
    if world > 1:
        import torch.distributed as dist

        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(res), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
