"""Throughput of the DDTree tree-verify step (mask + MLA-absorb attention) on B200.

One step = va_build_tree_mask + va_verify_attn (+ va_merge when split) over one
batch of synthetic requests, inputs resident in HBM.  Default workload:
bf16, B = 64 requests, H = 64 heads, prefix P ~ U[512, 8192] per request,
tree budget 32 (T = 33) best-first trees, 64-token shuffled pages.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--impl reference]

Prints one JSON line (rank 0).  `value` is TFLOP/s of algorithmic work
(visible keys only) over the whole job; `e2e` is the same metric through the
public binding with host buffers (pinned host -> device copies of the
step's queries and tree, result copied back, inside the timed region; the
KV cache stays resident).  `--impl reference` times the fp64 CPU oracle on a
bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from speculative_decoding_tree_va_b200 import synth  # noqa: E402

METRIC = ("verify-attn TFLOP/s & % of B200 roofline; µs per tree-verify step at B=64")
FP32_FFMA_PEAK = 148 * 128 * 2 * 1.965e9 / 1e12  # TFLOP/s, fp32 FFMA at the max SM clock
FLOP_PER_KEY = 2 * (synth.D_LATENT + synth.D_ROPE) + 2 * synth.D_LATENT  # QK + PV per (row, key)


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            m = json.load(f)
        return m["hbm_gbs"], m["bf16_tflops"], m.get("bf16_tflops_sustained"), "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


def recorded_traffic(kernel_src: str, workload: str):
    """DRAM bytes per launch of a kernel, from an ncu summary under profiles/.

    A summary records them on a line
    ``traffic-record: source_sha256=<hex> workload=<name> dram_bytes_per_launch=<int>``;
    the figure only counts while the kernel source still hashes to <hex>."""
    import glob
    import hashlib
    try:
        with open(os.path.join(ROOT, kernel_src), "rb") as f:
            sha = hashlib.sha256(f.read()).hexdigest()
    except OSError:
        return None
    for path in sorted(glob.glob(os.path.join(ROOT, "profiles", "*.md"))):
        with open(path) as f:
            for line in f:
                if not line.startswith("traffic-record:"):
                    continue
                kv = dict(x.split("=", 1) for x in line.split()[1:] if "=" in x)
                if kv.get("source_sha256") == sha and kv.get("workload") == workload:
                    return int(kv["dram_bytes_per_launch"])
    return None


def work(inp, depth):
    """Algorithmic flops and bytes of one step (visible keys only)."""
    B, T, H = inp.wl.B, inp.T, inp.wl.H
    e = 2 if inp.wl.dtype == "bf16" else 4
    ekv = 1 if inp.wl.kv == "fp8_e4m3" else e
    present = depth >= 0                                    # [B, T]
    vis = (inp.prefix[:, None].astype(np.int64) + depth + 1) * present
    flops = float(vis.sum()) * H * FLOP_PER_KEY
    kv_bytes = float(inp.kv_len.astype(np.int64).sum()) * (synth.D_LATENT + synth.D_ROPE) * ekv
    q_bytes = float(B * T * H) * (synth.D_LATENT + synth.D_ROPE) * e
    out_bytes = float(B * T * H) * (synth.D_LATENT * e + 4)
    return flops, kv_bytes + q_bytes + out_bytes


class Clocks:
    """Samples SM clocks and throttle reasons with nvidia-smi during a region.

    Every 20 ms: under continuous load the power cap engages after some tens
    of milliseconds (sw_power_cap, SM clock down from 1965 to ~1620 MHz), and
    a coarser sampling misses it inside a short timed region."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        import tempfile
        self.path = os.path.join(tempfile.gettempdir(), f"va_bench_clocks_{os.getpid()}.csv")

    def __enter__(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.Q}", "--format=csv,noheader",
                 "-lms", "20"], stdout=self.f, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.f.close()

    def summary(self):
        if self.proc is None or not os.path.exists(self.path):
            return None
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1].split()[0]))
                mx = float(f[2].split()[0])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        loaded = [s for s in sm if s > 0.5 * (mx or 1)] or sm
        return {"sm_mhz": float(np.median(loaded)), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def dist_setup(n_gpus, backend="nccl"):
    """One process per GPU under torchrun: (rank, local rank, torch.distributed or None).

    `backend` is "nccl" on GPUs; the rank plumbing is tested with "gloo" on CPU."""
    import torch
    import torch.distributed as dist
    if n_gpus > 1:
        import datetime
        rank = int(os.environ["RANK"])
        local = int(os.environ.get("LOCAL_RANK", rank))
        kw = {}
        if backend == "nccl":
            torch.cuda.set_device(local)
            kw["device_id"] = torch.device("cuda", local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120), **kw)
        return rank, local, dist
    if backend == "nccl":
        torch.cuda.set_device(0)
    return 0, 0, None


def max_over_ranks(x: float, dist, device="cuda") -> float:
    """The slowest rank's figure (every rank takes part; all get the same value)."""
    if dist is None:
        return x
    import torch
    t = torch.tensor([x], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_seed(wl, rank: int) -> int:
    """Each rank verifies its own independent batch (weak scaling)."""
    return wl.seed + 7919 * rank


def config_of(wl, S, world, flops, alg_bytes):
    """The workload description both arms print."""
    return {"workload": wl.name, "B": wl.B, "H": wl.H, "T": wl.T,
            "prefix": list(wl.P) if isinstance(wl.P, tuple) else wl.P,
            "tree": f"best-first top-{wl.topk}, depth<={wl.max_depth}, budget {wl.budget}",
            "kv": ("64-token pages, shuffled" if wl.paged else "contiguous")
                  + (f", FP8 E4M3 cache x {wl.kv_scale}" if wl.kv == "fp8_e4m3" else ""),
            "num_splits": S, "parallelism": f"replicas x{world} (independent requests)",
            "l2": ("inputs larger than the 126 MB L2, no flush" if alg_bytes > 126e6 else
                   "inputs fit in the 126 MB L2: value is the warm-cache figure, l2_flushed "
                   "the same steps after a 256 MB flush"),
            "gflop_per_step": round(flops / 1e9, 2), "alg_mb_per_step": round(alg_bytes / 1e6, 1)}


def run_gpu(args):
    import torch
    import speculative_decoding_tree_va_b200 as va

    rank, local, dist = dist_setup(args.gpus)
    wl = synth.WORKLOADS[args.workload]
    # every rank verifies its own batch (independent requests): weak scaling
    inp = synth.make_inputs(wl, seed=rank_seed(wl, rank))
    dev = torch.device("cuda", local)
    bf16 = wl.dtype == "bf16"
    fp8 = wl.kv == "fp8_e4m3"
    # bf16 queries run on the tensor cores (an FP8 cache is widened first)
    # unless --cuda-cores asks for the CUDA-core kernel
    tc = bf16 and not args.cuda_cores
    vflags = va.VA_FLAG_BF16_CUDA_CORES if (bf16 and args.cuda_cores) else 0
    tdt = torch.bfloat16 if bf16 else torch.float32

    def to_dev(a):
        t = torch.from_numpy(np.ascontiguousarray(a))
        if bf16:
            t = t.view(torch.int16).view(torch.bfloat16)
        return t.to(dev)

    q_nope, q_pe = to_dev(inp.q_nope), to_dev(inp.q_pe)
    if fp8:
        c_kv, k_pe = (torch.from_numpy(a).view(torch.float8_e4m3fn).to(dev) for a in (inp.c_kv, inp.k_pe))
    else:
        c_kv, k_pe = to_dev(inp.c_kv), to_dev(inp.k_pe)
    page_table = torch.from_numpy(inp.page_table).to(dev)
    kv_len = torch.from_numpy(inp.kv_len).to(dev)
    # draft trees from the library's GPU best-first builder
    parents, _, depth, _ = va.build_tree(torch.from_numpy(inp.lp).to(dev),
                                         torch.from_numpy(inp.tok).to(dev), wl.budget)
    depth_h = depth.cpu().numpy()
    flops, alg_bytes = work(inp, depth_h)
    B, T, H = wl.B, wl.T, wl.H
    out = torch.empty(B, T, H, synth.D_LATENT, device=dev, dtype=tdt)
    lse = torch.empty(B, T, H, device=dev, dtype=torch.float32)
    mask = torch.empty(B, T, (T + 63) // 64, device=dev, dtype=torch.int64)
    tstat = torch.empty(B, device=dev, dtype=torch.int32)
    splits = args.splits if args.splits is not None else wl.splits
    vargs = va.make_args(q_nope, q_pe, c_kv, k_pe, page_table, kv_len, mask, out, lse,
                         scale=synth.SCALE, num_splits=splits, kv_scale=wl.kv_scale,
                         flags=vflags)
    S = va.num_splits(vargs)
    wbytes = va.workspace_bytes(vargs)
    ws = torch.empty(max(wbytes, 256), device=dev, dtype=torch.uint8) if wbytes else None
    if ws is not None:
        vargs.workspace, vargs.workspace_bytes = ws.data_ptr(), wbytes
    lib = va.load_library()
    stream = torch.cuda.current_stream(dev)
    sptr = va._stream(stream)
    import ctypes

    def step(ev_a=None, ev_b=None, ev_s=None):
        if ev_s is not None:
            ev_s.record(stream)
        r = lib.va_build_tree_mask(ctypes.c_void_p(parents.data_ptr()), B, T,
                                   ctypes.c_void_p(mask.data_ptr()),
                                   ctypes.c_void_p(tstat.data_ptr()), sptr)
        if ev_a is not None:
            ev_a.record(stream)
        r |= lib.va_verify_attn(ctypes.byref(vargs), sptr)
        if ev_b is not None:
            ev_b.record(stream)
        if r:
            raise RuntimeError("library call failed")

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()

    # timed region: K back-to-back steps, inputs (> 126 MB L2) resident in HBM
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
            torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with Clocks(local) as clk:
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()
        t0.record(stream)
        for a, b, c in evs:
            step(a, b, c)
        t1.record(stream)
        torch.cuda.synchronize()
        if dist is not None:
            dist.barrier()
    ms_total = t0.elapsed_time(t1)
    ms_total = max_over_ranks(ms_total, dist)
    attn_ms = float(np.mean([a.elapsed_time(b) for a, b, _ in evs]))
    # per-step spread: step i runs from its first event to the next step's
    # first event (the last one to the end of the region)
    starts = [c for _, _, c in evs] + [t1]
    step_ms = [starts[i].elapsed_time(starts[i + 1]) for i in range(args.steps)]
    ms_step = ms_total / args.steps
    world = args.gpus
    value = flops * world / (ms_step * 1e-3) / 1e12

    # Inputs that fit in the 126 MB L2 are timed warm above; the same steps
    # with 256 MB written between them (evicting the inputs) give the cold
    # figure beside it.  Each step is timed alone, the flush outside it.
    l2_flushed = None
    if alg_bytes <= 126e6:
        flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
        pairs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                 for _ in range(min(args.steps, 20))]
        for a, b in pairs:
            flush.zero_()
            a.record(stream)
            step()
            b.record(stream)
        torch.cuda.synchronize()
        fl = [a.elapsed_time(b) * 1e3 for a, b in pairs]
        l2_flushed = {"us_per_step_median": round(float(np.median(fl)), 1),
                      "us_per_step_min": round(min(fl), 1), "us_per_step_max": round(max(fl), 1),
                      "steps": len(fl), "flush": "256 MB written to device memory before each step"}
        del flush

    # End to end through the binding with host buffers: every step copies its
    # queries, tree, kv_len and page table from pinned host memory and reads its
    # out / lse back.  Two device buffer sets and three streams let step i's
    # host->device copy, step i-1's compute and step i-2's device->host copy
    # overlap, as a serving loop would; the KV cache stays resident.
    def host(a):
        a = np.ascontiguousarray(a)
        return torch.from_numpy(a.view(np.int16) if bf16 else a).pin_memory()

    q_nope_h, q_pe_h = host(inp.q_nope), host(inp.q_pe)
    par_h = parents.cpu().pin_memory()
    kv_h = torch.from_numpy(inp.kv_len).pin_memory()
    pt_h = torch.from_numpy(inp.page_table).pin_memory()
    h2d = sum(x.numel() * x.element_size() for x in (q_nope_h, q_pe_h, par_h, kv_h, pt_h))
    d2h = out.numel() * out.element_size() + lse.numel() * 4

    sets = []
    for k in range(2):
        st_ = dict(q_nope=torch.empty_like(q_nope), q_pe=torch.empty_like(q_pe),
                   parents=torch.empty_like(parents), kv_len=torch.empty_like(kv_len),
                   page_table=torch.empty_like(page_table), mask=torch.empty_like(mask),
                   tstat=torch.empty_like(tstat), out=torch.empty_like(out), lse=torch.empty_like(lse),
                   out_h=torch.empty(out.numel() * out.element_size(), dtype=torch.uint8).pin_memory(),
                   lse_h=torch.empty(lse.numel(), dtype=torch.float32).pin_memory())
        st_["ws"] = torch.empty(max(wbytes, 256), device=dev, dtype=torch.uint8) if wbytes else None
        st_["args"] = va.make_args(st_["q_nope"], st_["q_pe"], c_kv, k_pe, st_["page_table"],
                                   st_["kv_len"], st_["mask"], st_["out"], st_["lse"],
                                   scale=synth.SCALE, num_splits=splits, workspace=st_["ws"],
                                   kv_scale=wl.kv_scale, flags=vflags)
        sets.append(st_)
    s_in, s_run, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = {n: [torch.cuda.Event() for _ in range(2)] for n in ("in", "run", "out")}
    run_ptr = va._stream(s_run)

    def e2e_step(i):
        k = i % 2
        b_ = sets[k]
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(ev["run"][k])          # step i-2 has read this set's inputs
            for d_, h_ in ((b_["q_nope"], q_nope_h), (b_["q_pe"], q_pe_h), (b_["parents"], par_h),
                           (b_["kv_len"], kv_h), (b_["page_table"], pt_h)):
                (d_.view(torch.int16) if d_.dtype == torch.bfloat16 else d_).copy_(h_, non_blocking=True)
            ev["in"][k].record(s_in)
        s_run.wait_event(ev["in"][k])
        if i >= 2:
            s_run.wait_event(ev["out"][k])             # step i-2's results have left this set
        r = lib.va_build_tree_mask(ctypes.c_void_p(b_["parents"].data_ptr()), B, T,
                                   ctypes.c_void_p(b_["mask"].data_ptr()),
                                   ctypes.c_void_p(b_["tstat"].data_ptr()), run_ptr)
        r |= lib.va_verify_attn(ctypes.byref(b_["args"]), run_ptr)
        if r:
            raise RuntimeError("library call failed")
        ev["run"][k].record(s_run)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev["run"][k])
            b_["out_h"].copy_(b_["out"].view(-1).view(torch.uint8), non_blocking=True)
            b_["lse_h"].copy_(b_["lse"].view(-1), non_blocking=True)
            ev["out"][k].record(s_out)

    for i in range(4):
        e2e_step(i)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n_e2e = max(4, min(args.steps, 20))
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    e0.record(s_in)
    for i in range(n_e2e):
        e2e_step(i)
    e1.record(s_out)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / n_e2e, dist)
    # the overlapped loop must produce the same result as the plain step
    assert torch.equal(sets[(n_e2e - 1) % 2]["lse"], lse) and torch.equal(sets[(n_e2e - 1) % 2]["out"], out)
    e2e_value = flops * world / (e2e_ms * 1e-3) / 1e12

    hbm, tc_peak, tc_sust, peak_src = peaks()
    kernel_src = "speculative_decoding_tree_va_b200/csrc/" + ("va_attn_tc.cu" if tc else "va_attn_simt.cu")
    traffic = recorded_traffic(kernel_src, wl.name) if S == 1 else None
    achieved = flops / (attn_ms * 1e-3) / 1e12
    roof_us = max(flops / ((tc_peak if tc else FP32_FFMA_PEAK) * 1e12), alg_bytes / (hbm * 1e9)) * 1e6
    clocks = clk.summary()
    # the split-KV long prefix and the deep-tree batch, timed in the same
    # process beside the headline (one GPU only; replicas skip them)
    others = None
    if world == 1 and not args.no_other_workloads and not args.cuda_cores:
        others = {}
        for name, sp in OTHER_WORKLOADS:
            if name == wl.name and sp == S:
                continue
            others[f"{name} S={sp}"] = time_workload(va, name, sp, dev, steps=20, warmup=5)
    if dist is not None:
        dist.destroy_process_group()
    if rank != 0:
        return
    cpu = None
    if not args.no_cpu_baseline:
        gpu_out = out.float().cpu().numpy().reshape(-1, synth.D_LATENT)
        gpu_lse = lse.cpu().numpy().reshape(-1)
        cpu = cpu_baseline(inp, depth_h, budget_s=args.cpu_seconds, gpu_out=gpu_out, gpu_lse=gpu_lse)
    line = {
        "metric": METRIC, "value": round(value, 3), "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 4),
        "us_per_step": round(ms_step * 1e3, 1),
        "us_per_step_spread": {"min": round(min(step_ms) * 1e3, 1),
                               "median": round(float(np.median(step_ms)) * 1e3, 1),
                               "max": round(max(step_ms) * 1e3, 1)},
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if tc else "f32", "data": "synthetic (seeded; no dataset or weights)",
        "config": config_of(wl, S, world, flops, alg_bytes),
        "roofline": {"bound": "tensor" if tc else "alu", "achieved": round(achieved, 2),
                     "peak": tc_peak if tc else FP32_FFMA_PEAK,
                     "unit": "TFLOP/s", "frac": round(achieved / (tc_peak if tc else FP32_FFMA_PEAK), 4),
                     "traffic": traffic,
                     "peak_source": (f"{peak_src} bf16 dense (burst); sustained {tc_sust}" if tc else
                                     "derived: 148 SMs x 128 fp32 lanes x 2 flop x 1.965 GHz"),
                     "kernel": (("kv_widen_kernel + attn_tc_kernel" if fp8 else "attn_tc_kernel")
                                if tc else "attn_simt_kernel"),
                     "kernel_us": round(attn_ms * 1e3, 1), "roofline_us": round(roof_us, 1),
                     "frac_of_step_roofline": round(roof_us / (ms_step * 1e3), 4)},
        "e2e": {"value": round(e2e_value, 3), "unit": "TFLOP/s", "ms_per_step": round(e2e_ms, 3),
                "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
                "pipelining": "2 buffer sets, copy-in / compute / copy-out on 3 streams"},
        "gpu_launches": args.steps * launches_per_step(tc, fp8, S),
        "clocks": clocks,
        "cpu_baseline": cpu,
    }
    if l2_flushed:
        line["l2_flushed"] = l2_flushed
    if others:
        line["other_workloads"] = others
    print(json.dumps(line), flush=True)


OTHER_WORKLOADS = [("bf16-long-prefix", 16), ("bf16-long-prefix", 64), ("bf16-deep", 1)]


def run_sharded(args):
    """One batch for the whole job, its split-KV partition shared out across the GPUs.

    Every rank holds the same batch; rank r computes its block of the S splits
    (va_verify_attn_partials), merges them locally, the ranks' partials are
    all-gathered (NCCL), and rank 0 merges them into out / lse.  Strong
    scaling: the work per step is fixed, `value` = its flops / the slowest
    rank's step time.  With one GPU the gather is skipped."""
    import ctypes

    import torch
    import speculative_decoding_tree_va_b200 as va
    from speculative_decoding_tree_va_b200.shard import ShardedStep

    rank, local, dist = dist_setup(args.gpus)
    world = args.gpus
    wl = synth.WORKLOADS[args.workload]
    S = args.splits if args.splits is not None else wl.splits
    if S < 1:
        raise SystemExit("--shard-prefix needs an explicit split count (--splits)")
    inp = synth.make_inputs(wl)                      # the same batch on every rank
    dev = torch.device("cuda", local)
    bf16 = wl.dtype == "bf16"
    tdt = torch.bfloat16 if bf16 else torch.float32

    def to_dev(a):
        t = torch.from_numpy(np.ascontiguousarray(a))
        return (t.view(torch.int16).view(torch.bfloat16) if bf16 else t).to(dev)

    parents, _, depth, _ = va.build_tree(torch.from_numpy(inp.lp).to(dev),
                                         torch.from_numpy(inp.tok).to(dev), wl.budget)
    flops, alg_bytes = work(inp, depth.cpu().numpy())
    B, T, H = wl.B, wl.T, wl.H
    q_nope, q_pe, c_kv, k_pe = (to_dev(a) for a in (inp.q_nope, inp.q_pe, inp.c_kv, inp.k_pe))
    page_table = torch.from_numpy(inp.page_table).to(dev)
    kv_len = torch.from_numpy(inp.kv_len).to(dev)
    mask = torch.empty(B, T, (T + 63) // 64, device=dev, dtype=torch.int64)
    tstat = torch.empty(B, device=dev, dtype=torch.int32)
    out = torch.empty(B, T, H, synth.D_LATENT, device=dev, dtype=tdt)
    lse = torch.empty(B, T, H, device=dev, dtype=torch.float32)
    vargs = va.make_args(q_nope, q_pe, c_kv, k_pe, page_table, kv_len, mask, out, lse,
                         scale=synth.SCALE, num_splits=S)
    lib = va.load_library()
    stream = torch.cuda.current_stream(dev)
    sptr = va._stream(stream)

    class _One:  # one rank: the gather is the identity
        @staticmethod
        def all_gather_into_tensor(o_all, o, group=None):
            o_all.copy_(o.reshape(o_all.shape))

    sharded = ShardedStep(va, vargs, rank, world, dist if dist is not None else _One(), dev)

    def step():
        if lib.va_build_tree_mask(ctypes.c_void_p(parents.data_ptr()), B, T,
                                  ctypes.c_void_p(mask.data_ptr()),
                                  ctypes.c_void_p(tstat.data_ptr()), sptr):
            raise RuntimeError("va_build_tree_mask failed")
        sharded()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with Clocks(local) as clk:
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()
        t0.record(stream)
        for _ in range(args.steps):
            step()
        t1.record(stream)
        torch.cuda.synchronize()
        if dist is not None:
            dist.barrier()
    ms_step = max_over_ranks(t0.elapsed_time(t1) / args.steps, dist) if dist is not None \
        else t0.elapsed_time(t1) / args.steps
    # rank 0 checks the sharded result against the one-GPU call of the same batch
    check = None
    if rank == 0:
        out1, lse1 = va.verify_attn(q_nope, q_pe, c_kv, k_pe, page_table, kv_len, mask,
                                    scale=synth.SCALE, num_splits=S)
        torch.cuda.synchronize()
        fin = torch.isfinite(lse1)
        check = {"out_max_abs_vs_one_gpu": float((out.float() - out1.float()).abs().max()),
                 "lse_max_abs_vs_one_gpu": float((lse[fin] - lse1[fin]).abs().max())}
    clocks = clk.summary()
    if dist is not None:
        dist.destroy_process_group()
    if rank != 0:
        return
    _, tc_peak, tc_sust, peak_src = peaks()
    value = flops / (ms_step * 1e-3) / 1e12
    cfg = config_of(wl, S, world, flops, alg_bytes)
    cfg["parallelism"] = f"split-KV partition of one batch across {world} GPU(s)"
    rows = B * T * H
    line = {
        "metric": METRIC, "value": round(value, 3), "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 4),
        "us_per_step": round(ms_step * 1e3, 1), "higher_is_better": True, "scaling": "strong",
        "vs_baseline": None, "dtype": "bf16" if bf16 else "f32",
        "data": "synthetic (seeded; no dataset or weights)", "config": cfg,
        "roofline": {"bound": "tensor", "achieved": round(value / world, 2), "per": "GPU",
                     "peak": tc_peak, "unit": "TFLOP/s", "frac": round(value / world / tc_peak, 4),
                     "traffic": None, "peak_source": f"{peak_src} bf16 dense (burst)"},
        "exchange_bytes_per_rank": rows * (synth.D_LATENT + 1) * 4,
        "check": check, "clocks": clocks,
        "gpu_launches": args.steps * (1 + 1 + 1 + (1 if sharded.count > 1 else 0) + 1),
        "e2e": {"value": None, "note": "not measured in the sharded mode (device-resident batch)"},
    }
    print(json.dumps(line), flush=True)


def launches_per_step(tc: bool, fp8: bool, S: int) -> int:
    """Library kernels one step launches: the tree mask, the request order
    (tensor cores), the FP8 widening pass (tensor cores with an FP8 cache),
    the attention kernel, and the merge when split."""
    return 2 + (1 if tc else 0) + (1 if tc and fp8 else 0) + (1 if S > 1 else 0)


def time_workload(va, name: str, splits: int, dev, steps: int = 10, warmup: int = 3) -> dict:
    """Device time of mask + verify steps of one more workload (CUDA events, per step)."""
    import ctypes

    import torch
    wl = synth.WORKLOADS[name]
    inp = synth.make_inputs(wl)

    def to_dev(a):
        t = torch.from_numpy(np.ascontiguousarray(a))
        return (t.view(torch.int16).view(torch.bfloat16) if wl.dtype == "bf16" else t).to(dev)

    parents, _, depth, _ = va.build_tree(torch.from_numpy(inp.lp).to(dev),
                                         torch.from_numpy(inp.tok).to(dev), wl.budget)
    flops, alg_bytes = work(inp, depth.cpu().numpy())
    B, T, H = wl.B, wl.T, wl.H
    tdt = torch.bfloat16 if wl.dtype == "bf16" else torch.float32
    out = torch.empty(B, T, H, synth.D_LATENT, device=dev, dtype=tdt)
    lse = torch.empty(B, T, H, device=dev, dtype=torch.float32)
    mask = torch.empty(B, T, (T + 63) // 64, device=dev, dtype=torch.int64)
    tstat = torch.empty(B, device=dev, dtype=torch.int32)
    q_nope, q_pe, c_kv, k_pe = (to_dev(a) for a in (inp.q_nope, inp.q_pe, inp.c_kv, inp.k_pe))
    del inp.c_kv, inp.k_pe
    page_table = torch.from_numpy(inp.page_table).to(dev)
    kv_len = torch.from_numpy(inp.kv_len).to(dev)
    vargs = va.make_args(q_nope, q_pe, c_kv, k_pe, page_table, kv_len, mask, out, lse,
                         scale=synth.SCALE, num_splits=splits)
    S = va.num_splits(vargs)
    wbytes = va.workspace_bytes(vargs)
    ws = torch.empty(max(wbytes, 256), device=dev, dtype=torch.uint8)
    vargs.workspace, vargs.workspace_bytes = ws.data_ptr(), wbytes
    lib = va.load_library()
    stream = torch.cuda.current_stream(dev)
    sptr = va._stream(stream)

    def step():
        r = lib.va_build_tree_mask(ctypes.c_void_p(parents.data_ptr()), B, T,
                                   ctypes.c_void_p(mask.data_ptr()),
                                   ctypes.c_void_p(tstat.data_ptr()), sptr)
        r |= lib.va_verify_attn(ctypes.byref(vargs), sptr)
        if r:
            raise RuntimeError("library call failed")

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(steps + 1)]
    evs[0].record(stream)
    for i in range(steps):
        step()
        evs[i + 1].record(stream)
    torch.cuda.synchronize()
    ms = [evs[i].elapsed_time(evs[i + 1]) for i in range(steps)]
    _, tc_peak, _, _ = peaks()
    mean = float(np.mean(ms))
    res = {"B": B, "H": H, "T": T, "prefix": list(wl.P) if isinstance(wl.P, tuple) else wl.P,
           "num_splits": S, "steps": steps,
           "us_per_step": round(mean * 1e3, 1),
           "us_per_step_spread": {"min": round(min(ms) * 1e3, 1),
                                  "median": round(float(np.median(ms)) * 1e3, 1),
                                  "max": round(max(ms) * 1e3, 1)},
           "tflops": round(flops / (mean * 1e-3) / 1e12, 2),
           "frac": round(flops / (mean * 1e-3) / 1e12 / tc_peak, 4),
           "gflop_per_step": round(flops / 1e9, 2), "alg_mb_per_step": round(alg_bytes / 1e6, 1),
           "l2": "inputs larger than the 126 MB L2, no flush" if alg_bytes > 126e6 else
                 "inputs fit in L2 (warm)"}
    del q_nope, q_pe, c_kv, k_pe, ws, out
    torch.cuda.empty_cache()
    return res


def host_cpu():
    """(logical cores, CPU model) of this host."""
    model = "unknown"
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return os.cpu_count(), model


def cpu_baseline(inp, depth, budget_s=15.0, gpu_out=None, gpu_lse=None):
    """fp64 oracle, single-threaded, on a seeded sample of whole rows.

    With the GPU's out / lse of the same workload (host numpy arrays, one row per
    (b, t, h)), the sampled rows are also compared with it element by element."""
    import oracle
    B, T, H = inp.wl.B, inp.T, inp.wl.H
    trees = oracle.build_trees(inp.lp, inp.tok, inp.wl.budget)
    mask, _ = oracle.ancestor_mask(trees["parent"])
    rng = np.random.default_rng(12345)
    order = rng.permutation(B * T * H).astype(np.int32)
    done_rows, flops, t_used = 0, 0.0, 0.0
    d_out = d_lse = 0.0
    kv_args = (dict(kv_dtype="fp8_e4m3", kv_scale=inp.wl.kv_scale) if inp.wl.kv == "fp8_e4m3"
               else {})
    chunk = 32
    while t_used < budget_s and done_rows < order.size:
        rows = order[done_rows:done_rows + chunk]
        t0 = time.perf_counter()
        ref_out, ref_lse = oracle.attention_rows(inp.q_nope, inp.q_pe, inp.c_kv, inp.k_pe,
                                                 inp.page_table, inp.kv_len, mask,
                                                 scale=synth.SCALE, dtype=inp.wl.dtype, rows=rows,
                                                 **kv_args)
        t_used += time.perf_counter() - t0
        if gpu_out is not None:
            live = np.isfinite(ref_lse)
            d_out = max(d_out, float(np.abs(gpu_out[rows] - ref_out).max()))
            if live.any():
                d_lse = max(d_lse, float(np.abs(gpu_lse[rows][live] - ref_lse[live]).max()))
        b = rows // (T * H)
        t = (rows // H) % T
        d = trees["depth"][b, t]
        flops += float(((inp.prefix[b].astype(np.int64) + d + 1) * (d >= 0)).sum()) * FLOP_PER_KEY
        done_rows += rows.size
    cores, model = host_cpu()
    res = {"value": round(flops / t_used / 1e12, 6), "unit": "TFLOP/s", "cores": 1,
           "kind": "oracle",
           "sample": (f"{done_rows} seeded (b,t,h) rows of {B * T * H}, {t_used:.1f} s, fp64 C++"
                      + (", extrapolated per flop" if done_rows < B * T * H else ", every row")),
           "host": f"{cores} logical cores, {model}"}
    if gpu_out is not None:
        res["parity_on_sample"] = {"rows": done_rows, "out_max_abs": d_out, "lse_max_abs": d_lse}
    return res


def run_reference(args):
    """The oracle as the reference arm: fp64 C++ on the host cores, rank 0 only."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    wl = synth.WORKLOADS[args.workload]
    inp = synth.make_inputs(wl)
    import oracle
    trees = oracle.build_trees(inp.lp, inp.tok, wl.budget)
    depth = trees["depth"]
    per_step = max(2.0, args.cpu_seconds / max(args.steps, 1))
    for _ in range(args.warmup):
        cpu_baseline(inp, depth, budget_s=0.2)
    vals = [cpu_baseline(inp, depth, budget_s=per_step) for _ in range(args.steps)]
    v = float(np.mean([x["value"] for x in vals]))
    flops, alg_bytes = work(inp, depth)
    ms = flops / (v * 1e12) * 1e3
    S = args.splits if getattr(args, "splits", None) is not None else wl.splits
    cfg = config_of(wl, S, args.gpus, flops, alg_bytes)  # the native arm's config, unchanged
    line = {
        "metric": METRIC, "value": round(v, 6), "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 1),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded; no dataset or weights)", "impl": "reference",
        "note": "each step = a bounded row sample; per-step time extrapolated per flop",
        "config": cfg,
        "cpu_baseline": {"value": round(v, 6), "unit": "TFLOP/s", "cores": 1, "kind": "oracle",
                         "sample": vals[0]["sample"], "host": vals[0]["host"]},
        "e2e": {"value": round(v, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default="bf16-b64-ragged", choices=list(synth.WORKLOADS))
    ap.add_argument("--splits", type=int, default=None)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-other-workloads", action="store_true",
                    help="skip the long-prefix and deep-tree figures printed beside the headline")
    ap.add_argument("--shard-prefix", action="store_true",
                    help="shard the workload's split-KV partition across the GPUs (one batch "
                         "for the whole job: strong scaling)")
    ap.add_argument("--cuda-cores", action="store_true",
                    help="run bf16 queries on the CUDA-core kernel (VA_FLAG_BF16_CUDA_CORES)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)  # at least 3 untimed warm-up steps
    if args.impl == "reference":
        run_reference(args)
    elif args.shard_prefix:
        run_sharded(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
