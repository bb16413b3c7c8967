"""Throughput of LSH self-attention forward + backward on B200.

One step = lsh_attn_fwd (hash, sort, attention, round merge) followed by
lsh_attn_bwd (backward prologue, attention backward, epilogue) on the
64K-token workload (B=1, H=8, L=65536, d=64, n_buckets=1024, n_hashes=4,
chunk 64, causal, bf16), inputs resident in HBM.  Prints one JSON line.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

Multi-GPU: launch one process per GPU with torch.distributed.run; each rank
runs an independent replica of the workload (the (batch, head) slices are
independent, so there is no data-path collective) and the time is the max
over ranks.  --impl reference times the CPU oracle on the host cores instead.
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

from lsh_attention_02_b200 import synth  # noqa: E402

METRIC = "LSH-attn fwd+bwd tokens/s at L=64K, 4 hashes; % of HBM/tensor roofline"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def bench_config(w: synth.Workload, world: int) -> dict:
    """The `config` object of both arms' JSON lines (identical for the same run shape)."""
    return {"workload": describe(w), "global_batch": w.B * world, "seq_len": w.L,
            "parallelism": f"{world} independent replica(s), no collective",
            "l2": "flushed between timed steps (256 MiB memset outside the step events)"}


def describe(w: synth.Workload) -> str:
    mode = "fwd+bwd" if w.backward else "fwd"
    extra = f" clustered{w.clustered}(sigma={w.sigma})" if w.clustered else ""
    return (f"{w.name}: B{w.B} H{w.H} L{w.L} d{w.d} n_buckets{w.n_buckets} n_hashes{w.n_hashes} "
            f"chunk{w.chunk} {'causal' if w.causal else 'non-causal'} {w.dtype} {mode}{extra}")


# ------------------------------------------------------------------ algorithmic bytes / flops
def algorithmic(w: synth.Workload) -> dict:
    """Per-step algorithmic HBM bytes and FLOPs (e = element bytes, R = n_hashes, d = 64).

    Whole step, staged formulation:      forward  L [d e (2 + 4R) + 24 R]
                                         backward L [4 d e + 8 + R (4 d e + 16 + 4 d 4)]
    per (batch, head).  Attention FLOPs: 4 (2m) d forward and 5 * 2 (2m) d backward per
    token, head and round; the hash GEMM d * n_buckets per token, head and round."""
    e = 2 if w.dtype == "bf16" else 4
    d, R, L, m = w.d, w.n_hashes, w.L, w.chunk
    bh = w.B * w.H
    fwd = L * (d * e * (2 + 4 * R) + 24 * R)
    bwd = L * (4 * d * e + 8 + R * (4 * d * e + 16 + 4 * d * 4)) if w.backward else 0
    attn_flops = bh * L * R * (4 * 2 * m * d + (10 * 2 * m * d if w.backward else 0))
    hash_flops = bh * L * R * d * w.n_buckets          # 2 flops x d x n_buckets/2 columns
    # per-kernel compulsory bytes (each input read once, each output written once)
    tok = bh * L
    kern = {
        "hash": tok * (d * e + 2 * R + 4),                              # x read, bucket ids and norms written
        "attn_fwd": tok * R * (2 * d * e + 4 + d * 2 + 4) + tok * 4,    # x, v rows + perm; o_r (bf16) + lse; norms
        "combine": tok * (R * (d * 2 + 4) + d * e),                     # o_r, lse read; out written
        "attn_bwd": tok * (3 * d * e + 12 + R * 4) + tok * 2 * d * 4 * 2,  # x, v, dY, LSE, delta, norms, perm;
                                                                          # fp32 dx, dv accumulators in and out
    }
    # the single-kernel forward of short segments: x and v read, the merged output
    # written, per round the lse, the permutation and the bucket ids written (the
    # rounds' outputs pass through L2 to the in-cluster merge)
    kern["fused_fwd"] = tok * (3 * d * e + R * (4 + 4 + 2))
    flops = {"hash": hash_flops, "fused_fwd": hash_flops + bh * L * R * 4 * 2 * m * d,
             "attn_fwd": bh * L * R * 4 * 2 * m * d,
             "attn_bwd": bh * L * R * 10 * 2 * m * d if w.backward else 0, "combine": 0}
    return {"bytes": bh * (fwd + bwd), "attn_flops": attn_flops, "hash_flops": hash_flops, "kernel_bytes": kern,
            "kernel_flops": flops}


# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) of one launch, from
# one ncu capture of the kernel on the named workload (summarised under
# profiles/).  A record counts only while the kernel's sources hash to the
# value taken with it; after any change the traffic is reported as null.
NCU_TRAFFIC = {
    ("long_64k", "attn_bwd"): {"bytes": 763_595_776, "files": ('attn_bwd_tc.cu', 'tc_common.cuh', 'common.cuh'),
                               "sha256": "bd2fe6864fa283d2da546f9f29634c18911c48ef364b9d4d20bca9ddd5952aff"},
    ("long_64k", "attn_fwd"): {"bytes": 368_641_024, "files": ('attn_fwd_tc.cu', 'attn_fwd_roles.cuh', 'tc_common.cuh', 'common.cuh'),
                               "sha256": "3574c081cae3bf556dea136f53c4727fdeff0fedd2183e3b459c46e680033229"},
    ("long_64k", "hash"): {"bytes": 67_439_872, "files": ('hash_tc.cu', 'tc_common.cuh', 'common.cuh'),
                           "sha256": "2e61e9680746c0fc3fee9fc9a7445655758a98a901f4f98dee20d76ece2e532f"},
    ("half_million", "hash"): {"bytes": 141_867_008, "files": ('hash_tc.cu', 'tc_common.cuh', 'common.cuh'),
                               "sha256": "2e61e9680746c0fc3fee9fc9a7445655758a98a901f4f98dee20d76ece2e532f"},
}


def ncu_traffic(workload: str, kernel: str):
    rec = NCU_TRAFFIC.get((workload, kernel))
    if rec is None:
        return None
    import hashlib
    h = hashlib.sha256()
    for f in rec["files"]:
        path = os.path.join(ROOT, "lsh_attention_02_b200", "csrc", f)
        if not os.path.exists(path):
            return None
        with open(path, "rb") as fh:
            h.update(fh.read())
    return float(rec["bytes"]) if h.hexdigest() == rec["sha256"] else None


def step_roofline(alg: dict, hbm_gbs: float, tflops: float, step_ms: float) -> dict:
    """Staged roofline of one step: the slower of the algorithmic bytes at the
    HBM peak and the chunk-attention FLOPs at the bf16 peak; also the
    hash-inclusive variant, which adds the rotation GEMM's FLOPs (it decides
    the bound when n_buckets is large, as for the 512K-token workload)."""
    t_bytes = alg["bytes"] / (hbm_gbs * 1e9)
    t_attn = alg["attn_flops"] / (tflops * 1e12)
    t_all = (alg["attn_flops"] + alg["hash_flops"]) / (tflops * 1e12)
    roof = max(t_bytes, t_attn) * 1e3
    roof_h = max(t_bytes, t_all) * 1e3
    return {"roofline_ms": roof, "frac": roof / step_ms,
            "roofline_ms_with_hash": roof_h, "frac_with_hash": roof_h / step_ms}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return json.load(f), "measured"
    return dict(PEAKS_FALLBACK), "fallback"


# ------------------------------------------------------------------ clocks
class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.QUERY}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        self.lines = []
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self) -> dict:
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in getattr(self, "lines", []):
            f = [s.strip() for s in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1])); mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------------ our arm
# ------------------------------------------------------------------ ranks
def init_ranks(backend: str, device=None, timeout_s: int = 120) -> None:
    """One process per GPU (or per CPU rank for gloo); rendezvous from the
    torch.distributed.run environment (MASTER_ADDR, MASTER_PORT, RANK, WORLD_SIZE)."""
    import datetime
    import torch.distributed as dist
    kw = {"device_id": device} if device is not None and backend == "nccl" else {}
    dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s), **kw)


def max_over_ranks(values, world: int, device) -> list[float]:
    """Element-wise maximum of `values` over all ranks (identity for one rank):
    a multi-GPU time is the slowest rank's."""
    import torch
    import torch.distributed as dist
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.cpu()]


def whole_job_tokens_per_s(w: synth.Workload, world: int, step_ms: float) -> float:
    """Every rank runs its own replica of the workload (weak scaling): all ranks'
    tokens over the slowest rank's step time."""
    return w.tokens * world / (step_ms / 1e3)


def run_ours(args, w: synth.Workload, rank: int, world: int) -> dict | None:
    import torch
    import torch.distributed as dist
    import lsh_attention_02_b200 as lsh

    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        init_ranks("nccl", dev)

    inp = synth.make_inputs(w.replace(seed=w.seed + 1000 * rank))
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    host = {k: torch.from_numpy(v).to(tdt).pin_memory() for k, v in inp.items()}
    x, v, R = host["x"].to(dev), host["v"].to(dev), host["R"].to(dev)
    dy = host["dy"].to(dev) if w.backward else None
    desc = lsh.desc_for(x, w.n_buckets, w.n_hashes, w.chunk, w.causal)
    out, lse, perm = lsh.outputs_like(desc, x)
    ws_f = lsh.workspace(desc, False, dev)
    ws_b = lsh.workspace(desc, True, dev) if w.backward else None
    dx = torch.empty_like(x); dv = torch.empty_like(v)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)   # > 126 MB L2
    torch.cuda.reset_peak_memory_stats(dev)

    def step():
        lsh.lsh_attn_fwd(desc, x, v, R, out, lse, perm, ws_f)
        if w.backward:
            lsh.lsh_attn_bwd(desc, x, v, R, out, lse, perm, dy, dx, dv, ws_b)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if lsh.lsh_attn_poll(ws_f) != 0 or (ws_b is not None and lsh.lsh_attn_poll(ws_b) != 0):
        raise RuntimeError("device-side timeout during warm-up")

    stream = torch.cuda.current_stream(dev)
    # Per-stage breakdown from a separate traced pass (an event pair around every
    # stage costs about 40 us per step, so the timed steps record events around the
    # dominant kernel alone).
    n_tr = max(1, min(args.steps, 10))
    lsh.trace_begin(64 * n_tr + 64)
    for _ in range(n_tr):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    traced = lsh.trace_end()
    alg0 = algorithmic(w)
    dom_name = max((k for k, (ms, c, _) in traced.items() if c and k in alg0["kernel_bytes"]),
                   key=lambda k: traced[k][0])
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        lsh.trace_stages([dom_name])
        lsh.trace_begin(4 * args.steps + 64)
        for k in range(args.steps):
            flush.zero_()
            starts[k].record(stream)
            step()
            ends[k].record(stream)
        torch.cuda.synchronize()
        timed = lsh.trace_end()
        lsh.trace_stages(None)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    step_ms = float(sum(s.elapsed_time(e) for s, e in zip(starts, ends))) / args.steps
    # device memory of the step: inputs, outputs, permutation, workspaces (the L2
    # flush buffer is not part of it)
    peak_bytes = int(torch.cuda.max_memory_allocated(dev)) - flush.numel()
    ws_bytes = {"fwd": int(ws_f.numel()), "bwd": int(ws_b.numel()) if ws_b is not None else 0}
    if lsh.lsh_attn_poll(ws_f) != 0 or (ws_b is not None and lsh.lsh_attn_poll(ws_b) != 0):
        raise RuntimeError("device-side timeout during the timed steps")

    # e2e: the same step through the C ABI's host-buffer entry point (lsh_attn_step_host:
    # pinned host inputs in, results out, copies pipelined with the kernels per chunk of
    # heads on three streams), copies inside the timed region
    e2e = None
    if not args.no_e2e:
        hout = torch.empty_like(out, device="cpu").pin_memory()
        hdx = torch.empty_like(dx, device="cpu").pin_memory(); hdv = torch.empty_like(dv, device="cpu").pin_memory()
        streams = [stream, torch.cuda.Stream(dev), torch.cuda.Stream(dev)]
        scratch = lsh.step_host_scratch(desc, 0, w.backward, dev)
        n_e2e = max(3, min(args.steps, 20))
        e_s = torch.cuda.Event(enable_timing=True); e_e = torch.cuda.Event(enable_timing=True)
        h2d = sum(t.numel() * t.element_size() for t in host.values())
        d2h = hout.numel() * hout.element_size() + (2 * hdx.numel() * hdx.element_size() if w.backward else 0)
        tot = 0.0
        for k in range(n_e2e + 1):
            flush.zero_()
            e_s.record(stream)
            lsh.lsh_attn_step_host(desc, host["x"], host["v"], host["R"], host["dy"] if w.backward else None, hout,
                                   None, hdx if w.backward else None, hdv if w.backward else None, scratch, streams)
            e_e.record(stream)
            torch.cuda.synchronize()
            if k > 0:
                tot += e_s.elapsed_time(e_e)
        if lsh.lsh_attn_poll(scratch) != 0:
            raise RuntimeError("device-side status set during the end-to-end steps")
        e2e_ms = tot / n_e2e
        e2e = {"value": None, "unit": "tokens/s", "ms_per_step": e2e_ms,
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "api": "lsh_attn_step_host (pipelined per chunk of heads)"}

    step_ms, e2e_max = max_over_ranks([step_ms, e2e["ms_per_step"] if e2e else 0.0], world, dev)
    if world > 1:
        dist.destroy_process_group()
    if e2e:
        e2e["ms_per_step"] = e2e_max
        e2e["value"] = whole_job_tokens_per_s(w, world, e2e_max)
    if rank != 0:
        return None

    peaks, peak_src = load_peaks()
    alg = algorithmic(w)
    per_stage = {k: {"ms_per_step": ms / n_tr, "calls": c // n_tr, "kernels": kk // n_tr}
                 for k, (ms, c, kk) in traced.items() if c}
    # our kernels in the timed region: the traced pass's launches per step, times the steps
    launches = sum(s["kernels"] for s in per_stage.values()) * args.steps
    # dominant kernel (the stage with the most time that is a single kernel we wrote),
    # its launch time from the events around it in the timed steps
    t_ms, t_calls, _ = timed[dom_name]
    dom = {"ms_per_step": t_ms / args.steps, "calls": t_calls // args.steps}
    dom_launch_ms = dom["ms_per_step"] / max(dom["calls"], 1)
    dom_bytes = alg["kernel_bytes"][dom_name] / max(dom["calls"], 1)
    dom_flops = alg["kernel_flops"].get(dom_name, 0.0) / max(dom["calls"], 1)
    hbm = float(peaks["hbm_gbs"])
    tensor = float(peaks["bf16_tflops_sustained"])
    # the bound is whichever of bytes at the HBM peak and FLOPs at the bf16 peak
    # takes longer for this kernel
    t_hbm, t_tc = dom_bytes / (hbm * 1e9), dom_flops / (tensor * 1e12)
    if t_tc > t_hbm:
        bound, achieved, peak, unit = "tensor", dom_flops / (dom_launch_ms / 1e3) / 1e12, tensor, "TFLOP/s"
    else:
        bound, achieved, peak, unit = "hbm", dom_bytes / (dom_launch_ms / 1e3) / 1e9, hbm, "GB/s"
    step_bytes_gbs = alg["bytes"] / (step_ms / 1e3) / 1e9
    roof = step_roofline(alg, hbm, float(peaks["bf16_tflops_sustained"]), step_ms)
    res = {
        "metric": METRIC, "value": whole_job_tokens_per_s(w, world, step_ms), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": w.dtype,
        "data": f"synthetic: seeded Philox4x32-10 + Box-Muller normals, rounded to {w.dtype}",
        "config": bench_config(w, world),
        "roofline": {"bound": bound, "kernel": dom_name, "achieved": achieved, "peak": peak, "unit": unit,
                     "frac": achieved / peak,
                     "peak_source": f"{peak_src} {'hbm_gbs' if bound == 'hbm' else 'bf16_tflops_sustained'}",
                     "traffic": ncu_traffic(w.name, dom_name),
                     "bytes_per_launch": dom_bytes, "flops_per_launch": dom_flops, "launch_ms": dom_launch_ms,
                     "hbm_frac": dom_bytes / (dom_launch_ms / 1e3) / 1e9 / hbm,
                     "tensor_frac": dom_flops / (dom_launch_ms / 1e3) / 1e12 / tensor},
        "roofline_step": {"algorithmic_bytes": alg["bytes"], "achieved_gbs": step_bytes_gbs,
                          "attn_flops": alg["attn_flops"], "hash_flops": alg["hash_flops"], **roof,
                          "peak_source": peak_src},
        "stages": per_stage,
        "stages_source": f"separate traced pass of {n_tr} steps (events around every stage); the timed steps "
                         f"record events around the dominant kernel ({dom_name}) only",
        "gpu_launches": int(launches),
        "memory": {"peak_device_bytes": peak_bytes, "workspace_bytes": ws_bytes,
                   "counts": "inputs, outputs, permutation and workspaces (torch allocator peak, "
                             "L2 flush buffer excluded)"},
        "e2e": e2e,
    }
    res["clocks"] = clk.summary()
    return res


# ------------------------------------------------------------------ oracle on the host cores
def oracle_slices(w: synth.Workload, n_slices: int, threads: int, L: int | None = None) -> float:
    """Runs the oracle forward (+ backward) on `n_slices` (batch, head) slices in
    parallel with `threads` OpenMP threads; returns wall seconds."""
    from oracle import oracle
    ws = w.replace(B=1, H=n_slices, L=L or w.L)
    inp = synth.make_inputs(ws)
    os.environ["OMP_NUM_THREADS"] = str(threads)
    t0 = time.perf_counter()
    res = oracle.fwd(inp["x"], inp["v"], inp["R"], ws.n_buckets, ws.chunk, ws.causal)
    if ws.backward:
        oracle.bwd(inp["x"], inp["v"], inp["dy"], res["perm"], ws.chunk, ws.causal)
    return time.perf_counter() - t0


def cpu_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


CPU_SAMPLE_S = 20.0      # target wall time of the CPU baseline's sample


def cpu_baseline(w: synth.Workload) -> dict:
    """The oracle on the host cores, one (batch, head) slice per OpenMP thread.
    A short probe (slices of min(L, 2048) tokens) sizes the sample: full-length
    slices when they finish in about CPU_SAMPLE_S seconds, else slices shortened
    (multiples of 128 tokens) to fit it -- the oracle's cost is linear in L, so
    the rate stands for the workload.  Tokens count sequence tokens as the
    metric does (a slice of Ls tokens of one head is Ls / H of them)."""
    cores = cpu_cores()
    n0 = max(1, min(cores, w.B * w.H * max(1, w.L // 4096)))
    Lp = min(w.L, 2048)
    tp = oracle_slices(w, n0, n0, Lp)
    est_full = tp * w.L / Lp                  # n0 full-length slices
    n, Ls = n0, w.L
    if Lp < w.L and est_full > CPU_SAMPLE_S:
        Ls = max(Lp, int(CPU_SAMPLE_S / tp * Lp) // 128 * 128)
    elif est_full * w.B * w.H / n0 <= CPU_SAMPLE_S:
        n = w.B * w.H                         # the whole workload fits the budget
    secs = tp if (n, Ls) == (n0, Lp) else oracle_slices(w, n, min(n, cores), Ls)
    value = n * Ls / w.H / secs
    return {"value": value, "unit": "tokens/s", "cores": min(n, cores), "kind": "oracle",
            "sample": f"{n} (batch, head) slices of {Ls} tokens (the workload: {w.B * w.H} x {w.L}) of {w.name}, "
                      f"fwd{'+bwd' if w.backward else ''}, {min(n, cores)} OpenMP threads; {secs:.1f} s wall"}


def run_reference(args, w: synth.Workload, world: int = 1) -> dict:
    """The oracle as it stands, timed on the host cores.  Each step is a bounded
    sample of the workload: min(cores, B*H) (batch, head) slices of
    min(L, 4096) tokens with the workload's buckets, rounds, chunk and mask, one
    slice per OpenMP thread (about a second of CPU work), so a --steps 200 run
    ends in a few minutes (the oracle's cost is linear in L).  ms_per_step is
    the measured time of one such sampled step; tokens/s counts sequence tokens
    as the metric does (a (batch, head) slice of Ls tokens is Ls / H of them)."""
    from oracle import oracle
    cores = cpu_cores() if args.ref_threads <= 0 else args.ref_threads
    n = max(1, min(cores, w.B * w.H))
    Ls = min(w.L, 4096)
    ws = w.replace(B=1, H=n, L=Ls)
    inp = synth.make_inputs(ws)
    os.environ["OMP_NUM_THREADS"] = str(n)

    def step() -> float:
        t0 = time.perf_counter()
        res = oracle.fwd(inp["x"], inp["v"], inp["R"], ws.n_buckets, ws.chunk, ws.causal)
        if ws.backward:
            oracle.bwd(inp["x"], inp["v"], inp["dy"], res["perm"], ws.chunk, ws.causal)
        return time.perf_counter() - t0

    for _ in range(args.warmup):
        step()
    times = [step() for _ in range(args.steps)]
    step_s = float(np.mean(times))
    seq_tokens = n * Ls / w.H                  # sequence tokens covered by one sampled step
    value = seq_tokens / step_s
    sample = (f"each step: {n} (batch, head) slices of {Ls} tokens (of {w.B * w.H} x {w.L} in {w.name}), "
              f"fwd{'+bwd' if w.backward else ''}, one slice per OpenMP thread = {seq_tokens:g} sequence tokens "
              f"in {step_s:.3f} s; ms_per_step is that sampled step")
    return {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": step_s * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic: seeded Philox4x32-10 + Box-Muller normals",
            "config": bench_config(w, world),
            "impl": "reference", "sampled": True,
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": n, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="long_64k", choices=sorted(synth.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--ref-threads", type=int, default=0,
                    help="--impl reference: OpenMP threads (0 = every host core the process may use)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    w = synth.WORKLOADS[args.workload]
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args, w, world)), flush=True)
        return
    res = run_ours(args, w, rank, world)
    if res is None:
        return
    if not args.no_cpu_baseline:
        res["cpu_baseline"] = cpu_baseline(w)
    print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
