#!/usr/bin/env python
"""Benchmark of relative-bias GQA decode attention on B200.

One step = one layer-call of the whole hot path (split plan, partial kernel,
LSE-merge combine) over one batch of synthetic inputs already resident in
HBM.  Default workload: batch 1, 1 decode token, 48 query / 8 KV heads,
head dim 128, full attention over a 100,000-token paged bf16 cache (64-token
pages in random order), relative table NB = 1,280 (1,024 exact + 256 log
buckets to 2^20).  The L2 cache is flushed (a 2 x L2-size write) before every
timed step; only the attention kernels sit between the CUDA events.

Prints one JSON line (rank 0).  `value` is achieved HBM throughput in GB/s
(algorithmic bytes: every visible K/V row once, every needed relative-table
row once, q/out/lse), aggregated over all ranks; `us_per_call` is the mean
device time per layer-call.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
  python bench.py --impl reference ...   # the fp64 CPU oracle as the baseline arm
Under torchrun every rank runs its own replica of the workload (independent
problems, no collective on the data path): weak scaling.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = ("µs/layer and achieved HBM GB/s (% of roofline), "
          "48/8-head d128 decode @100K ctx")
DEFAULT_WORKLOAD = "full_100k"
FALLBACK_HBM_GBS = 6650.0
# the sources of the decode kernels and their launches (the KV producer's
# own file is left out: no traffic entry covers it)
KERNEL_SOURCES = ("relative_bias_gqa_b200/csrc/rel_attn_kernels.cuh",
                  "relative_bias_gqa_b200/csrc/rel_attn_fp8.cuh",
                  "relative_bias_gqa_b200/csrc/sm100_ptx.cuh",
                  "relative_bias_gqa_b200/csrc/rel_attn.cu")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "partial_kernel_traffic.json")


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--num-splits", type=int, default=0)
    ap.add_argument("--kv-dtype", choices=("bf16", "e4m3"), default="bf16",
                    help="KV-cache format: bf16, or E4M3 codes with per-KV-head scales")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    return ap.parse_args()


def partial_kernel_name(e4m3: bool, q_tokens: int) -> str:
    """The partial kernel a decode call launches: over an E4M3 cache, up to
    three tokens run the FP8 kernel (one-token chunks), four and more the
    multi-token kernel with the codes widened to bf16 in shared memory."""
    if e4m3 and q_tokens <= 3:
        return "rel_attn_partial_fp8_kernel"
    return "rel_attn_partial_kernel (E4M3 codes widened)" if e4m3 else "rel_attn_partial_kernel"


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


# ------------------------------------------------------------ bookkeeping
def algorithmic_bytes(case, bucket_fn, out_bytes=2, kv_elem_bytes=2):
    """Bytes the call must move: visible K/V rows once (kv_elem_bytes per
    element: 2 for bf16, 1 for E4M3 plus the per-head scales), the
    relative-table rows [0, bucket(max distance)] of every KV head once, q,
    out, lse, the block-table entries read and seq_lens."""
    lens = case.seq_lens.cpu().tolist()
    T, Hq, Hkv, D, P = (case.q_tokens, case.num_q_heads, case.num_kv_heads,
                        case.head_dim, case.page_size)
    W = case.window
    kv = 0
    pages = 0
    d_max = 0
    for L in lens:
        lo = max(0, L - T - W + 1) if W > 0 else 0
        kv += (L - lo) * Hkv * D * 2 * kv_elem_bytes
        pages += (L - 1) // P - lo // P + 1
        d_max = max(d_max, min(W - 1, L - 1) if W > 0 else L - 1)
    r_rows = bucket_fn(d_max) + 1
    rel = r_rows * Hkv * D * 2
    small = len(lens) * T * Hq * (D * 2 + D * out_bytes + 4) + pages * 4 + len(lens) * 4
    if kv_elem_bytes == 1:
        small += 2 * Hkv * 4                          # K and V scales
    return kv + rel + small, dict(kv=kv, rel=rel, other=small)


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during a region."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu_id, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.2)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons, samples = [], None, set(), 0
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 8:
                continue
            try:
                sm.append(float(f[0]))
                mx = float(f[1])
            except ValueError:
                continue
            samples += 1
            for n, v in zip(names, f[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        loaded = [x for x in sm if mx and x > 0.5 * mx] or sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": samples}


def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


def load_traffic(src_hash, workload):
    """DRAM bytes per partial-kernel launch from the committed ncu capture of
    this workload, or None when the kernels changed since it was taken."""
    try:
        with open(TRAFFIC_FILE) as f:
            t = json.load(f)
    except (OSError, ValueError):
        return None
    if t.get("kernel_source_hash") != src_hash:
        return None
    entry = t.get("workloads", {}).get(workload)
    return entry.get("dram_bytes_per_launch_full_size") if entry else None


# ------------------------------------------------------------- CPU oracle
def head0_subcase(case, kv=None):
    """Sequence 0, KV head 0 of the workload as a compact host problem: its
    G query heads, the pages it walks (renumbered 0..n-1), relative table 0.
    ``kv`` = (k_codes, v_codes, k_scale, v_scale) for an E4M3 cache."""
    G = case.num_q_heads // case.num_kv_heads
    L = int(case.seq_lens[0])
    n_pages = math.ceil(L / case.page_size)
    pages = case.block_table[0, :n_pages].long()
    sub = dict(q=case.q[:1, :, :G].cpu(), bt=torch_arange_row(n_pages),
               sl=case.seq_lens[:1].cpu(), rel=case.rel_table[:1].cpu())
    if kv is None:
        sub["k"] = case.k_cache[pages][:, :1].cpu()
        sub["v"] = case.v_cache[pages][:, :1].cpu()
    else:
        kc, vc, ks, vs = kv
        sub["k"] = kc[pages][:, :1].cpu()
        sub["v"] = vc[pages][:, :1].cpu()
        sub["ks"], sub["vs"] = ks[:1].cpu(), vs[:1].cpu()
    return sub


def oracle_head0(case, sub):
    """The fp64 oracle, as it stands, on the head-0 sub-problem."""
    import oracle
    if "ks" in sub:
        return oracle.rel_attn_decode_fp8kv_ref(sub["q"], sub["k"], sub["v"], sub["ks"], sub["vs"],
                                                sub["bt"], sub["sl"], sub["rel"], case.window)
    return oracle.rel_attn_decode_ref(sub["q"], sub["k"], sub["v"], sub["bt"], sub["sl"],
                                      sub["rel"], case.window)


def oracle_throughput(case, sub, seconds: float):
    """The oracle on KV head 0 of sequence 0 (its G query heads over the
    whole visible context), repeated for ~`seconds`; returns the baseline
    record and the last result (for the parity sample)."""
    L = int(case.seq_lens[0])
    W = case.window
    lo = max(0, L - case.q_tokens - W + 1) if W > 0 else 0
    elem = 1 if "ks" in sub else 2
    nbytes = (L - lo) * 128 * 2 * elem
    G = case.num_q_heads // case.num_kv_heads
    t0 = time.perf_counter()
    calls = 0
    while True:
        res = oracle_head0(case, sub)
        calls += 1
        el = time.perf_counter() - t0
        if el >= seconds:
            break
    cores = len(os.sched_getaffinity(0))
    return {"value": calls * nbytes / el / 1e9, "unit": "GB/s", "cores": cores,
            "kind": "oracle",
            "sample": (f"KV head 0 of sequence 0 of {case.name} ({G} query heads x "
                       f"{case.q_tokens} token(s), {L - lo} visible keys), {calls} calls in "
                       f"{el:.1f} s; numpy fp64 with up to {cores} BLAS threads"),
            "seconds": el}, res


def torch_arange_row(n):
    import torch
    return torch.arange(n, dtype=torch.int32)[None]


# ------------------------------------------------------- multi-rank timing
def max_over_ranks(ms: float, world: int, device) -> float:
    """The slowest rank's device time: every rank contributes its own total and
    all receive the maximum (the process group's backend: NCCL on GPUs, gloo
    in the CPU tests)."""
    if world <= 1:
        return ms
    import torch
    import torch.distributed as dist
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_gbs(world: int, steps: int, bytes_per_step: int, total_ms: float) -> float:
    """Aggregate throughput: every rank moves `bytes_per_step` per step (weak
    scaling, one independent decode problem per rank), over the slowest
    rank's time."""
    return world * steps * bytes_per_step / (total_ms * 1e-3) / 1e9


# ---------------------------------------------------------------- our arm
def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    from relative_bias_gqa_b200 import rel_attn, workloads

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    case = workloads.make_workload(args.workload, seed=args.seed + rank, device=dev)
    e4m3 = args.kv_dtype == "e4m3"
    kc = vc = ks = vs = None
    if e4m3:
        kc, vc, ks, vs = workloads.to_e4m3(case)
        kv_args = dict(k_cache=kc, v_cache=vc, scales=dict(k_scale=ks, v_scale=vs))
    else:
        kv_args = dict(k_cache=case.k_cache, v_cache=case.v_cache, scales={})
    prep = rel_attn.Prepared(case.q, kv_args["k_cache"], kv_args["v_cache"], case.block_table,
                             case.seq_lens, case.rel_table, case.window, args.num_splits,
                             max_seq_len=case.max_seq_len, out_fp32=False, **kv_args["scales"])
    S = prep.num_splits
    bucket = lambda d: rel_attn.rel_attn_bucket(prep.shape, d)
    nbytes, parts = algorithmic_bytes(case, bucket, kv_elem_bytes=1 if e4m3 else 2)
    props = torch.cuda.get_device_properties(dev)
    flush = torch.empty(2 * max(props.L2_cache_size, 64 << 20), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step():
        prep.partial()
        prep.combine()

    for _ in range(max(3, args.warmup)):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    if prep.workspace.read_status() != rel_attn.REL_ATTN_OK:
        raise RuntimeError("device status error during warm-up")

    K = args.steps
    # Timed region: K calls of the fused entry point (partial kernel + the
    # PDL-chained combine, one rel_attn_decode call each), CUDA events on the
    # launching stream around each call.
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
    sampler = ClockSampler("GPU-" + str(props.uuid)) if rank == 0 else None
    if sampler:
        sampler.start()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    # A short device-side sleep after the flush keeps the GPU busy while the
    # host submits the step, so the events bracket device execution only.
    sleep_cycles = 200_000
    for i in range(K):
        flush.zero_()
        torch.cuda._sleep(sleep_cycles)
        ev[i][0].record(stream)
        prep.decode()
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop() if sampler else None
    t_step = [e[0].elapsed_time(e[1]) for e in ev]
    total_ms = max_over_ranks(sum(t_step), world, dev)
    status = prep.workspace.read_status()

    # Per-kernel durations: the same step with an event between the partial
    # kernel and the combine (which then cannot overlap its launch with the
    # partial kernel's tail).
    Kp = min(K, 2000)
    evp = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(Kp)]
    for i in range(Kp):
        flush.zero_()
        torch.cuda._sleep(sleep_cycles)
        evp[i][0].record(stream)
        prep.partial()
        evp[i][1].record(stream)
        prep.combine()
        evp[i][2].record(stream)
    torch.cuda.synchronize()
    t_part = [e[0].elapsed_time(e[1]) for e in evp]
    t_comb = [e[1].elapsed_time(e[2]) for e in evp]

    # End to end: the step's inputs (q, block table, seq_lens) live in one
    # pinned host buffer and cross in one copy; out and lse come back in one
    # copy.  The device side holds the same packed layout, and the library
    # reads and writes those views directly.
    def packed(parts, dev_or_pin):
        offs, total = [], 0
        for t in parts:
            offs.append(total)
            total = (total + t.numel() * t.element_size() + 255) // 256 * 256
        buf = (torch.empty(total, dtype=torch.uint8, device=dev) if dev_or_pin == "dev"
               else torch.empty(total, dtype=torch.uint8).pin_memory())
        views = [buf[o:o + t.numel() * t.element_size()].view(t.dtype).view(t.shape)
                 for o, t in zip(offs, parts)]
        return buf, views
    in_parts = (case.q, case.block_table, case.seq_lens)
    d_in, (d_q, d_bt, d_sl) = packed(in_parts, "dev")
    h_in, (h_q, h_bt, h_sl) = packed(in_parts, "pin")
    h_q.copy_(case.q.cpu()); h_bt.copy_(case.block_table.cpu()); h_sl.copy_(case.seq_lens.cpu())
    out_parts = (prep.out, prep.lse)
    d_res, (d_out, d_lse) = packed(out_parts, "dev")
    h_res, _ = packed(out_parts, "pin")
    prep_e2e = rel_attn.Prepared(d_q, kv_args["k_cache"], kv_args["v_cache"], d_bt, d_sl,
                                 case.rel_table, case.window, S, out=d_out, lse=d_lse,
                                 max_seq_len=case.max_seq_len, out_fp32=False, **kv_args["scales"])
    Ke = min(K, 2000)
    eve = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(Ke)]
    for i in range(Ke):
        flush.zero_()
        eve[i][0].record(stream)
        d_in.copy_(h_in, non_blocking=True)
        prep_e2e.decode()
        h_res.copy_(d_res, non_blocking=True)
        eve[i][1].record(stream)
    torch.cuda.synchronize()
    t_e2e = [e[0].elapsed_time(e[1]) for e in eve]
    # Breakdown of the same step with the device held by a short sleep while
    # the host queues it (as in the main loop), events between the parts:
    # copy in, call, copy out; the rest of the end-to-end time is the device
    # waiting for the host to submit the next part.
    Kb = min(K, 500)
    evb = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(Kb)]
    for i in range(Kb):
        flush.zero_()
        torch.cuda._sleep(sleep_cycles)
        evb[i][0].record(stream)
        d_in.copy_(h_in, non_blocking=True)
        evb[i][1].record(stream)
        prep_e2e.decode()
        evb[i][2].record(stream)
        h_res.copy_(d_res, non_blocking=True)
        evb[i][3].record(stream)
    torch.cuda.synchronize()
    t_in = statistics.fmean(e[0].elapsed_time(e[1]) for e in evb) * 1e3
    t_call = statistics.fmean(e[1].elapsed_time(e[2]) for e in evb) * 1e3
    t_out = statistics.fmean(e[2].elapsed_time(e[3]) for e in evb) * 1e3
    # The same step with the result written by the kernels straight into a
    # pinned host buffer (mapped host memory: under unified addressing its
    # host address is valid on the device), instead of a device-to-host copy
    # after the call; taken only when the runtime confirms the mapping.
    h_zc, (h_out_zc, h_lse_zc) = packed(out_parts, "pin")
    try:
        try:
            from cuda.bindings import runtime as cudart
        except ImportError:
            from cuda import cudart
        err, dptr = cudart.cudaHostGetDevicePointer(h_zc.data_ptr(), 0)
        mapped = int(err) == 0 and int(dptr) == h_zc.data_ptr()
    except Exception:
        mapped = False
    t_zc = None
    if mapped:
        prep_zc = rel_attn.Prepared(d_q, kv_args["k_cache"], kv_args["v_cache"], d_bt, d_sl,
                                    case.rel_table, case.window, S, out=h_out_zc, lse=h_lse_zc,
                                    max_seq_len=case.max_seq_len, out_fp32=False, **kv_args["scales"])
        evz = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(Ke)]
        for i in range(Ke):
            flush.zero_()
            evz[i][0].record(stream)
            d_in.copy_(h_in, non_blocking=True)
            prep_zc.decode()
            evz[i][1].record(stream)
        torch.cuda.synchronize()
        t_zc = [e[0].elapsed_time(e[1]) for e in evz]
    prep.decode()
    torch.cuda.synchronize()
    if not (torch.equal(prep.out, d_out) and torch.equal(prep.lse, d_lse)):
        raise RuntimeError("packed end-to-end call disagrees with the resident-input call")
    if mapped and not (torch.equal(prep.out.cpu(), h_out_zc) and torch.equal(prep.lse.cpu(), h_lse_zc)):
        raise RuntimeError("zero-copy end-to-end call disagrees with the resident-input call")
    h2d = h_in.numel()
    d2h = h_res.numel()

    # Parity sample on the timed inputs: the same call with an fp32 output
    # (the tolerance's reference point) against the oracle's rows for KV head
    # 0 of sequence 0; outside every timed region.
    parity = None
    cpu = None
    if rank == 0:
        G = case.num_q_heads // case.num_kv_heads
        prep32 = rel_attn.Prepared(case.q, kv_args["k_cache"], kv_args["v_cache"], case.block_table,
                                   case.seq_lens, case.rel_table, case.window, S,
                                   max_seq_len=case.max_seq_len, out_fp32=True, **kv_args["scales"])
        o32, l32 = prep32.decode()
        torch.cuda.synchronize()
        sub = head0_subcase(case, (kc, vc, ks, vs) if e4m3 else None)
        if not args.no_cpu_baseline and world == 1:
            cpu, (ref_o, ref_l) = oracle_throughput(case, sub, args.cpu_seconds)
        else:
            ref_o, ref_l = oracle_head0(case, sub)
        import numpy as np
        eo = float(np.abs(o32[:1, :, :G].double().cpu().numpy() - ref_o).max())
        el = float(np.abs(l32[:1, :, :G].double().cpu().numpy() - ref_l).max())
        parity = {"max_abs_err_out_fp32": eo, "max_abs_err_lse": el,
                  "tolerance": {"out": 2e-3, "lse": 1e-3}, "pass": eo <= 2e-3 and el <= 1e-3,
                  "rows": f"sequence 0, KV head 0 ({G} query heads x {case.q_tokens} token(s)) "
                          f"of the timed inputs, against the fp64 oracle"}

    result = None
    if rank == 0:
        peak, peak_kind = measured_peak()
        mean_step = total_ms / K
        mean_part = statistics.fmean(t_part)
        # the dominant kernel: the partial kernel (the whole call when S = 1)
        kernel_ms = mean_step if S == 1 else mean_part
        achieved = nbytes / (kernel_ms * 1e-3) / 1e9
        value = whole_job_gbs(world, K, nbytes, total_ms)
        src_hash = kernel_source_hash()
        t_best = t_zc if (t_zc is not None and statistics.fmean(t_zc) < statistics.fmean(t_e2e)) else t_e2e
        e2e_gbs = world * nbytes / (statistics.fmean(t_best) * 1e-3) / 1e9
        result = {
            "metric": METRIC, "value": round(value, 1), "unit": "GB/s",
            "n_gpus": world, "steps": K, "warmup": args.warmup,
            "ms_per_step": round(mean_step, 6),
            "us_per_call": round(mean_step * 1e3, 2),
            "us_per_call_p10_p50_p90": [round(x * 1e3, 2) for x in
                                        statistics.quantiles(t_step, n=10)[0:9:4]],
            "us_partial_kernel": round(mean_part * 1e3, 2),
            "us_combine_kernel_after_event": round(statistics.fmean(t_comb) * 1e3, 2),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16" if not e4m3 else (
                "bf16 q, e4m3 kv (e4m3 tensor-core MMAs)" if case.q_tokens <= 3 else
                "bf16 q, e4m3 kv (widened to bf16 in shared memory, bf16 tensor-core MMAs)"),
            "data": "synthetic (seeded N(0,1) q/k/v, N(0,0.02) relative table)" +
                    ("; K/V quantised to E4M3 with per-KV-head amax/448 scales" if e4m3 else ""),
            "config": {"workload": args.workload, "kv_dtype": args.kv_dtype,
                       "batch": case.batch, "q_tokens": case.q_tokens,
                       "num_q_heads": case.num_q_heads, "num_kv_heads": case.num_kv_heads,
                       "head_dim": case.head_dim, "seq_lens_max": case.max_seq_len,
                       "window": case.window, "num_buckets": case.num_buckets,
                       "page_size": case.page_size, "num_splits": S,
                       "algorithmic_bytes_per_call": nbytes, "bytes_breakdown": parts,
                       "l2": "flushed before every timed step (2 x L2 write)",
                       "parallelism": f"replicas x{world}"},
            "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak,
                         "unit": "GB/s", "frac": round(achieved / peak, 4),
                         "peak_source": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)" if peak_kind == "measured"
                         else "fallback 6.65 TB/s",
                         "kernel": partial_kernel_name(e4m3, case.q_tokens),
                         "traffic": load_traffic(src_hash, args.workload + ("_e4m3" if e4m3 else "")),
                         "frac_of_8TBps_nominal": round(achieved / 8000.0, 4),
                         "frac_per_call": round(value / world / peak, 4),
                         "frac_per_call_of_8TBps_nominal": round(value / world / 8000.0, 4),
                         "note": "achieved/frac: the partial kernel alone; frac_per_call: the "
                                 "whole layer-call (partial + combine) per GPU"},
            "parity": parity,
            "e2e": {"value": round(e2e_gbs, 1), "unit": "GB/s",
                    "us_per_call": round(statistics.fmean(t_best) * 1e3, 2),
                    "result_to_host": "kernel stores into mapped pinned memory" if t_best is t_zc
                                      else "one device-to-host copy",
                    "us_per_call_copy_out": round(statistics.fmean(t_e2e) * 1e3, 2),
                    "us_per_call_zero_copy_out": (round(statistics.fmean(t_zc) * 1e3, 2)
                                                  if t_zc is not None else None),
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "breakdown_us": {"copy_in": round(t_in, 2), "call": round(t_call, 2),
                                     "copy_out": round(t_out, 2),
                                     "rest": round(statistics.fmean(t_e2e) * 1e3
                                                   - t_in - t_call - t_out, 2)},
                    "note": "q, block table and seq_lens copied in from one pinned host buffer "
                            "inside each timed step; out + lse reach pinned host memory either by "
                            "one copy after the call (us_per_call_copy_out) or written there by "
                            "the kernels themselves (mapped memory, us_per_call_zero_copy_out); "
                            "us_per_call is the faster. The KV cache and relative table are "
                            "resident model state. breakdown_us (copy-out form): the same step "
                            "queued ahead behind a device sleep, events between its parts (each "
                            "event pair adds about 2 us); rest = us_per_call_copy_out minus the "
                            "three parts"},
            "gpu_launches": K * (2 if S > 1 else 1),
            "timed_region": "K rel_attn_decode calls (partial kernel + PDL-chained combine kernel); "
                            "us_partial_kernel from a second loop with an event between the kernels",
            "clocks": clocks,
            "device_status": rel_attn.error_string(status),
            "kernel_source_hash": src_hash,
            "library": rel_attn.version(),
        }
        if cpu is not None:
            result["cpu_baseline"] = cpu
    return result


# ------------------------------------------- producer and prefill rows
def _timed_loop(fn, K, flush, stream, sleep_cycles=200_000):
    import torch
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
    for i in range(K):
        flush.zero_()
        torch.cuda._sleep(sleep_cycles)
        ev[i][0].record(stream)
        fn()
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    return [e[0].elapsed_time(e[1]) for e in ev]


def run_side_row(args, rank, world, local_rank):
    """The KV-cache producer step (kv_write_8k: an 8,192-token prefill chunk;
    kv_write_decode: one token at 100K) and the chunked prefill (prefill_8k:
    8,192 query tokens over an 8,192-token context), 48 query / 8 KV heads,
    inputs resident in HBM, L2 flushed before every step."""
    import math
    import torch
    import numpy as np
    from relative_bias_gqa_b200 import rel_attn, workloads
    import oracle
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    props = torch.cuda.get_device_properties(dev)
    flush = torch.empty(2 * max(props.L2_cache_size, 64 << 20), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    g = torch.Generator(device=dev).manual_seed(args.seed + rank)
    K = args.steps
    peak, peak_kind = measured_peak()
    sampler = ClockSampler("GPU-" + str(props.uuid)) if rank == 0 else None
    e4m3 = args.kv_dtype == "e4m3"
    if args.workload.startswith("kv_write"):
        T, L = (8192, 8192) if args.workload == "kv_write_8k" else (1, 100_000)
        Hkv, P, D = 8, 64, 128
        pages = math.ceil(L / P)
        bt = torch.randperm(pages, generator=torch.Generator().manual_seed(args.seed + 1)).int()[None].to(dev)
        bf = lambda *sh, std=1.0: (torch.randn(*sh, generator=g, device=dev) * std).to(torch.bfloat16)
        c = dict(k_new=bf(1, T, Hkv, D), v_new=bf(1, T, Hkv, D), conv_w=bf(2, Hkv, D, 4, std=0.5),
                 k_raw=bf(pages, Hkv, P, D), v_raw=bf(pages, Hkv, P, D),
                 block_table=bt, seq_lens=torch.tensor([L], dtype=torch.int32, device=dev))
        if e4m3:
            c["k_cache"] = torch.zeros(pages, Hkv, P, D, dtype=torch.uint8, device=dev)
            c["v_cache"] = torch.zeros(pages, Hkv, P, D, dtype=torch.uint8, device=dev)
            c["k_scale"] = torch.full((Hkv,), 0.01, device=dev)
            c["v_scale"] = torch.full((Hkv,), 0.01, device=dev)
        else:
            c["k_cache"] = bf(pages, Hkv, P, D)
            c["v_cache"] = bf(pages, Hkv, P, D)
        # per new token and KV head: K and V in (512 B), raw K/V out (512 B),
        # cache out (512 B bf16 / 256 B E4M3); three older raw vectors once
        nbytes = T * Hkv * (512 + 512 + (256 if e4m3 else 512)) + min(3, L - T) * Hkv * 512 + \
            2 * Hkv * D * 4 * 2 + 8
        fn = lambda: rel_attn.rel_attn_kv_write(**c, stream=stream)
        for _ in range(max(3, args.warmup)):
            fn()
        torch.cuda.synchronize()
        # parity sample: a copy of the inputs, one step, against the oracle
        c2 = {k: v.clone() for k, v in c.items()}
        want = oracle.kv_write_ref(**c2)
        rel_attn.rel_attn_kv_write(**c2)
        torch.cuda.synchronize()
        exact = all(np.array_equal(c2[n].cpu().numpy() if c2[n].dtype == torch.uint8
                                   else c2[n].float().cpu().numpy(), w)
                    for n, w in zip(("k_raw", "v_raw", "k_cache", "v_cache"), want))
        if sampler:
            sampler.start()
        t = _timed_loop(fn, K, flush, stream)
        clocks = sampler.stop() if sampler else None
        ms = statistics.fmean(t)
        gbs = nbytes / (ms * 1e-3) / 1e9
        return {"metric": f"KV-cache producer step ({'8,192-token prefill chunk' if T > 1 else 'one decode token at 100K'}): "
                          "short conv + paged write" + (" + E4M3 quantisation" if e4m3 else ""),
                "value": round(gbs, 1), "unit": "GB/s", "n_gpus": world, "steps": K,
                "warmup": args.warmup, "ms_per_step": round(ms, 6), "us_per_call": round(ms * 1e3, 2),
                "us_per_call_p10_p50_p90": [round(x * 1e3, 2) for x in statistics.quantiles(t, n=10)[0:9:4]],
                "higher_is_better": True, "dtype": "bf16 in, fp32 taps, " + ("e4m3" if e4m3 else "bf16") + " out",
                "data": "synthetic", "config": {"workload": args.workload, "new_tokens": T, "seq_len": L,
                                                "num_kv_heads": Hkv, "algorithmic_bytes_per_call": nbytes,
                                                "l2": "flushed before every timed step"},
                "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": peak, "unit": "GB/s",
                             "frac": round(gbs / peak, 4), "peak_source": peak_kind,
                             "kernel": "rel_attn_kv_write_kernel"},
                "parity": {"bit_exact_vs_oracle": exact}, "clocks": clocks,
                "gpu_launches": K, "library": rel_attn.version()}
    # prefill_8k
    C = L = 8192
    case = workloads.make_case(seq_lens=[L], q_tokens=C, num_q_heads=48, num_kv_heads=8, window=0,
                               num_buckets=1280, seed=args.seed + rank, device=dev, name="prefill_8k")
    shape = rel_attn.shape_of(case.q, case.k_cache, case.block_table, case.rel_table, max_seq_len=L)
    ws = rel_attn.Workspace(rel_attn.prefill_workspace_bytes(shape, max(1, args.num_splits)), dev)
    out = torch.empty_like(case.q)
    lse = torch.empty(case.q.shape[:3], dtype=torch.float32, device=dev)
    fn = lambda: rel_attn.rel_attn_prefill(case.q, case.k_cache, case.v_cache, case.block_table,
                                           case.seq_lens, case.rel_table, 0, args.num_splits,
                                           out=out, lse=lse, workspace=ws, max_seq_len=L)
    for _ in range(max(3, args.warmup)):
        fn()
    torch.cuda.synchronize()
    # useful FLOPs: q.k and p.v over every visible key of every query row
    keys = C * (C + 1) // 2
    flops = 4 * 48 * 128 * keys
    if sampler:
        sampler.start()
    t = _timed_loop(fn, K, flush, stream)
    clocks = sampler.stop() if sampler else None
    ms = statistics.fmean(t)
    tflops = flops / (ms * 1e-3) / 1e12
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            tpeak, tkind = float(json.load(f)["bf16_tflops"]), "measured"
    except (OSError, KeyError, ValueError):
        tpeak, tkind = 1590.0, "fallback"
    # parity sample: KV head 0's query rows of the last 64 tokens against the oracle
    sub = dict(q=case.q[:, -64:, :6].cpu(), k=case.k_cache[:, :1].cpu(), v=case.v_cache[:, :1].cpu())
    ref_o, ref_l = oracle.rel_attn_decode_ref(sub["q"], sub["k"], sub["v"], case.block_table.cpu(),
                                              case.seq_lens.cpu(), case.rel_table[:1].cpu(), 0)
    o32 = torch.empty(case.q.shape, dtype=torch.float32, device=dev)
    rel_attn.rel_attn_prefill(case.q, case.k_cache, case.v_cache, case.block_table, case.seq_lens,
                              case.rel_table, 0, args.num_splits, out=o32, lse=lse, workspace=ws,
                              max_seq_len=L, out_fp32=True)
    torch.cuda.synchronize()
    eo = float(np.abs(o32[:, -64:, :6].double().cpu().numpy() - ref_o).max())
    el = float(np.abs(lse[:, -64:, :6].double().cpu().numpy() - ref_l).max())
    return {"metric": "chunked prefill attention, 8,192 query tokens over an 8,192-token context, 48/8 heads",
            "value": round(tflops, 2), "unit": "TFLOP/s", "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": round(ms, 4), "us_per_call": round(ms * 1e3, 1),
            "higher_is_better": True, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": "prefill_8k", "query_tokens": C, "seq_len": L, "num_q_heads": 48,
                       "num_kv_heads": 8, "useful_flops_per_call": flops,
                       "l2": "flushed before every timed step"},
            "roofline": {"bound": "tensor", "achieved": round(tflops, 2), "peak": tpeak, "unit": "TFLOP/s",
                         "frac": round(tflops / tpeak, 4), "peak_source": tkind,
                         "kernel": "rel_attn_partial_kernel (8-token chunks)"},
            "parity": {"max_abs_err_out_fp32": eo, "max_abs_err_lse": el,
                       "rows": "KV head 0, last 64 query tokens"},
            "clocks": clocks, "gpu_launches": K, "library": rel_attn.version()}


# ----------------------------------------------------------- reference arm
def run_reference(args, rank, world):
    """The fp64 CPU oracle timed on this host's cores, as the baseline arm."""
    if rank != 0:
        return None
    import torch
    from relative_bias_gqa_b200 import workloads
    import oracle
    case = workloads.make_workload(args.workload, seed=args.seed, device="cpu")
    G = case.num_q_heads // case.num_kv_heads
    L = int(case.seq_lens[0])
    W = case.window
    budget = 150.0 / max(1, args.steps + args.warmup)        # seconds per step
    # a bounded sample: KV head 0, the last n visible keys of sequence 0,
    # at their true positions (so the log buckets are exercised)
    lo = max(0, L - case.q_tokens - W + 1) if W > 0 else 0
    P = case.page_size
    first = lo // P
    n_pages_all = (L - 1) // P - first + 1
    pages = case.block_table[0, first:first + n_pages_all].long()
    k_all = case.k_cache[pages][:, :1].float().numpy()
    v_all = case.v_cache[pages][:, :1].float().numpy()
    q = case.q[0, :, :G].float().numpy()
    rel = case.rel_table[0].float().numpy()
    key_pos_all = __import__("numpy").arange(first * P, first * P + n_pages_all * P)
    keep = (key_pos_all >= lo) & (key_pos_all < L)
    keys = k_all.reshape(-1, 128)[keep]
    vals = v_all.reshape(-1, 128)[keep]
    key_pos = key_pos_all[keep]
    q_pos = L - case.q_tokens + __import__("numpy").arange(case.q_tokens)

    def one(n):
        oracle.attend_at_positions(q, q_pos, keys[-n:], vals[-n:], key_pos[-n:], rel, W,
                                   case.num_buckets)

    n = min(len(keys), 4096)
    t0 = time.perf_counter()
    one(n)
    dt = time.perf_counter() - t0
    n = int(min(len(keys), max(1024, n * budget / max(dt, 1e-6))))   # never past the visible keys
    for _ in range(args.warmup):
        one(n)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        one(n)
    el = time.perf_counter() - t0
    nbytes = n * 128 * 2 * 2
    value = args.steps * nbytes / el / 1e9
    cores = len(os.sched_getaffinity(0))
    sample = (f"KV head 0 of {args.workload}: the last {n} visible keys at their true positions, "
              f"{case.q_tokens} token(s) x {G} query heads per step (fp64 numpy oracle)")
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(el / args.steps * 1e3, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": args.workload, "sample": sample},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": cores,
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main():
    args = parse_args()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        res = run_reference(args, rank, world)
        if res is not None:
            print(json.dumps(res), flush=True)
        return
    dist_init = False
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
        dist_init = True
    try:
        if args.workload in ("kv_write_8k", "kv_write_decode", "prefill_8k"):
            res = run_side_row(args, rank, world, local_rank) if rank == 0 else None
        else:
            res = run_ours(args, rank, world, local_rank)
        if res is not None:
            print(json.dumps(res), flush=True)
    finally:
        if dist_init:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
