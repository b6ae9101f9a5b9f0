#!/usr/bin/env python
"""MLA decode benchmark: us/call and KV GB/s of one decode step on B200.

A step is one pass of the whole hot path over one batch: the split-KV
schedule, the persistent decode kernel and the LSE combine, launched by one
mla_decode_fwd call through the C ABI (libmla_decode.so) with
MLA_FLAG_INLINE_PLAN (the decode kernel builds the schedule from the lengths
in its prologue; for the 128-column CTA-pair kernel the call enqueues the
schedule kernel first), captured once as a CUDA graph that every timed step
replays.  Default workload: batch 16, s_q 1,
16 heads, KV length 65536 (1.21 GB of latent cache per step, larger than L2,
so no flush is needed between steps).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
  python bench.py --impl reference ...   # the fp64 CPU oracle, timed on this host

With N > 1 (torchrun, one process per GPU) every rank decodes its own batch
(weak scaling: data-parallel over requests, no collective on the data path);
rank 0 prints one JSON line with the whole-job throughput.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from mla_decode_attention_15_b200 import _build, binding as bd, workloads  # noqa: E402

METRIC = "MLA decode µs/call & KV GB/s (bs16, 64K ctx, 16 heads) vs roofline"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
NOMINAL_HBM_GBS = 8000.0


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=workloads.HEADLINE, choices=list(workloads.WORKLOADS))
    ap.add_argument("--batch", type=int, default=0,
                    help="decode only the first BATCH requests of the workload (small profiling case)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cases", action="store_true",
                    help="leave out the per-workload cases (every named workload: timing and all-rows parity)")
    ap.add_argument("--gqa", action="store_true",
                    help="GQA path over a group-expanded cache (bs16, s_q 2 causal, 8 KV groups = 128 query "
                         "heads, 16K context): one JSON line")
    ap.add_argument("--absorb", action="store_true",
                    help="absorbed projections q_nope.W_UK and O.W_UV at decode sizes (bs16 x 16 heads, "
                         "bs32 x s_q 2 x 128 heads): one JSON line")
    ap.add_argument("--sweep", action="store_true",
                    help="context/batch sweep (bs x L grid, 16 heads, s_q 1): one JSON line per point "
                         "instead of the single bench line")
    return ap.parse_args()


# ---------------------------------------------------------------- accounting
def flush_l2(flush: torch.Tensor, i: int) -> None:
    """Untimed, before a timed replay: overwrite L2 with a buffer larger than
    it, then hold the GPU for ~50 us so that the host has enqueued the start
    event and the replay before the GPU reaches them; the timed interval then
    holds the replay's own execution and no host enqueue latency."""
    flush.fill_(i & 0xFF)
    torch.cuda._sleep(100_000)


def kv_tokens(seqlens: torch.Tensor) -> int:
    return int(seqlens.clamp(min=0).to(torch.int64).sum())


def algorithmic_bytes(seqlens, s_q, heads):
    """Minimum bytes of one decode call: every cached row once (576 bf16 =
    1152 B per token), Q once, O once (bf16), LSE once (fp32)."""
    B = int(seqlens.numel())
    kv = kv_tokens(seqlens) * 576 * 2
    q = B * s_q * heads * 576 * 2
    o = B * s_q * heads * 512 * 2
    lse = B * s_q * heads * 4
    return dict(kv=kv, q=q, o=o, lse=lse, total=kv + q + o + lse)


def algorithmic_flops(seqlens, s_q, heads):
    """2 * h * s_q * L * (576 + 512) per request (both contractions)."""
    return 2 * heads * s_q * kv_tokens(seqlens) * (576 + 512)


def kernel_roofline(byt, flops, kernel_ms, hbm_peak, tf_peak, peak_kind, traffic):
    """Roofline object of the decode kernel: whichever of HBM bytes / bandwidth
    and FLOPs / dense bf16 peak takes longer binds (both contractions are
    counted; 2*h*s_q*L*1088 FLOPs)."""
    t_hbm = byt["total"] / (hbm_peak * 1e9)
    t_tc = flops / (tf_peak * 1e12)
    sec = kernel_ms * 1e-3
    if t_hbm >= t_tc:
        achieved = byt["total"] / sec / 1e9
        return {"kernel": "mla_decode_fwd_kernel", "bound": "hbm", "achieved": achieved, "peak": hbm_peak,
                "unit": "GB/s", "frac": achieved / hbm_peak, "peak_kind": peak_kind + " (copy bandwidth, burst)",
                "traffic": traffic, "algorithmic_bytes_per_launch": byt["total"]}
    achieved = flops / sec / 1e12
    return {"kernel": "mla_decode_fwd_kernel", "bound": "tensor", "achieved": achieved, "peak": tf_peak,
            "unit": "TFLOP/s", "frac": achieved / tf_peak, "peak_kind": peak_kind + " (cuBLAS bf16 GEMM, burst)",
            "traffic": traffic, "algorithmic_flops_per_launch": flops,
            "algorithmic_bytes_per_launch": byt["total"]}


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(path))
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, "fallback"


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    for p in _build.sources():
        h.update(open(p, "rb").read())
    return h.hexdigest()[:16]


def ncu_traffic(workload: str, kv_bytes: int):
    """DRAM bytes per launch of the decode kernel from the committed ncu
    summary, if it was taken on the current kernel source; else None."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    try:
        d = json.load(open(path))
    except Exception:
        return None
    if d.get("kernel_source_hash") != kernel_source_hash():
        return None
    per_kv_byte = d.get("dram_bytes_per_kv_byte")
    if per_kv_byte is None:
        return None
    return int(per_kv_byte * kv_bytes)


# ---------------------------------------------------------------- clocks
REASON_BITS = {
    0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
    0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
    0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting",
}


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML every ~10 ms."""

    def __init__(self, device_index: int):
        self.samples = []
        self._stop = threading.Event()
        self._ok = False
        self.max_mhz = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self._ok = True
        except Exception:
            self._ok = False
        self._t = threading.Thread(target=self._run, daemon=True)

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM)
                try:
                    reasons = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                except Exception:
                    reasons = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self._h)
                self.samples.append((time.perf_counter(), mhz, int(reasons)))
            except Exception:
                pass
            time.sleep(0.01)

    def start(self):
        if self._ok:
            self._t.start()
        return self

    def stop(self):
        self._stop.set()
        if self._ok:
            self._t.join(timeout=1.0)

    def summary(self, t0: float, t1: float):
        if not self._ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0,
                    "note": "NVML unavailable"}
        win = [s for s in self.samples if t0 <= s[0] <= t1]
        window = "timed"
        if not win:
            win = self.samples
            window = "warmup+timed (timed region shorter than the sampling period)"
        reasons = set()
        for _, _, r in win:
            for bit, name in REASON_BITS.items():
                if r & bit and name != "gpu_idle":
                    reasons.add(name)
        return {"sm_mhz": statistics.median([s[1] for s in win]) if win else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(reasons), "samples": len(win),
                "window": window}


# ---------------------------------------------------------------- dist
def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", str(rank)))
    return world, rank, local


def rank_seed(base_seed: int, rank: int) -> int:
    """Rank 0 decodes exactly the named workload; rank r a fresh draw of it."""
    return base_seed + 7919 * rank


def aggregate_over_ranks(times_ms, kv_bytes: float, device) -> tuple:
    """Whole-job view of a weak-scaling run: every time is the slowest rank's
    (MAX over ranks), the KV bytes are summed over ranks.  Single process:
    returned unchanged."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return list(times_ms), float(kv_bytes)
    t = torch.tensor(list(times_ms), dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    b = torch.tensor([float(kv_bytes)], dtype=torch.float64, device=device)
    dist.all_reduce(b, op=dist.ReduceOp.SUM)
    return [float(x) for x in t.tolist()], float(b[0])


# ---------------------------------------------------------------- oracle arm
def oracle_sample_rate(d, w, budget_s: float, max_requests=None, collect=None):
    """Times the fp64 oracle on whole requests (all heads x s_q rows of each)
    until about budget_s of wall time; returns (GB/s of KV, seconds, sample text, cores).
    With ``collect`` (a list), appends (rows, out, lse) of every request done."""
    import oracle
    oracle.build()
    cores = oracle.max_threads()
    rows_per_req = w.s_q * w.heads
    B = w.batch if max_requests is None else min(w.batch, max_requests)
    done_bytes = 0
    elapsed = 0.0
    n_req = 0
    for b in range(B):
        rows = list(range(b * rows_per_req, (b + 1) * rows_per_req))
        t = time.perf_counter()
        res = oracle.mla_oracle_fwd(d["q"], d["kv_cache"], d["block_table"], d["cache_seqlens"],
                                    d["softmax_scale"], causal=d["causal"], rows=rows)
        elapsed += time.perf_counter() - t
        if collect is not None:
            collect.append((rows, res[0], res[1]))
        done_bytes += int(max(int(d["cache_seqlens"][b]), 0)) * 576 * 2
        n_req += 1
        if elapsed >= budget_s:
            break
    sample = "%d of %d requests (all %d heads x s_q %d rows each, %d KV tokens)" % (
        n_req, w.batch, w.heads, w.s_q, done_bytes // 1152)
    return done_bytes / elapsed / 1e9, elapsed, sample, cores


def parity_metrics(ref, ref_l, got, got_l):
    """max|err| relative to max|ref|, RMSE (with the bf16 rounding floor of
    the exact result), LSE relative error of ``got`` rows against the fp64
    oracle's ``ref`` rows."""
    import numpy as np
    err = got.astype(np.float64) - ref
    got_l = got_l.astype(np.float64)
    bf = torch.from_numpy(ref).to(torch.bfloat16).double().numpy()
    fin = np.isfinite(ref_l)
    return {"rows": int(ref.shape[0]), "oracle": "fp64",
            "max_abs_err_over_max_ref": float(np.abs(err).max() / max(np.abs(ref).max(), 1e-30)),
            "rmse": float(np.sqrt(np.mean(err ** 2))),
            "bf16_floor_rmse": float(np.sqrt(np.mean((bf - ref) ** 2))),
            "lse_rel_err": float((np.abs(got_l[fin] - ref_l[fin]) / np.maximum(1.0, np.abs(ref_l[fin]))).max())
            if fin.any() else 0.0,
            "lse_neginf_match": bool(np.array_equal(np.isneginf(got_l), np.isneginf(ref_l)))}


def bench_parity(done, out_rows, lse_rows):
    """Outputs of the timed launch configuration against the oracle rows the
    CPU baseline computed."""
    import numpy as np
    if not done:
        return None
    rows = np.concatenate([np.asarray(r) for r, _, _ in done])
    ref = np.concatenate([o for _, o, _ in done])
    ref_l = np.concatenate([l for _, _, l in done])
    return parity_metrics(ref, ref_l, out_rows[rows], lse_rows[rows])


def run_reference(args, w):
    world, rank, _ = dist_env()
    if rank != 0:
        return 0
    d = workloads.make_inputs(w)
    budget = max(0.5, 120.0 / max(1, args.steps + args.warmup))
    rates, times = [], []
    sample = ""
    cores = 0
    for i in range(args.warmup + args.steps):
        r, t, sample, cores = oracle_sample_rate(d, w, budget)
        if i >= args.warmup:
            rates.append(r)
            times.append(t)
    value = statistics.median(rates)
    kv = algorithmic_bytes(d["cache_seqlens"], w.s_q, w.heads)["kv"]
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1e3 * kv / (value * 1e9),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "impl": "reference",
        "config": workload_config(w, d, args.gpus),
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": cores, "kind": "oracle",
                         "sample": sample + "; ms_per_step extrapolates the sample rate to the whole batch"},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def workload_config(w, d, n_gpus):
    lens = d["cache_seqlens"]
    byt = algorithmic_bytes(lens, w.s_q, w.heads)
    return {
        "workload": "%s: %s" % (w.name, w.description),
        "batch": w.batch, "s_q": w.s_q, "heads": w.heads, "d_qk": 576, "d_v": 512,
        "kv_len": w.lens[1] if w.lens[0] == "fixed" else "U[%d,%d] (sum %d)" % (w.lens[1], w.lens[2], kv_tokens(lens)),
        "page_size": 64, "causal": w.causal, "softmax_scale": "192^-0.5",
        "kv_bytes_per_step": byt["kv"],
        "l2": "inputs larger than L2 (%.2f GB KV per step): no flush" % (byt["kv"] / 1e9)
              if byt["kv"] > 2 * 126e6 else "L2 flushed between steps (256 MB write and a 50 us GPU wait, untimed)",
        "plan": "built every step from cache_seqlens (MLA_FLAG_INLINE_PLAN)",
        "parallelism": "dp%d: independent request batches per GPU, no collective" % n_gpus,
    }


# ---------------------------------------------------------------- our arm
def run_ours(args, w):
    world, rank, local = dist_env()
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(dev)
    _build.build()
    bd.lib()

    seed = rank_seed(w.seed, rank)
    d = workloads.make_inputs(w, seed=seed)
    q = d["q"].to(dev)
    kv = d["kv_cache"].to(dev)
    bt = d["block_table"].to(dev)
    sl = d["cache_seqlens"].to(dev)
    B, s_q, h = w.batch, w.s_q, w.heads
    num_sms = torch.cuda.get_device_properties(dev).multi_processor_count
    # The step is one mla_decode_fwd call that builds its split-KV plan from
    # the lengths itself (MLA_FLAG_INLINE_PLAN); mla_decode_get_schedule runs
    # once, before the warm-up, to clear the new buffer's status word.
    dims = bd.make_dims(B, s_q, h, kv.shape[0], bt.shape[1], w.causal, num_sms, bd.MLA_FLAG_INLINE_PLAN)
    sched = torch.empty(bd.mla_decode_schedule_bytes(dims), dtype=torch.uint8, device=dev)
    ws = torch.empty(bd.mla_decode_workspace_bytes(dims), dtype=torch.uint8, device=dev)
    out = torch.empty(B, s_q, h, 512, dtype=torch.bfloat16, device=dev)
    lse = torch.empty(B, h, s_q, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    byt = algorithmic_bytes(d["cache_seqlens"], s_q, h)
    flops = algorithmic_flops(d["cache_seqlens"], s_q, h)
    flush = None
    if byt["kv"] <= 2 * 126e6:
        flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)

    # The decode kernel and the combine are launched as programmatic
    # dependents (PDL) of the kernel before them, so the timed loop records
    # no events between the kernels of a step.
    dims_nc = bd.make_dims(B, s_q, h, kv.shape[0], bt.shape[1], w.causal, num_sms,
                           bd.MLA_FLAG_NO_COMBINE | bd.MLA_FLAG_INLINE_PLAN)
    bd.mla_decode_get_schedule(dims, sl, sched, stream)

    def step():
        bd.mla_decode_fwd(dims, sched, ws, q, kv, bt, sl, d["softmax_scale"], out, lse, stream)

    def decode_only():
        bd.mla_decode_fwd(dims_nc, sched, ws, q, kv, bt, sl, d["softmax_scale"], out, lse, stream)

    # A step whose device status reports MLA_STATUS_TIMEOUT (a bounded wait
    # in the decode kernel ran out; its outputs are undefined) is not a
    # measurement.  On one GPU the warm-up and the timed region are each run
    # once more after one, and the line says so ("status_retries"); a second
    # one, or one on several ranks, ends the run.
    status_retries = []

    def retry_after_timeout(where, status):
        if world == 1 and status == bd.MLA_STATUS_TIMEOUT and not status_retries:
            status_retries.append({"where": where, "status": "%#x" % status})
            bd.mla_decode_get_schedule(dims, sl, sched, stream)  # clears the status word
            torch.cuda.synchronize()
            return True
        return False

    for attempt in range(2):
        for _ in range(args.warmup):
            if flush is not None:
                flush.fill_(1)
            step()
        torch.cuda.synchronize()
        status = bd.mla_decode_get_status(sched)
        if attempt == 0 and retry_after_timeout("warm-up", status):
            continue
        break
    assert status == 0, "device status after warm-up %#x" % status

    # One step (the decode kernel, which builds its plan from the lengths, and
    # the combine as its programmatic dependent) is captured as a CUDA graph
    # and replayed, as a serving loop would; likewise the decode kernel alone
    # for its roofline timing.
    g_step = torch.cuda.CUDAGraph()
    g_dec = torch.cuda.CUDAGraph()
    cap = torch.cuda.Stream(dev)
    cap.wait_stream(stream)
    with torch.cuda.stream(cap):
        with torch.cuda.graph(g_step, stream=cap):
            bd.mla_decode_fwd(dims, sched, ws, q, kv, bt, sl, d["softmax_scale"], out, lse, cap)
        with torch.cuda.graph(g_dec, stream=cap):
            bd.mla_decode_fwd(dims_nc, sched, ws, q, kv, bt, sl, d["softmax_scale"], out, lse, cap)
    stream.wait_stream(cap)
    for _ in range(max(3, args.warmup)):
        if flush is not None:
            flush.fill_(1)
        g_step.replay()
    torch.cuda.synchronize()

    for attempt in range(2):
        clocks = ClockSampler(dev.index if world == 1 else local).start()
        steps_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                    for _ in range(args.steps)]
        t_start = torch.cuda.Event(enable_timing=True)
        t_end = torch.cuda.Event(enable_timing=True)
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize()
        wall0 = time.perf_counter()
        t_start.record(stream)
        for i in range(args.steps):
            if flush is not None:
                flush_l2(flush, i)
                steps_ev[i][0].record(stream)
            g_step.replay()
            if flush is not None:
                steps_ev[i][1].record(stream)
        t_end.record(stream)
        torch.cuda.synchronize()
        if world > 1:
            torch.distributed.barrier()
        wall1 = time.perf_counter()
        clocks.stop()
        if flush is not None:
            ms_step = sum(a.elapsed_time(b) for a, b in steps_ev) / args.steps
        else:
            ms_step = t_start.elapsed_time(t_end) / args.steps

        # Decode kernel alone (same plan, combine left out), for the kernel's
        # roofline fraction.
        kern = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                for _ in range(args.steps)]
        for i in range(args.steps):
            if flush is not None:
                flush_l2(flush, i)
            kern[i][0].record(stream)
            g_dec.replay()
            kern[i][1].record(stream)
        torch.cuda.synchronize()
        kernel_ms = sum(a.elapsed_time(b) for a, b in kern) / args.steps
        status = bd.mla_decode_get_status(sched)
        if attempt == 0 and retry_after_timeout("timed region", status):
            continue
        break
    assert status == 0, "device status %#x" % status
    del g_step, g_dec
    # One more full step (outside the timed region): its outputs are checked
    # against the oracle rows that the CPU baseline computes.
    step()
    torch.cuda.synchronize()
    out_check = out.float().cpu().numpy().reshape(-1, 512)
    lse_check = lse.cpu().numpy().transpose(0, 2, 1).reshape(-1)  # rows (b*s_q+s)*h+head

    (ms_step, kernel_ms), total_kv = aggregate_over_ranks([ms_step, kernel_ms], byt["kv"], dev)

    # ---- end to end through the public API with host buffers ----
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(args, w, d, dims, kv, sched, ws, stream, dev, world)
    del q, kv, bt, sl, sched, ws, out, lse, flush
    torch.cuda.empty_cache()

    if rank != 0:
        if world > 1:
            torch.distributed.destroy_process_group()
        return 0

    hbm_peak, tf_peak, peak_kind = measured_peaks()
    traffic = ncu_traffic(w.name, byt["kv"])
    value = total_kv / (ms_step * 1e-3) / 1e9
    roof_us_meas = max(byt["total"] / (hbm_peak * 1e9), flops / (tf_peak * 1e12)) * 1e6
    roof_us_nom = max(byt["total"] / (NOMINAL_HBM_GBS * 1e9), flops / (tf_peak * 1e12)) * 1e6
    cpu = None
    parity = None
    if world == 1 and not args.no_cpu_baseline:
        done = []
        r, t, sample, cores = oracle_sample_rate(d, w, budget_s=15.0, collect=done)
        cpu = {"value": r, "unit": "GB/s", "cores": cores, "kind": "oracle",
               "sample": sample + " (%.1f s)" % t}
        parity = bench_parity(done, out_check, lse_check)
    cases = None
    if world == 1 and not args.no_cases:
        cases = run_cases(args, dev, w, d, hbm_peak, tf_peak)
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "us_per_call": ms_step * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic", "impl": "ours",
        "config": workload_config(w, d, world),
        "kernel_us": kernel_ms * 1e3,
        "tflops": flops / (ms_step * 1e-3) / 1e12,
        "roofline_us": {"at_measured_hbm": roof_us_meas, "at_8tbs": roof_us_nom},
        "frac_of_roofline_step": {"measured_hbm": roof_us_meas / (ms_step * 1e3),
                                  "at_8tbs": roof_us_nom / (ms_step * 1e3)},
        "roofline": kernel_roofline(byt, flops, kernel_ms, hbm_peak, tf_peak, peak_kind, traffic),
        "cpu_baseline": cpu,
        "parity": parity,
        "e2e": e2e,
        "clocks": clocks.summary(wall0, wall1),
        "gpu_launches": 2 * args.steps,
        "status_retries": status_retries,
        "cases": cases,
    }
    print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()
    return 0


def run_e2e(args, w, d, dims, kv, sched, ws, stream, dev, world):
    """Per step: pinned host q / block_table / seqlens -> device, decode
    (plan built in the kernel), combine, out / lse -> pinned host, stream
    synchronised (the caller
    reads the result).  The KV cache stays resident: it is the model's state,
    not a per-step input.  The inputs travel as one packed host->device copy
    and the outputs as one packed device->host copy (the API calls take views
    into the packed buffers); each step, copies included, is one CUDA-graph
    replay followed by a stream synchronisation."""
    B, s_q, h = w.batch, w.s_q, w.heads

    def layout(parts):
        offs, off = [], 0
        for nbytes in parts:
            offs.append(off)
            off += (nbytes + 255) // 256 * 256
        return offs, off

    q_bytes = d["q"].numel() * 2
    bt_bytes = d["block_table"].numel() * 4
    sl_bytes = d["cache_seqlens"].numel() * 4
    (o_q, o_bt, o_sl), in_bytes = layout([q_bytes, bt_bytes, sl_bytes])
    out_bytes = B * s_q * h * 512 * 2
    lse_bytes = B * h * s_q * 4
    (o_out, o_lse), res_bytes = layout([out_bytes, lse_bytes])
    in_h = torch.empty(in_bytes, dtype=torch.uint8).pin_memory()
    in_h[o_q:o_q + q_bytes].view(torch.bfloat16).copy_(d["q"].reshape(-1))
    in_h[o_bt:o_bt + bt_bytes].view(torch.int32).copy_(d["block_table"].reshape(-1))
    in_h[o_sl:o_sl + sl_bytes].view(torch.int32).copy_(d["cache_seqlens"].reshape(-1))
    res_h = torch.empty(res_bytes, dtype=torch.uint8).pin_memory()
    in_d = torch.empty(in_bytes, dtype=torch.uint8, device=dev)
    res_d = torch.empty(res_bytes, dtype=torch.uint8, device=dev)
    q = in_d[o_q:o_q + q_bytes].view(torch.bfloat16).view(d["q"].shape)
    bt = in_d[o_bt:o_bt + bt_bytes].view(torch.int32).view(d["block_table"].shape)
    sl = in_d[o_sl:o_sl + sl_bytes].view(torch.int32).view(d["cache_seqlens"].shape)
    out = res_d[o_out:o_out + out_bytes].view(torch.bfloat16).view(B, s_q, h, 512)
    lse = res_d[o_lse:o_lse + lse_bytes].view(torch.float32).view(B, h, s_q)

    def step(st):
        in_d.copy_(in_h, non_blocking=True)
        bd.mla_decode_fwd(dims, sched, ws, q, kv, bt, sl, d["softmax_scale"], out, lse, st)
        res_h.copy_(res_d, non_blocking=True)

    g = torch.cuda.CUDAGraph()
    cap = torch.cuda.Stream()
    cap.wait_stream(stream)
    with torch.cuda.stream(cap):
        step(cap)
        with torch.cuda.graph(g, stream=cap):
            step(cap)
    stream.wait_stream(cap)
    torch.cuda.synchronize()

    def one():
        g.replay()
        stream.synchronize()

    with torch.cuda.stream(stream):
        for _ in range(max(3, args.warmup)):
            one()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize()
        a.record(stream)
        for _ in range(args.steps):
            one()
        b.record(stream)
        torch.cuda.synchronize()
    ms = a.elapsed_time(b) / args.steps
    # the result read back is the one the kernels computed
    o_chk = res_h[o_out:o_out + out_bytes].view(torch.bfloat16)
    assert torch.isfinite(o_chk.float()).all()
    del g
    (ms,), kvb = aggregate_over_ranks([ms], algorithmic_bytes(d["cache_seqlens"], s_q, h)["kv"], dev)
    return {"value": kvb / (ms * 1e-3) / 1e9, "unit": "GB/s", "ms_per_step": ms,
            "h2d_bytes_per_step": in_bytes, "d2h_bytes_per_step": res_bytes,
            "note": "q, block_table, cache_seqlens uploaded (one packed copy) and out, lse read back (one packed "
                    "copy) every step, inside one CUDA-graph replay per step, then a stream sync; KV cache resident"}


def measure_case(w, d, dev, steps, warmup, hbm_peak, tf_peak):
    """One named workload on this GPU: the step (plan + decode + combine)
    and the decode kernel alone, each graph-replayed with CUDA events around
    every replay (L2 flushed before each replay, untimed, where the KV fits
    twice into L2); median and best per call.  Then one more step in bf16 and
    one with MLA_FLAG_FP32_OUT, both checked against the fp64 oracle on every
    row of the workload."""
    import numpy as np
    import oracle
    stream = torch.cuda.current_stream(dev)
    q = d["q"].to(dev)
    kv = d["kv_cache"].to(dev)
    bt = d["block_table"].to(dev)
    sl = d["cache_seqlens"].to(dev)
    B, s_q, h = w.batch, w.s_q, w.heads
    num_sms = torch.cuda.get_device_properties(dev).multi_processor_count
    mk = lambda flags=0: bd.make_dims(B, s_q, h, kv.shape[0], bt.shape[1], w.causal, num_sms,
                                      flags | bd.MLA_FLAG_INLINE_PLAN)
    dims, dims_nc, dims_f32 = mk(), mk(bd.MLA_FLAG_NO_COMBINE), mk(bd.MLA_FLAG_FP32_OUT)
    sched = torch.empty(bd.mla_decode_schedule_bytes(dims), dtype=torch.uint8, device=dev)
    ws = torch.empty(bd.mla_decode_workspace_bytes(dims), dtype=torch.uint8, device=dev)
    out = torch.empty(B, s_q, h, 512, dtype=torch.bfloat16, device=dev)
    out32 = torch.empty(B, s_q, h, 512, dtype=torch.float32, device=dev)
    lse = torch.empty(B, h, s_q, dtype=torch.float32, device=dev)
    byt = algorithmic_bytes(d["cache_seqlens"], s_q, h)
    flops = algorithmic_flops(d["cache_seqlens"], s_q, h)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev) if byt["kv"] <= 2 * 126e6 else None
    scale = d["softmax_scale"]

    graphs = []
    for dm in (dims, dims_nc):
        g = torch.cuda.CUDAGraph()
        cap = torch.cuda.Stream(dev)
        cap.wait_stream(stream)
        with torch.cuda.stream(cap):
            bd.mla_decode_get_schedule(dims, sl, sched, cap)  # clears the status word once
            bd.mla_decode_fwd(dm, sched, ws, q, kv, bt, sl, scale, out, lse, cap)
            with torch.cuda.graph(g, stream=cap):
                bd.mla_decode_fwd(dm, sched, ws, q, kv, bt, sl, scale, out, lse, cap)
        stream.wait_stream(cap)
        graphs.append(g)
    times = []
    for g in graphs:
        n_it = max(3, warmup) + steps
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n_it)]
        ev = []
        for i in range(n_it):
            a, b = evs[i]
            if flush is not None:
                flush_l2(flush, i)
            a.record(stream)
            g.replay()
            b.record(stream)
            if i >= max(3, warmup):
                ev.append((a, b))
        torch.cuda.synchronize()
        times.append(sorted(x.elapsed_time(y) for x, y in ev))
    del graphs
    status = bd.mla_decode_get_status(sched)
    (step_ms, kern_ms) = times
    med = lambda t: statistics.median(t)

    # parity, every row: the bf16 output and the fp32 output before the cast
    bd.mla_decode_fwd(dims, sched, ws, q, kv, bt, sl, scale, out, lse, stream)
    torch.cuda.synchronize()
    o16 = out.float().cpu().numpy().reshape(-1, 512)
    l16 = lse.cpu().numpy().transpose(0, 2, 1).reshape(-1)
    bd.mla_decode_fwd(dims_f32, sched, ws, q, kv, bt, sl, scale, out32, lse, stream)
    torch.cuda.synchronize()
    status |= bd.mla_decode_get_status(sched)
    o32 = out32.cpu().numpy().reshape(-1, 512)
    l32 = lse.cpu().numpy().transpose(0, 2, 1).reshape(-1)
    del q, kv, bt, sl, sched, ws, out, out32, lse, flush
    torch.cuda.empty_cache()
    t0 = time.perf_counter()
    ro, rl = oracle.mla_oracle_fwd(d["q"], d["kv_cache"], d["block_table"], d["cache_seqlens"], scale,
                                   causal=d["causal"])
    t_oracle = time.perf_counter() - t0
    par = parity_metrics(ro, rl, o16, l16)
    par["fp32_output"] = parity_metrics(ro, rl, o32, l32)
    par["note"] = ("every row; fp32_output is MLA_FLAG_FP32_OUT, the result before the bf16 cast, held to the "
                   "literal RMSE 5e-4")
    t_hbm = byt["total"] / (hbm_peak * 1e9)
    t_tc = flops / (tf_peak * 1e12)
    roof_s = max(t_hbm, t_tc)
    bound = "hbm" if t_hbm >= t_tc else "tensor"
    return {
        "workload": w.name, "description": w.description, "batch": B, "s_q": s_q, "heads": h,
        "kv_tokens": kv_tokens(d["cache_seqlens"]), "kv_bytes": byt["kv"], "algorithmic_bytes": byt["total"],
        "flops": flops,
        "us_per_call": {"median": 1e3 * med(step_ms), "best": 1e3 * step_ms[0]},
        "kernel_us": {"median": 1e3 * med(kern_ms), "best": 1e3 * kern_ms[0]},
        "kv_gbs": byt["kv"] / (med(step_ms) * 1e-3) / 1e9,
        "tflops": flops / (med(step_ms) * 1e-3) / 1e12,
        "roofline": {"bound": bound, "us": roof_s * 1e6,
                     "frac_step": roof_s / (med(step_ms) * 1e-3), "frac_kernel": roof_s / (med(kern_ms) * 1e-3),
                     "kernel_achieved": (byt["total"] / (med(kern_ms) * 1e-3) / 1e9) if bound == "hbm"
                     else flops / (med(kern_ms) * 1e-3) / 1e12,
                     "unit": "GB/s" if bound == "hbm" else "TFLOP/s",
                     "peak": hbm_peak if bound == "hbm" else tf_peak},
        "l2": "flushed before every replay (untimed)" if byt["kv"] <= 2 * 126e6 else "inputs larger than L2: no flush",
        "steps": steps, "parity": par, "oracle_s": t_oracle, "status": status,
    }


def run_cases(args, dev, main_w, main_d, hbm_peak, tf_peak):
    """Every named workload (the main one with the inputs already drawn)."""
    cases = []
    for name, w in workloads.WORKLOADS.items():
        d = main_d if name == main_w.name and main_w.batch == w.batch else workloads.make_inputs(w)
        cases.append(measure_case(w, d, dev, args.steps, args.warmup, hbm_peak, tf_peak))
        del d
    return cases


SWEEP_BATCH = (1, 4, 8, 16, 32)
SWEEP_LEN = (512, 1024, 2048, 4096, 8192, 16384, 32768, 65536, 131072)


def run_sweep(args):
    """Decode step and kernel time over a grid of batch x context length (16
    heads, s_q 1, permuted pages, N(0,1) inputs).  The page pool is drawn on
    the GPU; workloads whose KV fits in L2 are timed with an L2 flush between
    steps.  One JSON line per grid point."""
    dev = torch.device("cuda:0")
    torch.cuda.set_device(dev)
    bd.lib()
    stream = torch.cuda.current_stream(dev)
    hbm_peak, _, _ = measured_peaks()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    for B in SWEEP_BATCH:
        for L in SWEEP_LEN:
            d = workloads.build(B, 1, 16, ("fixed", L), seed=3000 + B, pool_device="cuda")
            q, kv = d["q"].to(dev), d["kv_cache"]
            bt, sl = d["block_table"].to(dev), d["cache_seqlens"].to(dev)
            dims = bd.make_dims(B, 1, 16, kv.shape[0], bt.shape[1], False, 0, bd.MLA_FLAG_INLINE_PLAN)
            dnc = bd.make_dims(B, 1, 16, kv.shape[0], bt.shape[1], False, 0,
                               bd.MLA_FLAG_NO_COMBINE | bd.MLA_FLAG_INLINE_PLAN)
            sched = torch.empty(bd.mla_decode_schedule_bytes(dims), dtype=torch.uint8, device=dev)
            ws = torch.empty(bd.mla_decode_workspace_bytes(dims), dtype=torch.uint8, device=dev)
            out = torch.empty(B, 1, 16, 512, dtype=torch.bfloat16, device=dev)
            lse = torch.empty(B, 16, 1, dtype=torch.float32, device=dev)
            byt = algorithmic_bytes(d["cache_seqlens"], 1, 16)
            use_flush = byt["total"] < (512 << 20)

            bd.mla_decode_get_schedule(dims, sl, sched, stream)  # clears the status word once

            def step(st, dm=dims):
                bd.mla_decode_fwd(dm, sched, ws, q, kv, bt, sl, d["softmax_scale"], out, lse, st)

            times = []
            for dm in (dims, dnc):
                g = torch.cuda.CUDAGraph()
                cap = torch.cuda.Stream()
                cap.wait_stream(stream)
                with torch.cuda.stream(cap):
                    step(cap, dm)
                    with torch.cuda.graph(g, stream=cap):
                        step(cap, dm)
                stream.wait_stream(cap)
                ts = []
                evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                       for _ in range(3 + args.steps)]
                for i in range(3 + args.steps):
                    a, b = evs[i]
                    if use_flush:
                        flush_l2(flush, i)
                    a.record(stream)
                    g.replay()
                    b.record(stream)
                    if i >= 3:
                        ts.append((a, b))
                torch.cuda.synchronize()
                times.append(sum(x.elapsed_time(y) for x, y in ts) / len(ts))
                del g
            status = bd.mla_decode_get_status(sched)
            ms_step, ms_kernel = times
            print(json.dumps({"sweep": "context x batch", "batch": B, "kv_len": L, "heads": 16, "s_q": 1,
                              "kv_bytes": byt["kv"], "us_per_call": ms_step * 1e3, "kernel_us": ms_kernel * 1e3,
                              "kv_gbs": byt["kv"] / (ms_step * 1e-3) / 1e9,
                              "kernel_frac_hbm": byt["total"] / (ms_kernel * 1e-3) / 1e9 / hbm_peak,
                              "l2_flush": use_flush, "status": status}), flush=True)
            del d, q, kv, bt, sl, sched, ws, out, lse
            torch.cuda.empty_cache()
    return 0


def run_gqa_bench(args):
    """The GQLA GQA path (group-expanded cache: per token 8 groups of 128-wide
    keys and values plus a 64-wide shared RoPE key) at bs16, s_q 2 causal,
    128 query heads, 16K context: step (decode with its plan built in the
    kernel, then the combine) and decode kernel alone, graph-replayed; bytes = every cache row once + Q + O
    + LSE, FLOPs = 2 * h_q * s_q * L * (192 + 128)."""
    dev = torch.device("cuda:0")
    torch.cuda.set_device(dev)
    bd.lib()
    stream = torch.cuda.current_stream(dev)
    B, s_q, groups, L = 16, 2, 8, 16384
    h = 16 * groups
    d = workloads.build_gqa(B, s_q, groups, ("fixed", L), seed=1005, causal=True, pool_device="cuda")
    q, kv = d["q"].to(dev), d["kv_cache"]
    bt, sl = d["block_table"].to(dev), d["cache_seqlens"].to(dev)
    dims = bd.make_gqa_dims(B, s_q, groups, kv.shape[0], bt.shape[1], True, 0, bd.MLA_FLAG_INLINE_PLAN)
    dnc = bd.make_gqa_dims(B, s_q, groups, kv.shape[0], bt.shape[1], True, 0,
                           bd.MLA_FLAG_NO_COMBINE | bd.MLA_FLAG_INLINE_PLAN)
    sched = torch.empty(bd.mla_gqa_decode_schedule_bytes(dims), dtype=torch.uint8, device=dev)
    ws = torch.empty(bd.mla_gqa_decode_workspace_bytes(dims), dtype=torch.uint8, device=dev)
    out = torch.empty(B, s_q, h, 128, dtype=torch.bfloat16, device=dev)
    lse = torch.empty(B, h, s_q, dtype=torch.float32, device=dev)
    tokens = kv_tokens(d["cache_seqlens"])
    kv_bytes = tokens * (2 * groups * 128 + 64) * 2
    total_bytes = kv_bytes + q.numel() * 2 + out.numel() * 2 + lse.numel() * 4
    flops = 2 * h * s_q * tokens * (192 + 128)

    bd.mla_gqa_decode_get_schedule(dims, sl, sched, stream)  # clears the status word once

    def step(st, dm):
        bd.mla_gqa_decode_fwd(dm, sched, ws, q, kv, bt, sl, d["softmax_scale"], out, lse, st)

    times = []
    for dm in (dims, dnc):
        g = torch.cuda.CUDAGraph()
        cap = torch.cuda.Stream()
        cap.wait_stream(stream)
        with torch.cuda.stream(cap):
            step(cap, dm)
            with torch.cuda.graph(g, stream=cap):
                step(cap, dm)
        stream.wait_stream(cap)
        for _ in range(max(3, args.warmup)):
            g.replay()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        a.record(stream)
        for _ in range(args.steps):
            g.replay()
        b.record(stream)
        torch.cuda.synchronize()
        times.append(a.elapsed_time(b) / args.steps)
        del g
    status = bd.mla_decode_get_status(sched)
    assert status == 0, "device status %#x" % status
    ms_step, ms_kernel = times
    hbm_peak, tf_peak, peak_kind = measured_peaks()
    line = {
        "metric": "GQA-path decode (group-expanded cache) KV GB/s", "value": kv_bytes / (ms_step * 1e-3) / 1e9,
        "unit": "GB/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "us_per_call": ms_step * 1e3, "higher_is_better": True, "dtype": "bf16", "data": "synthetic",
        "impl": "ours",
        "config": {"workload": "gqa_b16_sq2_g8_l16k: batch 16, s_q 2 causal, 8 KV groups x 16 query heads, "
                               "KV len 16384, d_head 128 + shared RoPE 64, permuted pages",
                   "kv_bytes_per_step": kv_bytes, "l2": "inputs larger than L2 (1.1 GB): no flush"},
        "kernel_us": ms_kernel * 1e3, "tflops": flops / (ms_step * 1e-3) / 1e12,
        "roofline": kernel_roofline({"total": total_bytes}, flops, ms_kernel, hbm_peak, tf_peak, peak_kind, None),
        "gpu_launches": 2 * args.steps,
    }
    print(json.dumps(line), flush=True)
    return 0


def run_composed(args, dev, stream):
    """One absorbed-MLA layer at the bs16 x 4K x 16-head decode batch (16
    tokens x 16 heads): mla_absorb_q -> mla_decode_fwd (inline plan, combine)
    -> mla_absorb_o, each a programmatic dependent of the kernel before it,
    against mla_decode_fwd alone on the same inputs.  Both graph-replayed
    with L2 flushed before each replay (the layer's 4 MB of weights then come
    from HBM, as they do when a model's layers run in turn); medians."""
    w = workloads.WORKLOADS["b16_l4096_h16"]
    d = workloads.make_inputs(w)
    q, kv = d["q"].to(dev), d["kv_cache"].to(dev)
    bt, sl = d["block_table"].to(dev), d["cache_seqlens"].to(dev)
    B, s_q, h = w.batch, w.s_q, w.heads
    x = workloads.build_absorb(B * s_q, h, seed=1400)
    q_in = x["q_in"].view(B, s_q, h, 192).to(dev)
    w_uk, w_uv = x["w_uk"].to(dev), x["w_uv"].to(dev)
    dims = bd.make_dims(B, s_q, h, kv.shape[0], bt.shape[1], w.causal, 0, bd.MLA_FLAG_INLINE_PLAN)
    sched = torch.empty(bd.mla_decode_schedule_bytes(dims), dtype=torch.uint8, device=dev)
    ws = torch.empty(bd.mla_decode_workspace_bytes(dims), dtype=torch.uint8, device=dev)
    out = torch.empty(B, s_q, h, 512, dtype=torch.bfloat16, device=dev)
    lse = torch.empty(B, h, s_q, dtype=torch.float32, device=dev)
    q_lat = torch.empty(B, s_q, h, 576, dtype=torch.bfloat16, device=dev)
    y = torch.empty(B, s_q, h, 128, dtype=torch.bfloat16, device=dev)
    status = torch.zeros(4, dtype=torch.int32, device=dev)
    adims = bd.make_absorb_dims(B * s_q, h)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    bd.mla_decode_get_schedule(dims, sl, sched, stream)

    def decode_only(st):
        bd.mla_decode_fwd(dims, sched, ws, q, kv, bt, sl, d["softmax_scale"], out, lse, st)

    def layer(st):
        bd.mla_absorb_q(adims, q_in, w_uk, q_lat, status, st)
        bd.mla_decode_fwd(dims, sched, ws, q_lat, kv, bt, sl, d["softmax_scale"], out, lse, st)
        bd.mla_absorb_o(adims, out, w_uv, y, status, st)

    res = {}
    for tag, fn in (("decode_us", decode_only), ("layer_us", layer)):
        g = torch.cuda.CUDAGraph()
        cap = torch.cuda.Stream(dev)
        cap.wait_stream(stream)
        with torch.cuda.stream(cap):
            fn(cap)
            with torch.cuda.graph(g, stream=cap):
                fn(cap)
        stream.wait_stream(cap)
        n = max(3, args.warmup) + args.steps
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
        for i in range(n):
            flush_l2(flush, i)
            evs[i][0].record(stream)
            g.replay()
            evs[i][1].record(stream)
        torch.cuda.synchronize()
        res[tag] = statistics.median(a.elapsed_time(b) * 1e3 for a, b in evs[max(3, args.warmup):])
        del g
    assert int(status.max()) == 0 and bd.mla_decode_get_status(sched) == 0
    res["projections_us"] = res["layer_us"] - res["decode_us"]
    res["config"] = ("b16_l4096_h16 decode with its 16 tokens x 16 heads projected: W_UK [16,128,512], "
                     "W_UV [16,512,128]; L2 flushed before each replay")
    return res


def run_absorb_bench(args):
    """The absorbed projections around the decode (GQLA summary, "Caminho
    MQA-Absorvido") at the decode batches of the two measured configurations.
    Each case holds the weights of 61 layers and calls layer i for call i, the
    way one decode step runs through a model, so the weights (4 or 32 MB per
    layer) come from HBM, not L2.  Graph-replayed; per-call time = replay time
    / 61.  Algorithmic bytes: weights + input rows + output rows, once."""
    dev = torch.device("cuda:0")
    torch.cuda.set_device(dev)
    bd.lib()
    stream = torch.cuda.current_stream(dev)
    hbm_peak, _, peak_kind = measured_peaks()
    layers = 61
    cases = []
    for name, T, h in (("b16_sq1_h16", 16, 16), ("b32_sq2_h128", 64, 128)):
        x = workloads.build_absorb(T, h, seed=1200 + h)
        q_in, o = x["q_in"].to(dev), x["o"].to(dev)
        g = torch.Generator(device=dev)
        g.manual_seed(1300 + h)
        w_uk = (torch.randn(layers, h, 128, 512, generator=g, device=dev) / 128 ** 0.5).to(torch.bfloat16)
        w_uv = (torch.randn(layers, h, 512, 128, generator=g, device=dev) / 512 ** 0.5).to(torch.bfloat16)
        q_out = torch.empty(T, h, 576, dtype=torch.bfloat16, device=dev)
        out = torch.empty(T, h, 128, dtype=torch.bfloat16, device=dev)
        status = torch.zeros(4, dtype=torch.int32, device=dev)
        dims = bd.make_absorb_dims(T, h)
        res = {}
        for kind in ("absorb_q", "absorb_o"):
            def calls(st, kind=kind):
                for i in range(layers):
                    if kind == "absorb_q":
                        bd.mla_absorb_q(dims, q_in, w_uk[i], q_out, status, st)
                    else:
                        bd.mla_absorb_o(dims, o, w_uv[i], out, status, st)
            graph = torch.cuda.CUDAGraph()
            cap = torch.cuda.Stream()
            cap.wait_stream(stream)
            with torch.cuda.stream(cap):
                calls(cap)
                with torch.cuda.graph(graph, stream=cap):
                    calls(cap)
            stream.wait_stream(cap)
            for _ in range(max(3, args.warmup)):
                graph.replay()
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            torch.cuda.synchronize()
            a.record(stream)
            for _ in range(args.steps):
                graph.replay()
            b.record(stream)
            torch.cuda.synchronize()
            us = a.elapsed_time(b) * 1e3 / (args.steps * layers)
            del graph
            w_bytes = h * 128 * 512 * 2
            io = T * h * (192 + 576) * 2 if kind == "absorb_q" else T * h * (512 + 128) * 2
            byt = w_bytes + io
            achieved = byt / (us * 1e-6) / 1e9
            res[kind] = {"us_per_call": us, "algorithmic_bytes": byt, "achieved_gbs": achieved,
                         "frac": achieved / hbm_peak, "tflops": 2 * T * h * 128 * 512 / (us * 1e-6) / 1e12}
        assert int(status.max()) == 0, "device status %#x" % int(status.max())
        cases.append({"case": name, "tokens": T, "heads": h, **res})
    traffic = None
    try:
        tj = json.load(open(os.path.join(ROOT, "profiles", "ncu_traffic_absorb.json")))
        if tj.get("kernel_source_hash") == kernel_source_hash():
            traffic = sum(tj[k]["dram_bytes_read"] + tj[k]["dram_bytes_write"] for k in ("absorb_q", "absorb_o"))
    except Exception:
        traffic = None
    main_case = cases[1]
    us = main_case["absorb_q"]["us_per_call"] + main_case["absorb_o"]["us_per_call"]
    byt = main_case["absorb_q"]["algorithmic_bytes"] + main_case["absorb_o"]["algorithmic_bytes"]
    line = {
        "metric": "absorbed projections (q_nope.W_UK + O.W_UV) GB/s", "value": byt / (us * 1e-6) / 1e9,
        "unit": "GB/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": us * 1e-3,
        "higher_is_better": True, "dtype": "bf16", "data": "synthetic", "impl": "ours",
        "config": {"workload": "absorb_b32_sq2_h128: 64 tokens x 128 heads, W_UK [128,128,512] + "
                               "W_UV [128,512,128] per layer, 61 layers in rotation",
                   "l2": "61 layers of weights (244 MB / 2 GB) rotate: no flush"},
        "roofline": {"kernel": "mla_absorb_kernel", "bound": "hbm", "achieved": byt / (us * 1e-6) / 1e9,
                     "peak": hbm_peak, "unit": "GB/s", "frac": byt / (us * 1e-6) / 1e9 / hbm_peak,
                     "peak_kind": peak_kind + " (copy bandwidth, burst)", "traffic": traffic,
                     "traffic_note": "DRAM bytes of one absorb_q + one absorb_o launch (ncu, 1 pass)"},
        "cases": cases, "gpu_launches": 2 * layers * args.steps,
        "composed_layer": run_composed(args, dev, stream),
    }
    print(json.dumps(line), flush=True)
    return 0


def main():
    args = parse_args()
    if args.absorb:
        return run_absorb_bench(args)
    if args.sweep:
        return run_sweep(args)
    if args.gqa:
        return run_gqa_bench(args)
    w = workloads.WORKLOADS[args.workload]
    if args.batch:
        import dataclasses
        w = dataclasses.replace(w, batch=args.batch,
                                description=w.description + "; first %d requests only" % args.batch)
    if args.impl == "reference":
        return run_reference(args, w)
    return run_ours(args, w)


if __name__ == "__main__":
    sys.exit(main())
