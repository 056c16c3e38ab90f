"""QSA hot-path benchmark (one JSON line on rank 0).

Headline: QSA prefill tokens/s at a 128K context (batch 1, T=131072, 16 q
heads / 2 KV heads, d=128, 64-token blocks, top-32), one step = compress
the new key blocks -> pool/score/select -> sparse attention, with inputs
resident in HBM.  Also reported: decode microseconds per token at 128K
(32 sequences x 131072-token caches, top-64 per token; one step =
per-token selection + split-K attention; the cache summaries are the
persistent state and are built before timing).

Timing: W untimed warm-up steps, then exactly K steps between a barrier
and a device synchronise on both sides; each step is bracketed by CUDA
events on the launching stream and an L2 flush runs between steps outside
the events (a 256 MiB write, then a 256 MiB read, so every step starts
with a cold L2 that holds none of the flush's dirty lines).  The decode
step (selection + attention) is captured once as a CUDA graph and
replayed, as a serving loop would run it, so host launch gaps stay out of
its device time.  Multi-GPU: one process per GPU, each
rank runs its own sequence (weak scaling, no data-path collective); the
time is the max over ranks.

--impl reference times the fp64 CPU oracle (the path's reference
implementation here) on a bounded sample of the same workload.
"""
import argparse
import json
import math
import os
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synthetic  # noqa: E402

PREFILL = "prefill_128k"
DECODE = "decode_128k"
METRIC = "QSA prefill tokens/s and decode us/token at 128K ctx; % of TC / HBM roofline"
UNIT = "tokens/s"


# ------------------------------------------------------------ utilities

class L2Flush:
    """L2 eviction between timed steps: a 256 MiB write, then a 256 MiB read
    of another buffer, so a step starts with a cold L2 that holds none of the
    flush's dirty lines (whose write-back would otherwise land on the step)."""
    DESCRIPTION = ("flushed between steps (256 MiB write, then 256 MiB read: cold, no dirty "
                   "lines); inputs also exceed L2")

    def __init__(self, dev):
        self.w = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
        self.r = torch.zeros(64 << 20, dtype=torch.int32, device=dev)

    def __call__(self, k):
        self.w.fill_(k & 0xFF)
        torch.sum(self.r)

def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        p = json.load(open(path))
        return {"hbm_gbs": p["hbm_gbs"], "bf16_tflops": p["bf16_tflops"],
                "bf16_tflops_sustained": p.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


class ClockSampler:
    """SM clocks and throttle reasons sampled during the timed region: NVML
    read every few milliseconds from a thread (read-only queries), else
    nvidia-smi at its shortest interval.  Entering waits for the first sample,
    so that even a short timed region is covered."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def __init__(self, gpu_index, period_s=0.002):
        self.gpu = gpu_index
        self.period = period_s
        self.proc = None
        self.nvml = None
        self.samples = []          # (sm_mhz, max_mhz, set of reasons)
        self.stop = threading.Event()

    def _nvml_loop(self):
        nv, h = self.nvml
        bits = {"hw_slowdown": nv.nvmlClocksEventReasonHwSlowdown,
                "hw_thermal_slowdown": nv.nvmlClocksEventReasonHwThermalSlowdown,
                "sw_thermal_slowdown": nv.nvmlClocksEventReasonSwThermalSlowdown,
                "sw_power_cap": nv.nvmlClocksEventReasonSwPowerCap}
        mx = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
        while not self.stop.is_set():
            try:
                sm = float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                self.samples.append((sm, mx, {n for n, bit in bits.items() if r & bit}))
            except Exception:
                break
            time.sleep(self.period)

    def _smi_read(self):
        for line in self.proc.stdout:
            f = [x.strip() for x in line.strip().split(",")]
            if len(f) < 9:
                continue
            try:
                sm, mx = float(f[1]), float(f[2])
            except ValueError:
                continue
            self.samples.append((sm, mx, {n for n, v in zip(self.NAMES, f[5:9]) if v.lower() == "active"}))

    def __enter__(self):
        try:
            import pynvml as nv
            nv.nvmlInit()
            self.nvml = (nv, nv.nvmlDeviceGetHandleByIndex(self.gpu))
            self.t = threading.Thread(target=self._nvml_loop, daemon=True)
            self.t.start()
        except Exception:
            self.nvml = None
            try:
                self.proc = subprocess.Popen(
                    ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                     "--format=csv,noheader,nounits", "-lms", "100"],
                    stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
                self.t = threading.Thread(target=self._smi_read, daemon=True)
                self.t.start()
            except (OSError, FileNotFoundError):
                self.proc = None
        t0 = time.time()
        while (self.nvml or self.proc) and not self.samples and time.time() - t0 < 3.0:
            time.sleep(0.005)
        self.first = len(self.samples)
        return self

    def __exit__(self, *a):
        self.stop.set()
        if self.nvml is not None:
            self.t.join(timeout=1.0)
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        # the samples taken once the timed region was under way (the last
        # one before it, if the region was shorter than the interval)
        s = self.samples[max(self.first - 1, 0):] if self.samples else []
        if not s:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        reasons = set().union(*(x[2] for x in s))
        return {"sm_mhz": float(np.median([x[0] for x in s])), "sm_max_mhz": float(max(x[1] for x in s)),
                "reasons": sorted(reasons), "samples": len(s),
                "source": "nvml" if self.nvml is not None else "nvidia-smi"}


def job_throughput(ms_local, units_local, device):
    """Whole-job throughput over all ranks: sum of the ranks' units divided
    by the slowest rank's step time.  Returns (units/s, max ms)."""
    t = torch.tensor([ms_local, float(units_local)], dtype=torch.float64, device=device)
    if torch.distributed.is_available() and torch.distributed.is_initialized():
        ws = torch.distributed.get_world_size()
        mx = t[:1].clone()
        torch.distributed.all_reduce(mx, op=torch.distributed.ReduceOp.MAX)
        tot = t[1:].clone()
        torch.distributed.all_reduce(tot, op=torch.distributed.ReduceOp.SUM)
        ms_max, units = float(mx.item()), float(tot.item())
    else:
        ms_max, units = ms_local, float(units_local)
    return units / (ms_max * 1e-3), ms_max


def prefill_flops(w):
    """Algorithmic FLOPs of the sparse attention: 4*d*Hq per unmasked
    (query, key) pair inside the selected blocks (masked half of the
    diagonal block excluded)."""
    pairs = 0
    for i in range(w.n_rows):
        t0, t1 = i * 64, min((i + 1) * 64, w.Tq)
        D = (w.q_pos0 + t1 - 1) // 64
        nsel = min(w.topk, D + 1)
        full = nsel - 1                      # fully visible non-diagonal blocks
        for t in range(t0, t1):
            p = w.q_pos0 + t
            pairs += 64 * full + (p - 64 * D + 1)
    return 4.0 * w.d * w.Hq * pairs * w.B


def decode_bytes(w):
    """Selected K+V bytes per decode step (all sequences)."""
    D = (w.q_pos0) // 64
    nsel = min(w.topk, D + 1)
    keys = 64 * (nsel - 1) + (w.q_pos0 - 64 * D + 1)
    return 2 * 2 * w.d * w.Hkv * keys * w.B


# ------------------------------------------------------------- our arm
def bench_prefill(args, qsa, dev, wname, ws, rank, flush, keep=False, clocks=False):
    """One prefill workload: W untimed warm-up steps, then exactly K steps
    (compress of the step's new key blocks -> pool/score/select ->
    attention), each bracketed by CUDA events on the launching stream, the L2
    flushed between steps.  Returns a dict with the workload, the per-part
    times, the launches in the timed region, the clock record (when asked)
    and, with keep, host copies of the inputs and outputs for the oracle's
    parity check (taken after the timed region)."""
    wp = synthetic.CONFIGS[wname]
    if ws > 1:
        wp = synthetic.Workload(**{**wp.__dict__, "seed": wp.seed + 1000 * rank})
    x = synthetic.generate(wp, dev)
    Q, K, V = x["Q"], x["K"], x["V"]
    run = qsa.QSAPrefill(wp.B, wp.Tq, wp.Hq, wp.Hkv, wp.d, wp.T_kv, wp.topk, wp.q_pos0, device=dev)
    run.precompress_cache(K)           # the cache's summaries: persistent state (untimed)
    stream = torch.cuda.current_stream()

    def step(ev=None):
        if ev is None:
            return run(Q, K, V)
        ev[0].record(stream)
        qsa.compress_keys(K, run.Kc, run.blk_begin, run.blk_end)
        ev[1].record(stream)
        qsa.score_select(Q, run.Kc, run.idx, run.topk, run.q_pos0, 64, run.sm_scale, run.ws)
        ev[2].record(stream)
        qsa.sparse_attn_prefill(Q, K, V, run.idx, run.O, run.q_pos0, run.sm_scale, run.lse)
        ev[3].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    st, det = qsa.device_status()
    if st != "QSA_OK":
        raise RuntimeError(f"{wname}: device status {st} ({det})")

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    if ws > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    n0 = qsa.launch_count()
    clk = ClockSampler(dev.index) if clocks else None
    if clk:
        clk.__enter__()
    for k in range(args.steps):
        flush(k)
        step(evs[k])
    torch.cuda.synchronize()
    if clk:
        clk.__exit__(None, None, None)
    n_launch = qsa.launch_count() - n0
    if ws > 1:
        torch.distributed.barrier()
    st, det = qsa.device_status()
    if st != "QSA_OK":
        raise RuntimeError(f"{wname}: device status {st} ({det})")
    t = {"compress": np.array([e[0].elapsed_time(e[1]) for e in evs]),
         "score_select": np.array([e[1].elapsed_time(e[2]) for e in evs]),
         "attention": np.array([e[2].elapsed_time(e[3]) for e in evs]),
         "step": np.array([e[0].elapsed_time(e[3]) for e in evs])}
    out = {"w": wp, "t": t, "launches": int(n_launch), "clocks": clk.summary() if clk else None}
    if keep:
        out["kept"] = {"w": wp, "x": {k: x[k].cpu() for k in ("Q", "K", "V")},
                       "idx": run.idx.cpu().numpy(), "O": run.O.cpu()}
    del Q, K, V, x, run
    torch.cuda.empty_cache()
    return out


# DRAM bytes (read + written) per launch of the prefill attention kernel,
# from one-pass ncu captures (dram__bytes_read.sum + dram__bytes_write.sum)
# of this kernel on the workload itself, recorded with the command that
# took them among the repository's ncu summaries.  A workload without a
# capture reports null.
ATTN_TRAFFIC = {"prefill_128k": 899.11e6 + 519.84e6, "prefill_32k": 168.17e6 + 98.41e6}


def prefill_roofline(wp, att_ms, peaks):
    flops = prefill_flops(wp)
    achieved = flops / (att_ms * 1e-3) / 1e12
    return {"bound": "tensor", "kernel": "sparse_attn_prefill_kernel",
            "achieved": achieved, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
            "frac": achieved / peaks["bf16_tflops"],
            "frac_of_sustained": (achieved / peaks["bf16_tflops_sustained"]
                                  if peaks.get("bf16_tflops_sustained") else None),
            "peak_source": peaks["source"] + " bf16 burst", "flops_per_launch": flops,
            "traffic": ATTN_TRAFFIC.get(wp.name)}


def prefill_subline(pr, peaks):
    """A further prefill workload's part of the line (timed like the headline)."""
    wp, t = pr["w"], pr["t"]
    ms = float(t["step"].mean())
    return {"workload": wp.name, "batch": wp.B, "new_tokens": wp.Tq, "context": wp.q_pos0 + wp.Tq,
            "topk": wp.topk, "tokens_per_s": wp.B * wp.Tq / (ms * 1e-3), "ms_per_step": ms,
            "breakdown_ms": {k: float(t[k].mean()) for k in ("compress", "score_select", "attention")},
            "roofline": prefill_roofline(wp, float(t["attention"].mean()), peaks)}


def run_qsa(args, ws, rank, local, kept):
    """Our arm.  Appends to `kept` the host copies the parity check needs
    (rank 0 at N=1 only)."""
    import block_sparse_long_compress_b200 as qsa

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    peaks = load_peaks()
    flush = L2Flush(dev)
    want_keep = ws == 1 and not args.no_cpu_baseline
    pr = bench_prefill(args, qsa, dev, args.workload, ws, rank, flush, keep=want_keep, clocks=True)
    wp, t = pr["w"], pr["t"]
    if want_keep:
        kept.append(("prefill", pr["kept"]))
    ms = float(t["step"].sum() / args.steps)
    value, ms_max = job_throughput(ms, wp.B * wp.Tq, dev)
    result = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_max, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": wp.name, "batch": wp.B, "seq_len": wp.Tq, "q_heads": wp.Hq,
                   "kv_heads": wp.Hkv, "head_dim": wp.d, "block": 64, "topk": wp.topk,
                   "parallelism": f"dp{ws} (independent sequences)",
                   "l2": L2Flush.DESCRIPTION},
        "breakdown_ms": {k: float(t[k].mean()) for k in ("compress", "score_select", "attention")},
        "roofline": prefill_roofline(wp, float(t["attention"].mean()), peaks),
        "gpu_launches": pr["launches"],
        "clocks": pr["clocks"],
    }

    # ---- the other prefill workloads, timed the same way
    for name in filter(None, args.prefill_more.split(",")):
        sub = bench_prefill(args, qsa, dev, name, ws, rank, flush, keep=want_keep)
        if want_keep:
            kept.append(("prefill", sub["kept"]))
        result.setdefault("prefill_more", {})[name] = prefill_subline(sub, peaks)

    if args.prefill_max:
        x = synthetic.generate(wp, dev)
        result["prefill_max_selection"] = bench_prefill_agg(args, qsa, dev, peaks, wp, x["Q"], x["K"], flush, "max")
        result["prefill_softmax_sum_selection"] = bench_prefill_agg(args, qsa, dev, peaks, wp, x["Q"], x["K"],
                                                                    flush, "softmax_sum")
        del x
        torch.cuda.empty_cache()

    # ---- decode at 128K (same process, after the prefill tensors are freed)
    if not args.no_decode:
        if args.paged:
            result["prefill_ragged_paged"] = bench_prefill_paged(args, qsa, dev, peaks, ws, rank, flush)
            torch.cuda.empty_cache()
        result["decode"] = bench_decode(args, qsa, dev, peaks, ws, rank, flush, kept=kept if want_keep else None)
        if args.bf16_summaries:
            result["decode"]["bf16_summaries"] = bench_decode(args, qsa, dev, peaks, ws, rank, flush,
                                                              summary="bf16")
        if args.fp8_kv:
            torch.cuda.empty_cache()
            result["decode"]["fp8_kv"] = bench_decode(args, qsa, dev, peaks, ws, rank, flush,
                                                      summary="bf16", kv="fp8")
        if args.softmax_sum:
            torch.cuda.empty_cache()
            result["decode"]["softmax_sum_selection"] = bench_decode(args, qsa, dev, peaks, ws, rank, flush,
                                                                     agg="softmax_sum")
        if args.paged:
            torch.cuda.empty_cache()
            result["decode"]["ragged_paged"] = bench_decode_paged(args, qsa, dev, peaks, ws, rank, flush)
            if args.fp8_kv:
                torch.cuda.empty_cache()
                result["decode"]["ragged_paged"]["fp8_kv"] = bench_decode_paged(args, qsa, dev, peaks, ws, rank,
                                                                                flush, kv="fp8")
        for name in filter(None, args.decode_more.split(",")):
            torch.cuda.empty_cache()
            result.setdefault("decode_more", {})[name] = bench_decode(args, qsa, dev, peaks, ws,
                                                                      rank, flush, name,
                                                                      kept=kept if want_keep else None)
            if args.bf16_summaries:
                result["decode_more"][name]["bf16_summaries"] = bench_decode(
                    args, qsa, dev, peaks, ws, rank, flush, name, summary="bf16")

    # ---- e2e through the public API with host buffers
    if not args.no_e2e:
        result["e2e"] = bench_e2e(args, qsa, dev, wp, ws)
    return result


def decode_timings(args, qsa, dev, ws, flush, run_parts):
    """Times a decode step whose kernels run_parts(parts, stream) launches
    (parts from "select", "attention"): in-graph events and the differential
    per-step cost, for the whole step and each part.  Returns (events us,
    differential us, launches per step)."""
    stream = torch.cuda.current_stream()
    steps = max(args.steps, 20)

    def capture(parts, events=True):
        """flush [-> event] -> the step's kernels [-> event], as one CUDA
        graph; with events, they sit inside the graph so the graph's own
        launch stays outside the measured interval."""
        e0 = torch.cuda.Event(enable_timing=True, external=True)
        e1 = torch.cuda.Event(enable_timing=True, external=True)
        side = torch.cuda.Stream(device=dev)
        side.wait_stream(stream)
        g = torch.cuda.CUDAGraph()
        n0 = qsa.launch_count()
        with torch.cuda.graph(g, stream=side):
            flush(0)
            if events:
                e0.record(side)
            run_parts(parts, side)
            if events:
                e1.record(side)
        stream.wait_stream(side)
        return g, e0, e1, qsa.launch_count() - n0

    def timed_events(parts):
        g, e0, e1, launches = capture(parts)
        for _ in range(args.warmup):
            g.replay()
        torch.cuda.synchronize()
        if ws > 1:
            torch.distributed.barrier()
        out = []
        for _ in range(steps):
            g.replay()
            torch.cuda.synchronize()
            out.append(e0.elapsed_time(e1) * 1e3)   # us
        return np.array(out), launches

    def timed_differential(parts):
        """R back-to-back replays of (flush, kernels) minus R replays of
        (flush) alone, both between events on the stream: the kernels' cost
        per step as a stream of steps sees it."""
        g, _, _, _ = capture(parts, events=False)
        gf, _, _, _ = capture((), events=False)
        res = {}
        for name, gg in (("with", g), ("flush", gf)):
            for _ in range(args.warmup):
                gg.replay()
            torch.cuda.synchronize()
            if ws > 1:
                torch.distributed.barrier()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(steps):
                gg.replay()
            e1.record(stream)
            torch.cuda.synchronize()
            res[name] = e0.elapsed_time(e1) * 1e3 / steps
        return res["with"] - res["flush"]

    t = {}
    t["step"], launches_step = timed_events(("select", "attention"))
    t["select"], _ = timed_events(("select",))
    t["attention"], _ = timed_events(("attention",))
    d = {part: timed_differential(parts) for part, parts in
         (("step", ("select", "attention")), ("select", ("select",)), ("attention", ("attention",)))}
    st, det = qsa.device_status()
    if st != "QSA_OK":
        raise RuntimeError(f"decode device status {st} ({det})")
    return t, d, launches_step


def decode_result(wname, B, context, topk, t, d, launches, by, sel_bytes, peaks, extra=None):
    """The decode part of the JSON line (differential times reported, the
    in-graph event times kept beside them)."""
    us_step, us_att, us_sel = d["step"], d["attention"], d["select"]
    att_gbs = by / (us_att * 1e-6) / 1e9
    r = {"workload": wname, "batch": B, "context": context, "topk": topk}
    r.update(extra or {})
    r.update({
        "us_per_step": us_step, "us_per_token": us_step / B,
        "timing": ("per step: R back-to-back replays of a CUDA graph (L2 flush, step kernels) "
                   "minus R replays of (L2 flush) alone, events around each set"),
        "breakdown_us": {"score_select": us_sel, "attention": us_att},
        "in_graph_events_us": {"step": float(t["step"].mean()),
                               "score_select": float(t["select"].mean()),
                               "attention": float(t["attention"].mean())},
        "roofline": {"bound": "hbm", "kernel": "decode_kernel", "achieved": att_gbs,
                     "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": att_gbs / peaks["hbm_gbs"], "bytes_per_launch": by,
                     "traffic": None},
        "select_gbs": sel_bytes / (us_sel * 1e-6) / 1e9,
        "select_hbm_frac": sel_bytes / (us_sel * 1e-6) / 1e9 / peaks["hbm_gbs"],
        "gpu_launches_per_step": int(launches)})
    return r


def bench_decode(args, qsa, dev, peaks, ws, rank, flush, workload=None, summary="fp32", kv="bf16", agg="mean",
                 kept=None):
    wd = synthetic.CONFIGS[workload or args.decode_workload]
    if args.decode_batch:
        wd = synthetic.Workload(**{**wd.__dict__, "B": args.decode_batch})
    if ws > 1:
        wd = synthetic.Workload(**{**wd.__dict__, "seed": wd.seed + 1000 * rank})
    x = synthetic.generate(wd, dev)
    q = x["Q"].view(wd.B, wd.Hq, wd.d)
    K, V = x["K"], x["V"]
    L = wd.q_pos0 + 1
    sdt = torch.bfloat16 if summary == "bf16" else torch.float32
    dec = qsa.QSADecode(wd.B, wd.Hq, wd.Hkv, wd.d, wd.T_kv, wd.topk, device=dev, summary_dtype=sdt)
    dec.compress(K, 0, L // 64)           # persistent summaries (untimed)
    for _ in range(args.warmup):
        dec(q, K, V, L)
    torch.cuda.synchronize()
    sel_ws = dec._sel_ws[L]
    q4 = q.view(wd.B, 1, wd.Hq, wd.d)
    by = decode_bytes(wd)
    extra = {"summaries": summary}
    if kv == "fp8":
        # the cache as rotated e4m3 codes + per-row scales (written untimed,
        # as the cache write path would); summaries stay those of the keys
        Kq, Ks = qsa.quantize_kv_fp8(K)
        Vq, Vs = qsa.quantize_kv_fp8(V)
        del K, V, x
        torch.cuda.synchronize()
        torch.cuda.empty_cache()
        by = by // (2 * wd.d) * (wd.d + 4)      # per selected key and head: d code bytes + a 4-byte scale
        extra["kv_cache"] = "fp8 e4m3, Walsh-Hadamard rotated, per-row fp32 scale"

    if agg != "mean":
        extra["aggregator"] = agg

    def run_parts(parts, s):
        if "select" in parts:
            if agg == "mean":
                qsa.score_select(q4, dec.Kc, dec.idx, wd.topk, L - 1, 1, dec.sm_scale, sel_ws, s)
            else:
                qsa.score_select_token_agg(q4, dec.Kc, dec.idx, wd.topk, L - 1, agg, dec.sm_scale, stream=s)
        if "attention" in parts:
            if kv == "fp8":
                qsa.decode_fp8(q, Kq, Ks, Vq, Vs, dec.idx, dec.o, L, dec.sm_scale, s)
            else:
                qsa.decode(q, K, V, dec.idx, dec.o, L, dec.sm_scale, dec.ws_dec, s)

    t, d, launches = decode_timings(args, qsa, dev, ws, flush, run_parts)
    if kept is not None:
        # host copies for the oracle's parity check: the last replayed step's
        # indices and outputs, the queries, and two sequences' caches
        seqs = sorted({0, wd.B - 1})
        kept.append(("decode", {"w": wd, "q": x["Q"].cpu(), "idx": dec.idx.cpu().numpy(),
                                "o": dec.o.float().cpu().numpy(),
                                "seqs": {b: (K[b:b + 1].cpu(), V[b:b + 1].cpu()) for b in seqs}}))
    # summaries read by scoring (fp32, or bf16 for the bf16-summary option)
    sel_bytes = wd.B * wd.Hkv * ((L - 1) // 64) * wd.d * (2 if summary == "bf16" else 4)
    return decode_result(wd.name, wd.B, L, wd.topk, t, d, launches, by, sel_bytes, peaks, extra)


def bench_prefill_agg(args, qsa, dev, peaks, wp, Q, K, flush, agg):
    """Selection of the prefill workload's rows under the max-over-tokens or
    the softmax-sum aggregator: per-(head, token) logits of every candidate
    on the tensor cores (bf16 summaries, written untimed), then the chunked
    selection.  The FLOP rate is over the whole call (scoring, for the
    softmax-sum both passes, + selection)."""
    nblk = wp.T_kv // 64
    Kc = torch.empty((wp.B, wp.Hkv, nblk, wp.d), dtype=torch.bfloat16, device=dev)
    qsa.compress_keys(K, Kc, 0, (wp.q_pos0 + wp.Tq) // 64)
    NR = -(-wp.Tq // 64)
    idx = torch.empty((wp.B, wp.Hkv, NR, wp.topk), dtype=torch.int32, device=dev)
    need = qsa.score_select_prefill_agg_workspace(wp.B, wp.Hq, wp.Hkv, wp.Tq, wp.q_pos0, wp.T_kv, wp.d, wp.topk, agg)
    wsb = torch.empty(need, dtype=torch.uint8, device=dev)

    def call():
        qsa.score_select_prefill_agg(Q, Kc, idx, wp.topk, wp.q_pos0, agg, wp.sm_scale, wsb)

    for _ in range(args.warmup):
        call()
    torch.cuda.synchronize()
    # R calls back to back between two events: the host's per-call work
    # (tensor maps, argument checks) overlaps the previous call's kernels
    # instead of landing inside a timed interval; the queries (512 MiB at
    # prefill_128k) exceed L2 on their own
    R = max(args.steps, 5)
    flush(0)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(R):
        call()
    e1.record()
    torch.cuda.synchronize()
    ts = [e0.elapsed_time(e1) / R]
    st, det = qsa.device_status()
    if st != "QSA_OK":
        raise RuntimeError(f"prefill {agg} selection device status {st} ({det})")
    G = wp.Hq // wp.Hkv
    flops = 0
    for i in range(NR):
        t0, t1 = 64 * i, min(64 * (i + 1), wp.Tq)
        D = (wp.q_pos0 + t1 - 1) // 64
        # logits of the candidates (and, for the softmax-sum's statistics
        # pass, of every block before the diagonal)
        flops += 2 * wp.d * (t1 - t0) * G * (max(D - 1, 0) + (D if agg == "softmax_sum" and D > 1 else 0))
    flops *= wp.B * wp.Hkv
    ms = float(np.mean(ts))
    achieved = flops / (ms * 1e-3) / 1e12
    return {"workload": wp.name, "aggregator": agg, "summaries": "bf16",
            "ms": ms, "rows": wp.B * wp.Hkv * NR, "timing": f"{R} calls back to back between two events",
            "roofline": {"bound": "tensor",
                         "kernel": ("block_max_scores_kernel" if agg == "max" else
                                    "block_softmax_stats_kernel + block_softmax_scores_kernel")
                         + " (+ selection, in the time)",
                         "achieved": achieved, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                         "frac": achieved / peaks["bf16_tflops"], "flops_per_launch": flops, "traffic": None}}


def bench_prefill_paged(args, qsa, dev, peaks, ws, rank, flush):
    """Chunked prefill of a ragged batch over paged caches: 8 requests of
    4096 new tokens at positions uniform in [64K, 512K], top-64 per query
    block; selection and attention timed per step (L2 flushed)."""
    topk, Tq, Hq, Hkv, d = 64, 4096, 16, 2, 128
    x = synthetic.paged_prefill(B=8, Tq=Tq, Hq=Hq, Hkv=Hkv, d=d, seed=1008 + 1000 * rank, device=dev)
    B, max_blocks = x["Q"].shape[0], x["max_blocks"]
    seq_lens = x["q_pos"] + Tq
    Kc = torch.zeros((B, Hkv, max_blocks, d), dtype=torch.float32, device=dev)
    qsa.compress_keys_paged(x["K_pages"], x["block_table"], seq_lens, Kc)   # cache + chunk (untimed)
    NR = Tq // 64
    idx = torch.empty((B, Hkv, NR, topk), dtype=torch.int32, device=dev)
    O = torch.empty_like(x["Q"])
    ws_sel = torch.empty(max(1, qsa.score_select_workspace(B, Hq, Hkv, Tq, x["max_pos"], 64, d, topk)),
                         dtype=torch.uint8, device=dev)
    sm = d ** -0.5

    def select():
        qsa.score_select_ragged_prefill(x["Q"], Kc, x["q_pos"], idx, topk, x["max_pos"], sm, ws_sel)

    def attend():
        qsa.sparse_attn_prefill_paged(x["Q"], x["K_pages"], x["V_pages"], x["block_table"], x["q_pos"], idx, O,
                                      sm)

    for _ in range(args.warmup):
        select()
        attend()
    torch.cuda.synchronize()
    t_sel, t_att = [], []
    for _ in range(max(args.steps, 5)):
        flush(0)
        e = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        e[0].record()
        select()
        e[1].record()
        attend()
        e[2].record()
        torch.cuda.synchronize()
        t_sel.append(e[0].elapsed_time(e[1]))
        t_att.append(e[1].elapsed_time(e[2]))
    st, det = qsa.device_status()
    if st != "QSA_OK":
        raise RuntimeError(f"paged prefill device status {st} ({det})")
    pos = x["q_pos"].cpu().tolist()
    flops = sum(prefill_flops(synthetic.custom(B=1, Tq=Tq, T_kv=qp + Tq, q_pos0=qp, qblk=64, Hq=Hq, Hkv=Hkv,
                                               d=d, topk=topk)) for qp in pos)
    att = float(np.mean(t_att))
    achieved = flops / (att * 1e-3) / 1e12
    return {"workload": "chunked_ragged_paged", "batch": B, "chunk": Tq, "positions": f"{min(pos)}-{max(pos)}",
            "topk": topk, "layout": "paged: [pages][Hkv][64][d], random block table",
            "ms": {"score_select": float(np.mean(t_sel)), "attention": att},
            "tokens_per_s": B * Tq / ((float(np.mean(t_sel)) + att) * 1e-3),
            "roofline": {"bound": "tensor", "kernel": "sparse_attn_prefill_kernel", "achieved": achieved,
                         "peak": peaks["bf16_tflops"], "unit": "TFLOP/s", "frac": achieved / peaks["bf16_tflops"],
                         "flops_per_launch": flops, "traffic": None}}


def bench_decode_paged(args, qsa, dev, peaks, ws, rank, flush, kv="bf16"):
    """Ragged batch over a paged cache: 32 sequences of 64K-256K tokens
    (uniform), blocks in randomly placed pages, top-64 per token; kv="fp8":
    the pages hold the rotated fp8 cache (written untimed)."""
    topk, Hq, Hkv, d = 64, 16, 2, 128
    x = synthetic.paged_decode(B=32, min_len=65536, max_len=262144, Hq=Hq, Hkv=Hkv, d=d,
                               seed=1007 + 1000 * rank, device=dev)
    B = x["q"].shape[0]
    dec = qsa.QSADecodePaged(B, Hq, Hkv, d, x["max_blocks"], topk, device=dev)
    dec.compress(x["K_pages"], x["block_table"], x["seq_lens"])   # persistent summaries (untimed)
    args_ = (x["q"], x["K_pages"], x["V_pages"], x["block_table"], x["seq_lens"])
    for _ in range(args.warmup):
        dec(*args_, x["max_len"])
    torch.cuda.synchronize()
    q4 = x["q"].view(B, 1, Hq, d)
    if kv == "fp8":
        kc, ks = qsa.quantize_kv_fp8(x["K_pages"])
        vc, vs = qsa.quantize_kv_fp8(x["V_pages"])
        del args_
        x["K_pages"] = x["V_pages"] = None
        torch.cuda.synchronize()
        torch.cuda.empty_cache()

    def run_parts(parts, s):
        if "select" in parts:
            qsa.score_select_ragged(q4, dec.Kc, x["seq_lens"], dec.idx, topk, x["max_len"], dec.sm_scale, s)
        if "attention" in parts:
            if kv == "fp8":
                qsa.decode_fp8_paged(x["q"], kc, ks, vc, vs, x["block_table"], x["seq_lens"], dec.idx, dec.o,
                                     dec.sm_scale, s)
            else:
                qsa.decode_paged(*args_, dec.idx, dec.o, dec.sm_scale, s)

    t, d_, launches = decode_timings(args, qsa, dev, ws, flush, run_parts)
    lens = x["seq_lens"].cpu().numpy().astype(np.int64)
    # selected K + V bytes as decode_bytes counts them: full selected blocks
    # plus the visible keys of each sequence's diagonal block
    Dg = (lens - 1) // 64
    nsel = np.minimum(topk, Dg + 1)
    keys = 64 * (nsel - 1) + (lens - 64 * Dg)
    # per selected key and head: K and V rows of d bf16 values, or of d
    # fp8 codes plus a 4-byte scale
    by = int(keys.sum()) * 2 * Hkv * ((d + 4) if kv == "fp8" else 2 * d)
    sel_bytes = int(((lens - 1) // 64).sum()) * Hkv * d * 4
    extra = {"layout": "paged: [pages][Hkv][64][d], random block table; lengths uniform 64K-256K"}
    if kv == "fp8":
        extra["kv_cache"] = "fp8 e4m3, Walsh-Hadamard rotated, per-row fp32 scale"
    return decode_result("decode_ragged_paged", B, f"{int(lens.min())}-{int(lens.max())}", topk, t, d_,
                         launches, by, sel_bytes, peaks, extra)


def bench_e2e(args, qsa, dev, wp, ws):
    """Same metric through the public API, host buffers in and out: every
    step copies its Q, K, V from pinned host memory and reads its O back
    (PrefillHostPipeline: uploads, compute and downloads of neighbouring
    steps overlap on three streams, as a serving loop would run them)."""
    g = synthetic.generate(wp, dev)
    x = {k: g[k].cpu() for k in ("Q", "K", "V")}
    del g
    hQ, hK, hV = (x[k].pin_memory() for k in ("Q", "K", "V"))
    hO = torch.empty((wp.B, wp.Tq, wp.Hq, wp.d), dtype=torch.bfloat16).pin_memory()
    pipe = qsa.PrefillHostPipeline(wp.B, wp.Tq, wp.Hq, wp.Hkv, wp.d, wp.T_kv, wp.topk, wp.q_pos0,
                                   device=dev)
    for _ in range(args.warmup):
        pipe.submit(hQ, hK, hV, hO)
    pipe.synchronize()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if ws > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    e0.record(pipe.s_in)
    for _ in range(args.steps):
        pipe.submit(hQ, hK, hV, hO)
    e1.record(pipe.s_out)
    torch.cuda.synchronize()
    value, ms = job_throughput(e0.elapsed_time(e1) / args.steps, wp.B * wp.Tq, dev)
    h2d = sum(a.numel() * a.element_size() for a in (hQ, hK, hV))
    d2h = hO.numel() * hO.element_size()
    st, det = qsa.device_status()
    if st != "QSA_OK":
        raise RuntimeError(f"e2e device status {st} ({det})")
    return {"value": value, "unit": UNIT, "ms_per_step": ms,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "pipeline": "upload / compute / download of neighbouring steps on three streams"}


# ----------------------------------------------------- CPU oracle timing
def oracle_sample(wp, x_cpu, budget_s):
    """Time the fp64 oracle (as it stands) on a bounded sample of the
    workload: all summaries up to the sampled rows, the pooled queries, the
    selection of the sampled query blocks and the attention of all their
    tokens.  Returns (tokens/s, description, threads)."""
    import oracle

    nthreads = oracle.threads()
    # rows taken from the end of the sequence (full top-k), one per group
    # pair, as many as fit the budget after a one-row probe
    def run(rows):
        t0 = time.perf_counter()
        n_complete = (wp.q_pos0 + wp.Tq) // 64
        Kc = oracle.compress_keys(x_cpu["K"], 0, n_complete)
        Qbar = oracle.pool_queries(x_cpu["Q"], wp.Hkv, wp.qblk)
        flat = [(b * wp.Hkv + g) * wp.n_rows + i
                for b in range(wp.B) for g in range(wp.Hkv) for i in rows]
        sel = oracle.select(Qbar, Kc, wp.Tq, wp.q_pos0, wp.qblk, wp.topk, wp.sm_scale, rows=flat)
        idx = np.full((wp.B * wp.Hkv * wp.n_rows, wp.topk), -1, dtype=np.int32)
        idx[flat] = sel["idx"]
        idx = idx.reshape(wp.B, wp.Hkv, wp.n_rows, wp.topk)
        toks = [b * wp.Tq + t for b in range(wp.B) for i in rows
                for t in range(i * wp.qblk, min((i + 1) * wp.qblk, wp.Tq))]
        oracle.attend(x_cpu["Q"], x_cpu["K"], x_cpu["V"], idx, wp.q_pos0, wp.qblk,
                      wp.sm_scale, tokens=toks)
        return time.perf_counter() - t0, len(toks)

    t1, n1 = run([wp.n_rows - 1])
    nrows = max(1, min(wp.n_rows, int(budget_s / max(t1, 1e-3))))
    rows = list(range(wp.n_rows - nrows, wp.n_rows))
    t, n = run(rows)
    desc = (f"{len(rows)} query blocks x {wp.B} seq ({n} query tokens, all {wp.Hq} heads) of "
            f"{wp.name}: whole-cache compress + pooling of all rows + selection and attention of the "
            f"sampled rows, fp64")
    return n / t, desc, nthreads


def parity_check(kept, rng_seed=5):
    """The oracle against the GPU's outputs of the timed runs (part of the
    CPU-baseline leg, after every timed region): for each prefill workload,
    a sample of selection rows (exact-match and Jaccard overlap, the
    indices required to match wherever the oracle's gap exceeds 1e-3) and
    the outputs of a sample of their tokens over the GPU's own selection;
    for each decode workload, the rows and outputs of two sequences."""
    import oracle

    def jaccard(a, b):
        A, B = {int(v) for v in a if v >= 0}, {int(v) for v in b if v >= 0}
        return len(A & B) / len(A | B) if (A or B) else 1.0

    rng = np.random.RandomState(rng_seed)
    out = {}
    for kind, k in kept:
        w = k["w"]
        t0 = time.perf_counter()
        if kind == "prefill":
            x, idx = k["x"], k["idx"]
            NR = w.n_rows
            n_complete = (w.q_pos0 + w.Tq) // 64
            Kc = oracle.compress_keys(x["K"], 0, n_complete)
            Qbar = oracle.pool_queries(x["Q"], w.Hkv, w.qblk)
            nrows = w.B * w.Hkv * NR
            rows = np.unique(np.concatenate([[0, NR - 1, nrows - 1],
                                             rng.choice(nrows, size=min(nrows, 61), replace=False)]))
            sel = oracle.select(Qbar, Kc, w.Tq, w.q_pos0, w.qblk, w.topk, w.sm_scale, rows=rows)
            gidx = idx.reshape(-1, w.topk)[rows]
            # tokens: the first and the last 8 of up to 16 of the sampled rows (b = row // (Hkv NR))
            toks = []
            for r in rows[:16]:
                b, i = r // (w.Hkv * NR), r % NR
                t0_, t1_ = i * 64, min((i + 1) * 64, w.Tq)
                toks += [b * w.Tq + t for t in list(range(t0_, min(t0_ + 8, t1_))) + list(range(max(t1_ - 8, t0_), t1_))]
            toks = np.unique(np.array(toks, dtype=np.int64))
            O_ref = oracle.attend(x["Q"], x["K"], x["V"], idx, w.q_pos0, w.qblk, w.sm_scale, tokens=toks)
            O_gpu = k["O"].reshape(w.B * w.Tq, w.Hq, w.d)[torch.from_numpy(toks)].float().numpy()
        else:
            L = w.q_pos0 + 1
            sels, gl, O_ref, O_gpu = [], [], [], []
            for b, (Kb, Vb) in k["seqs"].items():
                qb = k["q"][b:b + 1]
                Kc = oracle.compress_keys(Kb, 0, L // 64)
                sel = oracle.select(oracle.pool_queries(qb, w.Hkv, 1), Kc, 1, w.q_pos0, 1, w.topk, w.sm_scale,
                                    rows=np.arange(w.Hkv))
                sels.append(sel)
                gl.append(k["idx"][b].reshape(-1, w.topk))
                O_ref.append(oracle.attend(qb, Kb, Vb, k["idx"][b:b + 1], w.q_pos0, 1, w.sm_scale)[0, 0])
                O_gpu.append(k["o"][b])
            sel = {"idx": np.concatenate([s_["idx"] for s_ in sels]), "gap": np.concatenate([s_["gap"] for s_ in sels])}
            gidx = np.concatenate(gl)
            O_ref, O_gpu = np.stack(O_ref), np.stack(O_gpu)
            rows, toks = np.arange(len(gidx)), np.arange(len(O_gpu))
        same = np.all(gidx == sel["idx"], axis=1)
        clear = sel["gap"] > 1e-3
        err = np.abs(O_gpu - O_ref)
        out[w.name] = {"rows": int(len(rows)), "gap_checked": float(clear.mean()),
                       "exact_where_gap_checked": float(same[clear].mean()) if clear.any() else None,
                       "identical": float(same.mean()),
                       "jaccard": float(np.mean([jaccard(a, b) for a, b in zip(gidx, sel["idx"])])),
                       "outputs": int(err.size), "max_abs_err": float(err.max()),
                       "mean_abs_err": float(err.mean()), "oracle_s": time.perf_counter() - t0}
    return out


def headline(res):
    """The line's key numbers in a few hundred characters, as its last key."""
    r = lambda v: None if v is None else float(f"{v:.4g}")
    h = {"prefill_128k" if res["config"]["workload"] == "prefill_128k" else res["config"]["workload"]: {
        "Mtok_s": r(res["value"] / 1e6), "select_ms": r(res["breakdown_ms"]["score_select"]),
        "attn_ms": r(res["breakdown_ms"]["attention"]), "attn_frac": r(res["roofline"]["frac"])}}
    for name, sub in res.get("prefill_more", {}).items():
        h[name] = {"Mtok_s": r(sub["tokens_per_s"] / 1e6), "select_ms": r(sub["breakdown_ms"]["score_select"]),
                   "attn_ms": r(sub["breakdown_ms"]["attention"]), "attn_frac": r(sub["roofline"]["frac"])}
    decs = [res["decode"]] if "decode" in res else []
    decs += list(res.get("decode_more", {}).values())
    for d in decs:
        h[d["workload"]] = {"us_per_token": r(d["us_per_token"]), "us_step": r(d["us_per_step"]),
                            "select_us": r(d["breakdown_us"]["score_select"]),
                            "attn_us": r(d["breakdown_us"]["attention"]), "attn_frac": r(d["roofline"]["frac"]),
                            "select_frac": r(d["select_hbm_frac"])}
    par = res.get("cpu_baseline", {}).get("parity")
    if par:
        h["parity"] = {n: {"max": r(p["max_abs_err"]), "mean": r(p["mean_abs_err"]), "identical": r(p["identical"]),
                           "jaccard": r(p["jaccard"])} for n, p in par.items()}
    return h


def run_reference(args, ws, rank):
    if rank != 0:
        return None
    wp = synthetic.CONFIGS[args.workload]
    x = synthetic.generate(wp, "cuda" if torch.cuda.is_available() else "cpu")
    x_cpu = {k: x[k].cpu() for k in ("Q", "K", "V")}
    del x
    per_step = []
    desc = threads = None
    budget = max(2.0, args.ref_budget / max(1, args.steps + args.warmup))
    for k in range(args.warmup + args.steps):
        v, desc, threads = oracle_sample(wp, x_cpu, budget)
        if k >= args.warmup:
            per_step.append(v)
    value = float(np.mean(per_step))
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": None,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": {"workload": wp.name, "batch": wp.B, "seq_len": wp.Tq, "q_heads": wp.Hq,
                       "kv_heads": wp.Hkv, "head_dim": wp.d, "block": 64, "topk": wp.topk},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                             "sample": desc},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="qsa", choices=["qsa", "reference"])
    ap.add_argument("--workload", default=PREFILL, choices=sorted(synthetic.CONFIGS))
    ap.add_argument("--decode-workload", default=DECODE, choices=sorted(synthetic.CONFIGS))
    ap.add_argument("--decode-more", default="decode_262k",
                    help="comma list of further decode workloads reported under decode_more")
    ap.add_argument("--prefill-more", default="prefill_32k,chunked_1m",
                    help="comma list of further prefill workloads reported under prefill_more")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-paged", dest="paged", action="store_false",
                    help="skip the ragged-batch, paged-cache decode run (reported beside the contiguous one)")
    ap.add_argument("--no-bf16-summaries", dest="bf16_summaries", action="store_false",
                    help="skip the decode run with the bf16-summary option (reported beside the fp32 one)")
    ap.add_argument("--no-fp8-kv", dest="fp8_kv", action="store_false",
                    help="skip the decode run over the rotated fp8 cache (reported beside the bf16 one)")
    ap.add_argument("--only-decode", action="store_true",
                    help="skip the prefill measurement (profiling the decode kernels)")
    ap.add_argument("--no-prefill-max", dest="prefill_max", action="store_false",
                    help="skip the prefill selections with the max-over-tokens and softmax-sum aggregators")
    ap.add_argument("--no-softmax-sum", dest="softmax_sum", action="store_false",
                    help="skip the decode run with the softmax-sum selection aggregator")
    ap.add_argument("--decode-variants", default="fp32,bf16,fp8,paged,softmax_sum",
                    help="with --only-decode: which decode runs (fp32 / bf16 summaries, fp8 cache, paged)")
    ap.add_argument("--decode-batch", type=int, default=None,
                    help="override the decode batch (smaller profiling captures)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=12.0, help="seconds of oracle work")
    ap.add_argument("--ref-budget", type=float, default=60.0)
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    ws, rank, local = dist_env()
    if ws > 1:
        import datetime
        backend = "nccl" if args.impl == "qsa" else "gloo"
        if args.impl == "reference" and rank != 0:
            return
        if args.impl == "qsa":
            torch.cuda.set_device(local)
            torch.distributed.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    if args.impl == "reference":
        res = run_reference(args, ws, rank)
        if res is not None:
            print(json.dumps(res), flush=True)
        return

    if args.only_decode:
        import block_sparse_long_compress_b200 as qsa
        dev = torch.device("cuda", local)
        torch.cuda.set_device(dev)
        flush = L2Flush(dev)
        variants = set(filter(None, args.decode_variants.split(",")))
        res = bench_decode(args, qsa, dev, load_peaks(), ws, rank, flush) if "fp32" in variants else {}
        if args.bf16_summaries and "bf16" in variants:
            res["bf16_summaries"] = bench_decode(args, qsa, dev, load_peaks(), ws, rank, flush, summary="bf16")
        if args.fp8_kv and "fp8" in variants:
            torch.cuda.empty_cache()
            res["fp8_kv"] = bench_decode(args, qsa, dev, load_peaks(), ws, rank, flush, summary="bf16", kv="fp8")
        if args.softmax_sum and "softmax_sum" in variants:
            torch.cuda.empty_cache()
            res["softmax_sum_selection"] = bench_decode(args, qsa, dev, load_peaks(), ws, rank, flush,
                                                        agg="softmax_sum")
        if args.paged and "paged" in variants:
            torch.cuda.empty_cache()
            res["ragged_paged"] = bench_decode_paged(args, qsa, dev, load_peaks(), ws, rank, flush)
            if args.fp8_kv and "fp8" in variants:
                torch.cuda.empty_cache()
                res["ragged_paged"]["fp8_kv"] = bench_decode_paged(args, qsa, dev, load_peaks(), ws, rank, flush,
                                                                   kv="fp8")
        for name in filter(None, args.decode_more.split(",")):
            torch.cuda.empty_cache()
            res.setdefault("decode_more", {})[name] = bench_decode(args, qsa, dev, load_peaks(), ws,
                                                                   rank, flush, name)
            if args.bf16_summaries:
                res["decode_more"][name]["bf16_summaries"] = bench_decode(
                    args, qsa, dev, load_peaks(), ws, rank, flush, name, summary="bf16")
        if rank == 0:
            print(json.dumps(res), flush=True)
        return
    kept = []
    res = run_qsa(args, ws, rank, local, kept)
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        wp = synthetic.CONFIGS[args.workload]
        x_cpu = next(k["x"] for kind, k in kept if kind == "prefill" and k["w"].name == wp.name)
        v, desc, threads = oracle_sample(wp, x_cpu, args.cpu_budget)
        res["cpu_baseline"] = {"value": v, "unit": UNIT, "cores": threads, "kind": "oracle",
                               "sample": desc, "parity": parity_check(kept)}
    del kept
    res["headline"] = headline(res)
    if ws > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
