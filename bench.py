#!/usr/bin/env python
"""Benchmark of one absorbed-MLA decode step on B200, through the C ABI.

A step is one pass of the whole decode path over one batch of synthetic input:
  mla_cache_append (RoPE on the new keys + paged scatter),
  mla_absorb_q (W^UK folded into the query, RoPE on q^R),
  mla_decode_attention (split-KV attention + log-sum-exp combine),
  mla_out_absorb (W^UV applied to the latent output).
Default workload: DeepSeek-V3-shaped decode, 64 sequences x 4096 cached tokens,
128 heads, one query token each ("v3").

Prints one JSON line (rank 0). Multi-GPU (torchrun): every rank runs its own
replica of the workload (the path shards by sequence with no exchange), the
device time is the max over ranks and ``value`` counts all ranks' tokens.

``--impl reference`` times the CPU fp64 oracle (the only reference that exists
for this method) on the host cores, on a bounded sample of the same workload.
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
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MLA decode tokens/sec and cache GB/s (% of HBM/bf16 roofline) on 1 B200"
UNIT = "tokens/s"
ROW_BYTES = 1152                 # 576 bf16 per cached token
FP8_TOKEN_BYTES = 644            # FP8 cache: 512 E4M3 + 64 bf16 + a float32 scale
# independent batches in flight in the end-to-end loop: with two, each
# stream's upload -> step -> download chain (~0.26 ms on v3) paced the loop
# at 0.23 ms per step; with three the step's compute does (0.14 ms)
E2E_SESSIONS = 3
FLOP_PER_TOKEN_HEAD = 2 * 576 + 2 * 512
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# B200 data-sheet figures (dense bf16), reported beside the measured peaks
SPEC_PEAKS = {"hbm_gbs": 8000.0, "bf16_tflops": 2250.0}


def dist_stats(xs):
    """median / min / p90 of a list of per-call times (ms)."""
    ys = sorted(xs)
    p90 = ys[min(len(ys) - 1, int(math.ceil(0.9 * len(ys))) - 1)]
    return {"median": statistics.median(ys), "min": ys[0], "p90": p90}

# DRAM traffic per launch of mla_decode_attention measured by ncu
# (dram__bytes_read.sum + dram__bytes_write.sum), keyed by the SHA-256 of the
# decode sources it was measured on, the workload and the cache format;
# reported only while the sources match (the combine kernel's few MB are not
# included).
TRAFFIC = {
    # decode_pair_kernel<bf16>: 1.054 x the cache bytes
    ("d754049324a228ee", "v3", "bf16"): 318256128,
    # decode_pair_kernel<fp8>: 1.066 x the cache bytes read, 8.6 MB written
    ("d754049324a228ee", "v3", "fp8"): 188447232,
}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--workload", default="v3")
    ap.add_argument("--cache", default="bf16", choices=["bf16", "fp8"],
                    help="latent cache format of the timed workload")
    ap.add_argument("--batch", type=int, default=0,
                    help="override the workload's batch (a smaller case of the same "
                         "workload, e.g. for profiling)")
    ap.add_argument("--num-ctas", type=int, default=0)
    ap.add_argument("--max-split", type=int, default=-1)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=200,
                    help="end-to-end steps timed (at least --steps)")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the per-workload lines (ragged, long_mtp, mtp8, layer_v3, tiny)")
    ap.add_argument("--configs",
                    default="tiny,ragged,long_mtp,mtp8,prefill,layer_v3,tiny:folded,"
                            "layer_v3:folded,v3:fp8,ragged:fp8",
                    help="comma-separated workloads measured besides the headline one "
                         "(':folded' = the layer with folded weights)")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--ramp-seconds", type=float, default=0.3,
                    help="back-to-back untimed steps before timing, so the clocks leave "
                         "their idle state (0: none, e.g. under a profiler)")
    ap.add_argument("--rows-only", default="",
                    help="with --rows: comma-separated row names to run (e.g. a1,a9)")
    ap.add_argument("--rows", action="store_true",
                    help="time every library call of the decode step (v3) and of the "
                         "full layer (layer_v3) alone against its own roofline; one JSON "
                         "line per call")
    return ap.parse_args()


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def decode_sources_hash():
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "mla_latent_kv_32_b200", "csrc")
    for name in sorted(os.listdir(csrc)):
        if name.startswith("decode") or name in ("plan.h", "common.cuh"):
            with open(os.path.join(csrc, name), "rb") as f:
                h.update(f.read())
    return h.hexdigest()[:16]


class ClockSampler:
    """Samples nvidia-smi SM clocks and throttle reasons every 20 ms while
    running. ``mark_start``/``mark_end`` bound the window the summary covers
    (the clock ramp and the timed loops); samples whose active reasons include
    GPU idle are left out, so the median is the clock under load."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    IDLE = 0x1

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []        # (host time, line)
        self.thread = None
        self.t0 = None
        self.t1 = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "20"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
            time.sleep(0.25)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.monotonic(), line.strip()))

    def mark_start(self):
        self.t0 = time.monotonic()

    def mark_end(self):
        self.t1 = time.monotonic()

    def __exit__(self, *a):
        if self.proc is not None:
            time.sleep(0.05)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            if self.thread:
                self.thread.join(timeout=2)

    def summary(self):
        if not self.lines:
            return None
        mhz, max_mhz, reasons, power, idle = [], 0.0, set(), [], 0
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        lo = self.t0 if self.t0 is not None else -math.inf
        hi = self.t1 if self.t1 is not None else math.inf
        for t, ln in self.lines:
            if t < lo or t > hi:
                continue
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                active = int(parts[4], 16)
                m, mx, pw = float(parts[1]), float(parts[2]), float(parts[3])
            except ValueError:
                continue
            max_mhz = max(max_mhz, mx)
            if active & self.IDLE:
                idle += 1
                continue
            mhz.append(m)
            power.append(pw)
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not mhz:
            return {"sm_mhz": None, "sm_max_mhz": max_mhz or None, "reasons": [],
                    "samples": 0, "idle_samples": idle,
                    "note": "no nvidia-smi sample under load in the window"}
        return {"sm_mhz": statistics.median(mhz), "sm_max_mhz": max_mhz,
                "reasons": sorted(reasons), "samples": len(mhz), "idle_samples": idle,
                "power_w_max": max(power) if power else None,
                "window": "clock ramp + timed loops, 20 ms samples, GPU-idle samples dropped"}


def ramp_clocks(fn, seconds=0.3, sync_every=16):
    """Runs fn() back to back for ~seconds (synchronising every sync_every
    calls) so that the GPU's clocks reach their loaded steady state before
    anything is timed; from idle they take a few ms to climb."""
    import torch
    t_end = time.monotonic() + seconds
    n = 0
    while time.monotonic() < t_end:
        for _ in range(sync_every):
            fn()
        torch.cuda.synchronize()
        n += sync_every
    return n


def cpu_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


def oracle_sample(w, inp, budget_s=12.0, max_seqs=None):
    """Time the absorbed fp64 oracle on whole sequences of the workload until
    ~budget_s of CPU work (at least one sequence). Returns (tokens/s, desc)."""
    from oracle import mla_oracle as O
    table = O.rope_table(int(inp.lens.max()))
    scale = 1.0 / math.sqrt(192)
    done, t_tot, cache_bytes = 0, 0.0, 0
    order = list(range(w.B))
    for b in order:
        L = int(inp.lens[b])
        n_pref = L - w.q_len
        prefix = (O.gather_rows(inp.pool, inp.table, b, n_pref) if n_pref > 0
                  else np.zeros((0, 576), np.uint16))
        t0 = time.perf_counter()
        O.decode_sequence(prefix, inp.c_new[b], inp.k_new[b], inp.q_nope[b], inp.q_pe[b],
                          inp.w_uk, inp.w_uv, L, table, scale)
        t_tot += time.perf_counter() - t0
        done += 1
        cache_bytes += L * ROW_BYTES
        if t_tot >= budget_s or (max_seqs and done >= max_seqs):
            break
    tokens = done * w.q_len
    desc = (f"absorbed fp64 oracle (numpy), {done} of {w.B} sequences of workload "
            f"'{w.name}' ({tokens} query tokens, {cache_bytes / 1e6:.1f} MB of cache rows), "
            f"{t_tot:.2f} s")
    return tokens / t_tot, desc, t_tot


def run_reference(args, rank, world):
    import synth
    if rank != 0:
        return 0
    w = synth.WORKLOADS[args.workload]
    inp = synth.make_decode_inputs(w)
    per_step = []
    desc = ""
    budget = max(1.0, 120.0 / max(1, args.steps + args.warmup))
    for s in range(args.warmup + args.steps):
        tps, desc, t = oracle_sample(w, inp, budget_s=budget)
        if s >= args.warmup:
            per_step.append(tps)
    v = statistics.median(per_step)
    cores = cpu_threads()
    out = {
        "impl": "reference", "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * w.B * w.q_len / v,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": workload_config(w, inp, None),
        "cpu_baseline": {"value": v, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(out), flush=True)
    return 0


def max_over_ranks(values, dist, device, world):
    """Element-wise maximum of per-rank timings (the slowest rank sets the job
    time). ``dist`` is torch.distributed; with one rank it is not touched."""
    import torch
    if world <= 1:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def whole_job_rate(world, units_per_rank, t_ms):
    """Units processed by all ranks per second, given the max-over-ranks time."""
    return world * units_per_rank / (t_ms / 1e3)


def workload_config(w, inp, sess, ramp_seconds=0.0):
    cfg = {"workload": f"{w.name}: absorbed MLA decode, batch {w.B}, {w.q_len} query token(s) "
                       f"per sequence, context {'U[1,%d]' % w.L if w.lens == 'ragged' else w.L}, "
                       f"n_h {w.n_h}, d_c 512, d_R 64, paged cache of 64-token pages",
           "batch": w.B, "q_len": w.q_len, "n_h": w.n_h,
           "context_tokens": int(inp.lens.sum()),
           "cache_bytes": int(inp.lens.sum()) * ROW_BYTES}
    if sess is not None:
        cfg["l2"] = ("flushed before every timed step and every timed attention call, "
                     "outside the events: a 256 MiB write, then a 256 MiB read of another "
                     "buffer so that no dirty lines of the flush remain in L2")
        cfg["timing"] = ("each step one CUDA graph replay of the four library calls; the "
                         "attention call timed alone in a second loop for the roofline; "
                         f"before timing, flush + step run back to back for "
                         f"{ramp_seconds:g} s so the clocks reach their loaded steady "
                         f"state")
        cfg["plan"] = {"work_lists": int(sess.info.num_ctas), "items": int(sess.info.num_items),
                       "partials": int(sess.info.num_partials)}
    return cfg


class L2Flush:
    """Empties L2 of the timed work's data between timed calls: writes a
    256 MiB buffer (L2 is 126 MB), then reads another 256 MiB buffer. The
    read leaves L2 holding clean lines unrelated to the timed call; a write
    alone would leave ~126 MB of dirty lines whose write-back to HBM would
    land inside the next timed call."""

    def __init__(self, dev):
        import torch
        self.w = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
        # float32: the sum reduces the buffer in place (an int32 sum would
        # first write a 512 MB int64 copy of it)
        self.r = torch.ones(64 << 20, dtype=torch.float32, device=dev)

    def __call__(self):
        self.w.zero_()
        self.r.sum()


def run_rows(args):
    """Each call of the path alone, L2 flushed before every call: time, its
    algorithmic bytes (weights and activations read once, outputs written
    once) and FLOPs, and the fraction of the roofline (the slower of bytes ÷
    measured HBM bandwidth and FLOPs ÷ measured bf16 peak). Each call is
    captured in a CUDA graph and timed as one replay: a call's host-side
    argument checks and tensor-map encoding are not in the time, the replay's
    own launch latency is."""
    import torch
    import synth
    from mla_latent_kv_32_b200 import build as build_mod
    from mla_latent_kv_32_b200 import mla
    from mla_latent_kv_32_b200.runtime import DecodeSession, LayerSession

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    build_mod.build()
    mla.load()
    peaks, peak_src = load_peaks()
    flush = L2Flush(dev)
    stream = torch.cuda.current_stream()

    def timed(fn, K):
        for _ in range(3):
            fn()
        side = torch.cuda.Stream()
        side.wait_stream(stream)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=side):
            fn(side)
        stream.wait_stream(side)
        if args.ramp_seconds > 0:
            ramp_clocks(lambda: (flush(), graph.replay()), seconds=min(0.2, args.ramp_seconds))
        ts = []
        for _ in range(K):
            flush()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            graph.replay()
            b.record(stream)
            torch.cuda.synchronize()
            ts.append(a.elapsed_time(b) * 1e3)
        return statistics.median(ts)

    only = {r for r in args.rows_only.split(",") if r}

    def want(row):
        return not only or row in only

    def line(workload, row, call, us, nbytes, flops):
        t_mem = nbytes / (peaks["hbm_gbs"] * 1e9) * 1e6
        t_tc = flops / (peaks["bf16_tflops"] * 1e12) * 1e6
        out = {"mode": "rows", "workload": workload, "row": row, "call": call, "us": us,
               "bytes": int(nbytes), "flops": float(flops),
               "gbs": nbytes / us / 1e3, "tflops": flops / us / 1e6,
               "bound": "hbm" if t_mem >= t_tc else "tensor",
               "roofline_us": max(t_mem, t_tc), "frac": max(t_mem, t_tc) / us,
               "peak_source": peak_src}
        print(json.dumps(out), flush=True)

    K = max(5, args.steps)
    bf = 2
    # decode step rows on v3
    if any(want(r) for r in ("a3+a4", "a3+a5", "a6+a7", "a8")):
        w = synth.WORKLOADS["v3"]
        inp = synth.make_decode_inputs(w)
        sess = DecodeSession(inp, dev)
        T, H = w.B * w.q_len, w.n_h
        if want("a3+a4"):
            line("v3", "a3+a4", "mla_cache_append", timed(sess.append, K),
                 T * (576 * bf + 1152 + 256), 0)
        if want("a3+a5"):
            line("v3", "a3+a5", "mla_absorb_q", timed(sess.absorb, K),
                 H * 128 * 512 * bf + T * H * (128 + 64 + 576) * bf + T * 256,
                 2.0 * T * H * 128 * 512)
        cache = int(inp.lens.sum()) * ROW_BYTES
        vis = sum(int(L) - w.q_len + j + 1 for L in inp.lens for j in range(w.q_len))
        if want("a6+a7"):
            line("v3", "a6+a7", "mla_decode_attention", timed(sess.attend, K), cache,
                 float(vis) * H * FLOP_PER_TOKEN_HEAD)
        if want("a8"):
            line("v3", "a8", "mla_out_absorb", timed(sess.expand, K),
                 H * 128 * 512 * bf + T * H * (512 + 128) * bf, 2.0 * T * H * 128 * 512)
        del sess, inp
        torch.cuda.empty_cache()
    if not any(want(r) for r in ("a1", "a2", "a6+a7", "a9")):
        return 0
    # the whole layer's projections on layer_v3
    w = synth.WORKLOADS["layer_v3"]
    inp = synth.make_layer_inputs(w)
    ls = LayerSession(inp, dev)
    Tq, Tk, H, d, ql = ls.Tq, ls.T, w.n_h, w.hidden, w.q_lora
    nq = H * 192
    if want("a1"):
        line("layer_v3", "a1", "mla_gemm_bf16 x2 (W_DQ, [W_UQ|W_QR])", timed(ls.project_q, K),
             (ql * d + Tq * d + Tq * ql) * bf + (nq * ql + Tq * ql + Tq * nq) * bf,
             2.0 * Tq * ql * d + 2.0 * Tq * nq * ql)
    if want("a2"):
        line("layer_v3", "a2", "mla_gemm_bf16 ([W_DKV|W_KR])", timed(ls.project_kv, K),
             (576 * d + Tk * d + Tk * 576) * bf, 2.0 * Tk * 576 * d)
    ls.project_q(); ls.project_kv(); ls.append(); ls.absorb()
    if want("a6+a7"):
        line("layer_v3", "a6+a7", "mla_decode_attention", timed(ls.attend, K),
             int(ls.lens.sum()) * ROW_BYTES,
             float(sum(int(L) for L in ls.lens)) * H * FLOP_PER_TOKEN_HEAD)
    if want("a9"):
        line("layer_v3", "a9", "mla_gemm_bf16 (W_O, fp32 out)", timed(ls.project_out, K),
             (d * H * 128 + Tq * H * 128) * bf + Tq * d * 4, 2.0 * Tq * d * H * 128)
    return 0


def timed_calls(run, flush, stream, K):
    """K calls of run(), L2 flushed before each outside the events; per-call
    device milliseconds (CUDA events on ``stream``)."""
    import torch
    ev = []
    for _ in range(K):
        if flush is not None:
            flush()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        run()
        b.record(stream)
        ev.append((a, b))
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in ev]


def attention_work(inp, w):
    """(cache bytes read once, FLOPs) of one attention call: 1152 B per cached
    token, 2176 FLOP per (visible cached token, head, query token)."""
    cache_bytes = int(inp.lens.sum()) * ROW_BYTES
    vis = sum(int(L) - w.q_len + j + 1 for L in inp.lens for j in range(w.q_len))
    return cache_bytes, float(vis) * w.n_h * FLOP_PER_TOKEN_HEAD


def roofline_of(nbytes, flops, t_ms, peaks):
    t_mem = nbytes / (peaks["hbm_gbs"] * 1e9)
    t_tc = flops / (peaks["bf16_tflops"] * 1e12)
    t = t_ms / 1e3
    return {"bound": "hbm" if t_mem >= t_tc else "tensor", "roofline_us": max(t_mem, t_tc) * 1e6,
            "measured_us": t_ms * 1e3, "frac_of_roofline": max(t_mem, t_tc) / t,
            "gbs": nbytes / t / 1e9, "tflops": flops / t / 1e12,
            "frac_spec": max(nbytes / (SPEC_PEAKS["hbm_gbs"] * 1e9),
                             flops / (SPEC_PEAKS["bf16_tflops"] * 1e12)) / t}


def measure_decode_config(name, dev, flush, stream, K, peaks, args, fp8=False):
    """One attention-only workload: the whole step (one graph replay) and the
    attention call alone, each after an L2 flush; the roofline of the call.
    fp8: the same workload over the FP8 cache (644 bytes per cached token)."""
    import torch
    import synth
    from mla_latent_kv_32_b200.runtime import DecodeSession
    w = synth.WORKLOADS[name]
    inp = synth.make_decode_inputs(w)
    sess = DecodeSession(inp, dev, fp8=fp8)
    for _ in range(3):
        sess.step()
    torch.cuda.synchronize()
    assert sess.read_status() == 0, f"{name}: device status during warm-up"
    sess.capture()
    sess.replay(stream)
    step = timed_calls(lambda: sess.replay(stream), flush, stream, K)
    attn = timed_calls(sess.attend, flush, stream, K)
    assert sess.read_status() == 0, f"{name}: device status in the timed calls"
    nbytes, flops = attention_work(inp, w)
    if fp8:
        nbytes = int(inp.lens.sum()) * FP8_TOKEN_BYTES
    t_step, t_attn = statistics.median(step), statistics.median(attn)
    out = {"workload": workload_config(w, inp, None)["workload"]
           + (", FP8 (E4M3) latent cache, bf16 k^R, per-token power-of-two scale" if fp8 else ""),
           "tokens_per_s": w.B * w.q_len / (t_step / 1e3), "step_ms": t_step,
           "attention_ms": t_attn, "step_ms_stats": dist_stats(step),
           "attention_ms_stats": dist_stats(attn), "cache_bytes": nbytes, "flops": flops,
           "cache_gbs_attention": nbytes / (t_attn / 1e3) / 1e9,
           "roofline": roofline_of(nbytes, flops, t_attn, peaks),
           "plan": {"work_lists": int(sess.info.num_ctas), "items": int(sess.info.num_items),
                    "partials": int(sess.info.num_partials),
                    "combine": int(sess.info.num_combine)},
           "launches_per_step": 3 + (1 if sess.info.num_combine else 0)}
    if w.q_len > 16:
        # the same attention in the expanded (non-absorbed) form: 2*(128+64)
        # + 2*128 FLOP per (visible token, head, query) plus expanding K^C and
        # V (2 * 2 * 512 * 128 per cached token and head); for context only
        vis = flops / (w.n_h * FLOP_PER_TOKEN_HEAD)
        out["flops_expanded_form"] = (vis * w.n_h * (2 * 192 + 2 * 128)
                                      + float(inp.lens.sum()) * w.n_h * 4 * 512 * 128)
    del sess
    torch.cuda.empty_cache()
    return out


def measure_layer_config(name, dev, flush, stream, K, peaks, folded=False):
    """A whole decode layer from hidden states: the step (one graph replay of
    the seven library calls) and the attention call alone. For the step the
    roofline counts the cache, every weight and the activations once, and the
    projection FLOPs besides the attention's; a launch-bound layer (the tiny
    one) reports microseconds per step only."""
    import torch
    import synth
    from mla_latent_kv_32_b200.runtime import LayerSession
    w = synth.WORKLOADS[name]
    inp = synth.make_layer_inputs(w)
    ls = LayerSession(inp, dev, folded=folded)
    for _ in range(3):
        ls.step()
    torch.cuda.synchronize()
    assert ls.read_status() == 0, f"{name}: device status during warm-up"
    ls.capture()
    ls.replay(stream)
    big = w.name != "tiny"
    step = timed_calls(lambda: ls.replay(stream), flush if big else None, stream, K)
    attn = timed_calls(ls.attend, flush if big else None, stream, K)
    assert ls.read_status() == 0, f"{name}: device status in the timed calls"
    t_step, t_attn = statistics.median(step), statistics.median(attn)
    cache_bytes = int(inp.lens.sum()) * ROW_BYTES
    attn_flops = float(sum(int(L) for L in inp.lens)) * w.n_h * FLOP_PER_TOKEN_HEAD
    Tq, T, H, d = ls.Tq, ls.T, w.n_h, w.hidden
    ql = w.q_lora
    q_in = ql or d
    if folded:
        # weights the folded step reads: W_DQ, W_QR, W~QK, W_DKV|W_KR, W~O
        wbytes = 2 * ((ql * d if ql else 0) + H * 64 * q_in + H * 512 * q_in + 576 * d
                      + d * H * 512)
        proj_flops = ((2.0 * Tq * ql * d if ql else 0.0) + 2.0 * Tq * H * 64 * q_in
                      + 2.0 * T * 576 * d + 2.0 * Tq * d * H * 512)
        absorb_flops = 2.0 * Tq * H * 512 * q_in
    else:
        wbytes = sum(int(v.size) for v in inp.weights.values()) * 2
        if ql:
            proj_flops = (2.0 * Tq * ql * d + 2.0 * Tq * H * 192 * ql + 2.0 * T * 576 * d
                          + 2.0 * Tq * d * H * 128)
        else:
            proj_flops = 2.0 * Tq * H * 192 * d + 2.0 * T * 576 * d + 2.0 * Tq * d * H * 128
        absorb_flops = 2.0 * 2 * Tq * H * 128 * 512
    act_bytes = (T * d + Tq * d * 2 + T * 576) * 2
    out = {"workload": (f"{w.name}: whole MLA decode layer, batch {w.B}, context {w.L}, hidden "
                        f"{w.hidden}, q_lora {w.q_lora or 'none'}, n_h {w.n_h}"
                        + (", folded weights W~QK = W^UK^T W^UQ and W~O = W^O W^UV per head"
                           if folded else "")),
           "weight_bytes": wbytes,
           "tokens_per_s": Tq / (t_step / 1e3), "step_ms": t_step, "attention_ms": t_attn,
           "step_ms_stats": dist_stats(step), "attention_ms_stats": dist_stats(attn)}
    if big:
        out["l2"] = "flushed before every timed call"
        out["roofline_attention"] = roofline_of(cache_bytes, attn_flops, t_attn, peaks)
        out["roofline_step"] = roofline_of(cache_bytes + wbytes + act_bytes,
                                           attn_flops + proj_flops + absorb_flops, t_step, peaks)
        out["step_bytes"] = cache_bytes + wbytes + act_bytes
        out["step_flops"] = attn_flops + proj_flops + absorb_flops
    else:
        out["us_per_step_graph_replay"] = t_step * 1e3
        out["l2"] = "not flushed: the layer is launch-bound (0.3 MB of cache)"
        out["roofline"] = None
    del ls
    torch.cuda.empty_cache()
    return out


def main():
    args = parse()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        return run_reference(args, rank, world)
    if args.rows:
        return run_rows(args) if rank == 0 else 0

    import torch
    import torch.distributed as dist
    import synth
    from mla_latent_kv_32_b200 import build as build_mod
    from mla_latent_kv_32_b200 import mla
    from mla_latent_kv_32_b200.runtime import (DecodeSession, capture_io_step,
                                               run_e2e_graphs)

    assert torch.cuda.is_available(), "bench.py needs a CUDA device"
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    if rank == 0 or not os.path.exists(mla.LIB_PATH):
        build_mod.build()
    if world > 1:
        dist.barrier()
    mla.load()

    w = synth.WORKLOADS[args.workload]
    if args.batch:
        import dataclasses
        w = dataclasses.replace(w, B=args.batch)
    assert not w.layer, "bench.py times the attention-only decode workloads"
    inp = synth.make_decode_inputs(w)
    fp8 = args.cache == "fp8"
    sess = DecodeSession(inp, dev, num_ctas=args.num_ctas, max_split=args.max_split, fp8=fp8)
    flush = L2Flush(dev)
    stream = torch.cuda.current_stream()
    peaks, peak_src = load_peaks()

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    for _ in range(max(3, args.warmup)):
        sess.step()
    torch.cuda.synchronize()
    bits = sess.read_status()
    assert bits == 0, f"device status 0x{bits:x} during warm-up"

    # Timed steps: each step is one replay of a CUDA graph holding the four
    # library calls (append, absorb, attention, expand); L2 flushed before
    # each step, outside the events. Then the attention call alone, timed the
    # same way, for the roofline of the decode kernel.
    sess.capture()
    for _ in range(2):
        sess.replay(stream)
    torch.cuda.synchronize()
    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
    ea = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
    with ClockSampler(local) as clocks:
        clocks.mark_start()
        if args.ramp_seconds > 0:
            ramp_clocks(lambda: (flush(), sess.replay(stream)), seconds=args.ramp_seconds)
        barrier()
        for k in range(K):
            flush()
            ev[k][0].record(stream)
            sess.replay(stream)
            ev[k][1].record(stream)
        for k in range(K):
            flush()
            ea[k][0].record(stream)
            sess.attend()
            ea[k][1].record(stream)
        barrier()
        bits = sess.read_status()
        assert bits == 0, f"device status 0x{bits:x} in the timed steps"
        step_ms = [a.elapsed_time(b) for a, b in ev]
        attn_ms = [a.elapsed_time(b) for a, b in ea]
        t_step = sum(step_ms) / K
        t_attn = sum(attn_ms) / K
        t_step, t_attn = max_over_ranks([t_step, t_attn], dist, dev, world)

        tokens = w.B * w.q_len
        value = whole_job_rate(world, tokens, t_step)
        cache_bytes, flops = attention_work(inp, w)
        if fp8:
            cache_bytes = int(inp.lens.sum()) * FP8_TOKEN_BYTES

        # e2e: per-step inputs uploaded from pinned host memory and the result
        # read back to pinned host memory, through the library's calls. Three
        # independent sessions (each with its own cache, weights and I/O
        # buffers) each hold one CUDA graph of upload + the step's calls +
        # download and take turns on three streams, so one batch's copies
        # overlap the others' compute, and one batch's GEMMs run on the SMs
        # another batch's attention leaves idle. Every step touches more than
        # L2 holds, so no flush runs in this loop.
        e2e = None
        if not args.no_e2e:
            sessions = [sess] + [DecodeSession(inp, dev, num_ctas=args.num_ctas,
                                               max_split=args.max_split, fp8=fp8)
                                 for _ in range(E2E_SESSIONS - 1)]
            ins, host_in, host_out0 = sess.pinned_step_buffers()
            host_outs = [host_out0] + [torch.empty_like(host_out0).pin_memory()
                                       for _ in range(E2E_SESSIONS - 1)]
            h2d, d2h = DecodeSession.step_io_bytes(ins, host_out0)
            graphs = [capture_io_step(s_, host_in, host_outs[i])
                      for i, s_ in enumerate(sessions)]
            streams = [torch.cuda.Stream() for _ in sessions]
            run_e2e_graphs(graphs, streams, 8)
            torch.cuda.synchronize()
            E = max(args.e2e_steps, K)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            barrier()
            e0.record(stream)
            for s_ in streams:
                s_.wait_stream(stream)
            host_s = run_e2e_graphs(graphs, streams, E)
            for s_ in streams:
                stream.wait_stream(s_)
            e1.record(stream)
            barrier()
            t_e2e = e0.elapsed_time(e1) / E
            (t_e2e,) = max_over_ranks([t_e2e], dist, dev, world)
            for s_ in sessions:
                assert s_.read_status() == 0, "device status in the end-to-end loop"
            # the host link alone: the same per-step copies timed by themselves
            def copy_ms(fn, n=20):
                a_, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                fn()
                a_.record(stream)
                for _ in range(n):
                    fn()
                b_.record(stream)
                torch.cuda.synchronize()
                return a_.elapsed_time(b_) / n

            dev_in = sess.io_inputs()
            t_h2d = copy_ms(lambda: [d.copy_(h_, non_blocking=True) for d, h_ in zip(dev_in, host_in)])
            t_d2h = copy_ms(lambda: host_outs[0].copy_(sess.u, non_blocking=True))
            e2e = {"value": whole_job_rate(world, tokens, t_e2e), "unit": UNIT,
                   "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
                   "host_link": {"h2d_ms": t_h2d, "d2h_ms": t_d2h,
                                 "h2d_gbs": h2d / t_h2d / 1e6, "d2h_gbs": d2h / t_d2h / 1e6},
                   "ms_per_step": t_e2e, "steps": E,
                   "host_enqueue_us_per_step": host_s / E * 1e6,
                   "method": f"{E2E_SESSIONS} sessions (independent batches), each one "
                             "CUDA graph of upload (pinned host -> device) + the step's "
                             "library calls + download (device -> pinned host); steps take "
                             f"turns on {E2E_SESSIONS} streams so one batch's copies and "
                             "GEMMs overlap another's attention; no L2 flush (each step "
                             "touches > L2)"}
            del graphs, sessions

        configs = {}
        if not args.no_configs and world == 1:
            for key in [c for c in args.configs.split(",") if c and c != args.workload]:
                name, _, variant = key.partition(":")
                wc = synth.WORKLOADS[name]
                if wc.layer:
                    configs[key] = measure_layer_config(name, dev, flush, stream, max(5, K // 2),
                                                        peaks, folded=variant == "folded")
                else:
                    configs[key] = measure_decode_config(name, dev, flush, stream,
                                                         max(5, K // 2), peaks, args,
                                                         fp8=variant == "fp8")
        clocks.mark_end()

    gbs = cache_bytes / (t_attn / 1e3) / 1e9
    tfs = flops / (t_attn / 1e3) / 1e12
    t_mem = cache_bytes / (peaks["hbm_gbs"] * 1e9)
    t_tc = flops / (peaks["bf16_tflops"] * 1e12)
    src_hash = decode_sources_hash()
    traffic = TRAFFIC.get((src_hash, args.workload, args.cache))
    roof = {
        "kernel": "mla_decode_attention (decode + combine kernels)",
        "bound": "hbm" if t_mem >= t_tc else "tensor",
        "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
        "frac": gbs / peaks["hbm_gbs"], "traffic": traffic,
        "algorithmic_bytes": cache_bytes, "algorithmic_flops": flops,
        "tensor": {"achieved": tfs, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                   "frac": tfs / peaks["bf16_tflops"]},
        "roofline_us": max(t_mem, t_tc) * 1e6, "measured_us": t_attn * 1e3,
        "frac_of_roofline": max(t_mem, t_tc) / (t_attn / 1e3),
        "spec": {"hbm_gbs": SPEC_PEAKS["hbm_gbs"], "bf16_tflops": SPEC_PEAKS["bf16_tflops"],
                 "frac_of_roofline": max(cache_bytes / (SPEC_PEAKS["hbm_gbs"] * 1e9),
                                         flops / (SPEC_PEAKS["bf16_tflops"] * 1e12))
                 / (t_attn / 1e3)},
        "peak_source": f"{peak_src} (MEASURED_PEAKS.json burst figures)"
        if peak_src == "measured" else "fallback", "sources": src_hash,
    }
    # the absorb GEMM (with the q RoPE pack and the cache append, bf16 or FP8,
    # in the same launch), decode, [combine], out_absorb per timed step, plus
    # decode [+ combine] per timed attention call
    combine = 1 if sess.info.num_combine > 0 else 0
    per_step = 3 + combine
    launches_timed = K * per_step + K * (1 + combine)
    out = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": t_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "cache": "FP8 (E4M3 latent, bf16 k^R, per-token scale)" if fp8 else "bf16",
        "config": workload_config(w, inp, sess, args.ramp_seconds),
        "cache_gbs": cache_bytes / (t_step / 1e3) / 1e9 * world,
        "attention_ms": t_attn,
        "step_ms_stats": dist_stats(step_ms), "attention_ms_stats": dist_stats(attn_ms),
        "roofline": roof,
        "e2e": e2e,
        "gpu_launches": launches_timed,
        "clocks": clocks.summary(),
        "configs": configs or None,
    }
    if rank == 0 and world == 1 and not args.no_cpu:
        tps, desc, _ = oracle_sample(w, inp, budget_s=12.0)
        out["cpu_baseline"] = {"value": tps, "unit": UNIT, "cores": cpu_threads(),
                               "kind": "oracle", "sample": desc}
    if rank == 0:
        print(json.dumps(out), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
