#!/usr/bin/env python
"""Benchmark of the paged MLA decode hot path on B200.

One step = one pass of the whole path over one batch: page table, int32 lengths and split
plan in one launch (build_decode_metadata: the work of build_block_table and
get_mla_metadata) and attention with its split merge (mla_decode_paged),
on inputs resident in HBM.  Default workload: the DeepSeek-V3-shaped decode (bs 64,
128 heads, q_len 1, L ~ U[1024, 4096], bf16 latent KV 576 wide, 64-token pages in a
shuffled pool 1.25x the need).  L2 is flushed (512 MB written, then 512 MB read) between timed steps,
outside the step's CUDA events.

Reported (one JSON line on rank 0):
  value        aggregate KV GB/s over all ranks: algorithmic KV bytes (each request's
               KV read once) per step x ranks / max-over-ranks step time;
  roofline     the attention call (decode kernel + merge) against the measured HBM peak:
               algorithmic (KV + Q) bytes / its CUDA-event time;
  e2e          the same metric through the public API with the step's inputs (q,
               seq_lens, req_pool_indices) copied from pinned host memory and
               the outputs (o, lse) copied back inside the timed region, the copies of
               neighbouring steps overlapping the step's compute on their own streams;
  per_config   every workload (tiny, DeepSeek-V3 decode, skewed long context, fp8 cache,
               target-verify): us per call, metadata us, roofline and clocks, from a short
               timed run each;
  cpu_baseline the CPU fp64 oracle on a bounded sample of the same workload (rank 0, N=1).
Multi-GPU: independent replicas (the path has no exchange step); NCCL is used only for
the barrier and the max-over-ranks reduction of the timings.

--impl reference times the CPU oracle (the reference arm) on the same workload.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "paged MLA decode: KV GB/s, TFLOP/s and % roofline; µs per call"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
KERNELS_PER_STEP = 3  # metadata (page table, lengths and plan in one launch), attention, split merge


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["b200", "reference"], default="b200")
    ap.add_argument("--config", type=int, default=2, choices=[1, 2, 3, 4, 5])
    ap.add_argument("--flush-mb", type=int, default=512)
    ap.add_argument("--e2e-steps", type=int, default=300)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="target CPU time of the oracle sample")
    ap.add_argument("--no-per-config", action="store_true",
                    help="time only the --config workload")
    ap.add_argument("--per-config-steps", type=int, default=50,
                    help="timed steps of each other workload in the per_config entries")
    ap.add_argument("--q-fp8", action="store_true",
                    help="the fp8-cache workload (--config 4) with its queries handed over as e4m3 "
                         "codes, the backend's fp8 recipe")
    args = ap.parse_args(argv)
    if args.q_fp8 and args.config != 4:
        ap.error("--q-fp8 applies to the fp8-cache workload, --config 4")
    return args


def dist_env():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def replica_seed(config: int, rank: int) -> int:
    """Each replica owns its own pool and batch: distinct seeds per rank."""
    return 1000 + config + 100 * rank


def reduce_max_over_ranks(values, device, world):
    """Every rank's timings -> the maximum over ranks (the slowest replica sets the job
    time).  One all-reduce on the default process group; identity for a single rank."""
    import torch
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def job_value(world, kv_bytes_per_replica, step_ms):
    """Whole-job KV GB/s: every replica's algorithmic KV bytes / the max-over-ranks step time."""
    return world * kv_bytes_per_replica / (step_ms * 1e-3) / 1e9


TRAFFIC_KEYS = {1: "tiny_decode", 2: "deepseek_v3_decode", 3: "skewed_long_context", 4: "fp8_kv_decode",
                "4q8": "fp8_kv_fp8_q_decode", 5: "target_verify"}


# The sources the decode kernel is built from: its body, the PTX helpers it inlines, and the
# translation unit with its tensor maps and launch configuration.
DECODE_KERNEL_SOURCES = ("decode.cuh", "combine.cuh", "ptx.cuh", "mla_b200.cu")


def kernel_sources_sha():
    import hashlib
    h = hashlib.sha256()
    for name in DECODE_KERNEL_SOURCES:
        with open(os.path.join(ROOT, "paged_kv_mla_create_b200", "csrc", name), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def captured_traffic(config):
    """DRAM bytes per decode launch from the committed ncu capture of this workload, or None
    when there is none or the kernel sources changed since it was taken."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            rec = json.load(f).get(TRAFFIC_KEYS.get(config, ""), None)
        if rec and rec["csrc_sha256_prefix"] == kernel_sources_sha():
            return float(rec["dram_bytes_per_launch"])
    except Exception:
        pass
    return None


def roofline_entry(kv_bytes, q_bytes, flops, attn_s, peaks, peak_src, is_fp8, traffic):
    """The bench line's roofline object for one attention call of attn_s seconds: the slower of
    the algorithmic KV + Q bytes at the measured HBM bandwidth and the algorithmic FLOPs at the
    dense tensor peak of the cache's precision -- the measured bf16 peak for a bf16 cache, the
    fp8 peak (the measured bf16 peak x the nominal fp8 / bf16 ratio 2) for an e4m3 cache.  An
    e4m3 cache is also reported against the bf16 peak, the rate of the f16 MMAs it runs."""
    tensor_peak = peaks["bf16_tflops"] * (2.0 if is_fp8 else 1.0)
    t_hbm = (kv_bytes + q_bytes) / (peaks["hbm_gbs"] * 1e9)
    t_tc = flops / (tensor_peak * 1e12)
    achieved_gbs = (kv_bytes + q_bytes) / attn_s / 1e9
    achieved_tf = flops / attn_s / 1e12
    if t_hbm >= t_tc:
        roof = {"bound": "hbm", "achieved": achieved_gbs, "peak": peaks["hbm_gbs"],
                "unit": "GB/s", "frac": achieved_gbs / peaks["hbm_gbs"]}
    else:
        roof = {"bound": "tensor", "achieved": achieved_tf, "peak": tensor_peak,
                "unit": "TFLOP/s", "frac": achieved_tf / tensor_peak}
    roof.update({"traffic": traffic, "traffic_unit": "bytes per launch",
                 "peak_source": f"{peak_src} (MEASURED_PEAKS.json burst)"
                 if peak_src == "measured" else "fallback",
                 "kernel": "mla_decode_paged call (decode kernel + split merge)",
                 "roofline_time_us": max(t_hbm, t_tc) * 1e6,
                 "frac_of_roofline_time": max(t_hbm, t_tc) / attn_s,
                 "tensor_peak_dtype": "fp8" if is_fp8 else "bf16"})
    if is_fp8:
        roof.update({"tensor_peak_tflops": tensor_peak,
                     "tensor_peak_source": "measured bf16 peak x 2 (nominal fp8 / bf16 ratio)",
                     "frac_of_bf16_peak": achieved_tf / peaks["bf16_tflops"]})
    return roof


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def algorithmic(wl):
    """KV bytes (each request's KV once), Q bytes and FLOPs of one attention call."""
    elem = 1 if wl.is_fp8 else 2
    L = [int(x) for x in wl.cache_seqlens.tolist()]
    kv = sum(L) * 576 * elem
    qb = wl.bs * wl.q_len * wl.h * 576 * 2
    flops = 0
    for Lb in L:
        for i in range(wl.q_len):
            allowed = max(0, min(Lb, Lb - wl.q_len + i + 1)) if wl.causal else Lb
            flops += 2 * wl.h * allowed * (576 + 512)
    return kv, qb, flops


def workload_config(cfg_index, wl, world, flush_mb):
    from paged_kv_mla_create_b200.workloads import CONFIGS
    c = CONFIGS[cfg_index]
    return {"workload": wl.name if wl.q_is_fp8 else c["name"], "batch": wl.bs, "heads": wl.h,
            "q_len": wl.q_len, "kv_dtype": "fp8_e4m3" if wl.is_fp8 else "bf16",
            "q_dtype": "fp8_e4m3" if wl.q_is_fp8 else "bf16", "page": 64,
            "head_dim": 576, "head_dim_v": 512,
            "l2": f"flushed between timed steps ({flush_mb} MB written, then another {flush_mb} MB read, "
                  "outside the step events: no input of the step and no dirty line left in L2)",
            "launch": "each step replays one CUDA graph of the metadata call (page table, lengths "
                      "and plan in one launch) and the attention call, the attention kernel a "
                      "programmatic dependent of the metadata kernel",
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU"}


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 100 ms while running."""
    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None
        self.out = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", self.gpu_id], stdout=self.out, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.out.flush()
        self.out.seek(0)
        rows = [l.strip().split(",") for l in self.out.read().splitlines() if l.strip()]
        os.unlink(self.out.name)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            r = [x.strip() for x in r]
            if len(r) < 10:
                continue
            try:
                sm.append(float(r[2]))
                smax.append(float(r[3]))
            except ValueError:
                continue
            for n, v in zip(names, r[6:10]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None, "reasons": sorted(reasons),
                "samples": len(sm)}


def gpu_id_for(device) -> str:
    import torch
    try:
        u = torch.cuda.get_device_properties(device).uuid
        s = str(u)
        return s if s.startswith("GPU-") else "GPU-" + s
    except Exception:
        return str(device.index or 0)


def _oracle_rows(wl, rows):
    import oracle
    t0 = time.perf_counter()
    oracle.mla_decode_rows(wl.q, wl.kv_cache, wl.req_to_token, wl.req_pool_indices,
                           wl.cache_seqlens, rows, wl.softmax_scale, wl.causal,
                           kv_is_fp8=wl.is_fp8,
                           descale_q=float(wl.descale_q[0]) if wl.descale_q is not None else 1.0,
                           descale_k=float(wl.descale_k[0]) if wl.descale_k is not None else 1.0,
                           q_is_fp8=wl.q_is_fp8)
    return time.perf_counter() - t0


def _row_sample(wl, n):
    """n query rows spread evenly over all requests and heads."""
    import numpy as np
    total = wl.bs * wl.q_len * wl.h
    n = int(max(1, min(total, n)))
    return np.unique(np.linspace(0, total - 1, n).round().astype(np.int64))


def _calibrate(wl):
    """Rows per second of the oracle on this host (one row per request)."""
    rows = _row_sample(wl, wl.bs)
    return len(rows) / max(_oracle_rows(wl, rows), 1e-6)


def cpu_baseline(wl, seconds):
    """The oracle as it stands on the host cores, on a bounded sample of rows spread over
    all requests and heads, scaled to KV GB/s by the fraction of rows processed."""
    import oracle
    kv_bytes, _, _ = algorithmic(wl)
    total = wl.bs * wl.q_len * wl.h
    rows = _row_sample(wl, _calibrate(wl) * seconds)
    dt = _oracle_rows(wl, rows)
    frac = len(rows) / total
    return {"value": kv_bytes * frac / dt / 1e9, "unit": "GB/s", "cores": oracle.num_threads(),
            "kind": "oracle",
            "sample": f"{len(rows)} of {total} query rows spread over all {wl.bs} requests, "
                      f"{dt:.1f} s; KV bytes scaled by the row fraction {frac:.4f}"}


def run_reference(args):
    """The reference arm: the CPU oracle, K timed steps of a bounded row sample each,
    sized so that warm-up plus timed steps take about two minutes of host time."""
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    import oracle
    from paged_kv_mla_create_b200 import workloads as W
    wl = W.make_workload(args.config, seed=replica_seed(args.config, 0), q_fp8=args.q_fp8)
    kv_bytes, _, _ = algorithmic(wl)
    total = wl.bs * wl.q_len * wl.h
    per_step = 120.0 / max(1, args.steps + args.warmup)
    rows = _row_sample(wl, _calibrate(wl) * per_step)
    for _ in range(args.warmup):
        _oracle_rows(wl, rows)
    times = [_oracle_rows(wl, rows) for _ in range(args.steps)]
    sec = statistics.median(times)
    frac = len(rows) / total
    value = kv_bytes * frac / sec / 1e9
    sample = (f"{len(rows)} of {total} query rows per step spread over all {wl.bs} requests; "
              f"KV bytes scaled by the row fraction {frac:.5f}")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": sec * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(args.config, wl, world, args.flush_mb),   # the GPU arm's config
            "cpu_baseline": {"value": value, "unit": "GB/s", "cores": oracle.num_threads(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


class Case:
    """One workload resident on the device, with its metadata / attention steps captured as
    CUDA graphs the way a serving engine replays them."""

    def __init__(self, cfg, seed, dev, flush_mb, q_fp8=False):
        import torch
        import paged_kv_mla_create_b200 as mla
        from paged_kv_mla_create_b200 import workloads as W
        self.mla, self.dev, self.cfg = mla, dev, cfg
        # the committed DRAM capture that belongs to this workload's kernel
        self.traffic_key = f"{cfg}q8" if q_fp8 else cfg
        self.host = host = W.make_workload(cfg, seed=seed, q_fp8=q_fp8)
        self.wl = host.to(dev)
        self.kv_bytes, self.q_bytes, self.flops = algorithmic(host)
        bs, q_len, h = host.bs, host.q_len, host.h
        self.parts = mla.num_sm_parts(q_len * h, 1, mla.sm_count(dev))
        self.bt = torch.empty((bs, host.max_pages), dtype=torch.int32, device=dev)
        self.md = torch.empty((self.parts, 8), dtype=torch.int32, device=dev)
        self.ns = torch.empty((bs + 1,), dtype=torch.int32, device=dev)
        self.cl = torch.empty((bs,), dtype=torch.int32, device=dev)
        self.o = torch.empty((bs, q_len, h, 512), dtype=torch.bfloat16, device=dev)
        self.lse = torch.empty((bs, q_len, h), dtype=torch.float32, device=dev)
        self.ws = torch.zeros((mla.workspace_bytes(bs, q_len, h, self.parts),), dtype=torch.uint8,
                              device=dev)
        self.flush = torch.empty((flush_mb << 20,), dtype=torch.uint8, device=dev)
        self.flush_rd = torch.ones((flush_mb << 20,), dtype=torch.uint8, device=dev)

    def flush_l2(self, i):
        self.flush.fill_(i & 0xFF)
        self.flush_rd.max()   # evicts the written lines while still outside the timed region

    def metadata(self, w):
        """Page table, int32 cache_seqlens and split plan: one launch."""
        host = self.host
        self.mla.build_decode_metadata(w.req_to_token, w.req_pool_indices, w.seq_lens, host.max_pages,
                                       host.q_len * host.h, 1, host.is_fp8,
                                       seq_len_add=host.num_draft_tokens,
                                       out=(self.bt, self.cl, self.md, self.ns))

    def attention(self, w, o=None, lse=None):
        host = self.host
        self.mla.mla_decode_paged(w.q, w.kv_cache, self.bt, self.cl, 512, self.md, self.ns,
                                  host.softmax_scale, host.causal, w.descale_q, w.descale_k,
                                  out=self.o if o is None else o, lse=self.lse if lse is None else lse,
                                  workspace=self.ws)

    def capture(self):
        import torch
        stream = torch.cuda.current_stream(self.dev)
        cap = torch.cuda.Stream(self.dev)
        cap.wait_stream(stream)
        with torch.cuda.stream(cap):
            self.metadata(self.wl)
            self.attention(self.wl)
        stream.wait_stream(cap)
        torch.cuda.synchronize(self.dev)
        self.g_step, self.g_meta, self.g_attn = (torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph(),
                                                 torch.cuda.CUDAGraph())
        with torch.cuda.graph(self.g_step):
            self.metadata(self.wl)
            self.attention(self.wl)
        with torch.cuda.graph(self.g_meta):
            self.metadata(self.wl)
        with torch.cuda.graph(self.g_attn):
            self.attention(self.wl)

    def release(self):
        for name in ("g_step", "g_meta", "g_attn"):
            if hasattr(self, name):
                delattr(self, name)

    def time_steps(self, steps, warmup, world, clocks=None):
        """Warm-up, then `steps` timed steps, each a replay of one graph holding the metadata
        call and the attention call (L2 flushed before each, outside its events), timed by an
        event pair around the step; then as many steps again as two graphs, the metadata call's
        and the attention call's, with an event between them, for the split into metadata and
        attention.  Returns (step_ms, attn_ms, meta_ms, clock record)."""
        import torch
        import torch.distributed as dist
        for i in range(warmup):
            self.flush_l2(i)
            self.metadata(self.wl)
            self.attention(self.wl)
        torch.cuda.synchronize(self.dev)
        if self.mla.read_device_error(self.dev) != 0:
            raise RuntimeError("device error word set during warm-up")
        self.capture()
        for i in range(3):
            self.flush_l2(i)
            self.g_step.replay()
            self.g_meta.replay()
            self.g_attn.replay()
        torch.cuda.synchronize(self.dev)
        stream = torch.cuda.current_stream(self.dev)
        # The timed steps: an event pair around each whole step (metadata then attention, one
        # graph, so that the attention kernel's set-up overlaps the metadata kernel).  The split
        # into metadata and attention needs an event between the two calls, which takes them
        # apart into two graphs and costs the step ~2.5 us by itself: it comes from a second
        # pass over as many steps.
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(steps)]
        ev3 = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(self.dev)
        if clocks is not None:
            clocks.start()
        for k in range(steps):
            self.flush_l2(k)
            ev[k][0].record(stream)
            self.g_step.replay()
            ev[k][1].record(stream)
        torch.cuda.synchronize(self.dev)
        if world > 1:
            dist.barrier()
        for k in range(steps):
            self.flush_l2(k)
            ev3[k][0].record(stream)
            self.g_meta.replay()
            ev3[k][1].record(stream)
            self.g_attn.replay()
            ev3[k][2].record(stream)
        torch.cuda.synchronize(self.dev)
        if world > 1:
            dist.barrier()
        clk = clocks.stop() if clocks is not None else None
        self.release()
        step_ms = sum(e[0].elapsed_time(e[1]) for e in ev) / steps
        attn_ms = sum(e[1].elapsed_time(e[2]) for e in ev3) / steps
        meta_ms = sum(e[0].elapsed_time(e[1]) for e in ev3) / steps
        return step_ms, attn_ms, meta_ms, clk

    def time_e2e(self, steps):
        """The same step end to end through the public API, from pinned host buffers: step k's
        inputs (q, seq_lens, req_pool_indices) are copied in on a copy stream
        while step k - 1 computes, and step k's o and lse are copied out on another while step
        k + 1 computes (two device buffer sets).  Every step's copies lie inside the timed
        region, which runs from the first copy in to the last copy out.  No L2 flush: the KV
        cache every step streams is larger than L2.  (cache_seqlens is not an input: the
        metadata launch derives it from seq_lens.)  Returns (ms per step, h2d, d2h bytes)."""
        import dataclasses
        import torch
        host, wl, dev = self.host, self.wl, self.dev
        pin = [t.pin_memory() for t in (host.q, host.seq_lens, host.req_pool_indices)]
        outs_h = [(torch.empty(self.o.shape, dtype=self.o.dtype, pin_memory=True),
                   torch.empty(self.lse.shape, dtype=self.lse.dtype, pin_memory=True)) for _ in range(2)]
        ins_d, outs_d, wls = [], [], []
        for _ in range(2):
            d = [torch.empty_like(t, device=dev) for t in pin]
            ins_d.append(d)
            outs_d.append((torch.empty_like(self.o), torch.empty_like(self.lse)))
            wls.append(dataclasses.replace(wl, q=d[0], seq_lens=d[1], req_pool_indices=d[2]))
        h2d = sum(t.numel() * t.element_size() for t in pin)
        d2h = sum(t.numel() * t.element_size() for t in outs_h[0])
        comp = torch.cuda.current_stream(dev)
        s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_comp = [torch.cuda.Event() for _ in range(2)]
        ev_out = [torch.cuda.Event() for _ in range(2)]
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

        def run(n, timed):
            torch.cuda.synchronize(dev)
            if timed:
                t0.record(comp)
            s_in.wait_stream(comp)
            s_out.wait_stream(comp)
            for k in range(n):
                j = k & 1
                if k >= 2:
                    s_in.wait_event(ev_comp[j])      # step k - 2 is done with input set j
                with torch.cuda.stream(s_in):
                    for dst, src in zip(ins_d[j], pin):
                        dst.copy_(src, non_blocking=True)
                    ev_in[j].record(s_in)
                comp.wait_event(ev_in[j])
                if k >= 2:
                    comp.wait_event(ev_out[j])       # step k - 2's outputs have left set j
                self.metadata(wls[j])
                self.attention(wls[j], o=outs_d[j][0], lse=outs_d[j][1])
                ev_comp[j].record(comp)
                s_out.wait_event(ev_comp[j])
                with torch.cuda.stream(s_out):
                    outs_h[j][0].copy_(outs_d[j][0], non_blocking=True)
                    outs_h[j][1].copy_(outs_d[j][1], non_blocking=True)
                    ev_out[j].record(s_out)
            comp.wait_stream(s_out)
            comp.wait_stream(s_in)
            if timed:
                t1.record(comp)
            torch.cuda.synchronize(dev)

        run(4, False)
        run(steps, True)
        return t0.elapsed_time(t1) / steps, h2d, d2h


class _NoGraph:
    def replay(self):
        pass


class ExtendCase(Case):
    """Extend with a cached prefix (ragged causal part over the new rows, paged part over the
    prefix, merge_state): 4 requests of the DeepSeek-V3 decode shape (128 heads, prefixes
    ~U[1024, 4096]) with 64 new tokens each.  One call is the whole extend (its page tables and
    plans are built inside it), so the metadata step is empty."""

    def __init__(self, seed, dev, flush_mb):
        import numpy as np
        import torch
        import paged_kv_mla_create_b200 as mla
        from paged_kv_mla_create_b200 import workloads as W
        self.mla, self.dev, self.cfg = mla, dev, "extend"
        self.traffic_key = None
        rng = np.random.default_rng(seed)
        prefix = [int(x) for x in rng.integers(1024, 4097, size=4)]
        e = 64
        self.host = host = W.make_case(prefix, h=128, q_len=e, verify=True, seed=seed,
                                       name="extend with cached prefix (bs 4, h 128, prefix ~U[1024, 4096], 64 new tokens, bf16)")
        self.wl = host.to(dev)
        pool = host.kv_cache.reshape(-1, 576)
        slots = torch.tensor([[int(host.req_to_token[host.req_pool_indices[b], prefix[b] + i]) for i in range(e)]
                              for b in range(host.bs)], dtype=torch.int64)
        self.k_new = pool[slots.reshape(-1)].reshape(host.bs, e, 576).contiguous().to(dev)
        self.prefix = torch.tensor(prefix, dtype=torch.int32, device=dev)
        self.mpp = max(-(-p // 64) for p in prefix)
        # the prefix rows once, the new rows once, q once; FLOPs of the causal new tokens over both
        self.kv_bytes, self.q_bytes, self.flops = algorithmic(host)
        self.o = torch.empty((host.bs, e, host.h, 512), dtype=torch.bfloat16, device=dev)
        self.lse = torch.empty((host.bs, e, host.h), dtype=torch.float32, device=dev)
        self.ws = torch.zeros((mla.extend_workspace_bytes(host.bs, e, host.h, self.mpp, mla.sm_count(dev)),),
                              dtype=torch.uint8, device=dev)
        self.flush = torch.empty((flush_mb << 20,), dtype=torch.uint8, device=dev)
        self.flush_rd = torch.ones((flush_mb << 20,), dtype=torch.uint8, device=dev)

    def metadata(self, w):
        pass

    def attention(self, w, o=None, lse=None):
        self.mla.extend_paged_prefix(w.q, self.k_new, w.kv_cache, w.req_to_token, w.req_pool_indices, self.prefix,
                                     self.mpp, self.host.softmax_scale, out=self.o if o is None else o,
                                     lse=self.lse if lse is None else lse, workspace=self.ws)

    def capture(self):
        import torch
        stream = torch.cuda.current_stream(self.dev)
        cap = torch.cuda.Stream(self.dev)
        cap.wait_stream(stream)
        with torch.cuda.stream(cap):
            self.attention(self.wl)
        stream.wait_stream(cap)
        torch.cuda.synchronize(self.dev)
        self.g_meta, self.g_attn = _NoGraph(), torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.g_attn):
            self.attention(self.wl)
        self.g_step = self.g_attn


def config_entry(case, step_ms, attn_ms, meta_ms, clk, peaks, peak_src):
    attn_s = attn_ms * 1e-3
    # metadata_us: the metadata call alone (its own graph, events around it); metadata_exposed_us:
    # what it adds to a step replayed as one graph, where it overlaps the attention kernel's set-up
    return {"workload": case.host.name, "us_per_call": attn_ms * 1e3,
            "metadata_us": meta_ms * 1e3, "us_per_step": step_ms * 1e3,
            "metadata_exposed_us": (step_ms - attn_ms) * 1e3,
            "kv_gbs_per_call": case.kv_bytes / attn_s / 1e9, "tflops": case.flops / attn_s / 1e12,
            "kv_bytes": case.kv_bytes, "q_bytes": case.q_bytes, "flops": case.flops,
            "roofline": roofline_entry(case.kv_bytes, case.q_bytes, case.flops, attn_s, peaks,
                                       peak_src, case.host.is_fp8, captured_traffic(case.traffic_key)),
            "clocks": clk}


def run_b200(args):
    import torch
    import torch.distributed as dist

    import paged_kv_mla_create_b200 as mla

    rank, world, local = dist_env()
    if world > 1:
        torch.cuda.set_device(local)
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local if world > 1 else torch.cuda.current_device())
    torch.cuda.set_device(dev)
    mla.library()
    peaks, peak_src = load_peaks()

    case = Case(args.config, replica_seed(args.config, rank), dev, args.flush_mb, q_fp8=args.q_fp8)
    K = args.steps
    clocks = ClockSampler(gpu_id_for(dev))
    step_ms, attn_ms, meta_ms, clk = case.time_steps(K, args.warmup, world, clocks)
    e2e_ms, h2d, d2h = case.time_e2e(max(1, min(args.e2e_steps, K)))
    err = mla.read_device_error(dev)
    step_ms, attn_ms, meta_ms, e2e_ms, err = reduce_max_over_ranks(
        [step_ms, attn_ms, meta_ms, e2e_ms, float(err)], dev, world)
    if err:
        raise RuntimeError(f"device error word {int(err)} after the timed run")
    head = config_entry(case, step_ms, attn_ms, meta_ms, clk, peaks, peak_src)
    host = case.host
    kv_bytes = case.kv_bytes
    del case
    torch.cuda.empty_cache()

    # every other workload, with a short timed run each (its own clock record)
    per_config = {f"{args.config}q8" if args.q_fp8 else str(args.config): head}
    if not args.no_per_config:
        # the five workloads, and the fp8-cache one with e4m3 queries (the backend's fp8 recipe)
        for cfg, q8 in ((1, False), (2, False), (3, False), (4, False), (4, True), (5, False)):
            if cfg == args.config and q8 == args.q_fp8:
                continue
            c = Case(cfg, replica_seed(cfg, rank), dev, args.flush_mb, q_fp8=q8)
            sm, am, mm, ck = c.time_steps(max(1, min(K, args.per_config_steps)), max(3, min(args.warmup, 5)),
                                          world, ClockSampler(gpu_id_for(dev)))
            e = mla.read_device_error(dev)
            sm, am, mm, e = reduce_max_over_ranks([sm, am, mm, float(e)], dev, world)
            if e:
                raise RuntimeError(f"device error word {int(e)} after workload {cfg}")
            per_config[f"{cfg}q8" if q8 else str(cfg)] = config_entry(c, sm, am, mm, ck, peaks, peak_src)
            del c
            torch.cuda.empty_cache()
        # the extend piece (new tokens over their own rows and a cached prefix, merged)
        c = ExtendCase(replica_seed(2, rank) + 7, dev, args.flush_mb)
        sm, am, mm, ck = c.time_steps(max(1, min(K, args.per_config_steps)), max(3, min(args.warmup, 5)), world,
                                      ClockSampler(gpu_id_for(dev)))
        e = mla.read_device_error(dev)
        sm, am, mm, e = reduce_max_over_ranks([sm, am, mm, float(e)], dev, world)
        if e:
            raise RuntimeError(f"device error word {int(e)} after the extend workload")
        per_config["extend"] = config_entry(c, sm, am, mm, ck, peaks, peak_src)
        del c
        torch.cuda.empty_cache()

    if rank != 0:
        if world > 1:
            dist.destroy_process_group()
        return 0
    value = job_value(world, kv_bytes, step_ms)
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None,
        "dtype": ("e4m3/f16" if host.q_is_fp8 else "f16") if host.is_fp8 else "bf16",
        "data": "synthetic",
        "config": workload_config(args.config, host, world, args.flush_mb),
        "us_per_call": head["us_per_call"], "metadata_us": head["metadata_us"],
        "metadata_exposed_us": head["metadata_exposed_us"],
        "kv_gbs_per_call": head["kv_gbs_per_call"], "tflops": head["tflops"],
        "tensor_frac": head["tflops"] / peaks["bf16_tflops"],
        "roofline": head["roofline"],
        "e2e": {"value": job_value(world, kv_bytes, e2e_ms), "unit": "GB/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
                "overlap": "inputs of step k+1 copied in and outputs of step k-1 copied out on "
                           "their own streams while step k computes"},
        "gpu_launches": KERNELS_PER_STEP * K,
        "clocks": clk,
        "per_config": per_config,
    }
    if world == 1 and not args.no_cpu_baseline:
        cb = cpu_baseline(host, args.cpu_seconds)
        line["cpu_baseline"] = cb
    print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        return run_reference(args)
    return run_b200(args)


if __name__ == "__main__":
    sys.exit(main())
