#!/usr/bin/env python
"""Decode-attention throughput on B200: KV GB/s, % of measured HBM peak, us/step.

One step = one gqa_decode call (one layer's decode attention for one batch) on a
seeded synthetic workload already resident in HBM.  Default workload: the
Llama-3-8B-shaped decode step (B=16, Hq=32, Hkv=8, D=128, L=8192, contiguous,
1% of keys x8).  L2 is flushed (256 MiB write) before every timed step, and
each step is timed with CUDA events on the launching stream.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
  python bench.py --impl reference ...     # the fp64 CPU oracle on host cores

Under torchrun every rank runs the same workload on its own GPU (independent
batches: weak scaling, no collective on the data path); rank 0 prints one JSON
line with the whole-job throughput computed from the slowest rank.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import workloads  # noqa: E402

METRIC = "decode-attn KV GB/s & % of B200 HBM peak; µs/step at 1 GPU"
SPEC_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
L2_FLUSH_BYTES = 256 << 20
_CSRC = "gqa_decode_attention_attn_b200/csrc/"
# The sources each kernel is compiled from (a traffic record is valid while they
# are unchanged).
KERNEL_SOURCES = {
    "tc": [_CSRC + f for f in ("decode_tc.cuh", "gather_merge.cuh", "schedule.cuh", "tc.cuh",
                               "ptx.cuh")],
    "simt": [_CSRC + f for f in ("decode_simt.cuh", "schedule.cuh", "ptx.cuh")],
    "wide": [_CSRC + f for f in ("decode_tc_wide.cuh", "decode_tc.cuh", "gather_merge.cuh",
                                 "schedule.cuh", "tc.cuh", "ptx.cuh")],
}


def plan_for(gq, p, num_splits: int, device: int) -> dict:
    """What the library launches for this problem and schedule (gqa_decode_plan):
    the kernel, its template parameters, grid and LeanTiles."""
    return gq.decode_plan(p.B, p.Hq, p.Hkv, p.D, p.block_size, p.paged, p.num_blocks,
                          kv_fp8=p.meta.get("kv_elem_bytes") == 1, num_splits=num_splits,
                          seq_lens_host=p.seq_lens.to(torch.int32), device=device)


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="llama3_8b", choices=sorted(workloads.WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--schedule", choices=["auto", "streamk", "fixed"], default="auto",
                    help="auto: gqa_decode_auto (the library's runtime schedule selection); "
                         "streamk: gqa_decode; fixed: the fixed-split comparator "
                         "(gqa_decode_fixed_split) with --splits chunks per segment")
    ap.add_argument("--splits", type=int, default=0,
                    help="chunks per segment for --schedule fixed (0: enough chunks for "
                         "one CTA per SM, FlashDecoding's usual choice)")
    ap.add_argument("--cpu-seconds", type=float, default=10.0,
                    help="target duration of the CPU-baseline sample")
    ap.add_argument("--workloads", default="default",
                    help="comma-separated workloads timed after the headline in the same run "
                         "(default: the other configurations and sweep points when the "
                         "headline is the default llama3_8b at 1 GPU; '' for none)")
    return ap.parse_args()


def hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


def kernel_source_hash(kernel: str) -> str:
    """Hash of the sources of the named kernel (a gqa_decode_plan kernel name)."""
    h = hashlib.sha256()
    kind = "wide" if "tc_wide_kernel" in kernel else "tc" if "tc_kernel" in kernel else "simt"
    for rel in KERNEL_SOURCES[kind]:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(workload: str, kernel: str):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on the
    current source of the kernel (else None)."""
    path = os.path.join(ROOT, "profiles", f"decode_{workload}_traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
    except (OSError, ValueError):
        return None
    if rec.get("kernel_source_sha256_16") != kernel_source_hash(kernel):
        return None
    return rec.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled every 100 ms."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.samples = []
        self.proc = None
        self.gpu = gpu_index
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", str(self.gpu)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) >= 9:
                self.samples.append((time.time(), parts))

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        if self.thread is not None:
            self.thread.join(timeout=5)

    def summary(self, t0: float, t1: float):
        inside = [s for t, s in self.samples if t0 <= t <= t1]
        window = "timed"
        if not inside:
            inside = [s for _, s in self.samples]
            window = "whole run (timed region shorter than the sampling period)"
        if not inside:
            return None

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None

        sm = [num(s[1]) for s in inside if num(s[1]) is not None]
        smax = [num(s[2]) for s in inside if num(s[2]) is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for s in inside for i in range(4)
                          if s[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": reasons, "samples": len(inside), "window": window,
                "power_w_max": max((num(s[3]) or 0.0) for s in inside)}


def workload_config(p) -> dict:
    lens = p.seq_lens.tolist()
    cfg = {"workload": p.name, "B": p.B, "Hq": p.Hq, "Hkv": p.Hkv, "D": p.D,
           "kv_len": lens[0] if len(set(lens)) == 1 else
           {"min": min(lens), "max": max(lens), "mean": sum(lens) / len(lens)},
           "cache": f"paged, {p.block_size}-token blocks" if p.paged else "contiguous",
           "algorithmic_bytes_per_step": p.algorithmic_bytes(),
           "block_table_bytes_per_step": p.block_table_bytes(),
           "l2": "flushed before every timed step (256 MiB write)"}
    return cfg


def _oracle_chunk(p, threads: int) -> int:
    """Whole requests per oracle call so that every host thread gets query rows."""
    return max(1, min(p.B, -(-threads // p.Hq)))


def _sample_bytes(p, b0: int, b1: int) -> int:
    L = sum(int(x) for x in p.seq_lens[b0:b1])
    eb = int(p.meta.get("kv_elem_bytes", 2))
    return 2 * eb * p.Hkv * p.D * L + 4 * (b1 - b0) * p.Hq * p.D


def cpu_oracle_sample(p, target_s: float, gpu_out=None):
    """Time the fp64 oracle as it stands on a bounded sample of the workload: groups
    of whole requests, in order, until about target_s seconds have passed.  With
    gpu_out (the timed steps' output), the oracle rows it computed are also compared
    with it: max-abs and rel-RMS error over the sampled requests."""
    import oracle
    threads = oracle.host_threads()
    oracle.default()
    chunk = _oracle_chunk(p, threads)
    got = None if gpu_out is None else gpu_out.float().cpu().double().numpy().reshape(-1, p.D)
    max_abs, sq_err, sq_ref, rows_cmp = 0.0, 0.0, 0.0, 0
    done_bytes, reqs, b = 0, 0, 0
    t0 = time.perf_counter()
    while True:
        b1 = min(p.B, b + chunk)
        ref = oracle.gqa_decode(p.q, p.k_cache, p.v_cache, p.block_table, p.seq_lens, p.scale,
                                rows=(b * p.Hq, b1 * p.Hq), threads=threads)
        if got is not None and reqs < p.B:  # each request compared once
            d = got[b * p.Hq:b1 * p.Hq] - ref
            max_abs = max(max_abs, float(np.abs(d).max()) if d.size else 0.0)
            sq_err += float((d * d).sum())
            sq_ref += float((ref * ref).sum())
            rows_cmp += (b1 - b) * p.Hq
        done_bytes += _sample_bytes(p, b, b1)
        reqs += b1 - b
        b = 0 if b1 == p.B else b1
        if time.perf_counter() - t0 >= target_s:
            break
    dt = time.perf_counter() - t0
    res = {"value": done_bytes / dt / 1e9, "unit": "GB/s",
           "cores": min(threads, chunk * p.Hq), "kind": "oracle",
           "sample": f"{reqs} whole requests (all {p.Hq} heads each) of {p.name}, "
                     f"{done_bytes / 1e6:.1f} MB of K+V+Q+O in {dt:.1f} s"}
    if got is not None:
        res["parity_of_sample"] = {
            "rows": rows_cmp, "max_abs": max_abs,
            "rel_rms": (sq_err / sq_ref) ** 0.5 if sq_ref > 0 else 0.0,
            "bar": "max-abs <= 1e-2, rel-RMS <= 2e-3 (gpu bf16 output vs fp64 oracle)"}
    return res


def run_reference(args, rank: int):
    """The reference arm: the fp64 CPU oracle on the host cores, one bounded sample
    of the workload (a group of whole requests) per step."""
    if rank != 0:
        return
    import oracle
    p = workloads.workload(args.workload)
    threads = oracle.host_threads()
    oracle.default()
    chunk = _oracle_chunk(p, threads)
    per_step, total_bytes = [], 0
    fp8 = workloads.fp8_caches(p) if p.meta.get("kv_elem_bytes") == 1 else None

    def step(i):
        b0 = (i * chunk) % p.B
        b1 = min(p.B, b0 + chunk)
        if fp8:
            oracle.gqa_decode_fp8(p.q, fp8[0], fp8[1], fp8[2], fp8[3], p.block_table, p.seq_lens,
                                  p.scale, rows=(b0 * p.Hq, b1 * p.Hq), threads=threads)
        else:
            oracle.gqa_decode(p.q, p.k_cache, p.v_cache, p.block_table, p.seq_lens, p.scale,
                              rows=(b0 * p.Hq, b1 * p.Hq), threads=threads)
        return _sample_bytes(p, b0, b1)

    for i in range(args.warmup):
        step(i)
    for i in range(args.steps):
        t = time.perf_counter()
        total_bytes += step(i)
        per_step.append(time.perf_counter() - t)
    secs = sum(per_step)
    ms = 1e3 * secs / len(per_step)
    value = total_bytes / secs / 1e9
    cores = min(threads, chunk * p.Hq)
    sample = f"{chunk} whole request(s) (all {p.Hq} heads) of {p.name} per step"
    line = {"metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded N(0,1) bf16 q/K/V; no trained weights)",
            "impl": "reference", "config": workload_config(p),
            "cpu_baseline": {"value": value, "unit": "GB/s", "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# Workloads the default run times after the headline, each in the same process and
# on the same GPU (the other configurations of the metric and the sweep points).
EXTRA_WORKLOADS = ("long_256k", "varlen_paged", "llama3_8b_fp8", "tiny", "sweep_32_32_128",
                   "sweep_32_8_128", "sweep_64_4_128", "sweep_64_1_128", "sweep_32_8_64",
                   "sweep_16_4_256")
EXTRA_STEPS = 200


class Runner:
    """One workload resident on the GPU and the call that runs one decode step of it
    (the schedule as the library plans it: gqa_decode_plan)."""

    def __init__(self, gq, p, dev, args, flush):
        self.gq, self.p, self.dev, self.flush = gq, p, dev, flush
        self.fp8 = p.meta.get("kv_elem_bytes") == 1
        self.d = p.to(dev)
        if self.fp8:  # the cache as FP8 E4M3 bytes with per-tensor scales
            k8, v8, self.k_scale, self.v_scale = workloads.fp8_caches(p)
            self.d.k_cache, self.d.v_cache = k8.to(dev), v8.to(dev)
        self.out = torch.empty_like(self.d.q)
        self.ws = gq.Workspace(dev)
        self.stream = torch.cuda.current_stream(dev)
        self.lens_host = p.seq_lens.to(torch.int32).contiguous()
        sms = torch.cuda.get_device_properties(dev).multi_processor_count
        # FP8 caches: gqa_decode_fp8_auto, or gqa_decode_fp8 (stream-K) for any other
        # --schedule (the fixed-split comparator has no FP8 form).
        self.mode = ("auto" if args.schedule == "auto" else "streamk") if self.fp8 \
            else args.schedule
        if self.mode == "fixed":
            segs = p.B * p.Hkv * -(-p.G // 16)
            self.splits = args.splits if args.splits > 0 else max(1, -(-sms // segs))
        else:
            self.splits = -1 if self.mode == "auto" else 0
        self.plan = plan_for(gq, p, self.splits, dev.index)
        ns = self.plan["num_splits"]
        what = ("stream-K" if ns == 0 else "one CTA per (request, KV head)" if ns == 1
                else f"fixed split x{ns}")
        self.schedule = (f"auto: {what}" if self.mode == "auto" else what) + \
            (" (FP8 cache)" if self.fp8 else "")

    def launches_per_step(self) -> int:
        return 2 if self.plan["merge_launch"] else 1

    def step(self):
        gq, d, p = self.gq, self.d, self.p
        kw = dict(out=self.out, scale=p.scale, workspace=self.ws, stream=self.stream)
        if self.fp8 and self.mode == "auto":
            gq.gqa_decode_fp8_auto(d.q, d.k_cache, d.v_cache, self.k_scale, self.v_scale,
                                   d.block_table, d.seq_lens, self.lens_host, **kw)
        elif self.fp8:
            gq.gqa_decode_fp8(d.q, d.k_cache, d.v_cache, self.k_scale, self.v_scale,
                              d.block_table, d.seq_lens, **kw)
        elif self.mode == "fixed":
            gq.gqa_decode_fixed_split(d.q, d.k_cache, d.v_cache, d.block_table, d.seq_lens,
                                      self.splits, **kw)
        elif self.mode == "auto":
            gq.gqa_decode_auto(d.q, d.k_cache, d.v_cache, d.block_table, d.seq_lens,
                               self.lens_host, **kw)
        else:
            gq.gqa_decode(d.q, d.k_cache, d.v_cache, d.block_table, d.seq_lens, **kw)

    def warm(self, n: int):
        for _ in range(max(3, n)):
            self.flush.fill_(1)
            self.step()
        torch.cuda.synchronize(self.dev)
        if self.ws.status():
            raise SystemExit(f"{self.p.name}: device status error during warm-up")

    def timed(self, steps: int):
        """Per-step milliseconds (CUDA events on the launching stream around each
        step; L2 flushed by a 256 MiB write before each) and the whole region's."""
        starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
        ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
        region0 = torch.cuda.Event(enable_timing=True)
        region1 = torch.cuda.Event(enable_timing=True)
        region0.record(self.stream)
        for i in range(steps):
            self.flush.fill_(i & 0xFF)
            starts[i].record(self.stream)
            self.step()
            ends[i].record(self.stream)
        region1.record(self.stream)
        torch.cuda.synchronize(self.dev)
        if self.ws.status():
            raise SystemExit(f"{self.p.name}: device status error during the timed steps")
        return [s.elapsed_time(e) for s, e in zip(starts, ends)], region0.elapsed_time(region1)

    def floor(self, steps: int):
        """The streaming floor of this step: gqa_stream_floor over the same number of
        K and V bytes, read from the workload's own cache buffers, on every SM, timed
        like the step (L2 flushed before each, CUDA events).  Mean and median us."""
        gq, d, p = self.gq, self.d, self.p
        tile = gq.FLOOR_TILE_BYTES
        kv = (p.algorithmic_bytes() - 4 * p.B * p.Hq * p.D) // 2  # bytes of K (= of V)
        nbytes = max(tile, kv // tile * tile)
        sms = torch.cuda.get_device_properties(self.dev).multi_processor_count
        run = lambda: gq.stream_floor(d.k_cache, d.v_cache, nbytes, sms, self.ws, self.stream)
        for _ in range(3):
            self.flush.fill_(1)
            run()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(steps)]
        for i, (a, b) in enumerate(ev):
            self.flush.fill_(i & 0xFF)
            a.record(self.stream)
            run()
            b.record(self.stream)
        torch.cuda.synchronize(self.dev)
        if self.ws.status():
            raise SystemExit(f"{p.name}: device status error in the streaming floor")
        us = [a.elapsed_time(b) * 1e3 for a, b in ev]
        return sum(us) / len(us), statistics.median(us), 2 * nbytes, sms

    def timeline(self):
        """One more step, untimed and after an L2 flush, through gqa_decode_timeline
        with the schedule the timed steps ran: per-CTA start/end (%globaltimer) and
        SM, summed up as span, busy fraction and tail idle, plus the phase times of
        the tensor-core CTAs."""
        if self.fp8:
            return None
        ns = self.plan["num_splits"]
        d, p = self.d, self.p
        self.flush.fill_(0)
        _, tl = self.gq.gqa_decode_timeline(d.q, d.k_cache, d.v_cache, d.block_table,
                                            d.seq_lens, num_splits=ns, out=self.out,
                                            scale=p.scale, workspace=self.ws,
                                            stream=self.stream)
        torch.cuda.synchronize(self.dev)
        if self.ws.status():
            raise SystemExit(f"{p.name}: device status error during the timeline step")
        summary = self.gq.timeline_summary(tl)
        summary["source"] = ("one untimed step through gqa_decode_timeline, same schedule: "
                             "per-CTA %globaltimer at entry and exit, %smid")
        return summary


def extra_entry(r: Runner, steps: int, warmup: int, peak: float) -> dict:
    """One workload of the multi-workload block: timed like the headline, fewer steps."""
    r.warm(warmup)
    per, _ = r.timed(steps)
    ms = sum(per) / len(per)
    gbs = r.p.algorithmic_bytes() / (ms / 1e3) / 1e9
    tl = r.timeline()
    floor_us, _, _, _ = r.floor(steps)
    e = {"us_per_step": ms * 1e3, "us_per_step_median": statistics.median(per) * 1e3,
         "GB_per_s": gbs, "frac": gbs / peak, "steps": steps,
         "algorithmic_bytes": r.p.algorithmic_bytes(), "kernel": r.plan["kernel_name"],
         "schedule": r.schedule, "grid": r.plan["grid"], "tiles": r.plan["tiles"],
         "gpu_launches": steps * r.launches_per_step(),
         "traffic": profiled_traffic(r.p.name, r.plan["kernel_name"]),
         "floor_us": floor_us, "floor_frac": floor_us / (ms * 1e3)}
    if tl:
        e["tail_idle"] = tl["tail_idle"]
        e["span_us"] = tl["span_us"]
        if tl.get("phases_us"):
            e["phases_us_median"] = {k: v["median"] for k, v in tl["phases_us"].items()}
    return e


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank)
        return

    import gqa_decode_attention_attn_b200 as gq
    gq.load_library()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
        pg = dist

    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    p = workloads.workload(args.workload)
    r = Runner(gq, p, dev, args, flush)
    if r.fp8:
        args.no_e2e = True  # the host-buffer entry point takes bf16 caches
        args.no_cpu_baseline = True  # (bench.py --impl reference times the FP8 oracle)
    r.warm(args.warmup)

    props = torch.cuda.get_device_properties(dev)
    uuid = getattr(props, "uuid", None)
    sampler = ClockSampler(f"GPU-{uuid}" if uuid is not None else str(local_rank))
    sampler.start()
    time.sleep(0.3)
    if pg:
        pg.barrier()
    torch.cuda.synchronize(dev)
    t0 = time.time()
    per, region_ms = r.timed(args.steps)
    if pg:
        pg.barrier()
    t1 = time.time()
    sampler.stop()

    ms = sum(per) / len(per)
    if pg:
        tt = torch.tensor([ms], device=dev)
        pg.all_reduce(tt, op=pg.ReduceOp.MAX)
        ms = float(tt.item())

    bytes_step = p.algorithmic_bytes()
    value = world * bytes_step / (ms / 1e3) / 1e9
    peak, peak_kind = hbm_peak()
    achieved = bytes_step / (ms / 1e3) / 1e9
    clocks = sampler.summary(t0, t1)
    plan = r.plan

    line = None
    if rank == 0:
        traffic = profiled_traffic(p.name, plan["kernel_name"])
        line = {
            "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "us_per_step": ms * 1e3, "us_per_step_median": statistics.median(per) * 1e3,
            "pct_of_hbm_peak": 100.0 * achieved / peak,
            "pct_of_spec_8tbs": 100.0 * achieved / SPEC_HBM_GBS,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded N(0,1) bf16 q/K/V; no trained weights)",
            "config": dict(workload_config(p), schedule=r.schedule),
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "traffic": traffic,
                         "peak_source": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs, burst copy)"
                         if peak_kind == "measured" else
                         "fallback (MEASURED_PEAKS.json absent: the recipe's 6.65 TB/s)",
                         "kernel": plan["kernel_name"], "grid": plan["grid"],
                         "tiles": plan["tiles"],
                         "algorithmic_bytes_per_launch": bytes_step},
            "gpu_launches": args.steps * r.launches_per_step(),
            "timed_region_ms": region_ms,
            "clocks": clocks,
        }
        tl = r.timeline()
        if tl:
            line["timeline"] = tl
        f_mean, f_med, f_bytes, f_ctas = r.floor(args.steps)
        line["stream_floor"] = {
            "us_per_step": f_mean, "us_per_step_median": f_med, "kv_bytes": f_bytes,
            "ctas": f_ctas, "GB_per_s": f_bytes / (f_mean / 1e6) / 1e9,
            "floor_frac": f_mean / (ms * 1e3),
            "what": ("gqa_stream_floor: the same K and V bytes through the decode kernel's "
                     "TMA boxes and rings with no arithmetic, timed like the step; "
                     "floor_frac = floor time / step time")}
    if r.mode == "fixed":  # comparator runs report the kernel numbers only
        args.no_e2e = args.no_cpu_baseline = True
    if rank == 0 and not args.no_e2e:
        line["e2e"] = measure_e2e(gq, p, dev, args, r.stream)
    if rank == 0 and not args.no_cpu_baseline and world == 1:
        line["cpu_baseline"] = cpu_oracle_sample(p, args.cpu_seconds, gpu_out=r.out)
    extras = [w for w in (args.workloads.split(",") if args.workloads else ()) if w]
    if args.workloads == "default":
        extras = list(EXTRA_WORKLOADS) if (world == 1 and args.workload == "llama3_8b"
                                           and r.mode == "auto") else []
    if rank == 0 and extras:
        del r
        block = {}
        for name in extras:
            rr = Runner(gq, workloads.workload(name), dev, args, flush)
            block[name] = extra_entry(rr, min(args.steps, EXTRA_STEPS), args.warmup, peak)
            del rr
            torch.cuda.empty_cache()
        line["workloads"] = block
        line["workloads_note"] = ("other configurations timed in the same run, same method "
                                  "(L2 flushed before each step, CUDA events), "
                                  f"min(steps, {EXTRA_STEPS}) steps each; frac of the same peak")
    if rank == 0:
        print(json.dumps(line), flush=True)
    if pg:
        pg.barrier()
        pg.destroy_process_group()


def measure_e2e(gq, p, dev, args, stream):
    """Same metric through the host-buffer C-ABI call: every step copies the inputs
    from pinned host memory, runs the kernel and copies the output back."""
    dec = gq.HostDecoder(p.B, p.Hq, p.Hkv, p.D, p.block_size, p.max_blocks, p.num_blocks,
                         p.paged, device=dev)
    pin = [t.pin_memory() if t is not None else None
           for t in (p.q, p.k_cache, p.v_cache, p.block_table, p.seq_lens)]
    out = torch.empty_like(p.q).pin_memory()
    steps = max(3, min(args.steps, 20))
    for _ in range(3):
        dec(*pin, out, scale=p.scale, stream=stream)
    times = []
    for _ in range(steps):
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record(stream)
        dec(*pin, out, scale=p.scale, stream=stream)
        e.record(stream)
        e.synchronize()
        times.append(s.elapsed_time(e))
    ms = sum(times) / len(times)
    return {"value": p.algorithmic_bytes() / (ms / 1e3) / 1e9, "unit": "GB/s",
            "ms_per_step": ms, "steps": steps,
            "h2d_bytes_per_step": dec.h2d_bytes(*pin), "d2h_bytes_per_step": out.numel() * 2}


if __name__ == "__main__":
    main()
