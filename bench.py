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
}


def kernel_for(p) -> str:
    """Which decode kernel the library runs for this problem (mirrors the library's
    dispatch: tensor cores for D = 64 or 128 (FP8 caches: D = 128) with at least 4
    query heads per KV head and pages that tile into 128-token boxes, CUDA cores
    otherwise)."""
    bs = p.block_size
    boxes = (not p.paged) or (bs % 128 == 0 if bs >= 128 else (bs >= 8 and 128 % bs == 0))
    if p.meta.get("kv_elem_bytes") == 1:
        if p.D == 128 and p.G >= 4 and p.B <= 1024 and boxes:
            nv = 4 if p.G <= 4 else (8 if p.G <= 8 else 16)
            return f"gqa_decode_tc_kernel<{nv}> (FP8 E4M3 cache)"
        return "gqa_decode_simt_kernel (FP8 E4M3 cache)"
    if p.D in (64, 128) and p.G >= 4 and p.B <= 1024 and boxes:
        nv = 4 if p.G <= 4 else (8 if p.G <= 8 else 16)
        return f"gqa_decode_tc_kernel<{nv}>"
    return "gqa_decode_simt_kernel"


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
    return ap.parse_args()


def hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


def kernel_source_hash(kernel: str) -> str:
    """Hash of the sources of the named kernel (a kernel_for() name)."""
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES["tc" if "tc_kernel" in kernel else "simt"]:
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


def step_timeline(gq, d, p, out, ws, stream, flush, splits, schedule):
    """One more step, untimed and after an L2 flush, through gqa_decode_timeline with
    the schedule the timed steps ran: per-CTA start/end (%globaltimer) and SM, summed
    up as span, busy fraction and tail idle."""
    ns = splits if splits else (1 if schedule.startswith("auto: one CTA") else 0)
    flush.fill_(0)
    _, tl = gq.gqa_decode_timeline(d.q, d.k_cache, d.v_cache, d.block_table, d.seq_lens,
                                   num_splits=ns, out=out, scale=p.scale, workspace=ws,
                                   stream=stream)
    torch.cuda.synchronize()
    if ws.status():
        raise SystemExit("device status error during the timeline step")
    summary = gq.timeline_summary(tl)
    summary["source"] = ("one untimed step through gqa_decode_timeline, same schedule: "
                         "per-CTA %globaltimer at entry and exit, %smid")
    return summary


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

    p = workloads.workload(args.workload)
    fp8 = p.meta.get("kv_elem_bytes") == 1
    d = p.to(dev)
    if fp8:  # the cache as FP8 E4M3 bytes with per-tensor scales
        k8, v8, k_scale, v_scale = workloads.fp8_caches(p)
        d.k_cache, d.v_cache = k8.to(dev), v8.to(dev)
        args.no_e2e = True  # the host-buffer entry point takes bf16 caches
        args.no_cpu_baseline = True  # (bench.py --impl reference times the FP8 oracle)
    out = torch.empty_like(d.q)
    ws = gq.Workspace(dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    splits = 0
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    lens_host = p.seq_lens.to(torch.int32).contiguous()
    if fp8:
        schedule = "stream-K (FP8 cache)"
    elif args.schedule == "fixed":
        segs = p.B * p.Hkv * -(-p.G // 16)
        splits = args.splits if args.splits > 0 else max(1, -(-sms // segs))
        schedule = f"fixed-split x{splits}"
    elif args.schedule == "auto":
        chosen, _ = gq.select_schedule(lens_host, p.Hq, p.Hkv, p.D, sms, max_splits=1)
        schedule = "auto: one CTA per (request, KV head)" if chosen else "auto: stream-K"
    else:
        schedule = "stream-K"

    def step():
        if fp8:
            gq.gqa_decode_fp8(d.q, d.k_cache, d.v_cache, k_scale, v_scale, d.block_table,
                              d.seq_lens, out=out, scale=p.scale, workspace=ws, stream=stream)
        elif splits:
            gq.gqa_decode_fixed_split(d.q, d.k_cache, d.v_cache, d.block_table, d.seq_lens,
                                      splits, out=out, scale=p.scale, workspace=ws, stream=stream)
        elif args.schedule == "auto":
            gq.gqa_decode_auto(d.q, d.k_cache, d.v_cache, d.block_table, d.seq_lens, lens_host,
                               out=out, scale=p.scale, workspace=ws, stream=stream)
        else:
            gq.gqa_decode(d.q, d.k_cache, d.v_cache, d.block_table, d.seq_lens, out=out,
                          scale=p.scale, workspace=ws, stream=stream)

    for _ in range(max(3, args.warmup)):
        flush.fill_(1)
        step()
    torch.cuda.synchronize(dev)
    if ws.status():
        raise SystemExit("device status error during warm-up")

    props = torch.cuda.get_device_properties(dev)
    uuid = getattr(props, "uuid", None)
    sampler = ClockSampler(f"GPU-{uuid}" if uuid is not None else str(local_rank))
    sampler.start()
    time.sleep(0.3)
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    if pg:
        pg.barrier()
    torch.cuda.synchronize(dev)
    t0 = time.time()
    region0 = torch.cuda.Event(enable_timing=True)
    region1 = torch.cuda.Event(enable_timing=True)
    region0.record(stream)
    for i in range(args.steps):
        flush.fill_(i & 0xFF)
        starts[i].record(stream)
        step()
        ends[i].record(stream)
    region1.record(stream)
    torch.cuda.synchronize(dev)
    if pg:
        pg.barrier()
    t1 = time.time()
    sampler.stop()
    if ws.status():
        raise SystemExit("device status error during the timed steps")

    per = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    ms = sum(per) / len(per)
    region_ms = region0.elapsed_time(region1)
    if pg:
        tt = torch.tensor([ms], device=dev)
        pg.all_reduce(tt, op=pg.ReduceOp.MAX)
        ms = float(tt.item())

    bytes_step = p.algorithmic_bytes()
    value = world * bytes_step / (ms / 1e3) / 1e9
    peak, peak_kind = hbm_peak()
    achieved = bytes_step / (ms / 1e3) / 1e9
    clocks = sampler.summary(t0, t1)

    line = None
    if rank == 0:
        traffic = profiled_traffic(p.name, kernel_for(p))
        line = {
            "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "us_per_step": ms * 1e3, "us_per_step_median": statistics.median(per) * 1e3,
            "pct_of_hbm_peak": 100.0 * achieved / peak,
            "pct_of_spec_8tbs": 100.0 * achieved / SPEC_HBM_GBS,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded N(0,1) bf16 q/K/V; no trained weights)",
            "config": dict(workload_config(p), schedule=schedule),
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "traffic": traffic,
                         "peak_source": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs, burst copy)",
                         "kernel": kernel_for(p),
                         "algorithmic_bytes_per_launch": bytes_step},
            "gpu_launches": args.steps * (2 if splits > 1 else 1),
            "timed_region_ms": region_ms,
            "clocks": clocks,
        }
    if rank == 0 and not fp8:
        line["timeline"] = step_timeline(gq, d, p, out, ws, stream, flush, splits, schedule)
    if splits:  # comparator runs report the kernel numbers only
        args.no_e2e = args.no_cpu_baseline = True
    if rank == 0 and not args.no_e2e:
        line["e2e"] = measure_e2e(gq, p, dev, args, stream)
    if rank == 0 and not args.no_cpu_baseline and world == 1:
        line["cpu_baseline"] = cpu_oracle_sample(p, args.cpu_seconds, gpu_out=out)
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
