#!/usr/bin/env python3
"""DCA prefill benchmark on B200.

One step = one whole prefill of the workload through the library's staged C
ABI (per query block: rotate the block's keys into the rotated-key cache, then
the fused attention kernel), inputs resident in HBM.  Default workload: the
1M-token chunked prefill of the 7B shape (32 query blocks of 32,768 tokens,
Hq 28 / Hkv 4, d 128, chunk 196,608, local window 32,768, pretraining window
262,144, YaRN 4, bf16), synthetic seeded inputs.

Prints one JSON line (rank 0):
  value        whole-job tokens/s (all ranks; replicas, weak scaling)
  tflops       algorithmic attention TFLOP/s of the whole step (4*d*Hq per causal pair)
  roofline     the attention kernel: algorithmic FLOPs / CUDA-event time of its launches
  e2e          same metric through the host-buffer C entry point (copies timed)
  cpu_baseline the fp64 oracle on a bounded sample, on the host cores (rank 0, N=1)
``--impl reference`` times that oracle alone as the reference arm.

Multi-GPU: ``torchrun --nproc-per-node N bench.py --gpus N``: N independent
replicas (the method has no exchange step), timed as the max over ranks.
"""
from __future__ import annotations

import argparse
import datetime
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

from length_extrapolation_b200.workloads import (DECODE_WORKLOADS, SPARSE_WORKLOADS,  # noqa: E402
                                                 WORKLOADS, generate, generate_decode,
                                                 generate_sparse, sample_heads)

METRIC = "DCA prefill tokens/s and attention TFLOP/s (fraction of B200 bf16 peak)"
DECODE_METRIC = "DCA decode tokens/s (KV-cache stream, fraction of B200 HBM bandwidth)"
SPARSE_METRIC = "vertical-slash sparse DCA prefill tokens/s (member-pair TFLOP/s)"
UNIT = "tokens/s"


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="qwen7b_1m_chunked",
                    choices=sorted(WORKLOADS) + sorted(DECODE_WORKLOADS) + sorted(SPARSE_WORKLOADS),
                    help="a prefill workload, or a decode step (*_decode*: the new tokens "
                         "against a full cache)")
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--cpu-seconds", type=float, default=20.0,
                    help="approximate CPU seconds for the oracle baseline sample")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--block", type=int, default=None, metavar="B",
                    help="profiling mode for a chunked workload: allocate only query block B "
                         "and the KV cache it attends (a few GB), time its attention launch "
                         "alone; prints a profiling line, not the workload's metric")
    ap.add_argument("--record-traffic", metavar="NCU_CSV",
                    help="store the attention kernel's DRAM bytes per launch from an ncu CSV "
                         "capture of --workload, then exit")
    return ap.parse_args(argv)


# ----------------------------------------------------------------------------- helpers
def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        return dict(bf16_tflops=float(pk["bf16_tflops"]),
                    bf16_tflops_sustained=float(pk.get("bf16_tflops_sustained", pk["bf16_tflops"])),
                    hbm_gbs=float(pk["hbm_gbs"]), source="measured")
    except (OSError, KeyError, ValueError):
        return dict(bf16_tflops=1590.0, bf16_tflops_sustained=1400.0, hbm_gbs=6650.0,
                    source="fallback")


KERNEL_SOURCES = ["length_extrapolation_b200/csrc/dca_fwd_sm100.cu",
                  "length_extrapolation_b200/csrc/dca_softmax.cuh",
                  "length_extrapolation_b200/csrc/sm100_ptx.cuh",
                  "length_extrapolation_b200/csrc/dca_plan.cuh"]
TRAFFIC_RECORD = os.path.join(ROOT, "profiles", "dca_fwd_kernel_traffic.json")


def kernel_source_hash():
    import hashlib
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def recorded_traffic(workload: str):
    """Average DRAM bytes (read + write) per attention launch from an ncu capture
    of this workload, or None when there is none for the current kernel source."""
    try:
        with open(TRAFFIC_RECORD) as f:
            rec = json.load(f)
    except (OSError, ValueError):
        return None
    ent = rec.get(workload)
    if not ent or ent.get("source_sha256") != kernel_source_hash():
        return None
    return ent.get("bytes_per_launch")


def write_traffic_record(workload: str, ncu_csv: str):
    """Store the average DRAM bytes per attention launch of an ncu CSV capture
    (metrics dram__bytes_read.sum, dram__bytes_write.sum) under the current
    kernel source hash."""
    import csv
    rows = list(csv.reader(open(ncu_csv)))
    hdr, per = None, {}
    for r in rows:
        if r and r[0] == "ID":
            hdr = r
            continue
        if hdr and len(r) == len(hdr):
            d = dict(zip(hdr, r))
            if "dca_fwd_kernel" not in d["Kernel Name"] or not d["Metric Name"].startswith("dram__bytes"):
                continue
            scale = {"byte": 1, "Kbyte": 1e3, "Mbyte": 1e6, "Gbyte": 1e9}[d["Metric Unit"]]
            per[d["ID"]] = per.get(d["ID"], 0.0) + float(d["Metric Value"].replace(",", "")) * scale
    if not per:
        raise SystemExit("no dca_fwd_kernel dram__bytes rows in " + ncu_csv)
    rec = {}
    if os.path.exists(TRAFFIC_RECORD):
        with open(TRAFFIC_RECORD) as f:
            rec = json.load(f)
    rec[workload] = {"bytes_per_launch": sum(per.values()) / len(per), "launches": len(per),
                     "source_sha256": kernel_source_hash()}
    with open(TRAFFIC_RECORD, "w") as f:
        json.dump(rec, f, indent=1)
    print(json.dumps({workload: rec[workload]}))


def causal_pairs(q0, lq):
    """Number of causal (query, key) pairs of rows q0 .. q0+lq-1 (key j <= i)."""
    return lq * q0 + lq * (lq + 1) // 2


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples every 200 ms while running."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.samples = []
        self.proc = None
        self.thread = None
        try:
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            sel = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
        except Exception:  # pragma: no cover
            sel = str(device_index)
        self.cmd = ["nvidia-smi", "-i", sel, f"--query-gpu={self.FIELDS}",
                    "--format=csv,noheader,nounits", "-lms", "200"]

    def start(self):
        try:
            self.proc = subprocess.Popen(self.cmd, stdout=subprocess.PIPE,
                                         stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return self
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()
        return self

    def _read(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 9:
                self.samples.append(parts)

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        if self.thread is not None:
            self.thread.join(timeout=5)
        return self.summary()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None

        sm = [num(s[1]) for s in self.samples if num(s[1]) is not None]
        smax = [num(s[2]) for s in self.samples if num(s[2]) is not None]
        load = [x for x in sm if smax and x > 0.3 * max(smax)] or sm
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[k] for s in self.samples for k in range(4)
                          if s[5 + k].lower().startswith("active")})
        return {"sm_mhz": statistics.median(load) if load else None,
                "sm_max_mhz": max(smax) if smax else None, "reasons": reasons,
                "samples": len(self.samples),
                "power_w_max": max((num(s[3]) or 0.0) for s in self.samples)}


def oracle_sample_rate(w, q_block, k, v, q0, lq, budget_s, rows_from_end=True):
    """Time the fp64 oracle on (row, head) samples of one block; returns
    (pairs*heads per second, description, threads used)."""
    import numpy as np

    import oracle
    threads = os.cpu_count() or 1
    heads = sample_heads(w).numpy()
    qc = q_block.cpu()
    lk = q0 + lq
    kc, vc = k[:lk].cpu(), v[:lk].cpu()
    # calibrate on one row, then size the sample to the time budget
    rows = np.array([lq - 1], dtype=np.int64)
    t0 = time.perf_counter()
    oracle.attention(qc, kc, vc, q_start=q0, rows=rows, heads=heads[:1], n_threads=threads,
                     **w.params())
    dt1 = max(time.perf_counter() - t0, 1e-3)
    n_rows = int(max(1, min(lq, budget_s / dt1 * threads / len(heads))))
    rows = np.arange(lq - n_rows, lq, dtype=np.int64) if rows_from_end else np.arange(n_rows)
    t0 = time.perf_counter()
    oracle.attention(qc, kc, vc, q_start=q0, rows=rows, heads=heads, n_threads=threads,
                     **w.params())
    dt = time.perf_counter() - t0
    pairs = sum(q0 + int(r) + 1 for r in rows) * len(heads)
    desc = (f"{len(rows)} rows x {len(heads)} heads of block q_start={q0} "
            f"({pairs:.3e} causal pair-heads in {dt:.1f} s)")
    return pairs / dt, desc, threads, dt


def total_pair_heads(w):
    return sum(causal_pairs(q0, lq) for q0, lq, _ in w.blocks()) * w.Hq


def init_dist(world: int, local: int):
    """Process group for N > 1 (one process per GPU; gloo when there is no GPU)."""
    if world <= 1:
        return None
    import torch.distributed as dist
    if torch.cuda.is_available():
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=900),
                                device_id=torch.device("cuda", local))
    else:
        dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=120))
    return dist


def max_over_ranks(values, dist, device="cpu"):
    """Element-wise max of a list of floats over all ranks (identity without dist)."""
    t = torch.tensor([float(x) for x in values], dtype=torch.float64, device=device)
    if dist is not None:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def whole_job_rate(tokens_per_rank: int, world: int, ms_per_step: float) -> float:
    """Replicas: every rank runs the whole workload; the job's rate divides all
    ranks' tokens by the slowest rank's step time."""
    return world * tokens_per_rank / (ms_per_step / 1e3)


# ----------------------------------------------------------------------------- reference arm
def run_reference(args, w, rank, world):
    """The oracle as it stands, on the host cores: each step times a bounded
    sample of the workload and reports extrapolated tokens/s."""
    if rank != 0:
        return 0
    import numpy as np  # noqa: F401
    q, k, v = generate(w, device="cpu")
    q0, lq, _ = w.blocks()[-1]
    budget = min(args.cpu_seconds, max(2.0, 120.0 / max(1, args.steps + args.warmup)))
    rates = []
    desc = threads = None
    for it in range(args.warmup + args.steps):
        rate, desc, threads, _ = oracle_sample_rate(w, q[q0:q0 + lq], k, v, q0, lq, budget)
        if it >= args.warmup:
            rates.append(rate)
    rate = statistics.median(rates)
    t_full = total_pair_heads(w) / rate
    value = w.L / t_full
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": t_full * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {**workload_config(w), "parallelism": f"replicas x{world}" if world > 1 else "1 GPU"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def workload_config(w):
    return {"workload": w.name, "L": w.L, "Hq": w.Hq, "Hkv": w.Hkv, "d": w.d,
            "chunk_size": w.chunk_size, "local_window": w.local_window,
            "pretrain_window": w.pretrain_window, "rope_base": w.rope_base,
            "yarn_scale": w.yarn_scale, "query_block": w.block or w.L,
            "global_batch": 1, "seq_len": w.L,
            "l2": "inputs larger than L2 (no flush)"}


# ----------------------------------------------------------------------------- decode
def decode_config(dw):
    w = dw.base
    return {"workload": dw.name, "kv_len": dw.Lk, "new_tokens": dw.Lq, "Hq": w.Hq,
            "Hkv": w.Hkv, "d": w.d, "chunk_size": w.chunk_size, "local_window": w.local_window,
            "pretrain_window": w.pretrain_window, "rope_base": w.rope_base,
            "yarn_scale": w.yarn_scale, "global_batch": 1, "seq_len": dw.Lk,
            "l2": "L2 flushed between steps (256 MiB write + 256 MiB read, untimed)"}


def oracle_decode_rate(dw, q, k, v, budget_s):
    """Time the fp64 oracle on the decode rows for a subset of heads; returns
    (seconds per whole step extrapolated to all heads, description, threads)."""
    import oracle
    w = dw.base
    threads = os.cpu_count() or 1
    heads = sample_heads(w).numpy()
    qc, kc, vc = q.cpu(), k.cpu(), v.cpu()
    t0 = time.perf_counter()
    n = 0
    while True:
        oracle.attention(qc, kc, vc, q_start=dw.Lk - dw.Lq, heads=heads, n_threads=threads,
                         **w.params())
        n += 1
        if time.perf_counter() - t0 > budget_s or n >= 50:
            break
    dt = (time.perf_counter() - t0) / n
    t_step = dt * w.Hq / len(heads)
    desc = (f"{dw.Lq} rows x {len(heads)} of {w.Hq} heads against {dw.Lk} keys, "
            f"{n} repetitions of {dt:.2f} s; extrapolated to all heads")
    return t_step, desc, threads


def run_decode_bench(args, dw, world, rank, local, dist):
    """One step = one generation step of the library: rotate the Lq new keys
    into the rotated-key cache (whose earlier rows are already there), then
    the split-KV decode kernel and its merge, inputs resident in HBM."""
    w = dw.base
    if args.impl == "reference":
        if rank != 0:
            return 0
        q, k, v = generate_decode(dw, device="cpu")
        budget = min(args.cpu_seconds, max(2.0, 120.0 / max(1, args.steps + args.warmup)))
        times, desc, threads = [], None, None
        for it in range(min(args.warmup, 1) + min(args.steps, 3)):
            t_step, desc, threads = oracle_decode_rate(dw, q, k, v, budget / 4)
            if it >= min(args.warmup, 1):
                times.append(t_step)
        t_step = statistics.median(times)
        value = dw.Lq / t_step
        print(json.dumps({
            "impl": "reference", "metric": DECODE_METRIC, "value": value, "unit": UNIT,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": t_step * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {**decode_config(dw), "parallelism": f"replicas x{world}" if world > 1 else "1 GPU"},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                             "sample": desc},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}), flush=True)
        return 0

    import length_extrapolation_b200 as dca
    from length_extrapolation_b200 import _native as N

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    peaks = load_peaks()
    q, k, v = generate_decode(dw, device=dev, seed=0)
    kw = dict(chunk_size=w.chunk_size, local_window=w.local_window,
              pretrain_window=w.pretrain_window)
    ws = dca.Workspace(dw.Lk, w.Hq, w.Hkv, w.d, w.chunk_size, w.local_window, w.pretrain_window,
                       q.dtype, dev)
    scratch = torch.empty(dca.decode_scratch_size(dw.Lq, w.Hq, w.Hkv), dtype=torch.uint8,
                          device=dev)
    out = torch.empty_like(q)
    # the earlier keys are in the rotated-key cache (the prefill before this step)
    dca.prepare(k, kv_len=dw.Lk - dw.Lq, k_rows_valid=0, rope_base=w.rope_base, workspace=ws,
                **kw)
    # L2 flush between steps: write a buffer larger than L2, then read another
    # one, so that L2 holds neither the cache nor dirty lines whose write-back
    # would land in the next timed step
    flush_w = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    flush_r = torch.zeros(64 << 20, dtype=torch.float32, device=dev)

    def flush_l2():
        flush_w.zero_()
        flush_r.sum()

    def prep():
        dca.prepare(k, kv_len=dw.Lk, k_rows_valid=dw.Lk - dw.Lq, rope_base=w.rope_base,
                    workspace=ws, **kw)

    def attend():
        dca.decode(q, v, out, q_start=dw.Lk - dw.Lq, kv_len=dw.Lk, yarn_scale=w.yarn_scale,
                   workspace=ws, scratch=scratch, **kw)

    # The two stages of a step are captured once as CUDA graphs and replayed,
    # as a serving loop issues a decode step: the device timeline then holds
    # the kernels alone, not the host's per-call argument marshalling.
    prep()
    attend()
    torch.cuda.synchronize()
    g_prep, g_dec = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_prep):
        prep()
    with torch.cuda.graph(g_dec):
        attend()

    def step(evs=None):
        if evs is not None:
            evs[0].record()
        g_prep.replay()
        if evs is not None:
            evs[1].record()
        g_dec.replay()
        if evs is not None:
            evs[2].record()

    for _ in range(args.warmup):
        flush_l2()
        step()
    torch.cuda.synchronize()
    if ws.status() != N.DCA_OK:
        raise RuntimeError("device status after warm-up")
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    clocks = ClockSampler(dev.index).start()
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    for e in evs:
        flush_l2()
        step(e)
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    clk = clocks.stop()
    if ws.status() != N.DCA_OK:
        raise RuntimeError("device status after timing")
    ms = sum(e[0].elapsed_time(e[2]) for e in evs)
    kern_ms = sum(e[1].elapsed_time(e[2]) for e in evs)
    ms, kern_ms = max_over_ranks([ms, kern_ms], dist, dev)
    ms_per_step = ms / args.steps
    esz = q.element_size()
    alg_bytes = dw.kv_bytes() + 2 * dw.Lq * w.Hq * w.d * esz   # K', V streamed once; q in, out
    achieved = alg_bytes / (kern_ms / args.steps / 1e3) / 1e9
    roofline = {"kernel": "dca_decode_kernel (split-KV, tcgen05) + merge",
                "bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / peaks["hbm_gbs"],
                "peak_kind": f"{peaks['source']} HBM copy bandwidth",
                "traffic": None, "traffic_unit": "bytes per launch (dram read + write, ncu)",
                "algorithmic_bytes_per_launch": alg_bytes,
                "avg_launch_ms": kern_ms / args.steps}

    e2e = None
    if not args.no_e2e:
        # host-side inputs of a step: the new tokens' q, k and v rows; result read back
        qh = q.cpu().pin_memory()
        knew = k[dw.Lk - dw.Lq:].cpu().pin_memory()
        vnew = v[dw.Lk - dw.Lq:].cpu().pin_memory()
        oh = torch.empty_like(qh).pin_memory()
        qd = torch.empty_like(q)

        def e2e_step():
            qd.copy_(qh, non_blocking=True)
            k[dw.Lk - dw.Lq:].copy_(knew, non_blocking=True)
            v[dw.Lk - dw.Lq:].copy_(vnew, non_blocking=True)
            dca.decode_step(qd, k, v, kv_len=dw.Lk, rope_base=w.rope_base,
                            yarn_scale=w.yarn_scale, workspace=ws, scratch=scratch, out=out, **kw)
            oh.copy_(out, non_blocking=True)

        e2e_step()
        torch.cuda.synchronize()
        tot = 0.0
        for _ in range(args.steps):
            flush_l2()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record()
            e2e_step()
            e1.record()
            torch.cuda.synchronize()
            tot += e0.elapsed_time(e1)
        ems = max_over_ranks([tot], dist, dev)[0] / args.steps
        e2e = {"value": world * dw.Lq / (ems / 1e3), "unit": UNIT, "ms_per_step": ems,
               "h2d_bytes_per_step": (qh.numel() + knew.numel() + vnew.numel()) * esz,
               "d2h_bytes_per_step": oh.numel() * esz,
               "path": "decode_step after pinned host->device copies of the new q/k/v rows; "
                       "out copied back"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        t_step, desc, threads = oracle_decode_rate(dw, q, k, v, args.cpu_seconds)
        cpu = {"value": dw.Lq / t_step, "unit": UNIT, "cores": threads, "kind": "oracle",
               "sample": desc}

    line = {
        "metric": DECODE_METRIC, "value": world * dw.Lq / (ms_per_step / 1e3), "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": w.dtype,
        "data": "synthetic",
        "config": {**decode_config(dw),
                   "parallelism": f"replicas x{world}" if world > 1 else "1 GPU"},
        "roofline": roofline, "e2e": e2e, "cpu_baseline": cpu, "clocks": clk,
        "gpu_launches": 3 * args.steps,   # key rotation, decode, merge
        "timing": "per step: CUDA graphs of the two stages replayed between CUDA events",
        "peaks_source": peaks["source"],
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return 0


# ----------------------------------------------------------------------------- sparse
def member_pairs(V, S, L, rows=None):
    """Sum over query heads and rows i of |{j <= i in V_h} U {i - o : o in S_h,
    o <= i} U {i}| (the sparse variant's attended pairs), in closed form:
    sum_v (L - v) + sum_o (L - o) - #{(v, o) : v + o < L} + the rows whose
    own key is in neither set.  `rows` = (r0, r1) restricts to rows [r0, r1)."""
    import numpy as np
    r0, r1 = (0, L) if rows is None else rows
    tot = 0
    for Vh, Sh in zip(V, S):
        Vh = np.asarray(Vh, dtype=np.int64)
        Sh = np.asarray(Sh, dtype=np.int64)
        a = np.clip(r1 - np.maximum(Vh, r0), 0, None).sum()
        b = np.clip(r1 - np.maximum(Sh, r0), 0, None).sum()
        both = np.add.outer(Vh, Sh)
        ov = np.count_nonzero((both >= r0) & (both < r1))
        own = 0 if (Sh.size and Sh[0] == 0) else (r1 - r0) - np.count_nonzero((Vh >= r0) & (Vh < r1))
        tot += int(a + b - ov + own)
    return tot


def sparse_config(sw):
    w = sw.base
    return {**workload_config(w), "workload": sw.name, "n_vertical": sw.n_vertical,
            "n_band": sw.n_band, "n_far": sw.n_far}


def run_sparse_bench(args, sw, world, rank, local, dist):
    """One step = one whole chunked sparse prefill: per query block, rotate
    the block's keys, prepare the pattern for the grown cache (copy, bitmaps,
    gather of the vertical rows), run the sparse attention kernel."""
    import numpy as np
    w = sw.base
    V, S = generate_sparse(sw)
    pairs = member_pairs(V, S, w.L)
    flops = 4.0 * w.d * pairs
    if args.impl == "reference" or (rank == 0 and world == 1 and not args.no_cpu_baseline):
        import oracle
        qc, kc, vc = generate(w, device="cpu")
        q0, lq, _ = w.blocks()[-1]
        heads = sample_heads(w).numpy()
        threads = os.cpu_count() or 1
        rows = np.arange(lq - 64, lq)
        t0 = time.perf_counter()
        oracle.sparse_attention(qc[q0:q0 + lq], kc, vc, vertical=V, slash=S, q_start=q0,
                                rows=rows, heads=heads, n_threads=threads, **w.params())
        dt = time.perf_counter() - t0
        done = member_pairs([V[h] for h in heads], [S[h] for h in heads], w.L,
                            rows=(q0 + lq - 64, q0 + lq))
        t_full = dt * pairs / done
        cpu = {"value": w.L / t_full, "unit": UNIT, "cores": threads, "kind": "oracle",
               "sample": f"64 rows x {len(heads)} heads of the last block ({done:.3e} member "
                         f"pairs in {dt:.1f} s); extrapolated by member pairs"}
        if args.impl == "reference":
            if rank == 0:
                print(json.dumps({
                    "impl": "reference", "metric": SPARSE_METRIC, "value": cpu["value"],
                    "unit": UNIT, "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
                    "ms_per_step": t_full * 1e3, "higher_is_better": True, "scaling": "weak",
                    "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                    "config": {**sparse_config(sw), "parallelism": f"replicas x{world}" if world > 1 else "1 GPU"}, "cpu_baseline": cpu,
                    "e2e": {"value": cpu["value"], "unit": UNIT, "h2d_bytes_per_step": 0,
                            "d2h_bytes_per_step": 0}}), flush=True)
            return 0
        del qc, kc, vc
    else:
        cpu = None

    import length_extrapolation_b200 as dca
    from length_extrapolation_b200 import _native as N
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    peaks = load_peaks()
    q, k, v = generate(w, device=dev, seed=0)
    out = torch.empty_like(q)
    pat = dca.SparsePattern(V, S)
    kw = dict(chunk_size=w.chunk_size, local_window=w.local_window,
              pretrain_window=w.pretrain_window)
    ws = dca.Workspace(w.L, w.Hq, w.Hkv, w.d, w.chunk_size, w.local_window, w.pretrain_window,
                       q.dtype, dev)
    sp = dca.SparseWorkspace(w.L, w.Hq, pat.max_vertical(), pat.max_slash(), dev)
    blocks = w.blocks()
    # the pattern restricted to each block's cache, built once (host lists)
    pats = [pat.restricted(lk) for _, _, lk in blocks]

    def step(evs=None):
        for b, (q0, lq, lk) in enumerate(blocks):
            dca.prepare(k, kv_len=lk, k_rows_valid=q0, rope_base=w.rope_base, workspace=ws, **kw)
            dca.sparse_prepare(pats[b], v, kv_len=lk, workspace=ws, sparse=sp, **kw)
            if evs is not None:
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record()
            dca.sparse_attend(q[q0:q0 + lq], v, out[q0:q0 + lq], q_start=q0, kv_len=lk,
                              yarn_scale=w.yarn_scale, workspace=ws, sparse=sp, **kw)
            if evs is not None:
                e1.record()
                evs.append((e0, e1))

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if ws.status() != N.DCA_OK:
        raise RuntimeError("device status after warm-up")
    clocks = ClockSampler(dev.index).start()
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    evs = []
    t0.record()
    for _ in range(args.steps):
        step(evs)
    t1.record()
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    clk = clocks.stop()
    if ws.status() != N.DCA_OK:
        raise RuntimeError("device status after timing")
    ms, attn_ms = max_over_ranks([t0.elapsed_time(t1), sum(a.elapsed_time(b) for a, b in evs)],
                                 dist, dev)
    ms_per_step = ms / args.steps
    # processed tiles: items x 128 x 128 pairs (host plan of every query tile and head)
    achieved = flops * args.steps / (attn_ms / 1e3) / 1e12
    roofline = {
        "kernel": "dca_sparse_kernel (tcgen05, vertical-slash)", "bound": "tensor",
        "achieved": achieved, "peak": peaks["bf16_tflops_sustained"], "unit": "TFLOP/s",
        "frac": achieved / peaks["bf16_tflops_sustained"],
        "peak_kind": f"{peaks['source']} sustained bf16 (cuBLAS, power-capped loop)",
        "algorithmic_flops_per_step": flops, "member_pairs_per_step": pairs,
        "dense_causal_pairs_per_step": total_pair_heads(w),
        "traffic": None, "launches_per_step": len(blocks),
        "avg_launch_ms": attn_ms / (args.steps * len(blocks)),
    }
    # the online key selection (continuous positions) of the last block, timed alone
    q0, lq, lk = blocks[-1]
    n_s = min(sw.n_band + sw.n_far, N.DCA_SPARSE_MAX_RUNS)
    sel_sp = dca.SparseWorkspace(w.L, w.Hq, sw.n_vertical, n_s, dev)
    sel_scratch = torch.empty(N.lib().dca_sparse_select_scratch_size(lk, w.Hq, w.chunk_size),
                              dtype=torch.uint8, device=dev)

    def select():
        dca.sparse_select(q[q0:q0 + lq], v, q_start=q0, kv_len=lk, rope_base=w.rope_base,
                          yarn_scale=w.yarn_scale, n_vertical=sw.n_vertical, n_slash=n_s,
                          n_last=64, continuous=True, workspace=ws, sparse=sel_sp,
                          scratch=sel_scratch, **kw)

    select()
    torch.cuda.synchronize()
    s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s0.record()
    for _ in range(3):
        select()
    s1.record()
    torch.cuda.synchronize()
    sel_ms = s0.elapsed_time(s1) / 3
    # one 2^x per (row, key) pair and pass on the exponential unit (16 per SM
    # per clock), the unit the score passes' softmax side is bound by
    sel_ex2 = 2.0 * 64 * lk * w.Hq
    ex2_peak = 148 * 16 * (clk.get("sm_mhz") or 1965.0) * 1e6 / 1e9
    sel_rate = sel_ex2 / (sel_ms / 1e3) / 1e9
    select_info = {"kv_len": lk, "n_last": 64, "n_vertical": sw.n_vertical, "n_slash": n_s,
                   "positions": "continuous", "ms": sel_ms,
                   "roofline": {"bound": "alu", "achieved": sel_rate, "peak": ex2_peak,
                                "unit": "G exp2/s", "frac": sel_rate / ex2_peak,
                                "peak_kind": "MUFU exp2: 148 SMs x 16 per clock x median SM clock"}}
    line = {
        "metric": SPARSE_METRIC, "value": whole_job_rate(w.L, world, ms_per_step), "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": w.dtype,
        "data": "synthetic",
        "config": {**sparse_config(sw), "parallelism": f"replicas x{world}" if world > 1 else "1 GPU"},
        "tflops_member_pairs": world * flops / (ms_per_step / 1e3) / 1e12,
        "roofline": roofline, "e2e": None, "cpu_baseline": cpu, "clocks": clk,
        "select": select_info,
        "gpu_launches": args.steps * len(blocks) * 5,  # rotate, 2 prep kernels, attend (+ memset)
        "peaks_source": peaks["source"],
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return 0


# ----------------------------------------------------------------------------- one block
def run_block_bench(args, w, local=0):
    """One query block of a chunked workload, alone on the device: q/out of
    that block and the keys/values it attends (seeded like the workload's
    inputs, but drawn for these rows only).  The keys are rotated once before
    timing; each step is one attention launch.  For ncu captures of a long
    block (the last block of the 1M workload holds about 3.6 GB on the device)."""
    import length_extrapolation_b200 as dca
    from length_extrapolation_b200 import _native as N
    from length_extrapolation_b200.workloads import _draw

    q0, lq, lk = w.blocks()[args.block]
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    peaks = load_peaks()
    g = torch.Generator(device=dev)
    g.manual_seed(0)
    k = _draw(w, g, lk, w.Hkv, dev)
    v = _draw(w, g, lk, w.Hkv, dev)
    q = _draw(w, g, lq, w.Hq, dev)
    out = torch.empty_like(q)
    p = w.params()
    ws = dca.Workspace(lk, w.Hq, w.Hkv, w.d, w.chunk_size, w.local_window, w.pretrain_window,
                       w.torch_dtype, dev)
    dca.prepare(k, kv_len=lk, k_rows_valid=0, chunk_size=p["chunk_size"],
                local_window=p["local_window"], pretrain_window=p["pretrain_window"],
                rope_base=p["rope_base"], workspace=ws)

    def step():
        dca.attend(q, v, out, q_start=q0, kv_len=lk, chunk_size=p["chunk_size"],
                   local_window=p["local_window"], pretrain_window=p["pretrain_window"],
                   yarn_scale=p["yarn_scale"], workspace=ws)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if ws.status() != N.DCA_OK:
        raise RuntimeError("device status after warm-up")
    clocks = ClockSampler(dev.index).start()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        step()
    e1.record()
    torch.cuda.synchronize()
    clk = clocks.stop()
    ms = e0.elapsed_time(e1) / args.steps
    flops = 4.0 * w.d * w.Hq * causal_pairs(q0, lq)
    print(json.dumps({
        "profiling": f"attention of query block {args.block} of {w.name} alone",
        "q_start": q0, "Lq": lq, "Lk": lk, "steps": args.steps, "warmup": args.warmup,
        "ms_per_launch": ms, "tflops": flops / (ms / 1e3) / 1e12,
        "frac_of_measured_sustained": flops / (ms / 1e3) / 1e12 / peaks["bf16_tflops_sustained"],
        "algorithmic_bytes": (2 * lq * w.Hq + 2 * lk * w.Hkv) * w.d * q.element_size(),
        "clocks": clk}), flush=True)
    return 0


# ----------------------------------------------------------------------------- our arm
def main(argv=None):
    args = parse_args(argv)
    if args.workload in SPARSE_WORKLOADS:
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        local = int(os.environ.get("LOCAL_RANK", "0"))
        dist = init_dist(world, local)
        return run_sparse_bench(args, SPARSE_WORKLOADS[args.workload], world, rank, local, dist)
    if args.workload in DECODE_WORKLOADS:
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        local = int(os.environ.get("LOCAL_RANK", "0"))
        dist = init_dist(world, local)
        return run_decode_bench(args, DECODE_WORKLOADS[args.workload], world, rank, local, dist)
    w = WORKLOADS[args.workload]
    if args.block is not None:
        return run_block_bench(args, w)
    if args.record_traffic:
        write_traffic_record(w.name, args.record_traffic)
        return 0
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dist = init_dist(world, local)
    if args.impl == "reference":
        rc = run_reference(args, w, rank, world)
        if dist is not None:
            dist.destroy_process_group()
        return rc

    import length_extrapolation_b200 as dca
    from length_extrapolation_b200 import _native as N
    from length_extrapolation_b200 import runner

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    peaks = load_peaks()
    q, k, v = generate(w, device=dev, seed=0)
    out = torch.empty_like(q)
    ws = runner.make_workspace(w, dev)
    blocks = w.blocks()
    attn_flops = [4.0 * w.d * w.Hq * causal_pairs(q0, lq) for q0, lq, _ in blocks]
    step_flops = sum(attn_flops)
    launches_per_step = 1 + 2 * len(blocks)  # RoPE table + (key rotation, attention) per block

    def barrier():
        if dist is not None:
            dist.barrier()

    for _ in range(args.warmup):
        runner.run_workload(w, q, k, v, out, ws)
    torch.cuda.synchronize()
    st = ws.status()
    if st != N.DCA_OK:
        raise RuntimeError(f"device status after warm-up: {N.status_string(st)}")

    clocks = ClockSampler(dev.index).start()
    ev_all = []
    barrier()
    torch.cuda.synchronize()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record()
    for _ in range(args.steps):
        runner.run_workload(w, q, k, v, out, ws, attn_events=ev_all)
    t_end.record()
    torch.cuda.synchronize()
    barrier()
    clk = clocks.stop()
    ms = t_start.elapsed_time(t_end)
    st = ws.status()
    if st != N.DCA_OK:
        raise RuntimeError(f"device status after timing: {N.status_string(st)}")
    attn_ms = sum(a.elapsed_time(b) for a, b in ev_all)
    ms_max, attn_ms_max = max_over_ranks([ms, attn_ms], dist, dev)
    ms_per_step = ms_max / args.steps
    value = whole_job_rate(w.L, world, ms_per_step)
    tflops = world * step_flops / (ms_per_step / 1e3) / 1e12

    achieved = step_flops * args.steps / (attn_ms_max / 1e3) / 1e12
    roofline = {
        "kernel": "dca_fwd_kernel (tcgen05 attention)" if w.dtype == "bf16" else "dca_fwd_f32_kernel",
        "bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops_sustained"],
        "unit": "TFLOP/s", "frac": achieved / peaks["bf16_tflops_sustained"],
        "peak_kind": f"{peaks['source']} sustained bf16 (cuBLAS, power-capped loop)",
        "frac_of_burst_peak": achieved / peaks["bf16_tflops"],
        "frac_of_datasheet_2250": achieved / 2250.0,
        "traffic": recorded_traffic(w.name),
        "traffic_unit": "bytes per launch (dram read + write, ncu)",
        "algorithmic_bytes_per_launch": sum(
            (2 * lq * w.Hq + 2 * lk * w.Hkv) * w.d * q.element_size() for q0, lq, lk in blocks)
            / len(blocks),
        "launches_per_step": len(blocks),
        "avg_launch_ms": attn_ms_max / (args.steps * len(blocks)),
    }

    # ---------------------------------------------------------------- end to end
    e2e = None
    if not args.no_e2e:
        qh = q.cpu().pin_memory()
        kh = k.cpu().pin_memory()
        vh = v.cpu().pin_memory()
        oh = torch.empty_like(qh).pin_memory()
        n = dca.host_arena_size(w.L, w.block or w.L, w.Hq, w.Hkv, w.d, w.chunk_size,
                                w.local_window, w.pretrain_window, w.torch_dtype)
        del out, ws
        torch.cuda.empty_cache()
        arena = torch.empty(n, dtype=torch.uint8, device=dev)
        dca.prefill_host(qh, kh, vh, oh, block=w.block or w.L, arena=arena, **w.params())
        torch.cuda.synchronize()
        barrier()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(args.e2e_steps):
            dca.prefill_host(qh, kh, vh, oh, block=w.block or w.L, arena=arena, **w.params())
        e1.record()
        torch.cuda.synchronize()
        barrier()
        ems_step = max_over_ranks([e0.elapsed_time(e1)], dist, dev)[0] / args.e2e_steps
        esz = q.element_size()
        h2d_bytes = (q.numel() + k.numel() + v.numel()) * esz
        d2h_bytes = q.numel() * esz
        # copy rates of the same bytes alone (one pinned copy each way, device timed)
        del arena
        torch.cuda.empty_cache()
        buf = torch.empty(q.numel() * esz, dtype=torch.uint8, device=dev)
        c0 = torch.cuda.Event(enable_timing=True)
        c1 = torch.cuda.Event(enable_timing=True)
        c2 = torch.cuda.Event(enable_timing=True)
        c0.record()
        for t in (qh, kh, vh):
            buf[:t.numel() * esz].copy_(t.view(-1).view(torch.uint8), non_blocking=True)
        c1.record()
        oh.view(-1).view(torch.uint8).copy_(buf[:d2h_bytes], non_blocking=True)
        c2.record()
        torch.cuda.synchronize()
        del buf
        e2e = {"value": whole_job_rate(w.L, world, ems_step), "unit": UNIT,
               "ms_per_step": ems_step,
               "h2d_bytes_per_step": h2d_bytes, "d2h_bytes_per_step": d2h_bytes,
               "h2d_gbs_alone": h2d_bytes / (c0.elapsed_time(c1) / 1e3) / 1e9,
               "d2h_gbs_alone": d2h_bytes / (c1.elapsed_time(c2) / 1e3) / 1e9,
               "path": "dca_prefill_host (pinned host buffers; copies on the library's copy "
                       "stream overlap the kernels on the caller's stream)"}

    # ---------------------------------------------------------------- CPU baseline
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        q0, lq, _ = blocks[-1]
        rate, desc, threads, _ = oracle_sample_rate(w, q[q0:q0 + lq], k, v, q0, lq,
                                                    args.cpu_seconds)
        t_full = total_pair_heads(w) / rate
        cpu = {"value": w.L / t_full, "unit": UNIT, "cores": threads, "kind": "oracle",
               "sample": desc + "; extrapolated to all causal pairs of the workload"}

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
        "config": {**workload_config(w), "parallelism": f"replicas x{world}" if world > 1 else "1 GPU"},
        "tflops": tflops,
        "tflops_frac_of_peak": {"measured_sustained": tflops / world / peaks["bf16_tflops_sustained"],
                                "measured_burst": tflops / world / peaks["bf16_tflops"],
                                "datasheet_2250": tflops / world / 2250.0},
        "roofline": roofline,
        "e2e": e2e,
        "cpu_baseline": cpu,
        "clocks": clk,
        "gpu_launches": launches_per_step * args.steps,
        "peaks_source": peaks["source"],
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
