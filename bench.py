#!/usr/bin/env python
"""Benchmark of the IsoQuant hot path on B200: packed 3-bit decode attention
KV GB/s (fraction of HBM peak) and quantize Mvec/s.

One step is one pass of the whole path over one batch of synthetic input:
  1. stage-1 round trip: isoq_quantize then isoq_dequantize of 2^20 float16
     unit vectors, d=128, 3-bit, IsoQuant-Full;
  2. long-context decode: isoq_decode_split + isoq_decode_combine for batch 32
     x 65,536 tokens, 16 query / 8 KV heads, d=256, 3-bit Full, over a packed
     cache compressed from Student-t (nu=4) K/V with outlier channels and RoPE.
The headline ``value`` is the decode's packed K/V bytes (codes + float16
norms) divided by the decode's device time (split + combine, CUDA events on
the launching stream, max over ranks).  Each step streams 3.3 GB of packed
K/V, more than 26x the 126 MB L2, so no step finds its inputs in L2.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl isoq|reference]

Multi-GPU runs are weak-scaled replicas: every rank runs the same per-GPU
workload on its own data; there is no data-path collective (the (b, kvh)
pairs are independent).  ``--impl reference`` times the float64 oracle on the
host cores on a bounded sample of the same decode workload.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "packed-3-bit decode attn KV GB/s (% of HBM peak); quantize Mvec/s"
FALLBACK_HBM_GBS = 6650.0
NOMINAL_HBM_GBS = 8000.0      # B200's nominal HBM3e bandwidth (~8 TB/s), reported beside the measured copy peak
# The files holding the decode split kernel's device code (its traffic in the
# committed ncu summary is valid only while they are unchanged).
KERNEL_SOURCES = ["compressed_space_attention_b200/csrc/decode_i8.cuh",
                  "compressed_space_attention_b200/csrc/common.cuh"]
TRAFFIC_FILE = "profiles/decode_split_traffic.json"

WORKLOADS = {
    # name: (B, Hq, Hkv, T, d)
    "long_context_decode_b32_gqa16_8_d256_t65536": (32, 16, 8, 65536, 256),
    "decode_b1_gqa32_4_d128_t32768": (1, 32, 4, 32768, 128),
    "decode_b16_gqa32_4_d128_t8192_ragged": (16, 32, 4, 8192, 128),
}
DEFAULT_WORKLOAD = "long_context_decode_b32_gqa16_8_d256_t65536"
STAGE1 = dict(n=1 << 20, d=128, bits=3)


def env_int(name, default):
    try:
        return int(os.environ.get(name, default))
    except ValueError:
        return default


def kv_bytes_per_token_head(d, bits=3):
    return 2 * (d * bits // 8 + 2)


def source_hash():
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def read_traffic():
    """Per-launch DRAM bytes of the decode split kernel, from the data file
    that ``--record-traffic`` wrote out of an ncu capture, if that capture
    was taken on the current kernel source."""
    path = os.path.join(ROOT, TRAFFIC_FILE)
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f)
    if rec.get("source_hash") != source_hash():
        return None
    return float(rec["traffic_bytes_per_launch"])


def record_traffic(csv_path, kernel_regex, scale, note):
    """Writes TRAFFIC_FILE from an ncu ``--page raw --csv`` export: the
    dram__bytes_read.sum + dram__bytes_write.sum of the launches whose name
    matches kernel_regex (averaged), times `scale` (the full launch's units
    over the captured launch's), with the current kernel source hash."""
    import csv

    with open(csv_path, newline="") as f:
        rows = list(csv.reader(f))
    header = rows[0]
    idx_name = header.index("Kernel Name")
    units = {}
    for unit_row in rows[1:2]:
        units = dict(zip(header, unit_row))
    cols = {m: header.index(m) for m in ("dram__bytes_read.sum", "dram__bytes_write.sum")}
    mult = {"byte": 1.0, "Kbyte": 1e3, "Mbyte": 1e6, "Gbyte": 1e9, "KB": 1e3, "MB": 1e6, "GB": 1e9}
    vals = []
    for r in rows[2:]:
        if len(r) <= max(cols.values()) or not re.search(kernel_regex, r[idx_name]):
            continue
        tot = 0.0
        for m, i in cols.items():
            tot += float(r[i].replace(",", "")) * mult.get(units.get(m, "byte"), 1.0)
        vals.append(tot)
    if not vals:
        raise SystemExit(f"no launch of {kernel_regex} in {csv_path}")
    rec = {"kernel": kernel_regex, "source_hash": source_hash(),
           "captured_bytes_per_launch": sum(vals) / len(vals), "scale": scale,
           "traffic_bytes_per_launch": sum(vals) / len(vals) * scale, "launches": len(vals), "note": note}
    with open(os.path.join(ROOT, TRAFFIC_FILE), "w") as f:
        json.dump(rec, f, indent=1)
        f.write("\n")
    print(json.dumps(rec))


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return json.load(f), "measured"
    return {"hbm_gbs": FALLBACK_HBM_GBS}, "fallback"


# ---------------------------------------------------------------------------
# Clock sampling during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    """Samples the SM clock and the clock-event reasons of one GPU while the
    timed region runs.

    An ``nvidia-smi -lms`` child process does the polling (no Python thread
    competes with the launch loop for the interpreter); each sample carries
    nvidia-smi's own timestamp, and only the samples inside the region (with
    one sampling interval of slack on each side) are kept.  Without
    nvidia-smi, a thread polls NVML instead.
    """
    REASONS = {
        "sw_power_cap": 0x4, "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20,
        "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80,
    }
    INTERVAL_MS = 20

    def __init__(self, torch_device_index):
        self.samples = []          # (datetime, sm_mhz, reason mask)
        self.max_mhz = None
        self.proc = None
        self.reader = None
        self.t0 = self.t1 = None
        self.uuid = None
        try:
            import torch
            u = str(torch.cuda.get_device_properties(torch_device_index).uuid)
            self.uuid = u if u.startswith("GPU-") else "GPU-" + u
        except Exception:
            self.uuid = None

    def _read(self):
        import datetime
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) != 4:
                continue
            try:
                ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f")
                sm, mx = float(parts[1]), float(parts[2])
                mask = int(parts[3], 16)
            except ValueError:
                continue
            self.max_mhz = mx
            self.samples.append((ts, sm, mask))

    def start(self):
        import shutil
        import subprocess
        exe = shutil.which("nvidia-smi")
        if exe is None or self.uuid is None:
            return
        cmd = [exe, "-i", self.uuid, "--query-gpu=timestamp,clocks.sm,clocks.max.sm,clocks_event_reasons.active",
               "--format=csv,noheader,nounits", "-lms", str(self.INTERVAL_MS)]
        self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True, bufsize=1)
        self.reader = threading.Thread(target=self._read, daemon=True)
        self.reader.start()
        # let the first samples arrive before the region starts
        deadline = time.time() + 3.0
        while not self.samples and time.time() < deadline and self.proc.poll() is None:
            time.sleep(0.01)

    def stop(self):
        if self.proc is not None:
            time.sleep(2 * self.INTERVAL_MS / 1000)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.reader.join(timeout=5)

    def __enter__(self):
        import datetime
        self.t0 = datetime.datetime.now()
        return self

    def __exit__(self, *exc):
        import datetime
        self.t1 = datetime.datetime.now()

    def summary(self):
        import datetime
        if not self.samples or self.t0 is None or self.t1 is None:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0,
                    "source": "nvidia-smi" if self.proc is not None else "unavailable"}
        slack = datetime.timedelta(milliseconds=self.INTERVAL_MS)
        inside = [(sm, m) for ts, sm, m in self.samples if self.t0 - slack <= ts <= self.t1 + slack]
        reasons = sorted({name for _, m in inside for name, bit in self.REASONS.items() if m & bit})
        return {"sm_mhz": float(statistics.median([sm for sm, _ in inside])) if inside else None,
                "sm_max_mhz": self.max_mhz, "reasons": reasons, "samples": len(inside),
                "source": f"nvidia-smi -lms {self.INTERVAL_MS}, samples inside the timed region"}


# ---------------------------------------------------------------------------
# CPU baseline: the float64 oracle on a bounded sample of the decode workload
# ---------------------------------------------------------------------------

def oracle_decode_sample(workload, budget_s=20.0, min_s=8.0, tokens=None, seed=1000):
    """Times the oracle's decode attention on one (b, kvh) pair of the
    workload (its G query heads), token count chosen to take ~min_s..budget_s.
    Returns (GB/s, seconds, description)."""
    from threadpoolctl import threadpool_limits

    import oracle as O
    import synth

    B, Hq, Hkv, T, d = WORKLOADS[workload]
    g = Hq // Hkv
    t = tokens or T
    k, v = synth.student_t_kv(1, t, d, seed=seed)
    prk = O.make_params(d, O.FULL, seed=1)
    prv = O.make_params(d, O.FULL, seed=2)
    pk, nk = O.quantize(k[0].astype(np.float64), prk, 3, O.FULL)
    pv, nv = O.quantize(v[0].astype(np.float64), prv, 3, O.FULL)
    q = synth.queries(1, g, d, seed=seed + 1)
    args = (q, pk[None], pv[None], nk[None], nv[None], [t], prk, prv, 3, O.FULL, 1 / math.sqrt(d))
    reps, elapsed = 0, 0.0
    with threadpool_limits(limits=1):
        while elapsed < min_s and elapsed < budget_s:
            t0 = time.perf_counter()
            O.decode_attention(*args)
            elapsed += time.perf_counter() - t0
            reps += 1
    nbytes = reps * t * kv_bytes_per_token_head(d)
    desc = (f"oracle decode of 1 of {B * Hkv} (b, kvh) pairs ({g} query heads, {t} tokens, d={d}), "
            f"{reps} repetitions, float64 NumPy, BLAS threads 1")
    return nbytes / elapsed / 1e9, elapsed, desc


def oracle_quantize_rate(n=4096, seed=77):
    from threadpoolctl import threadpool_limits

    import oracle as O
    import synth

    x = synth.unit_vectors(n, STAGE1["d"], seed=seed, dtype=np.float16).astype(np.float64)
    p = O.make_params(STAGE1["d"], O.FULL, seed=1)
    with threadpool_limits(limits=1):
        t0 = time.perf_counter()
        O.quantize(x, p, STAGE1["bits"], O.FULL)
        dt = time.perf_counter() - t0
    return n / dt / 1e6


# ---------------------------------------------------------------------------
# The oracle on all host cores: spawned worker processes (no CUDA in them),
# BLAS threads 1 each, released together by a barrier so that the timed parts
# overlap; the rate is the bytes (or vectors) of all workers over the
# slowest worker's timed seconds.
# ---------------------------------------------------------------------------

_POOL_BARRIER = None


def _pool_init(barrier):
    global _POOL_BARRIER
    _POOL_BARRIER = barrier
    for var in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS"):
        os.environ[var] = "1"


def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def _pool_run(fn, tasks, sync, workers=None):
    """Runs fn over tasks in spawned processes.  With sync, one task per
    worker, each waiting on a shared barrier before its timed part."""
    import multiprocessing as mp

    ctx = mp.get_context("spawn")
    n = len(tasks) if sync else max(1, min(len(tasks), workers or len(tasks)))
    barrier = ctx.Barrier(n) if sync else None
    with ctx.Pool(n, initializer=_pool_init, initargs=(barrier,)) as pool:
        return pool.map_async(fn, tasks, chunksize=1).get(timeout=900)


def _oracle_decode_task(task):
    """One (b, kvh) pair of the decode workload: its G query heads over
    `tokens` tokens; oracle decodes repeated for at least min_s seconds."""
    from threadpoolctl import threadpool_limits

    import oracle as O
    import synth

    workload, seed, tokens, min_s = task
    B, Hq, Hkv, T, d = WORKLOADS[workload]
    g = Hq // Hkv
    with threadpool_limits(limits=1):
        k, v = synth.student_t_kv(1, tokens, d, seed=seed)
        prk = O.make_params(d, O.FULL, seed=1)
        prv = O.make_params(d, O.FULL, seed=2)
        pk, nk = O.quantize(k[0].astype(np.float64), prk, 3, O.FULL)
        pv, nv = O.quantize(v[0].astype(np.float64), prv, 3, O.FULL)
        q = synth.queries(1, g, d, seed=seed + 1)
        args = (q, pk[None], pv[None], nk[None], nv[None], [tokens], prk, prv, 3, O.FULL, 1 / math.sqrt(d))
        if _POOL_BARRIER is not None:
            _POOL_BARRIER.wait(timeout=600)
        reps, elapsed = 0, 0.0
        while elapsed < min_s:
            t0 = time.perf_counter()
            O.decode_attention(*args)
            elapsed += time.perf_counter() - t0
            reps += 1
    return reps * tokens * kv_bytes_per_token_head(d), reps * tokens, elapsed


def _oracle_quantize_task(task):
    """Oracle quantize of one seeded chunk of stage-1 unit vectors, repeated
    for at least min_s seconds."""
    from threadpoolctl import threadpool_limits

    import oracle as O
    import synth

    n, d, bits, seed, min_s = task
    with threadpool_limits(limits=1):
        x = synth.unit_vectors(n, d, seed=seed, dtype=np.float16).astype(np.float64)
        p = O.make_params(d, O.FULL, seed=1)
        if _POOL_BARRIER is not None:
            _POOL_BARRIER.wait(timeout=600)
        reps, elapsed = 0, 0.0
        while elapsed < min_s:
            t0 = time.perf_counter()
            O.quantize(x, p, bits, O.FULL)
            elapsed += time.perf_counter() - t0
            reps += 1
    return reps * n, elapsed


def oracle_pool_rates(workload, cores, tokens=2048, min_s=6.0):
    """The oracle on `cores` host cores: decode GB/s and token-heads/s over
    one (b, kvh) pair per core, and quantize vectors/s over one 4,096-vector
    chunk per core (stage-1 setting, d=128, 3-bit, float16 input)."""
    dec = _pool_run(_oracle_decode_task, [(workload, 3000 + 7 * i, tokens, min_s) for i in range(cores)], True)
    qnt = _pool_run(_oracle_quantize_task,
                    [(4096, STAGE1["d"], STAGE1["bits"], 5000 + i, min_s / 2) for i in range(cores)], True)
    t_dec = max(r[2] for r in dec)
    t_q = max(r[1] for r in qnt)
    B, Hq, Hkv, T, d = WORKLOADS[workload]
    return {
        "cores": cores,
        "decode_gbs": sum(r[0] for r in dec) / t_dec / 1e9,
        "decode_token_heads_per_s": sum(r[1] for r in dec) / t_dec,
        "quantize_vec_per_s": sum(r[0] for r in qnt) / t_q,
        "sample": (f"one (b, kvh) pair per core ({Hq // Hkv} query heads, {tokens} tokens, d={d}) and one "
                   f"4,096-vector stage-1 chunk per core; {cores} spawned processes, BLAS threads 1 each, "
                   f"released together; rate = all workers' work / slowest worker's seconds"),
    }


def _oracle_check_task(task):
    """Oracle compression of one input chunk, compared with the GPU's codes
    and norms for the same chunk: (vectors, code mismatches inside the 1e-5
    boundary band, outside it, norm mismatches at an float16 midpoint, away
    from one, oracle reconstruction squared error, GPU reconstruction
    squared error, squared norm of the input)."""
    from threadpoolctl import threadpool_limits

    import oracle as O

    x, params, bits, variant, gcodes, gnorms, grecon = task
    with threadpool_limits(limits=1):
        d = x.shape[-1]
        x64 = np.asarray(x, dtype=np.float64)[None]
        oc, on, y = O.quantize(x64, params, bits, variant, return_rotated=True)
        _, thr = O.make_codebook(d, bits)
        gc = O.bitunpack(np.asarray(gcodes)[None], bits, d)
        rc = O.bitunpack(oc, bits, d)
        mism = gc != rc
        band = np.zeros(mism.sum(), dtype=bool)
        if mism.any():
            dist = np.min(np.abs(y[mism][:, None] - np.asarray(thr)[None, :]), axis=1)
            band = dist < 1e-5
        gn = np.asarray(gnorms, dtype=np.float16)[None]
        nm = gn.view(np.uint16) != on.view(np.uint16)
        s = np.sqrt(np.sum(x64 * x64, axis=-1))
        mid = 0.5 * (gn.astype(np.float64) + on.astype(np.float64))
        at_mid = np.abs(s - mid) <= 1e-6 * s
        orec = O.dequantize(oc, on, params, bits, variant, d)
        return (x64.shape[1], int(band.sum()), int((~band).sum()), int((nm & at_mid).sum()),
                int((nm & ~at_mid).sum()), float(np.sum((orec - x64) ** 2)),
                float(np.sum((np.asarray(grecon, dtype=np.float64)[None] - x64) ** 2)), float(np.sum(x64 * x64)))


def oracle_checks(tasks, cores):
    return _pool_run(_oracle_check_task, tasks, False, workers=cores) if tasks else []


def summarize_checks(rows):
    n = sum(r[0] for r in rows)
    return {"vectors": n, "code_mismatches_in_band": sum(r[1] for r in rows),
            "code_mismatches_outside_band": sum(r[2] for r in rows),
            "norm_mismatches_at_midpoint": sum(r[3] for r in rows),
            "norm_mismatches_elsewhere": sum(r[4] for r in rows),
            "rel_mse_oracle": sum(r[5] for r in rows) / sum(r[7] for r in rows),
            "rel_mse_gpu": sum(r[6] for r in rows) / sum(r[7] for r in rows)}


# ---------------------------------------------------------------------------
# Reference arm
# ---------------------------------------------------------------------------

def run_reference(args):
    rank = env_int("RANK", 0)
    if rank != 0:
        return 0
    workload = args.workload
    B, Hq, Hkv, T, d = WORKLOADS[workload]
    # Size each step so that warm-up + timed steps take about two minutes.
    rate_gbs, secs, _ = oracle_decode_sample(workload, budget_s=5, min_s=0.5, tokens=4096)
    tok_per_s = rate_gbs * 1e9 / kv_bytes_per_token_head(d)
    per_step_s = 120.0 / max(1, args.steps + args.warmup)
    t_step = int(min(T, max(1024, tok_per_s * per_step_s)) // 1024 * 1024)

    import oracle as O
    import synth
    from threadpoolctl import threadpool_limits

    g = Hq // Hkv
    k, v = synth.student_t_kv(1, t_step, d, seed=2000)
    prk = O.make_params(d, O.FULL, seed=1)
    prv = O.make_params(d, O.FULL, seed=2)
    pk, nk = O.quantize(k[0].astype(np.float64), prk, 3, O.FULL)
    pv, nv = O.quantize(v[0].astype(np.float64), prv, 3, O.FULL)
    q = synth.queries(1, g, d, seed=2001)
    call = (q, pk[None], pv[None], nk[None], nv[None], [t_step], prk, prv, 3, O.FULL, 1 / math.sqrt(d))
    with threadpool_limits(limits=1):
        for _ in range(args.warmup):
            O.decode_attention(*call)
        t0 = time.perf_counter()
        for _ in range(args.steps):
            O.decode_attention(*call)
        elapsed = time.perf_counter() - t0
    nbytes = args.steps * t_step * kv_bytes_per_token_head(d)
    value = nbytes / elapsed / 1e9
    sample = (f"per step: oracle decode of 1 of {B * Hkv} (b, kvh) pairs, {g} query heads, "
              f"{t_step} of {T} tokens, d={d}, float64 NumPy, BLAS threads 1")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": elapsed / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(workload, args.gpus),
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": 1, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def workload_config(workload, n_gpus, batch=0, context=0):
    B, Hq, Hkv, T, d = WORKLOADS[workload]
    B = batch or B
    T = context or T
    return {
        "workload": workload + "+stage1_quantize_dequantize_d128_b3_f16_n1048576",
        "batch": B, "context": T, "q_heads": Hq, "kv_heads": Hkv, "head_dim": d, "bits": 3,
        "variant": "IsoQuant-Full", "stage1_vectors": STAGE1["n"],
        "l2": ("inputs larger than L2: each step streams the whole 3.3 GB packed K/V cache; the stage-1 "
               "quantize input is evicted by that stream between steps, and the dequantize reads codes "
               "written two steps earlier (four rotating 50 MB code buffers)"),
        "parallelism": f"replicas x{n_gpus} (weak; no data-path collective)",
    }


# ---------------------------------------------------------------------------
# Multi-rank helpers (weak-scaled replicas)
# ---------------------------------------------------------------------------

def max_over_ranks(values, dist=None, device=None):
    """Element-wise max of per-rank timings (every rank gets the result)."""
    import torch

    t = torch.tensor(values, dtype=torch.float64, device=device)
    if dist is not None and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def aggregate_gbs(bytes_per_step_per_rank, steps, max_ms, n_ranks):
    """Whole-job GB/s: bytes of all ranks over the slowest rank's time."""
    return n_ranks * bytes_per_step_per_rank * steps / (max_ms * 1e-3) / 1e9


def rank_seed(rank):
    """Each replica draws its own data."""
    return 1000 * rank


# ---------------------------------------------------------------------------
# CUDA arm
# ---------------------------------------------------------------------------

class L2Flush:
    """Evicts the 126 MB L2 between timed repetitions: writes, then reads, a
    buffer of four times the L2 size, so that the lines it leaves behind are
    clean (no write-back traffic lands in the next timed launch)."""

    def __init__(self, torch, dev):
        l2 = torch.cuda.get_device_properties(dev).L2_cache_size or (126 << 20)
        self.buf = torch.empty(4 * l2, dtype=torch.uint8, device=dev)
        self.bytes = 4 * l2

    def __call__(self):
        self.buf.zero_()
        self.buf.max()


def timed_reps(torch, stream, fn, reps, flush=None):
    """Device times (ms) of `reps` calls of fn, each after an L2 flush when
    one is given, CUDA events on the launching stream around the call only."""
    out = []
    for _ in range(reps):
        if flush is not None:
            flush()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        fn()
        e1.record(stream)
        torch.cuda.synchronize()
        out.append(e0.elapsed_time(e1))
    return out


def med_cv(xs):
    m = float(statistics.median(xs))
    cv = float(statistics.pstdev(xs) / statistics.mean(xs)) if len(xs) > 1 and statistics.mean(xs) > 0 else 0.0
    return m, cv


STAGE1_SWEEP_SLICE = 4096


def measure_stage1_sweep(isoq, torch, dev, stream, flush, hbm, cores, n=1 << 20, reps=5):
    """The 36-setting stage-1 sweep: d in {128, 256, 512} x bits in {2, 3, 4}
    x {float16, float32} x {Full, Fast}, N = 2^20 normalised N(0, I_d)
    vectors.  Per setting: quantize and dequantize device time (median of
    `reps`, L2 flushed before each), vectors/s, quantize GB/s on input +
    packed codes + float16 norms and its fraction of HBM peak, the relative
    reconstruction MSE over all N; and on a seeded 4,096-vector slice, the
    codes and norms against the oracle (mismatch counts inside and outside
    the 1e-5 boundary band) and both reconstruction MSEs."""
    import synth

    rows, checks, gen = [], [], torch.Generator(device=dev)
    for d in (128, 256, 512):
        for var, vname in ((isoq.ISOQ_FULL, "Full"), (isoq.ISOQ_FAST, "Fast")):
            p_np = isoq.isoq_make_params(d, var, 1, 1)
            p = torch.from_numpy(p_np).to(dev)
            for dt, dname, np_dt in ((torch.float16, "f16", np.float16), (torch.float32, "f32", np.float32)):
                gen.manual_seed(1000 + d)
                x = torch.randn((1, n, d), generator=gen, device=dev)
                x = (x / x.norm(dim=-1, keepdim=True)).to(dt)
                r = torch.empty_like(x)
                nrm = torch.empty((1, n), dtype=torch.float16, device=dev)
                xs_np = synth.unit_vectors(STAGE1_SWEEP_SLICE, d, seed=d + var, dtype=np_dt)
                xs = torch.from_numpy(xs_np).to(dev)
                for bits in (2, 3, 4):
                    pb = isoq.isoq_packed_bytes(d, bits)
                    c = torch.empty((1, n, pb), dtype=torch.uint8, device=dev)
                    qf = lambda: isoq.isoq_quantize(x, p, bits, var, codes=c, norms=nrm)  # noqa: E731
                    df = lambda: isoq.isoq_dequantize(c, nrm, p, d, bits, var, out=r)  # noqa: E731
                    qf()
                    df()
                    tq = timed_reps(torch, stream, qf, reps, flush)
                    td = timed_reps(torch, stream, df, reps, flush)
                    xf = x.float()
                    mse = float(((r.float() - xf) ** 2).sum() / (xf * xf).sum())
                    mq, cvq = med_cv(tq)
                    md, cvd = med_cv(td)
                    qbytes = n * (d * x.element_size() + pb + 2)
                    row = {"d": d, "bits": bits, "dtype": dname, "variant": vname,
                           "quantize_ms": mq, "quantize_cv": cvq, "quantize_mvec_s": n / (mq * 1e-3) / 1e6,
                           "quantize_gbs": qbytes / (mq * 1e-3) / 1e9, "quantize_frac": qbytes / (mq * 1e-3) / 1e9 / hbm,
                           "dequantize_ms": md, "dequantize_cv": cvd, "dequantize_mvec_s": n / (md * 1e-3) / 1e6,
                           "rel_mse_gpu_all": mse}
                    sc, sn = isoq.isoq_quantize(xs, p, bits, var)
                    sr = isoq.isoq_dequantize(sc, sn, p, d, bits, var, out_dtype=torch.float32)
                    checks.append((xs_np[0], p_np, bits, var, sc[0].cpu().numpy(), sn[0].cpu().numpy(),
                                   sr[0].cpu().numpy()))
                    rows.append(row)
                    del c
                del x, r, nrm, xs
    torch.cuda.empty_cache()
    assert isoq.isoq_check_device_error() == 0
    results = oracle_checks(checks, cores)
    for row, res in zip(rows, results):
        row["oracle_slice"] = summarize_checks([res])
    return {"workload": "stage-1 sweep: 36 settings, 2^20 normalised N(0, I_d) vectors each (device-drawn); "
                        f"oracle comparison on a {STAGE1_SWEEP_SLICE}-vector seeded slice per setting",
            "timing": f"median of {reps} launches, L2 flushed before each (CUDA events around the launch)",
            "settings": rows,
            "all_slices": summarize_checks(results)}


def measure_prefill_compression(isoq, torch, dev, stream, flush, hbm, cores, reps=10):
    """The KV-cache prefill-compression workload: 4 KV heads x 32,768 tokens x
    d=128 float16 K and V (Student-t nu=4 with 4 outlier channels per head
    x10, RoPE at base 1e6 on K), 3-bit Full, K rotation seed 1, V seed 2.
    Throughput of isoq_quantize on K then V (80 MB, below L2: flushed before
    each repetition), and every code and norm against the oracle."""
    import synth

    h, t, d, bits = 4, 32768, 128, 3
    k, v = synth.student_t_kv(h, t, d, seed=3)
    k, v = k[0], v[0]
    pk_np = isoq.isoq_make_params(d, isoq.ISOQ_FULL, 1, h)
    pv_np = isoq.isoq_make_params(d, isoq.ISOQ_FULL, 2, h)
    kd, vd = torch.from_numpy(k).to(dev), torch.from_numpy(v).to(dev)
    pk, pv = torch.from_numpy(pk_np).to(dev), torch.from_numpy(pv_np).to(dev)
    ck = torch.empty((h, t, 48), dtype=torch.uint8, device=dev)
    cv = torch.empty_like(ck)
    nk = torch.empty((h, t), dtype=torch.float16, device=dev)
    nv = torch.empty_like(nk)

    def both():
        isoq.isoq_quantize(kd, pk, bits, isoq.ISOQ_FULL, codes=ck, norms=nk)
        isoq.isoq_quantize(vd, pv, bits, isoq.ISOQ_FULL, codes=cv, norms=nv)

    both()
    ts = timed_reps(torch, stream, both, reps, flush)
    m, cv_ = med_cv(ts)
    nvec = 2 * h * t
    nbytes = nvec * (2 * d + 48 + 2)
    rk = isoq.isoq_dequantize(ck, nk, pk, d, bits, isoq.ISOQ_FULL).cpu().numpy()
    rv = isoq.isoq_dequantize(cv, nv, pv, d, bits, isoq.ISOQ_FULL).cpu().numpy()
    assert isoq.isoq_check_device_error() == 0
    tasks = []
    step = 8192
    for x, par, codes, norms, rec in ((k, pk_np, ck, nk, rk), (v, pv_np, cv, nv, rv)):
        cc, nn = codes.cpu().numpy(), norms.cpu().numpy()
        for hh in range(h):
            for t0 in range(0, t, step):
                tasks.append((x[hh, t0:t0 + step], par[hh:hh + 1], bits, isoq.ISOQ_FULL, cc[hh, t0:t0 + step],
                              nn[hh, t0:t0 + step], rec[hh, t0:t0 + step]))
    checks = summarize_checks(oracle_checks(tasks, cores))
    return {"workload": "prefill compression: 4 KV heads x 32,768 tokens x d=128 float16 K and V (Student-t "
                        "nu=4, 4 outlier channels x10 per head, RoPE base 1e6 on K), 3-bit Full",
            "ms": m, "cv": cv_, "mvec_s": nvec / (m * 1e-3) / 1e6, "gbs": nbytes / (m * 1e-3) / 1e9,
            "frac": nbytes / (m * 1e-3) / 1e9 / hbm, "vectors": nvec, "bytes": nbytes,
            "timing": f"median of {reps} (K then V), L2 flushed before each", "oracle": checks}


VARIANT_NAMES = {0: "Full (WHT+SO(4), v3)", 1: "Fast (WHT+q_L)", 2: "2-D special case (WHT+planar)",
                 3: "v2: block SO(4), no WHT", 4: "v1: single quaternion, no WHT"}


def measure_variants(isoq, synth, torch, dev, stream, x1, seed0, reps=5):
    """Per rotation variant: quantize throughput on the stage-1 workload and
    the relative round-trip error on it and on outlier-channel keys."""
    n1, d1, bits = x1.shape[1], x1.shape[2], STAGE1["bits"]
    k, _ = synth.student_t_kv_torch(1, 1, 65536, d1, seed=seed0 + 31, device=dev)
    xk = k[0]
    out = {}
    for var, name in VARIANT_NAMES.items():
        p = torch.from_numpy(isoq.isoq_make_params(d1, var, 1, 1)).to(dev)
        codes = torch.empty((1, n1, d1 * bits // 8), dtype=torch.uint8, device=dev)
        norms = torch.empty((1, n1), dtype=torch.float16, device=dev)
        for _ in range(2):
            isoq.isoq_quantize(x1, p, bits, var, codes=codes, norms=norms)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            isoq.isoq_quantize(x1, p, bits, var, codes=codes, norms=norms)
        e1.record(stream)
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / reps
        rel = {}
        for label, x in (("unit_vectors", x1), ("outlier_keys", xk)):
            c, nrm = isoq.isoq_quantize(x, p, bits, var)
            r = isoq.isoq_dequantize(c, nrm, p, d1, bits, var, out_dtype=torch.float32)
            xf = x.float()
            rel[label] = float((((r - xf) ** 2).sum(-1) / (xf * xf).sum(-1)).mean())
        out[name] = {"quantize_mvec_s": n1 / (ms * 1e-3) / 1e6, "quantize_ms": ms,
                     "rel_mse_unit_vectors": rel["unit_vectors"], "rel_mse_outlier_keys": rel["outlier_keys"]}
    assert isoq.isoq_check_device_error() == 0
    return {"workload": f"2^20 float16 unit vectors (stage-1) and 65,536 Student-t keys with outlier "
                        f"channels and RoPE; d={d1}, {bits}-bit", "by_variant": out}


def measure_rotor_comparison(isoq, torch, dev, stream, n=1 << 20, reps=3):
    """IsoQuant-Full against the RotorQuant comparator on the stage-1 sweep:
    d in {128, 256, 512} x bits in {2, 3, 4} x {float16, float32}, N = 2^20
    normalised N(0, I_d) vectors; quantize + dequantize time of each, CUDA
    events on the launching stream."""
    rows = []
    gen = torch.Generator(device=dev)
    for d in (128, 256, 512):
        p = torch.from_numpy(isoq.isoq_make_params(d, isoq.ISOQ_FULL, 1, 1)).to(dev)
        rot = torch.from_numpy(isoq.isoq_rotor_make_params(d, 1, 1)).to(dev)
        for dt in (torch.float16, torch.float32):
            gen.manual_seed(1000 + d)
            x = torch.randn((1, n, d), generator=gen, device=dev)
            x = (x / x.norm(dim=-1, keepdim=True)).to(dt)
            r = torch.empty_like(x)
            nrm = torch.empty((1, n), dtype=torch.float16, device=dev)
            for bits in (2, 3, 4):
                # outputs allocated once per arm: the timed calls launch kernels only
                ci = torch.empty((1, n, isoq.isoq_packed_bytes(d, bits)), dtype=torch.uint8, device=dev)
                cr = torch.empty((1, n, isoq.isoq_rotor_packed_bytes(d, bits)), dtype=torch.uint8, device=dev)
                arms = {
                    "isoquant": (lambda b=bits: isoq.isoq_quantize(x, p, b, isoq.ISOQ_FULL, codes=ci, norms=nrm),
                                 lambda c, s, b=bits: isoq.isoq_dequantize(c, s, p, d, b, isoq.ISOQ_FULL, out=r)),
                    "rotorquant": (lambda b=bits: isoq.isoq_rotor_quantize(x, rot, b, codes=cr, norms=nrm),
                                   lambda c, s, b=bits: isoq.isoq_rotor_dequantize(c, s, rot, d, b, out=r)),
                }
                row = {"d": d, "bits": bits, "dtype": "f16" if dt == torch.float16 else "f32"}
                for name, (qf, df) in arms.items():
                    c, s_ = qf()
                    df(c, s_)
                    e = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
                    e[0].record(stream)
                    for _ in range(reps):
                        qf()
                    e[1].record(stream)
                    for _ in range(reps):
                        df(c, s_)
                    e[2].record(stream)
                    torch.cuda.synchronize()
                    xf = x.float()
                    mse = float(((r.float() - xf) ** 2).sum(-1).mean())
                    row[name] = {"quantize_ms": e[0].elapsed_time(e[1]) / reps,
                                 "dequantize_ms": e[1].elapsed_time(e[2]) / reps, "mse": mse}
                iq, rq = row["isoquant"], row["rotorquant"]
                row["speedup"] = (rq["quantize_ms"] + rq["dequantize_ms"]) / (iq["quantize_ms"] + iq["dequantize_ms"])
                rows.append(row)
                del ci, cr
            del x, r, nrm
    assert isoq.isoq_check_device_error() == 0
    speedups = [r["speedup"] for r in rows]
    return {"workload": "stage-1 sweep: d in {128,256,512} x bits in {2,3,4} x {f16,f32}, 2^20 unit "
                        "vectors; quantize + dequantize, IsoQuant-Full vs the RotorQuant comparator",
            "mean_speedup": sum(speedups) / len(speedups), "min_speedup": min(speedups),
            "max_speedup": max(speedups), "settings": rows}


PREFILL_WORKLOADS = [
    # (name, B, Hq, Hkv, context, chunk, d)
    ("chunk2048_ctx32768_gqa32_4_d128", 1, 32, 4, 32768, 2048, 128),
    ("chunk1024_ctx65536_gqa16_8_d256", 1, 16, 8, 65536, 1024, 256),
]


def measure_prefill(isoq, synth, torch, dev, stream, seed0, peak_tflops, reps=5):
    """Chunked prefill (causal attention of the chunk's queries over the packed
    cache that holds them) on each PREFILL_WORKLOADS shape: the cache is drawn
    with the Student-t generator and compressed by isoq_quantize, the queries
    are float16 N(0, 1).  Algorithmic FLOPs: 4 d per (query head, visible
    token) (QK and PV multiply-adds, the causal triangle included)."""
    out = {}
    for name, B, Hq, Hkv, ctx, tq, d in PREFILL_WORKLOADS:
        bits, variant, pb = 3, isoq.ISOQ_FULL, d * 3 // 8
        prk = torch.from_numpy(isoq.isoq_make_params(d, variant, 1, Hkv)).to(dev)
        prv = torch.from_numpy(isoq.isoq_make_params(d, variant, 2, Hkv)).to(dev)
        k, v = synth.student_t_kv_torch(B, Hkv, ctx, d, seed=seed0 + 51, device=dev)
        pk, nk = isoq.isoq_quantize(k.view(-1, ctx, d), prk.repeat(B, 1, 1), bits, variant)
        pv, nv = isoq.isoq_quantize(v.view(-1, ctx, d), prv.repeat(B, 1, 1), bits, variant)
        del k, v
        pk, pv = pk.view(B, Hkv, ctx, pb), pv.view(B, Hkv, ctx, pb)
        nk, nv = nk.view(B, Hkv, ctx), nv.view(B, Hkv, ctx)
        q = synth.queries_torch(B * tq, Hq, d, seed=seed0 + 52, device=dev).view(B, tq, Hq, d)
        lens = torch.full((B,), ctx, dtype=torch.int32, device=dev)
        o = torch.empty_like(q)
        for _ in range(2):
            isoq.isoq_prefill_attention(q, pk, pv, nk, nv, lens, prk, prv, bits, variant, out=o)
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            isoq.isoq_prefill_attention(q, pk, pv, nk, nv, lens, prk, prv, bits, variant, out=o)
        e1.record(stream)
        torch.cuda.synchronize()
        assert isoq.isoq_check_device_error() == 0
        ms = e0.elapsed_time(e1) / reps
        visible = sum(ctx - tq + t + 1 for t in range(tq))        # tokens seen by the chunk's queries
        flops = 4.0 * d * Hq * B * visible
        kv_bytes = B * Hkv * ctx * 2 * (pb + 2)
        tflops = flops / (ms * 1e-3) / 1e12
        out[name] = {"ms": ms, "tflops": tflops, "frac_of_tensor_peak": tflops / peak_tflops,
                     "queries_per_s": B * tq / (ms * 1e-3), "kv_bytes": kv_bytes,
                     "kernel": f"prefill_tc_kernel<__half, {d}, Full, GP={Hq // Hkv}>"}
        del pk, pv, nk, nv, q, o
    torch.cuda.empty_cache()
    return {"workloads": out, "peak_tflops": peak_tflops,
            "peak_source": "MEASURED_PEAKS.json bf16_tflops (burst; float16 runs at the bf16 rate)",
            "what": "isoq_prefill_attention: one chunk of float16 queries at the end of the context, "
                    "causal, 3-bit Full, tcgen05.mma kind::f16 with accumulators in tensor memory"}


DECODE_SWEEP = [
    # (name, B, Hq, Hkv, Tmax, d, ragged)
    ("b1_gqa32_4_d128_t32768", 1, 32, 4, 32768, 128, False),
    ("b16_gqa32_4_d128_t8192_ragged", 16, 32, 4, 8192, 128, True),
] + [(f"b32_gqa16_8_d256_t{t}", 32, 16, 8, t, 256, False) for t in (1024, 2048, 4096, 8192, 16384, 32768)]


def measure_decode_sweep(isoq, synth, torch, dev, seed0, hbm, flush, reps=20, runs=3):
    """Decode attention (query preparation + split + combine) on the small
    decode workloads and the long-context shape at shorter contexts: each
    call captured once in a CUDA graph, so host launch overhead does not
    enter the small cases; every replay follows an L2 flush (these working
    sets, 13-103 MB, fit in the 126 MB L2) and is timed alone.  `runs` runs
    of `reps` replays: the median over all replays, and the coefficient of
    variation of the runs' medians."""
    out = {}
    for name, B, Hq, Hkv, T, d, ragged in DECODE_SWEEP:
        bits, variant, pb = 3, isoq.ISOQ_FULL, d * 3 // 8
        prk = torch.from_numpy(isoq.isoq_make_params(d, variant, 1, Hkv)).to(dev)
        prv = torch.from_numpy(isoq.isoq_make_params(d, variant, 2, Hkv)).to(dev)
        k, v = synth.student_t_kv_torch(B, Hkv, T, d, seed=seed0 + 61, device=dev)
        pk, nk = isoq.isoq_quantize(k.view(-1, T, d), prk.repeat(B, 1, 1), bits, variant)
        pv, nv = isoq.isoq_quantize(v.view(-1, T, d), prv.repeat(B, 1, 1), bits, variant)
        del k, v
        pk, pv, nk, nv = pk.view(B, Hkv, T, pb), pv.view(B, Hkv, T, pb), nk.view(B, Hkv, T), nv.view(B, Hkv, T)
        q = synth.queries_torch(B, Hq, d, seed=seed0 + 62, device=dev)
        lens_np = synth.ragged_lengths(B, T // 2, T, seed=0) if ragged else np.full(B, T, dtype=np.int32)
        lens = torch.from_numpy(lens_np).to(dev)
        o = torch.empty((B, Hq, d), dtype=torch.float16, device=dev)
        ws = torch.empty(isoq.isoq_decode_workspace_size(B, Hq, Hkv, T, d), dtype=torch.uint8, device=dev)
        call = lambda: isoq.isoq_decode_attention(q, pk, pv, nk, nv, lens, prk, prv, bits, variant,  # noqa: E731
                                                  out=o, workspace=ws)
        for _ in range(3):
            call()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            call()
        g.replay()
        torch.cuda.synchronize()
        stream = torch.cuda.current_stream(dev)
        run_ms = [timed_reps(torch, stream, g.replay, reps, flush) for _ in range(runs)]
        assert isoq.isoq_check_device_error() == 0
        med, _ = med_cv([t for r in run_ms for t in r])
        _, cv = med_cv([statistics.median(r) for r in run_ms])
        us = med * 1e3
        kv_bytes = int(lens_np.clip(0, T).sum()) * Hkv * kv_bytes_per_token_head(d, bits)
        gbps = kv_bytes / (us * 1e-6) / 1e9
        out[name] = {"us": us, "gbps": gbps, "frac": gbps / hbm, "kv_bytes": kv_bytes, "cv_of_runs": cv,
                     "min_us": min(t for r in run_ms for t in r) * 1e3}
        del g, pk, pv, nk, nv, q, o, ws
        torch.cuda.empty_cache()
    return {"what": "isoq_decode_attention (prep + split + combine) replayed from a CUDA graph, L2 flushed "
                    f"before every replay; median of {runs} x {reps} replays; KV GB/s on the packed bytes of the "
                    "valid tokens", "by_workload": out}


def run_isoq(args):
    import torch

    import compressed_space_attention_b200 as isoq
    import synth

    world = env_int("WORLD_SIZE", 1)
    rank = env_int("RANK", 0)
    local_rank = env_int("LOCAL_RANK", 0)
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    else:
        torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    stream = torch.cuda.current_stream(dev)

    B, Hq, Hkv, T, d = WORKLOADS[args.workload]
    if args.batch:
        B = args.batch
    if args.context:
        T = args.context
    bits, variant = 3, isoq.ISOQ_FULL
    pb = d * bits // 8
    seed0 = rank_seed(rank)

    # ---- decode inputs: compress Student-t K/V into the packed cache ----
    prk = torch.from_numpy(np.tile(isoq.isoq_make_params(d, variant, 1, Hkv), (1, 1, 1))).to(dev)
    prv = torch.from_numpy(isoq.isoq_make_params(d, variant, 2, Hkv)).to(dev)
    pk = torch.empty((B, Hkv, T, pb), dtype=torch.uint8, device=dev)
    pv = torch.empty_like(pk)
    nk = torch.empty((B, Hkv, T), dtype=torch.float16, device=dev)
    nv = torch.empty_like(nk)
    bchunk = max(1, min(B, (1 << 28) // (Hkv * T * d)))  # bound the float16 staging size
    for b0 in range(0, B, bchunk):
        b1 = min(B, b0 + bchunk)
        k, v = synth.student_t_kv_torch(b1 - b0, Hkv, T, d, seed=seed0 + b0, device=dev)
        prk_t = prk.repeat(b1 - b0, 1, 1)
        prv_t = prv.repeat(b1 - b0, 1, 1)
        isoq.isoq_quantize(k.view(-1, T, d), prk_t, bits, variant,
                           codes=pk[b0:b1].view(-1, T, pb), norms=nk[b0:b1].view(-1, T))
        isoq.isoq_quantize(v.view(-1, T, d), prv_t, bits, variant,
                           codes=pv[b0:b1].view(-1, T, pb), norms=nv[b0:b1].view(-1, T))
        del k, v
    q = synth.queries_torch(B, Hq, d, seed=seed0 + 7, device=dev)
    if "ragged" in args.workload:
        lens_np = synth.ragged_lengths(B, T // 2, T, seed=0)
    else:
        lens_np = np.full(B, T, dtype=np.int32)
    lens = torch.from_numpy(lens_np).to(dev)
    out = torch.empty((B, Hq, d), dtype=torch.float16, device=dev)
    ws = torch.empty(isoq.isoq_decode_workspace_size(B, Hq, Hkv, T, d), dtype=torch.uint8, device=dev)
    kv_bytes = int(lens_np.clip(0, T).sum()) * Hkv * kv_bytes_per_token_head(d, bits)
    torch.cuda.synchronize()

    # ---- stage-1 inputs ----
    n1, d1 = STAGE1["n"], STAGE1["d"]
    gen = torch.Generator(device=dev)
    gen.manual_seed(seed0 + 11)
    x1 = torch.randn((1, n1, d1), generator=gen, device=dev)
    x1 = (x1 / x1.norm(dim=-1, keepdim=True)).half()
    p1 = torch.from_numpy(isoq.isoq_make_params(d1, variant, 1, 1)).to(dev)
    # Step i quantizes into code slot i % R and dequantizes slot (i + 2) % R,
    # written two steps (and 6.6 GB of decode reads) earlier, so the
    # dequantize does not read codes the quantize has just left in L2.
    n_slots = 4
    c1 = [torch.empty((1, n1, d1 * bits // 8), dtype=torch.uint8, device=dev) for _ in range(n_slots)]
    s1 = [torch.empty((1, n1), dtype=torch.float16, device=dev) for _ in range(n_slots)]
    for c_, s_ in zip(c1, s1):
        isoq.isoq_quantize(x1, p1, bits, variant, codes=c_, norms=s_)
    r1 = torch.empty((1, n1, d1), dtype=torch.float16, device=dev)
    q_bytes = n1 * (d1 * 2 + d1 * bits // 8 + 2)
    dq_bytes = n1 * (d1 * bits // 8 + 2 + d1 * 2)
    step_no = [0]

    def step(ev=None):
        i = step_no[0]
        step_no[0] += 1
        qs, ds = i % n_slots, (i + 2) % n_slots
        if ev:
            ev[0].record(stream)
        isoq.isoq_quantize(x1, p1, bits, variant, codes=c1[qs], norms=s1[qs])
        if ev:
            ev[1].record(stream)
        isoq.isoq_dequantize(c1[ds], s1[ds], p1, d1, bits, variant, out=r1)
        if ev:
            ev[2].record(stream)
        isoq.isoq_decode_split(q, pk, pv, nk, nv, lens, prk, bits, variant, ws)
        if ev:
            ev[3].record(stream)
        isoq.isoq_decode_combine(out, lens, B, Hq, Hkv, T, d, variant, prv, ws)
        if ev:
            ev[4].record(stream)

    sampler = ClockSampler(local_rank)
    sampler.start()
    try:
        for _ in range(args.warmup):
            step()
        torch.cuda.synchronize()
        assert isoq.isoq_check_device_error() == 0

        events = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
        start = torch.cuda.Event(enable_timing=True)
        end = torch.cuda.Event(enable_timing=True)
        if dist:
            dist.barrier()
        torch.cuda.synchronize()
        with sampler:
            start.record(stream)
            for i in range(args.steps):
                step(events[i])
            end.record(stream)
            torch.cuda.synchronize()
    finally:
        sampler.stop()
    if dist:
        dist.barrier()
    total_ms = start.elapsed_time(end)
    t_quant = sum(e[0].elapsed_time(e[1]) for e in events)
    t_deq = sum(e[1].elapsed_time(e[2]) for e in events)
    t_split = sum(e[2].elapsed_time(e[3]) for e in events)
    t_comb = sum(e[3].elapsed_time(e[4]) for e in events)
    t_decode = t_split + t_comb
    # three runs: the timed steps in three consecutive groups
    per_step_dec = [e[2].elapsed_time(e[4]) for e in events]
    groups = [per_step_dec[i * len(per_step_dec) // 3:(i + 1) * len(per_step_dec) // 3] for i in range(3)]
    run_gbs = [kv_bytes * len(gp) / (sum(gp) * 1e-3) / 1e9 for gp in groups if gp]
    split_ms = [e[2].elapsed_time(e[3]) for e in events]
    assert isoq.isoq_check_device_error() == 0

    # ---- end to end through the API with host buffers (decode half) ----
    e2e_steps = 0 if args.no_e2e else max(1, min(args.steps, 3))
    host = [t.cpu().pin_memory() for t in (q, pk, pv, nk, nv, lens)] if e2e_steps else []
    out_host = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in host)
    d2h = out_host.numel() * out_host.element_size()
    dev_bufs = [torch.empty_like(t, device=dev) for t in host]
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        for hb, db in zip(host, dev_bufs):
            db.copy_(hb, non_blocking=True)
        isoq.isoq_decode_attention(dev_bufs[0], dev_bufs[1], dev_bufs[2], dev_bufs[3], dev_bufs[4],
                                   dev_bufs[5], prk, prv, bits, variant, out=out, workspace=ws)
        out_host.copy_(out, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) if e2e_steps else 0.0
    if dist:
        dist.barrier()

    # ---- decode-step append, then the whole step (append + attention) ----
    # Timed after the main region on rows set to half their capacity, so the
    # appended positions never reach Tmax; the cache contents past the
    # original lengths do not affect the numbers above.
    kn = synth.queries_torch(B, Hkv, d, seed=seed0 + 21, device=dev)
    vn = synth.queries_torch(B, Hkv, d, seed=seed0 + 22, device=dev)
    lens_a = torch.full((B,), T // 2, dtype=torch.int32, device=dev)
    n_app = max(args.steps, 3)
    for _ in range(2):
        isoq.isoq_decode_append(kn, vn, pk, pv, nk, nv, lens_a, prk, prv, bits, variant)
    torch.cuda.synchronize()
    a0 = torch.cuda.Event(enable_timing=True)
    a1 = torch.cuda.Event(enable_timing=True)
    a2 = torch.cuda.Event(enable_timing=True)
    a0.record(stream)
    for _ in range(n_app):
        isoq.isoq_decode_append(kn, vn, pk, pv, nk, nv, lens_a, prk, prv, bits, variant)
    a1.record(stream)
    for _ in range(n_app):
        isoq.isoq_decode_step(q, kn, vn, pk, pv, nk, nv, lens_a, prk, prv, bits, variant, out=out,
                              workspace=ws)
    a2.record(stream)
    torch.cuda.synchronize()
    assert isoq.isoq_check_device_error() == 0
    t_app = a0.elapsed_time(a1) / n_app
    t_dstep = a1.elapsed_time(a2) / n_app
    app_bytes = 2 * B * Hkv * (2 * d + pb + 2)

    # ---- rotation variants (IsoQuant's 2-D case, RotaryQuant §4.6 v1, v2) ----
    variants = measure_variants(isoq, synth, torch, dev, stream, x1, seed0) if not args.no_variants else None
    comparator = measure_rotor_comparison(isoq, torch, dev, stream) if not args.no_comparator else None
    peaks_all, _ = measured_peaks()
    hbm_all = float(peaks_all.get("hbm_gbs", FALLBACK_HBM_GBS))
    flush = L2Flush(torch, dev)
    cores = host_cores()
    sweep = (measure_decode_sweep(isoq, synth, torch, dev, seed0, hbm_all, flush)
             if not args.no_sweep else None)
    stage1 = (measure_stage1_sweep(isoq, torch, dev, stream, flush, hbm_all, cores)
              if not args.no_stage1_sweep and rank == 0 else None)
    c3 = (measure_prefill_compression(isoq, torch, dev, stream, flush, hbm_all, cores)
          if not args.no_stage1_sweep and rank == 0 else None)
    prefill = (measure_prefill(isoq, synth, torch, dev, stream, seed0,
                               float(peaks_all.get("bf16_tflops", 1590.0))) if not args.no_prefill else None)

    # ---- reduce over ranks: max time, summed bytes ----
    total_ms, t_decode, t_split, t_quant, t_deq, t_comb, e2e_ms, t_app, t_dstep = max_over_ranks(
        [total_ms, t_decode, t_split, t_quant, t_deq, t_comb, e2e_ms, t_app, t_dstep], dist, dev)
    n_ranks = world

    peaks, peak_kind = measured_peaks()
    hbm = float(peaks.get("hbm_gbs", FALLBACK_HBM_GBS))
    value = aggregate_gbs(kv_bytes, args.steps, t_decode, n_ranks)
    split_avg_s = t_split / args.steps * 1e-3
    achieved = kv_bytes / split_avg_s / 1e9
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": n_ranks, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f16", "data": "synthetic",
        "config": workload_config(args.workload, n_ranks, args.batch, args.context),
        "frac_of_hbm_peak": value / n_ranks / hbm,
        "frac_of_nominal_8000_gbs": value / n_ranks / NOMINAL_HBM_GBS,
        "runs": {"what": "the timed steps in three consecutive groups: decode (split + combine) GB/s of each",
                 "gbs": run_gbs, "median_gbs": float(statistics.median(run_gbs)),
                 "cv": med_cv(run_gbs)[1] if len(run_gbs) > 1 else 0.0,
                 "split_ms_median": float(statistics.median(split_ms)), "split_ms_cv": med_cv(split_ms)[1]},
        "roofline": {"bound": "hbm", "kernel": "split_i8_kernel<256,Full,GP=2> (decode split)",
                     "achieved": achieved, "peak": hbm, "unit": "GB/s", "frac": achieved / hbm,
                     "frac_of_nominal_8000_gbs": achieved / NOMINAL_HBM_GBS,
                     "traffic": read_traffic(), "peak_source": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)",
                     "algorithmic_bytes_per_launch": kv_bytes},
        "quantize": {"value": n_ranks * n1 * args.steps / (t_quant * 1e-3) / 1e6, "unit": "Mvec/s",
                     "gbps": q_bytes * args.steps / (t_quant * 1e-3) / 1e9,
                     "frac": q_bytes * args.steps / (t_quant * 1e-3) / 1e9 / hbm,
                     "workload": "2^20 float16 unit vectors, d=128, 3-bit, Full"},
        "dequantize": {"value": n_ranks * n1 * args.steps / (t_deq * 1e-3) / 1e6, "unit": "Mvec/s",
                       "gbps": dq_bytes * args.steps / (t_deq * 1e-3) / 1e9,
                       "frac": dq_bytes * args.steps / (t_deq * 1e-3) / 1e9 / hbm},
        "step_ms": {"quantize": t_quant / args.steps, "dequantize": t_deq / args.steps,
                    "decode_split": t_split / args.steps, "decode_combine": t_comb / args.steps},
        "e2e": {"value": (n_ranks * kv_bytes * e2e_steps / (e2e_ms * 1e-3) / 1e9) if e2e_steps else None, "unit": "GB/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": e2e_steps,
                "path": "pinned host cache -> device copy -> isoq_decode_attention -> host copy of the output"},
        "decode_step": {"append_ms": t_app, "append_gbps": app_bytes / (t_app * 1e-3) / 1e9,
                        "append_bytes": app_bytes, "step_ms": t_dstep, "launches": n_app,
                        "what": "isoq_decode_append of one float16 K and V token per (b, kvh) "
                                "(append_kernel + length advance), and isoq_decode_step = append "
                                "then decode attention over the cache at half capacity; timed "
                                "outside the main region"},
        "variants": variants,
        "rotorquant_comparison": comparator,
        "prefill": prefill,
        "decode_sweep": sweep,
        "stage1_sweep": stage1,
        "prefill_compression": c3,
        # per step: quantize_kernel, dequantize_kernel, prep_i8_kernel +
        # split_i8_kernel (isoq_decode_split), combine_kernel
        "gpu_launches": 5 * args.steps,
        "clocks": sampler.summary(),
    }
    if rank == 0 and not args.no_cpu_baseline:
        gbs, secs, desc = oracle_decode_sample(args.workload)
        line["cpu_baseline"] = {"value": gbs, "unit": "GB/s", "cores": 1, "kind": "oracle",
                                "sample": desc, "seconds": secs,
                                "quantize_mvec_s": oracle_quantize_rate(),
                                "all_cores": oracle_pool_rates(args.workload, cores)}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["isoq", "reference"], default="isoq")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default=DEFAULT_WORKLOAD)
    ap.add_argument("--no-cpu-baseline", action="store_true",
                    help="skip the oracle CPU baseline (profiling runs)")
    ap.add_argument("--no-sweep", action="store_true",
                    help="skip the decode measurements at small batch and shorter contexts")
    ap.add_argument("--no-prefill", action="store_true",
                    help="skip the chunked-prefill attention measurement")
    ap.add_argument("--no-comparator", action="store_true",
                    help="skip the IsoQuant vs RotorQuant stage-1 sweep")
    ap.add_argument("--no-variants", action="store_true",
                    help="skip the rotation-variant measurements (2-D case, ablation v1/v2)")
    ap.add_argument("--no-e2e", action="store_true",
                    help="skip the host-buffer end-to-end leg (profiling runs)")
    ap.add_argument("--no-stage1-sweep", action="store_true",
                    help="skip the 36-setting stage-1 sweep and the prefill-compression line")
    ap.add_argument("--batch", type=int, default=0,
                    help="override the decode batch size (smaller profiling cases)")
    ap.add_argument("--context", type=int, default=0,
                    help="override the decode context length (the long-context sweep)")
    ap.add_argument("--record-traffic", metavar="NCU_RAW_CSV",
                    help="write the decode split's per-launch DRAM traffic from an ncu raw CSV export and exit")
    ap.add_argument("--traffic-scale", type=float, default=1.0,
                    help="full launch's units over the captured launch's (with --record-traffic)")
    ap.add_argument("--traffic-note", default="", help="how the capture was taken (with --record-traffic)")
    args = ap.parse_args()
    if args.record_traffic:
        record_traffic(args.record_traffic, r"split_i8_kernel", args.traffic_scale, args.traffic_note)
        return 0
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.impl == "reference":
        return run_reference(args)
    return run_isoq(args)


if __name__ == "__main__":
    sys.exit(main())
