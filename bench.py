#!/usr/bin/env python
"""QAM-W codec benchmark: encode/decode Gweights/s of one weight matrix per step.

A *step* is one pass of the whole hot path over one matrix:
qamw_calibrate_encode (channel scale and row norms once, then the sigma_k
calibration pass and the encode pass: rotation, nearest-centroid search,
packing) and qamw_decode (bf16 weights), all through the C ABI of libqamw.so. The default workload is the Llama-7B-shaped attention projection:
bf16 4096 x 4096, N(0, 0.02^2) with 0.5% outlier columns x20, act RMS
lognormal(0, 1), alpha 0.5, Hadamard block 128, 2048 centroids (11 bits per
pair). Inputs are synthetic (seeded); the codebook is the shipped Lloyd table.

Usage:
  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
  torchrun --nproc-per-node N bench.py --gpus N ...   (one replica per GPU)

Timing: inputs resident in HBM; L2 flushed (256 MiB write) before every timed
step; CUDA events on the launching stream around each C-ABI call; max over
ranks. Each rank codes its own matrix (independent problems, no collective on
the data path), so scaling is weak. ``--impl reference`` times the CPU oracle
(fp64 numpy) on bounded row samples of the same workload.
"""
from __future__ import annotations

import argparse
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
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "QAM-W encode/decode Gweights/s per matrix; decode % HBM roofline, encode % FP32"
FALLBACK_HBM_GBS = 6650.0
SM_COUNT_B200 = 148
FP32_LANES_PER_SM = 128
L2_FLUSH_BYTES = 256 << 20
# DRAM bytes (read + written) of one launch of the encode kernel on a
# workload, from one ncu capture of that kernel (dram__bytes_read.sum +
# dram__bytes_write.sum); an entry is removed whenever the kernel changes,
# until it is captured again. The default workload's figure: 33.81 MB read +
# 22.78 MB written (the written bytes include the previous step's L2-flush
# buffer written back while the kernel runs, under ncu's flushed replay).
ENCODE_TRAFFIC_BYTES = {"llama7b_attn": 56592384}


def parse_args(argv=None):
    p = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--impl", choices=("ours", "reference"), default="ours")
    p.add_argument("--workload", default="llama7b_attn",
                   choices=("llama7b_attn", "tiny", "decode_13b", "rate35", "rate4", "lloyd", "polar", "mlp",
                            "stack_1p1b", "decode_gemm"),
                   help="llama7b_attn: 4096x4096 bf16 at 2048 centroids (5.5 bits/weight; the default); "
                        "rate35 / rate4: the same matrix at 128 / 256 centroids (3.5 / 4 bits/weight); "
                        "decode_13b: decode-only sweep over the 13B shapes; tiny: 256x512 fp32; "
                        "lloyd: codebook training, one Lloyd iteration of 2048 centroids on 2^21 samples per step; "
                        "polar: the polar baseline codec on the 4096x4096 projection at 2048 points; "
                        "mlp: the 24 MLP runs (11008x4096 and 4096x11008, alpha x block x codebook); "
                        "stack_1p1b: the 154 matrices of the 22-layer 1.1B-shaped stack; "
                        "decode_gemm: the fused decode + matmul on the 13824x5120 matrix at 1..4096 tokens")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--cpu-rows", type=int, default=0, help="rows per oracle sample (0 = auto)")
    p.add_argument("--search", choices=("pruned", "brute"), default="pruned",
                   help="nearest-centroid search: exact pruned table (default) or brute force")
    p.add_argument("--no-graph", dest="graph", action="store_false",
                   help="time the step launched call by call only (default: also replay it as a CUDA graph, "
                        "which is the headline)")
    p.add_argument("--brute-steps", type=int, default=3,
                   help="extra brute-force encodes timed after the steps (FP32 roofline of that search)")
    return p.parse_args(argv)


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", str(rank)))
    return rank, world, local


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return json.load(f), "measured"
    return {"hbm_gbs": FALLBACK_HBM_GBS, "sm_max_mhz": 1965.0}, "fallback"


def workload_spec(name):
    import synth
    return synth.WORKLOADS[name]().specs[0], synth.WORKLOADS[name]().name


# ---------------------------------------------------------------------------
# clocks sampled during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("clocks.sm", "clocks.max.sm", "clocks_event_reasons.active", "clocks_event_reasons.hw_slowdown",
              "clocks_event_reasons.hw_thermal_slowdown", "clocks_event_reasons.sw_thermal_slowdown",
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), "--query-gpu=" + ",".join(self.FIELDS),
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, FileNotFoundError):
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)
        sm, mx, reasons = [], [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) != len(self.FIELDS):
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[3:]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------
# multi-rank helpers (also exercised by the gloo tests on CPU)
# ---------------------------------------------------------------------------

def max_over_ranks(value: float, device=None) -> float:
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_throughput(units_per_rank: float, seconds_max: float, world: int) -> float:
    """Whole-job rate: units all ranks processed / the slowest rank's time."""
    return units_per_rank * world / seconds_max


# ---------------------------------------------------------------------------
# CPU oracle on a bounded sample (cpu_baseline and the reference arm)
# ---------------------------------------------------------------------------

def oracle_sample_step(W32_rows, act, spec, C):
    """calibrate + encode + decode of a row sample with the oracle (fp64 numpy)."""
    from oracle import codec
    sig = codec.calibrate_sigma(W32_rows, act, spec.alpha, spec.block, spec.seed)
    enc = codec.encode(W32_rows, act, spec.alpha, spec.block, spec.seed, sig, C, spec.bits)
    codec.decode(enc["packed"], enc["r"], sig, act, spec.alpha, spec.K, spec.block, spec.seed, C, spec.bits)


_WORKER_LIMITS = None


def _oracle_worker_init():
    """Each oracle worker process runs numpy on one thread (the pool supplies the parallelism)."""
    global _WORKER_LIMITS
    from threadpoolctl import threadpool_limits
    _WORKER_LIMITS = threadpool_limits(limits=1)


def _oracle_task(job):
    W_rows, act, spec, C = job
    oracle_sample_step(W_rows, act, spec, C)
    return W_rows.shape[0]


class OraclePool:
    """The oracle on every host core: a pool of spawned worker processes (one
    numpy thread each), each running the whole calibrate + encode + decode
    of its own block of rows. Spawned, not forked, so that it is safe next to
    a CUDA context."""

    def __init__(self, workers=None):
        import multiprocessing as mp
        self.workers = int(workers or os.cpu_count() or 1)
        self.pool = mp.get_context("spawn").Pool(self.workers, initializer=_oracle_worker_init)

    def run(self, W32, act, spec, C, rows_per_worker, start=0):
        """One parallel step over workers x rows_per_worker rows; returns (rows, wall seconds)."""
        M = W32.shape[0]
        jobs = []
        for w in range(self.workers):
            r0 = (start + w * rows_per_worker) % M
            idx = (np.arange(rows_per_worker) + r0) % M
            jobs.append((np.ascontiguousarray(W32[idx]), act, spec, C))
        t0 = time.perf_counter()
        rows = sum(self.pool.map(_oracle_task, jobs))
        return rows, time.perf_counter() - t0

    def close(self):
        self.pool.close()
        self.pool.join()


def time_oracle_parallel(pool, W32, act, spec, C, rows_per_worker, repeats, warmup=1):
    for i in range(warmup):
        pool.run(W32, act, spec, C, rows_per_worker, start=i)
    walls, rows = [], 0
    for i in range(repeats):
        rows, wall = pool.run(W32, act, spec, C, rows_per_worker, start=warmup + i)
        walls.append(wall)
    return rows, walls


def auto_rows(spec):
    """Rows per oracle worker per step: ~1 s of single-core fp64 work (16 rows
    of the 4096-column, N = 2048 workload; the brute-force search dominates)."""
    per_row = spec.K / 2 * spec.N
    return max(1, min(spec.M, int(round(16 * 2048 * 2048 / per_row))))


def oracle_parity(W32, act, spec, C, sigma, r, s, packed):
    """Index parity of the whole matrix (every pair): the oracle's fp64
    rotation, sigma and exact nearest centroids (oracle.codec.nearest_centroid_kd)
    against the GPU's packed stream, sigma, row norms and channel scales."""
    from oracle import codec
    t0 = time.perf_counter()
    s_o, r_o, Y = codec.rotated_rows(W32, act, spec.alpha, spec.block, spec.seed)
    sig_o = codec.sigma_from_rotated(Y)
    X = codec.normalised_pairs(Y, sig_o)
    del Y
    idx, gap = codec.nearest_centroid_kd(X, C)
    gidx = codec.unpack_indices(packed, spec.K // 2, spec.bits)
    diff = gidx != idx
    near = diff & (gap < 1e-6)
    return {"scope": f"every pair of the {spec.M}x{spec.K} matrix", "pairs": int(idx.size),
            "near_tie_pairs": int(np.sum(gap < 1e-6)), "hard_mismatches": int(np.sum(diff & ~near)),
            "near_tie_mismatches": int(np.sum(near)), "sigma_mismatches": int(np.sum(sigma != sig_o)),
            "row_norm_mismatches": int(np.sum(r != r_o)), "scale_mismatches": int(np.sum(s != s_o)),
            "rule": "indices bit-exact unless the oracle's best-two gap is below 1e-6 (counted); sigma, r, s bit-exact",
            "oracle_seconds": round(time.perf_counter() - t0, 1)}


def _reference_line(args, metric, value, unit, config, sample, ms_per_step, cores=1):
    return {
        "impl": "reference", "metric": metric, "value": value, "unit": unit, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": config,
        "cpu_baseline": {"value": value, "unit": unit, "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def run_reference_special(args):
    """The oracle legs of the decode-only, polar and codebook-training workloads."""
    import synth
    import vector_codebook_codec_b200 as q
    from oracle import codec
    from oracle import lloyd as olloyd
    if args.workload == "lloyd":
        Ts = 1 << 18
        x = synth.gaussian_points(LLOYD_T, LLOYD_SEED)[:Ts]
        C = x[:LLOYD_N].copy()
        idx = olloyd.assign(x, C)
        for _ in range(args.warmup):
            C = olloyd.centroid_update(x, idx, C)
            idx = olloyd.assign(x, C)
        t0 = time.perf_counter()
        for _ in range(args.steps):
            C = olloyd.centroid_update(x, idx, C)
            idx = olloyd.assign(x, C)
        dt = (time.perf_counter() - t0) / args.steps
        value = (Ts / LLOYD_T) / dt
        return _reference_line(args, "QAM-W codebook training: Lloyd iterations per second", value, "iterations/s",
                               {"workload": "lloyd_N2048_T2097152", "N": LLOYD_N, "T": LLOYD_T},
                               f"{Ts} of {LLOYD_T} samples per iteration, scaled", 1e3 / value, os.cpu_count())
    if args.workload == "decode_gemm":
        spec = synth.decode_sweep_13b().specs[1]
        rows = args.cpu_rows or 8
        C = q.load_codebook(spec.N)
        idx = synth.make_indices(rows, spec.K // 2, spec.N, spec.seed)
        r = synth.make_row_norms(rows, spec.seed)
        sig = synth.make_sigma(spec.K // 2, spec.seed)
        s_ = synth.make_act_rms(spec.K, 0.5, spec.seed)
        X = synth.make_activations(1, spec.K, 901).astype(np.float64)
        ts = []
        for i in range(args.warmup + args.steps):
            t0 = time.perf_counter()
            Wh = codec.decode_with_scale(idx, r, sig, s_, spec.K, spec.block, spec.seed, C)
            X @ Wh.T
            if i >= args.warmup:
                ts.append(time.perf_counter() - t0)
        value = rows * spec.K * len(ts) / sum(ts) / 1e9
        return _reference_line(args, METRIC, value, "Gweights/s",
                               {"workload": "decode_gemm_13824x5120_bf16_b128_N2048", "op": "decode then X W^T"},
                               f"{rows} of {spec.M} rows per step, decoded and multiplied with one token",
                               1e3 * sum(ts) / len(ts))
    if args.workload == "polar":
        spec = synth.llama7b_attn().specs[0]
        _, W32 = synth.to_bf16(synth.make_matrix(spec))
        act = synth.act_for(spec)
        pol = q.load_polar(spec.N)
        rows = args.cpu_rows or 64
        sig = codec.calibrate_sigma(W32[:rows], act, spec.alpha, spec.block, spec.seed)
        ts = []
        for i in range(args.warmup + args.steps):
            t0 = time.perf_counter()
            e = codec.encode_polar(W32[:rows], act, spec.alpha, spec.block, spec.seed, sig, pol["amps"], pol["P"],
                                   spec.bits)
            codec.decode_with_scale(e["idx"], e["r"], sig, e["s"], spec.K, spec.block, spec.seed, pol["points"])
            if i >= args.warmup:
                ts.append(time.perf_counter() - t0)
        value = rows * spec.K * len(ts) / sum(ts) / 1e9
        return _reference_line(args, METRIC, value, "Gweights/s",
                               {"workload": "polar_4096x4096_bf16_b128_A32xP64", "codec": "polar baseline"},
                               f"{rows} of {spec.M} rows per step (polar encode + decode)", 1e3 * sum(ts) / len(ts))
    # decode_13b: decode only, on row samples of the three matrices
    wl = synth.decode_sweep_13b()
    rows = args.cpu_rows or 16
    ts, weights = [], 0
    for i in range(args.warmup + args.steps):
        t = 0.0
        for spec in wl.specs:
            idx = synth.make_indices(rows, spec.K // 2, spec.N, spec.seed)
            r = synth.make_row_norms(rows, spec.seed)
            sig = synth.make_sigma(spec.K // 2, spec.seed)
            s_ = synth.make_act_rms(spec.K, 0.5, spec.seed)
            C = q.load_codebook(spec.N)
            t0 = time.perf_counter()
            codec.decode_with_scale(idx, r, sig, s_, spec.K, spec.block, spec.seed, C)
            t += time.perf_counter() - t0
            if i == 0:
                weights += rows * spec.K
        if i >= args.warmup:
            ts.append(t)
    value = weights * len(ts) / sum(ts) / 1e9
    return _reference_line(args, METRIC, value, "Gweights/s",
                           {"workload": wl.name, "op": "decode only"},
                           f"{rows} rows of each 13B-shaped matrix per step (decode)", 1e3 * sum(ts) / len(ts))


def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    if args.workload in ("lloyd", "polar", "decode_13b", "decode_gemm"):
        print(json.dumps(run_reference_special(args)), flush=True)
        return 0
    import synth
    import vector_codebook_codec_b200 as q
    spec, wname = workload_spec(args.workload)
    W32 = synth.make_matrix(spec)
    if spec.dtype == "bf16":
        _, W32 = synth.to_bf16(W32)
    act = synth.act_for(spec)
    C = q.load_codebook(spec.N)
    rows = args.cpu_rows or auto_rows(spec)
    pool = OraclePool()
    try:
        nrows, walls = time_oracle_parallel(pool, W32, act, spec, C, rows, args.steps, warmup=max(1, args.warmup))
    finally:
        pool.close()
    tot = sum(walls)
    value = nrows * spec.K * args.steps / tot / 1e9
    sample = (f"{pool.workers} worker processes x {rows} rows (of {spec.M}) per step, each running calibrate + "
              f"encode + decode of its rows on one core" + (f"; {spec.name}, the first matrix of the workload"
                                                             if args.workload in ("mlp", "stack_1p1b") else ""))
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "Gweights/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": wname, "M": spec.M, "K": spec.K, "block": spec.block, "N": spec.N,
                   "bits": spec.bits, "alpha": spec.alpha, "weight_dtype": spec.dtype},
        "cpu_baseline": {"value": value, "unit": "Gweights/s", "cores": pool.workers, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "Gweights/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# work accounting of the pruned search (outside the timed region)
# ---------------------------------------------------------------------------

def pruned_evaluations(q, Wd, cscale, rnorm, sigma, table, spec) -> int:
    """Distance evaluations the exact pruned search performs on this matrix:
    three per pair (the inline entries of its cell's record, evaluated without
    a branch), plus the overflow entries of a longer list, or N for a pair
    outside the grid. x is recomputed through the library's fp64 rotation hook
    (qamw_rotate_rows) on U = w * s / r, in row blocks, and each pair's cell
    comes from the encode's own cell arithmetic (qamw_search_cells)."""
    import torch
    raw = table.cpu().numpy()
    G = int(raw[8:12].view(np.int32)[0])
    rec = raw[64:64 + 8 * G * G].view(np.uint64)
    ovf = raw[64 + 8 * G * G:].view(np.uint16).astype(np.int64)
    meta = (rec >> np.uint64(48)).astype(np.int64)
    extra = np.where((meta & 3) == 0, ovf[np.minimum(meta >> 2, ovf.size - 1)], 0)
    extra_t = torch.from_numpy(extra).to(Wd.device)
    M, K = Wd.shape
    sig = sigma.to(torch.float64)
    total = 0
    for r0 in range(0, M, 1024):
        r1 = min(M, r0 + 1024)
        U = Wd[r0:r1].to(torch.float64) * cscale.to(torch.float64)[None, :]
        rr = rnorm[r0:r1].to(torch.float64)[:, None]
        U = torch.where(rr > 0, U / torch.where(rr > 0, rr, torch.ones_like(rr)), torch.zeros_like(U))
        Y = q.rotate_rows(U.contiguous(), spec.block, spec.seed)
        x = (Y.view(-1, 2) / sig.repeat(r1 - r0)[:, None]).to(torch.float32).contiguous()
        cells = q.search_cells(x, table).to(torch.int64)
        n = 3 + torch.where(cells >= 0, extra_t[cells.clamp(min=0)], torch.full_like(cells, spec.N))
        total += int(n.sum().item())
    return total


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------

def run_decode_sweep(args):
    """Decode-only steps over the 13B-shaped matrices (5120x5120, 13824x5120,
    5120x13824), pre-encoded on the GPU outside the timed region; one step
    decodes all three to bf16."""
    import torch
    import torch.distributed as dist

    import synth
    import vector_codebook_codec_b200 as q
    from vector_codebook_codec_b200 import build as qbuild

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    qbuild.build()
    wl = synth.decode_sweep_13b()
    mats = []
    for spec in wl.specs:
        Wt, _ = synth.to_bf16(synth.make_matrix(spec))
        Wd = Wt.to(dev)
        act = torch.from_numpy(synth.act_for(spec)).to(dev)
        Cd = torch.from_numpy(q.load_codebook(spec.N)).to(dev)
        sig = q.calibrate_sigma(Wd, act, spec.alpha, spec.block, spec.seed)
        enc = q.encode(Wd, act, spec.alpha, spec.block, spec.seed, sig, Cd, spec.bits)
        del Wd
        out = torch.empty((spec.M, spec.K), dtype=torch.bfloat16, device=dev)
        mats.append((spec, enc, Cd, out))
    torch.cuda.synchronize(dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    nm = len(mats)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(nm + 1)] for _ in range(args.steps)]

    def one(evs=None):
        for j, (spec, enc, Cd, out) in enumerate(mats):
            if evs: evs[j].record(stream)
            q.decode(enc, Cd, out_dtype=torch.bfloat16, status=status, out=out)
        if evs: evs[nm].record(stream)

    for _ in range(args.warmup):
        flush.fill_(1.0)
        one()
    torch.cuda.synchronize(dev)
    # the step (three decodes) captured once as a CUDA graph: the headline
    graph = None
    if args.graph:
        side = torch.cuda.Stream(dev)
        graph = torch.cuda.CUDAGraph()
        torch.cuda.synchronize(dev)
        with torch.cuda.graph(graph, stream=side):
            for spec, enc, Cd, out in mats:
                q.decode(enc, Cd, out_dtype=torch.bfloat16, status=status, out=out, stream=side)
        for _ in range(args.warmup):
            flush.fill_(3.0)
            graph.replay()
        torch.cuda.synchronize(dev)
    gev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    for i in range(args.steps):
        flush.fill_(float(i))
        one(ev[i])
    torch.cuda.synchronize(dev)
    if graph is not None:
        if world > 1:
            dist.barrier()
        for i, (e0, e1) in enumerate(gev):
            flush.fill_(float(i) + 0.5)
            e0.record(stream)
            graph.replay()
            e1.record(stream)
        torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    time.sleep(0.2)
    clk = clocks.stop()
    if status.item() != 0:
        raise SystemExit(f"device status {status.item()}")
    per = [[ev[i][j].elapsed_time(ev[i][j + 1]) for i in range(args.steps)] for j in range(nm)]
    total_s = max_over_ranks(sum(ev[i][0].elapsed_time(ev[i][nm]) for i in range(args.steps)) / 1e3, dev)
    weights = sum(sp.M * sp.K for sp, _, _, _ in mats)
    value = aggregate_throughput(weights * args.steps, total_s, world) / 1e9
    eager = {"ms_per_step": 1e3 * total_s / args.steps, "value": value, "unit": "Gweights/s"}
    if graph is not None:
        total_s = max_over_ranks(sum(e0.elapsed_time(e1) for e0, e1 in gev) / 1e3, dev)
        value = aggregate_throughput(weights * args.steps, total_s, world) / 1e9
        del graph
    peaks, peak_kind = measured_peaks()
    hbm = float(peaks.get("hbm_gbs", FALLBACK_HBM_GBS))
    per_mat = []
    tot_bytes = 0
    for (spec, enc, _, _), t in zip(mats, per):
        wpr = q.words_per_row(spec.K, spec.bits)
        b = spec.M * spec.K * 2 + spec.M * wpr * 4 + 4 * spec.M + 4 * spec.K + 2 * spec.K + 8 * spec.N
        tot_bytes += b
        ms = statistics.mean(t)
        per_mat.append({"name": spec.name, "M": spec.M, "K": spec.K, "us": 1e3 * ms,
                        "gweights_per_s": spec.M * spec.K / (ms * 1e-3) / 1e9,
                        "gbs": b / (ms * 1e-3) / 1e9, "frac": b / (ms * 1e-3) / 1e9 / hbm})
    mean_step_s = total_s / args.steps
    roof = {"bound": "hbm", "achieved": tot_bytes / mean_step_s / 1e9, "peak": hbm, "unit": "GB/s",
            "frac": tot_bytes / mean_step_s / 1e9 / hbm, "traffic": None, "kernel": "decode_tma_kernel (3 launches per step)",
            "peak_source": f"{peak_kind} hbm_gbs"}
    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": "Gweights/s", "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": 1e3 * mean_step_s, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic (seeded; no checkpoint)",
                "config": {"workload": wl.name, "op": "decode only (bf16 out)", "matrices": [
                    f"{sp.M}x{sp.K}" for sp, _, _, _ in mats], "block": 128, "N": 2048, "bits": 11,
                    "l2": "flushed by a 256 MiB write before every timed step",
                    "parallelism": f"{world} independent replica(s)"},
                "roofline": roof, "per_matrix": per_mat, "gpu_launches": nm * args.steps, "clocks": clk,
                "timing": ("each step replays a CUDA graph of the three decodes; 'eager' and 'per_matrix' are the "
                           "decodes launched call by call" if args.graph else "each decode launched call by call"),
                "eager": eager}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


LLOYD_N, LLOYD_T, LLOYD_SEED = 2048, 1 << 21, 12345 + 2048
FP64_LANES_PER_SM = 64


def run_lloyd(args):
    """Steps of codebook training: one Lloyd iteration (qamw_lloyd_update then
    qamw_lloyd_assign) of 2048 centroids on 2^21 unit-Gaussian samples -- the
    size the shipped 2048-centroid codebook was trained at. Each iteration is
    timed with CUDA events; the start is the first 2048 samples."""
    import torch
    import synth
    import vector_codebook_codec_b200 as q
    from vector_codebook_codec_b200 import build as qbuild
    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    qbuild.build()
    x = synth.gaussian_points(LLOYD_T, LLOYD_SEED)
    pts = torch.from_numpy(x).to(dev)
    C = pts[:LLOYD_N].clone()
    lib = q.load_library()
    idx = torch.full((LLOYD_T,), -1, dtype=torch.int32, device=dev)
    ws = torch.empty(int(lib.qamw_lloyd_workspace_bytes(LLOYD_T, LLOYD_N)), dtype=torch.uint8, device=dev)
    changed = torch.zeros(1, dtype=torch.int64, device=dev)
    stream = torch.cuda.current_stream(dev)
    q.lloyd_assign(pts, C, idx=idx)

    def one():
        q._check("qamw_lloyd_update", lib.qamw_lloyd_update(q._ptr(pts), LLOYD_T, q._ptr(idx), LLOYD_N, q._ptr(C),
                                                            q._ptr(ws), ws.numel(), q._stream_ptr(stream)))
        q.lloyd_assign(pts, C, idx=idx, changed=changed)

    for _ in range(args.warmup):
        one()
    torch.cuda.synchronize(dev)
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    for e0, e1 in ev:
        e0.record(stream)
        one()
        e1.record(stream)
    torch.cuda.synchronize(dev)
    time.sleep(0.2)
    clk = clocks.stop()
    ms = [e0.elapsed_time(e1) for e0, e1 in ev]
    total_s = sum(ms) / 1e3
    value = args.steps / total_s
    peaks, peak_kind = measured_peaks()
    sm_max = float(peaks.get("sm_max_mhz", 1965.0))
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    fp64_peak = sms * FP64_LANES_PER_SM * sm_max * 1e6
    ops = 5.0 * LLOYD_T * LLOYD_N          # 2 fp64 subs, 2 muls, 1 add per (sample, centroid)
    mean_s = total_s / args.steps
    roof = {"bound": "alu", "achieved": ops / mean_s / 1e9, "peak": fp64_peak / 1e9, "unit": "Gop/s",
            "frac": ops / mean_s / fp64_peak, "traffic": None,
            "kernel": "lloyd_assign_kernel + lloyd_partial_kernel + lloyd_reduce_kernel (events span one iteration)",
            "peak_source": f"{sms} SMs x {FP64_LANES_PER_SM} FP64 lanes x {sm_max:.0f} MHz ({peak_kind} max clock)"}
    cpu = None
    if rank == 0 and not args.no_cpu_baseline:
        from oracle import lloyd as olloyd
        Ts = 1 << 18
        xs, Cs = x[:Ts], x[:LLOYD_N].copy()
        i0 = olloyd.assign(xs, Cs)
        t0 = time.perf_counter()
        reps = 3
        for _ in range(reps):
            Cs = olloyd.centroid_update(xs, i0, Cs)
            i0 = olloyd.assign(xs, Cs)
        dt = (time.perf_counter() - t0) / reps
        cpu = {"value": (Ts / LLOYD_T) / dt, "unit": "iterations/s", "cores": os.cpu_count(), "kind": "oracle",
               "sample": f"{Ts} of {LLOYD_T} samples per iteration (cKDTree assignment on all cores + bincount "
                         f"means), scaled to the full sample count"}
    if rank == 0:
        line = {"metric": "QAM-W codebook training: Lloyd iterations per second", "value": value,
                "unit": "iterations/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": 1e3 * mean_s, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "f64", "data": "synthetic (seeded unit circular Gaussian samples)",
                "config": {"workload": "lloyd_N2048_T2097152", "N": LLOYD_N, "T": LLOYD_T, "seed": LLOYD_SEED,
                           "l2": "samples (32 MB) stay in L2 between iterations; the work is ALU-bound"},
                "roofline": roof, "cpu_baseline": cpu, "gpu_launches": 3 * args.steps, "clocks": clk}
        print(json.dumps(line), flush=True)
    return 0


def run_polar(args):
    """Steps of the polar baseline codec on the 4096x4096 projection at 2048
    points (32 amplitude levels x 64 sectors): qamw_calibrate_sigma +
    qamw_encode_polar + qamw_decode (the polar points as codebook). Also
    reports the whole-matrix relative error of the joint and the polar codec."""
    import torch
    import synth
    import vector_codebook_codec_b200 as q
    from vector_codebook_codec_b200 import build as qbuild
    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    qbuild.build()
    spec = synth.llama7b_attn().specs[0]
    M, K = spec.M, spec.K
    Wt, W32 = synth.to_bf16(synth.make_matrix(spec))
    act = synth.act_for(spec)
    Wd, actd = Wt.to(dev), torch.from_numpy(act).to(dev)
    pol = q.load_polar(spec.N)
    amps = torch.from_numpy(pol["amps"]).to(dev)
    pts = torch.from_numpy(pol["points"]).to(dev)
    lib = q.load_library()
    ws = torch.empty(int(lib.qamw_calibrate_workspace_bytes(M, K)), dtype=torch.uint8, device=dev)
    wpr = q.words_per_row(K, spec.bits)
    sigma = torch.empty(K // 2, dtype=torch.float32, device=dev)
    packed = torch.empty((M, wpr), dtype=torch.int32, device=dev)
    rnorm = torch.empty(M, dtype=torch.float32, device=dev)
    cscale = torch.empty(K, dtype=torch.float32, device=dev)
    out = torch.empty((M, K), dtype=torch.bfloat16, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]

    def one(evs=None):
        if evs: evs[0].record(stream)
        sig = q.calibrate_sigma(Wd, actd, spec.alpha, spec.block, spec.seed, status=status, workspace=ws, out=sigma)
        if evs: evs[1].record(stream)
        enc = q.encode_polar(Wd, actd, spec.alpha, spec.block, spec.seed, sig, amps, pol["P"], spec.bits,
                             status=status, out=(packed, rnorm, cscale))
        if evs: evs[2].record(stream)
        q.decode(enc, pts, out_dtype=torch.bfloat16, status=status, out=out)
        if evs: evs[3].record(stream)
        return enc

    for _ in range(args.warmup):
        flush.fill_(1.0)
        one()
    torch.cuda.synchronize(dev)
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    for i in range(args.steps):
        flush.fill_(float(i))
        one(ev[i])
    torch.cuda.synchronize(dev)
    time.sleep(0.2)
    clk = clocks.stop()
    if status.item() != 0:
        raise SystemExit(f"device status {status.item()}")
    t = {k: statistics.mean(ev[i][j].elapsed_time(ev[i][j + 1]) for i in range(args.steps))
         for j, k in enumerate(("calibrate", "encode", "decode"))}
    step_ms = sum(ev[i][0].elapsed_time(ev[i][3]) for i in range(args.steps)) / args.steps
    peaks, peak_kind = measured_peaks()
    hbm = float(peaks.get("hbm_gbs", FALLBACK_HBM_GBS))
    enc_bytes = M * K * 2 + M * wpr * 4
    roof = {"bound": "hbm", "achieved": enc_bytes / (t["encode"] * 1e-3) / 1e9, "peak": hbm, "unit": "GB/s",
            "frac": enc_bytes / (t["encode"] * 1e-3) / 1e9 / hbm, "traffic": None,
            "kernel": "encode_polar_kernel (fp64 hypot / atan2 per pair; events span the qamw_encode_polar call)",
            "peak_source": f"{peak_kind} hbm_gbs"}
    # quality at equal rate: whole-matrix relative error of both codecs (fp32 decode)
    enc = one()
    wp = q.decode(enc, pts, out_dtype=torch.float32)
    C = torch.from_numpy(q.load_codebook(spec.N)).to(dev)
    joint = q.encode(Wd, actd, spec.alpha, spec.block, spec.seed, sigma, C, spec.bits,
                     search_table=q.build_search_table(C))
    wj = q.decode(joint, C, out_dtype=torch.float32)
    Wf = Wd.float()
    nrm = torch.sum(Wf * Wf).item()
    err = {"joint": torch.sum((wj - Wf) ** 2).item() / nrm, "polar": torch.sum((wp - Wf) ** 2).item() / nrm}
    cpu = None
    if not args.no_cpu_baseline:
        from oracle import codec
        rows = 64
        sig_h = sigma.cpu().numpy()
        t0 = time.perf_counter()
        codec.encode_polar(W32[:rows], act, spec.alpha, spec.block, spec.seed, sig_h, pol["amps"], pol["P"],
                           spec.bits)
        dt = time.perf_counter() - t0
        cpu = {"value": rows * K / dt / 1e9, "unit": "Gweights/s", "cores": 1, "kind": "oracle",
               "sample": f"polar encode of {rows} of {M} rows (fp64 numpy)"}
    if rank == 0:
        print(json.dumps({
            "metric": METRIC, "value": M * K / (step_ms * 1e-3) / 1e9, "unit": "Gweights/s", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded; no checkpoint)",
            "config": {"workload": "polar_4096x4096_bf16_b128_A32xP64", "codec": "polar baseline",
                       "A": int(amps.numel()), "P": pol["P"], "bits": spec.bits,
                       "l2": "flushed by a 256 MiB write before every timed step"},
            "roofline": roof, "ms": t, "relative_sq_error": err, "cpu_baseline": cpu,
            "gpu_launches": 8 * args.steps, "clocks": clk}), flush=True)
    return 0


def run_multi(args):
    """Steps over every matrix of a multi-matrix workload: the 24 MLP runs
    (11008x4096 and 4096x11008 Student-t matrices x alpha {0.25, 0.5, 0.75} x
    block {128, 256} x {1024, 2048} centroids) or the 154 matrices of the
    22-layer 1.1B-shaped stack. One step = qamw_calibrate_encode of every
    matrix, then qamw_decode (bf16) of every matrix, all through the C ABI.
    Matrices are spread over 4 streams so that small ones (the 256x2048 k and v
    projections) run beside others. The step is captured once as a CUDA graph
    and replayed (the headline); per-shape times come from an eager pass with
    one stream."""
    import torch
    import synth
    import vector_codebook_codec_b200 as q
    from vector_codebook_codec_b200 import build as qbuild
    rank, world, local = dist_env()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    qbuild.build()
    lib = q.load_library()
    wl = synth.mlp_runs() if args.workload == "mlp" else synth.stack_1p1b()
    specs = wl.specs
    n_streams = 4
    cache, host_w, ents = {}, {}, []
    cbs, tables = {}, {}
    for spec in specs:
        key = (spec.M, spec.K, spec.dist, spec.std, spec.outlier_frac, spec.outlier_scale, spec.seed)
        if key not in cache:
            Wt, _ = synth.to_bf16(synth.make_matrix(spec))
            cache[key] = Wt.to(dev)
            host_w[key] = Wt
        if spec.N not in cbs:
            cbs[spec.N] = torch.from_numpy(q.load_codebook(spec.N)).to(dev)
            tables[spec.N] = q.build_search_table(cbs[spec.N])
        M, K = spec.M, spec.K
        wpr = q.words_per_row(K, spec.bits)
        ents.append(dict(
            spec=spec, key=key, W=cache[key], act=torch.from_numpy(synth.act_for(spec)).to(dev),
            ws=torch.empty(int(lib.qamw_calibrate_workspace_bytes(M, K)), dtype=torch.uint8, device=dev),
            sigma=torch.empty(K // 2, dtype=torch.float32, device=dev),
            packed=torch.empty((M, wpr), dtype=torch.int32, device=dev),
            r=torch.empty(M, dtype=torch.float32, device=dev), s=torch.empty(K, dtype=torch.float32, device=dev),
            out=torch.empty((M, K), dtype=torch.bfloat16, device=dev)))
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    main = torch.cuda.current_stream(dev)
    streams = [torch.cuda.Stream(dev) for _ in range(n_streams)]

    def enc_call(e, st):
        sp = e["spec"]
        return q.calibrate_encode(e["W"], e["act"], sp.alpha, sp.block, sp.seed, cbs[sp.N], sp.bits, status=status,
                                  out=(e["packed"], e["r"], e["s"], e["sigma"]), search_table=tables[sp.N],
                                  workspace=e["ws"], stream=st)

    def dec_call(e, enc, st):
        q.decode(enc, cbs[e["spec"].N], out_dtype=torch.bfloat16, status=status, out=e["out"], stream=st)

    def step(origin):
        """All encodes, then all decodes, round-robin over the streams, forked from and joined to origin."""
        fork = torch.cuda.Event()
        fork.record(origin)
        for st in streams:
            st.wait_event(fork)
        encs = [enc_call(e, streams[i % n_streams]) for i, e in enumerate(ents)]
        for i, (e, enc) in enumerate(zip(ents, encs)):
            dec_call(e, enc, streams[i % n_streams])
        for st in streams:
            j = torch.cuda.Event()
            j.record(st)
            origin.wait_event(j)

    for _ in range(args.warmup):
        flush.fill_(1.0)
        step(main)
    torch.cuda.synchronize(dev)
    if status.item() != 0:
        raise SystemExit(f"device status {status.item()} after warm-up")
    graph = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream(dev)
    with torch.cuda.graph(graph, stream=side):
        step(side)
    for _ in range(args.warmup):
        flush.fill_(3.0)
        graph.replay()
    torch.cuda.synchronize(dev)
    # eager pass on one stream, each call timed: the per-shape figures
    per = []
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
            torch.cuda.Event(enable_timing=True)) for _ in ents]
    flush.fill_(4.0)
    for e, (a, b, c) in zip(ents, evs):
        a.record(main)
        enc = enc_call(e, main)
        b.record(main)
        dec_call(e, enc, main)
        c.record(main)
    torch.cuda.synchronize(dev)
    for e, (a, b, c) in zip(ents, evs):
        per.append((e["spec"], a.elapsed_time(b), b.elapsed_time(c)))

    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    gev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    torch.cuda.synchronize(dev)
    for i, (e0, e1) in enumerate(gev):
        flush.fill_(float(i))
        e0.record(main)
        graph.replay()
        e1.record(main)
    torch.cuda.synchronize(dev)
    time.sleep(0.2)
    clk = clocks.stop()
    if status.item() != 0:
        raise SystemExit(f"device status {status.item()} in the timed steps")
    total_s = max_over_ranks(sum(e0.elapsed_time(e1) for e0, e1 in gev) / 1e3, dev)
    weights = sum(sp.M * sp.K for sp in specs)
    value = aggregate_throughput(weights * args.steps, total_s, world) / 1e9
    mean_step_s = total_s / args.steps

    # per shape (or per run): mean eager time of the fused encode call and the decode
    groups = {}
    for sp, te, td in per:
        name = sp.name.split(".", 1)[1] if args.workload == "stack_1p1b" else sp.name
        g = groups.setdefault(name, {"M": sp.M, "K": sp.K, "N": sp.N, "block": sp.block, "alpha": sp.alpha,
                                     "n": 0, "enc_ms": 0.0, "dec_ms": 0.0})
        g["n"] += 1
        g["enc_ms"] += te
        g["dec_ms"] += td
    per_shape = []
    for name, g in groups.items():
        em, dm = g["enc_ms"] / g["n"], g["dec_ms"] / g["n"]
        w = g["M"] * g["K"]
        per_shape.append({"name": name, "M": g["M"], "K": g["K"], "N": g["N"], "block": g["block"],
                          "alpha": g["alpha"], "matrices": g["n"], "calibrate_encode_us": 1e3 * em,
                          "decode_us": 1e3 * dm, "gweights_per_s": w / ((em + dm) * 1e-3) / 1e9})

    # the dominant kernel alone on the workload's first matrix (as the default line)
    peaks, peak_kind = measured_peaks()
    hbm = float(peaks.get("hbm_gbs", FALLBACK_HBM_GBS))
    e = ents[0]
    sp = e["spec"]
    kev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(5)]
    for e0, e1 in kev:
        flush.fill_(5.0)
        e0.record(main)
        q.encode_prepared(e["W"], e["s"], e["r"], sp.block, sp.seed, e["sigma"], cbs[sp.N], sp.bits, status=status,
                          out=e["packed"], search_table=tables[sp.N])
        e1.record(main)
    torch.cuda.synchronize(dev)
    kern_ms = statistics.mean(e0.elapsed_time(e1) for e0, e1 in kev)
    wpr = q.words_per_row(sp.K, sp.bits)
    enc_bytes = sp.M * sp.K * 2 + sp.M * wpr * 4 + 4 * sp.M + 4 * sp.K + 2 * sp.K + 8 * sp.N
    roof = {"bound": "hbm", "achieved": enc_bytes / (kern_ms * 1e-3) / 1e9, "peak": hbm, "unit": "GB/s",
            "frac": enc_bytes / (kern_ms * 1e-3) / 1e9 / hbm, "traffic": None,
            "kernel": f"encode_pruned_kernel alone (qamw_encode_prepared) on {sp.name} {sp.M}x{sp.K}",
            "us_per_launch": 1e3 * kern_ms, "algorithmic_bytes_per_launch": enc_bytes,
            "peak_source": f"{peak_kind} hbm_gbs"}

    # end to end: every distinct matrix uploaded from pinned host memory, every
    # matrix's decoded weights and encoded artefact read back, inside the timing
    e2e = None
    if not args.no_e2e:
        pin_w = {k: v.pin_memory() for k, v in host_w.items()}
        pin_out = [torch.empty(e["out"].shape, dtype=torch.bfloat16).pin_memory() for e in ents]
        pin_pk = [torch.empty(e["packed"].shape, dtype=torch.int32).pin_memory() for e in ents]
        pin_meta = [[torch.empty(e[k].shape, dtype=torch.float32).pin_memory() for k in ("r", "s", "sigma")]
                    for e in ents]
        h2d = sum(v.numel() * 2 for v in pin_w.values())
        d2h = sum(o.numel() * 2 + p.numel() * 4 + 4 * (e["spec"].M + e["spec"].K + e["spec"].K // 2)
                  for o, p, e in zip(pin_out, pin_pk, ents))

        def e2e_step():
            for k, v in pin_w.items():
                cache[k].copy_(v, non_blocking=True)
            step(main)
            for e, o, p, mt in zip(ents, pin_out, pin_pk, pin_meta):
                o.copy_(e["out"], non_blocking=True)
                p.copy_(e["packed"], non_blocking=True)
                for h, k in zip(mt, ("r", "s", "sigma")):
                    h.copy_(e[k], non_blocking=True)
        e2e_step()
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(main)
        for _ in range(max(1, args.steps // 2)):
            e2e_step()
        e1.record(main)
        torch.cuda.synchronize(dev)
        n_e2e = max(1, args.steps // 2)
        e2e_s = max_over_ranks(e0.elapsed_time(e1) / 1e3, dev)
        e2e = {"value": aggregate_throughput(weights * n_e2e, e2e_s, world) / 1e9, "unit": "Gweights/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "pipelining": "none: uploads, the step on 4 streams, then the read-backs"}

    cpu, parity = None, None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        sp0 = specs[0]
        _, W32 = synth.to_bf16(synth.make_matrix(sp0))
        act0 = synth.act_for(sp0)
        C0 = q.load_codebook(sp0.N)
        rows = args.cpu_rows or auto_rows(sp0)
        pool = OraclePool()
        try:
            nrows, walls = time_oracle_parallel(pool, W32, act0, sp0, C0, rows, 3)
        finally:
            pool.close()
        cpu = {"value": nrows * sp0.K / statistics.median(walls) / 1e9, "unit": "Gweights/s",
               "cores": pool.workers, "kind": "oracle",
               "sample": f"{sp0.name} ({sp0.M}x{sp0.K}): {pool.workers} worker processes x {rows} rows per step, "
                         f"calibrate + encode + decode; median of 3 steps"}
        # whole-matrix parity of the first matrix (the MLP workload) or of
        # every matrix of layer 0 (the stack), from the last step's encodings
        chk = [ents[0]] if args.workload == "mlp" else [e for e in ents if e["spec"].name.startswith("L0.")]
        parity = {"matrices": [], "pairs": 0, "near_tie_pairs": 0, "hard_mismatches": 0, "near_tie_mismatches": 0,
                  "sigma_mismatches": 0, "row_norm_mismatches": 0, "scale_mismatches": 0}
        for e in chk:
            spx = e["spec"]
            _, Wx = synth.to_bf16(synth.make_matrix(spx))
            rec = oracle_parity(Wx, synth.act_for(spx), spx, q.load_codebook(spx.N), e["sigma"].cpu().numpy(),
                                e["r"].cpu().numpy(), e["s"].cpu().numpy(), e["packed"].cpu().numpy().view(np.uint32))
            parity["matrices"].append(f"{spx.name} {spx.M}x{spx.K}")
            for k in ("pairs", "near_tie_pairs", "hard_mismatches", "near_tie_mismatches", "sigma_mismatches",
                      "row_norm_mismatches", "scale_mismatches"):
                parity[k] += rec[k]
        parity["rule"] = "indices bit-exact unless the oracle's best-two gap is below 1e-6 (counted); sigma, r, s bit-exact"
    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": "Gweights/s", "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": 1e3 * mean_step_s, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic (seeded; no checkpoint)",
                "config": {"workload": wl.name, "matrices": len(specs), "weights_per_step": weights,
                           "weight_dtype": "bf16", "op": "calibrate + encode all, then decode all (bf16 out)",
                           "streams": n_streams, "l2": "flushed by a 256 MiB write before every timed step",
                           "parallelism": f"{world} independent replica(s)"},
                "roofline": roof, "per_shape": per_shape, "cpu_baseline": cpu, "parity": parity, "e2e": e2e,
                "gpu_launches": 6 * len(specs) * args.steps, "clocks": clk,
                "timing": "each step replays one CUDA graph of all calls (4 streams); per_shape: an eager pass"}
        print(json.dumps(line), flush=True)
    del graph
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


DG_TOKENS = (1, 16, 128, 4096)


def run_decode_gemm(args):
    """The fused decode + matmul (qamw_decode_matmul) on the 13B up projection
    (13824 x 5120, 2048 centroids, block 128), pre-encoded: Y = X W^T for T in
    {1, 16, 128, 4096} tokens, against the unfused path (qamw_decode to bf16,
    then torch's bf16 matmul, i.e. cuBLAS) and against cuBLAS alone on the
    already-decoded bf16 weights. A step runs every T once; the headline is
    the fused call's weight throughput at T = 1 (memory-bound: 0.69 bytes per
    weight read instead of 2)."""
    import torch
    import synth
    import vector_codebook_codec_b200 as q
    from vector_codebook_codec_b200 import build as qbuild
    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    qbuild.build()
    spec = synth.decode_sweep_13b().specs[1]
    M, K = spec.M, spec.K
    # pre-encode the matrix with the GPU encode (as the decode-only workload does)
    Wt, _ = synth.to_bf16(synth.make_matrix(spec))
    Wd = Wt.to(dev)
    act = torch.from_numpy(synth.act_for(spec)).to(dev)
    Cd = torch.from_numpy(q.load_codebook(spec.N)).to(dev)
    sig = q.calibrate_sigma(Wd, act, spec.alpha, spec.block, spec.seed)
    enc = q.encode(Wd, act, spec.alpha, spec.block, spec.seed, sig, Cd, spec.bits,
                   search_table=q.build_search_table(Cd))
    del Wd
    Wb = q.decode(enc, Cd, out_dtype=torch.bfloat16)          # for the cuBLAS-only reference
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    Xs = {T: torch.from_numpy(synth.make_activations(T, K, 900 + T)).to(torch.bfloat16).to(dev) for T in DG_TOKENS}
    Ys = {T: torch.empty((T, M), dtype=torch.float32, device=dev) for T in DG_TOKENS}
    Wtmp = torch.empty((M, K), dtype=torch.bfloat16, device=dev)
    Ws = {T: torch.empty(q.decode_matmul_workspace_bytes(M, K, T), dtype=torch.uint8, device=dev) for T in DG_TOKENS}

    def fused(T):
        q.decode_matmul(enc, Cd, Xs[T], status=status, out=Ys[T], workspace=Ws[T])

    def unfused(T):
        q.decode(enc, Cd, out_dtype=torch.bfloat16, status=status, out=Wtmp)
        torch.matmul(Xs[T], Wtmp.T)

    def cublas(T):
        torch.matmul(Xs[T], Wb.T)

    def timed(fn, T, reps):
        ts = []
        for i in range(reps):
            flush.fill_(float(i))
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            fn(T)
            e1.record(stream)
            torch.cuda.synchronize(dev)
            ts.append(e0.elapsed_time(e1))
        return statistics.median(ts)

    for T in DG_TOKENS:
        for fn in (fused, unfused, cublas):
            for _ in range(args.warmup):
                fn(T)
    torch.cuda.synchronize(dev)
    if status.item() != 0:
        raise SystemExit(f"device status {status.item()} after warm-up")
    # sanity at the smallest and largest T: fused vs decode to bf16 + matmul (the
    # parity tests hold the derived bound against the oracle)
    for T in (DG_TOKENS[0], DG_TOKENS[-1]):
        fused(T)
        ref = torch.matmul(Xs[T].float(), Wb.float().T)
        scale = torch.matmul(Xs[T].float().abs(), Wb.float().abs().T)
        if not bool(((Ys[T] - ref).abs() <= 2.0 ** -6 * scale + 1e-6).all()):
            raise SystemExit(f"fused decode + matmul differs from decode + matmul at T={T}")
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    rows = []
    total_ms = 0.0
    for T in DG_TOKENS:
        reps = max(args.steps, 3)
        tf, tu, tc = timed(fused, T, reps), timed(unfused, T, reps), timed(cublas, T, reps)
        total_ms += tf
        rows.append({"tokens": T, "fused_us": 1e3 * tf, "decode_then_cublas_us": 1e3 * tu,
                     "cublas_on_decoded_bf16_us": 1e3 * tc, "fused_speedup_vs_unfused": tu / tf,
                     "fused_tflops": 2.0 * M * K * T / (tf * 1e-3) / 1e12})
    time.sleep(0.2)
    clk = clocks.stop()
    if status.item() != 0:
        raise SystemExit(f"device status {status.item()} in the timed calls")
    # end to end at T = 1: the token's activations uploaded from pinned host
    # memory, the fused call, Y read back, all inside the timed region
    T1 = DG_TOKENS[0]
    x_host = Xs[T1].cpu().pin_memory()
    y_host = torch.empty((T1, M), dtype=torch.float32).pin_memory()
    x_dev = torch.empty_like(Xs[T1])
    e2e_ts = []
    for i in range(args.warmup + max(args.steps, 3)):
        flush.fill_(float(i))
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        x_dev.copy_(x_host, non_blocking=True)
        q.decode_matmul(enc, Cd, x_dev, status=status, out=Ys[T1], workspace=Ws[T1])
        y_host.copy_(Ys[T1], non_blocking=True)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        if i >= args.warmup:
            e2e_ts.append(e0.elapsed_time(e1))
    if not torch.equal(y_host, Ys[T1].cpu()):
        raise SystemExit("end-to-end read-back differs from the device result")
    e2e_ms = statistics.median(e2e_ts)
    e2e = {"value": M * K / (e2e_ms * 1e-3) / 1e9, "unit": "Gweights/s",
           "h2d_bytes_per_step": int(x_host.numel() * x_host.element_size()),
           "d2h_bytes_per_step": int(y_host.numel() * y_host.element_size()),
           "note": "T = 1 token: its activations uploaded, the fused call, Y read back (pinned host memory)"}
    # the oracle (decode then product, fp64 numpy) on a bounded sample of rows, one core
    cpu = None
    if not args.no_cpu_baseline and rank == 0:
        from oracle import codec as ocodec
        n_rows = args.cpu_rows or 64
        idx_o = ocodec.unpack_indices(enc.packed[:n_rows].cpu().numpy().view(np.uint32), K // 2, spec.bits)
        r_o, sig_o, s_o = enc.row_norm[:n_rows].cpu().numpy(), enc.sigma.cpu().numpy(), enc.col_scale.cpu().numpy()
        X1 = Xs[T1].double().cpu().numpy()
        C_o = Cd.cpu().numpy()
        ts_o = []
        for _ in range(3):
            t_a = time.perf_counter()
            Wh = ocodec.decode_with_scale(idx_o, r_o, sig_o, s_o, K, spec.block, spec.seed, C_o)
            X1 @ Wh.T
            ts_o.append(time.perf_counter() - t_a)
        cpu = {"value": n_rows * K / statistics.median(ts_o) / 1e9, "unit": "Gweights/s", "cores": 1,
               "kind": "oracle", "sample": f"{n_rows} of {M} rows decoded (fp64) and multiplied with one token; "
                                           "median of 3"}
    peaks, peak_kind = measured_peaks()
    hbm = float(peaks.get("hbm_gbs", FALLBACK_HBM_GBS))
    tc_peak = float(peaks.get("bf16_tflops", 1590.0))
    wpr = q.words_per_row(K, spec.bits)
    t1 = rows[0]["fused_us"] * 1e-6
    # both kernels of the call at T = 1: packed words, r, codebook, Y; x (bf16),
    # s, sigma, a (fp16, written then read), the token's power of two
    bytes1 = M * wpr * 4 + 4 * M + 8 * spec.N + 4 * M + 2 * K + 4 * K + 2 * K + 2 * K + 2 * K + 8
    t4 = rows[-1]["fused_us"] * 1e-6
    flops4 = 2.0 * M * K * DG_TOKENS[-1]
    value = M * K / t1 / 1e9
    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": "Gweights/s", "n_gpus": 1, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": total_ms, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "f16", "data": "synthetic (seeded; no checkpoint)",
                "config": {"workload": "decode_gemm_13824x5120_bf16_b128_N2048", "M": M, "K": K, "N": spec.N,
                           "bits": spec.bits, "tokens": list(DG_TOKENS),
                           "op": "Y[T x M] = X[T x K] decode(W)^T: decode's linear steps applied to X "
                                 "(fp32, stored fp16 with a power of two per token), fp16 centroids, "
                                 "fp32 accumulation on tcgen05",
                           "l2": "flushed by a 256 MiB write before every timed call",
                           "value_note": "weights per second of the fused call at T = 1"},
                "roofline": {"bound": "hbm", "achieved": bytes1 / t1 / 1e9, "peak": hbm, "unit": "GB/s",
                             "frac": bytes1 / t1 / 1e9 / hbm, "traffic": None,
                             "kernel": "prepare_x_kernel + decode_gemm_kernel at T = 1 (the whole call)",
                             "peak_source": f"{peak_kind} hbm_gbs"},
                "rooflines": {"tensor_at_4096_tokens": {
                    "bound": "tensor", "achieved": flops4 / t4 / 1e12, "peak": tc_peak, "unit": "TFLOP/s",
                    "frac": flops4 / t4 / 1e12 / tc_peak, "traffic": None,
                    "kernel": "prepare_x_kernel + decode_gemm_kernel at T = 4096",
                    "peak_source": f"{peak_kind} bf16_tflops (burst; fp16 runs at the bf16 rate)"}},
                "per_tokens": rows,
                "gpu_launches": len(DG_TOKENS) * 3 * max(args.steps, 3) + 2 * len(e2e_ts),
                "clocks": clk, "cpu_baseline": cpu, "e2e": e2e,
                "timing": "each call timed alone with events after an L2 flush; median of the repetitions"}
        print(json.dumps(line), flush=True)
    return 0


def run_ours(args):
    if args.workload == "decode_gemm":
        return run_decode_gemm(args)
    if args.workload in ("mlp", "stack_1p1b"):
        return run_multi(args)
    if args.workload == "polar":
        return run_polar(args)
    if args.workload == "decode_13b":
        return run_decode_sweep(args)
    if args.workload == "lloyd":
        return run_lloyd(args)
    import torch
    import torch.distributed as dist

    import synth
    import vector_codebook_codec_b200 as q
    from vector_codebook_codec_b200 import build as qbuild

    rank, world, local = dist_env()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    qbuild.build()
    q.load_library()

    spec, wname = workload_spec(args.workload)
    M, K = spec.M, spec.K
    w32 = synth.make_matrix(spec)
    if spec.dtype == "bf16":
        Wt, W32 = synth.to_bf16(w32)
    else:
        import torch as _t
        Wt, W32 = _t.from_numpy(w32), w32
    act = synth.act_for(spec)
    C = q.load_codebook(spec.N)
    Wd = Wt.to(dev)
    actd = torch.from_numpy(act).to(dev)
    Cd = torch.from_numpy(C).to(dev)
    table = q.build_search_table(Cd) if args.search == "pruned" else None   # once per codebook
    lib = q.load_library()
    wpr = q.words_per_row(K, spec.bits)
    ws = torch.empty(int(lib.qamw_calibrate_workspace_bytes(M, K)), dtype=torch.uint8, device=dev)
    sigma = torch.empty(K // 2, dtype=torch.float32, device=dev)
    packed = torch.empty((M, wpr), dtype=torch.int32, device=dev)
    rnorm = torch.empty(M, dtype=torch.float32, device=dev)
    cscale = torch.empty(K, dtype=torch.float32, device=dev)
    out = torch.empty((M, K), dtype=torch.bfloat16, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(max(args.steps, 1))]
    bd = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(max(args.steps, 1))]

    def one(evs=None):
        """The step: calibrate + encode in one call (s and r computed once), then decode."""
        if evs: evs[0].record(stream)
        enc = q.calibrate_encode(Wd, actd, spec.alpha, spec.block, spec.seed, Cd, spec.bits, status=status,
                                 out=(packed, rnorm, cscale, sigma), search_table=table, workspace=ws)
        if evs: evs[1].record(stream)
        q.decode(enc, Cd, out_dtype=torch.bfloat16, status=status, out=out)
        if evs: evs[2].record(stream)

    def separate(evs):
        """The same work as three separate calls, for the per-call breakdown."""
        evs[0].record(stream)
        sig = q.calibrate_sigma(Wd, actd, spec.alpha, spec.block, spec.seed, status=status, workspace=ws,
                                out=sigma)
        evs[1].record(stream)
        enc = q.encode(Wd, actd, spec.alpha, spec.block, spec.seed, sig, Cd, spec.bits, status=status,
                       out=(packed, rnorm, cscale), search_table=table)
        evs[2].record(stream)
        q.decode(enc, Cd, out_dtype=torch.bfloat16, status=status, out=out)
        evs[3].record(stream)

    for _ in range(args.warmup):
        flush.fill_(1.0)
        one()
    torch.cuda.synchronize(dev)
    if status.item() != 0:
        raise SystemExit(f"device status {status.item()} after warm-up")

    # The same step captured once as a CUDA graph (its 6 kernels replayed as one
    # graph launch: the launch gaps between dependent kernels shrink). The
    # headline is the replayed step; the eager calls below time it call by
    # call. Both run the same kernels on the same buffers.
    graph = None
    if args.graph:
        side = torch.cuda.Stream(dev)
        graph = torch.cuda.CUDAGraph()
        torch.cuda.synchronize(dev)
        with torch.cuda.graph(graph, stream=side):
            genc = q.calibrate_encode(Wd, actd, spec.alpha, spec.block, spec.seed, Cd, spec.bits, status=status,
                                      out=(packed, rnorm, cscale, sigma), search_table=table, workspace=ws,
                                      stream=side)
            q.decode(genc, Cd, out_dtype=torch.bfloat16, status=status, out=out, stream=side)
        for _ in range(args.warmup):
            flush.fill_(3.0)
            graph.replay()
        torch.cuda.synchronize(dev)
    gev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]

    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    for i in range(args.steps):
        flush.fill_(float(i))
        one(ev[i])
    torch.cuda.synchronize(dev)
    for i in range(args.steps):
        flush.fill_(float(i) + 0.25)
        separate(bd[i])
    torch.cuda.synchronize(dev)
    if graph is not None:
        if world > 1:
            dist.barrier()
        for i, (e0, e1) in enumerate(gev):
            flush.fill_(float(i) + 0.5)
            e0.record(stream)
            graph.replay()
            e1.record(stream)
        torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    time.sleep(0.2)
    clk = clocks.stop()
    if status.item() != 0:
        raise SystemExit(f"device status {status.item()} in the timed steps")

    t_cal = [bd[i][0].elapsed_time(bd[i][1]) for i in range(args.steps)]
    t_enc = [bd[i][1].elapsed_time(bd[i][2]) for i in range(args.steps)]
    t_dec = [bd[i][2].elapsed_time(bd[i][3]) for i in range(args.steps)]
    t_calenc = [ev[i][0].elapsed_time(ev[i][1]) for i in range(args.steps)]
    t_step = [ev[i][0].elapsed_time(ev[i][2]) for i in range(args.steps)]
    total_s = max_over_ranks(sum(t_step) / 1e3, dev)      # eager steps
    weights = M * K
    value = aggregate_throughput(weights * args.steps, total_s, world) / 1e9
    eager = {"ms_per_step": 1e3 * total_s / args.steps, "value": value, "unit": "Gweights/s"}
    if graph is not None:
        total_s = max_over_ranks(sum(e0.elapsed_time(e1) for e0, e1 in gev) / 1e3, dev)
        value = aggregate_throughput(weights * args.steps, total_s, world) / 1e9
        del graph

    peaks, peak_kind = measured_peaks()
    hbm = float(peaks.get("hbm_gbs", FALLBACK_HBM_GBS))
    sm_max = float(peaks.get("sm_max_mhz", 1965.0))
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    fp32_peak = sms * FP32_LANES_PER_SM * sm_max * 1e6  # FP32 lane-instructions per second
    P = M * K // 2
    es = 2 if spec.dtype == "bf16" else 4
    enc_ms = statistics.mean(t_enc)
    dec_ms = statistics.mean(t_dec)
    cal_ms = statistics.mean(t_cal)
    dec_bytes = M * K * 2 + M * wpr * 4 + 4 * M + 4 * K + 2 * K + 8 * spec.N
    cal_bytes = M * K * es * 2 + 4 * K + 4 * M
    fp32_src = f"{sms} SMs x 128 FP32 lanes x {sm_max:.0f} MHz ({peak_kind} max clock)"

    # The dominant kernel alone: the encode kernel, launched by
    # qamw_encode_prepared with the step's channel scales and row norms (the
    # same kernel and inputs as inside qamw_calibrate_encode), timed with
    # events on this stream after the steps, L2 flushed before each launch.
    kev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(max(args.steps, 3))]
    for e0, e1 in kev:
        flush.fill_(5.0)
        e0.record(stream)
        q.encode_prepared(Wd, cscale, rnorm, spec.block, spec.seed, sigma, Cd, spec.bits, status=status, out=packed,
                          search_table=table)
        e1.record(stream)
    torch.cuda.synchronize(dev)
    kern_ms = statistics.mean(e0.elapsed_time(e1) for e0, e1 in kev)
    enc_bytes = M * K * es + M * wpr * 4 + 4 * M + 4 * K + 4 * (K // 2) + 8 * spec.N
    evals = pruned_evaluations(q, Wd, cscale, rnorm, sigma, table, spec) if args.search == "pruned" else P * spec.N
    enc_roof = {"bound": "hbm", "achieved": enc_bytes / (kern_ms * 1e-3) / 1e9, "peak": hbm, "unit": "GB/s",
                "frac": enc_bytes / (kern_ms * 1e-3) / 1e9 / hbm,
                "traffic": ENCODE_TRAFFIC_BYTES.get(args.workload if args.search == "pruned" else "-"),
                "kernel": ("encode_pruned_kernel" if args.search == "pruned" else "encode_kernel (brute force)") +
                          " alone (qamw_encode_prepared)",
                "us_per_launch": 1e3 * kern_ms, "algorithmic_bytes_per_launch": enc_bytes,
                "bytes_note": "weights read + packed words written + r, s, sigma and codebook",
                "peak_source": f"{peak_kind} hbm_gbs",
                "fp32_issue": {"achieved": 4.0 * evals / (kern_ms * 1e-3) / 1e9, "peak": fp32_peak / 1e9,
                               "unit": "G lane-op/s", "frac": 4.0 * evals / (kern_ms * 1e-3) / fp32_peak,
                               "evaluations_per_pair": evals / P, "peak_source": fp32_src,
                               "note": "4 FP32 lane-ops (2 FSUB, FMUL, FFMA) per distance evaluation"}}
    # brute-force encode, timed on its own (not part of the step): its search is
    # FP32-bound, 4 FP32 operations (2 FSUB, FMUL, FFMA) per pair and centroid
    brute_ms = None
    if args.search == "pruned" and args.brute_steps > 0:
        bev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(args.brute_steps)]
        bpk = torch.empty_like(packed)
        q.encode_prepared(Wd, cscale, rnorm, spec.block, spec.seed, sigma, Cd, spec.bits, status=status, out=bpk)
        for e0, e1 in bev:
            flush.fill_(2.0)
            e0.record(stream)
            q.encode_prepared(Wd, cscale, rnorm, spec.block, spec.seed, sigma, Cd, spec.bits, status=status,
                              out=bpk)
            e1.record(stream)
        torch.cuda.synchronize(dev)
        brute_ms = statistics.mean(e0.elapsed_time(e1) for e0, e1 in bev)
        if not torch.equal(bpk, packed):
            raise SystemExit("brute-force and pruned encodes differ")
    elif args.search == "brute":
        brute_ms = kern_ms
    brute_roof = None
    if brute_ms is not None:
        ops = 4.0 * P * spec.N
        brute_roof = {"bound": "alu", "achieved": ops / (brute_ms * 1e-3) / 1e9, "peak": fp32_peak / 1e9,
                      "unit": "Gop/s", "frac": ops / (brute_ms * 1e-3) / fp32_peak, "traffic": None,
                      "kernel": "encode_kernel (brute-force search) alone (qamw_encode_prepared, no table)",
                      "ms": brute_ms, "peak_source": fp32_src}
    dec_roof = {"bound": "hbm", "achieved": dec_bytes / (dec_ms * 1e-3) / 1e9, "peak": hbm, "unit": "GB/s",
                "frac": dec_bytes / (dec_ms * 1e-3) / 1e9 / hbm, "traffic": None, "kernel": "decode_tma_kernel",
                "peak_source": f"{peak_kind} hbm_gbs", "gweights_per_s": weights / (dec_ms * 1e-3) / 1e9}
    cal_roof = {"bound": "hbm", "achieved": cal_bytes / (cal_ms * 1e-3) / 1e9, "peak": hbm, "unit": "GB/s",
                "frac": cal_bytes / (cal_ms * 1e-3) / 1e9 / hbm, "traffic": None,
                "kernel": "qamw_calibrate_sigma (4 kernels)"}
    rooflines = {"encode": enc_roof, "decode": dec_roof, "calibrate": cal_roof}
    if brute_roof is not None:
        rooflines["encode_brute_force"] = brute_roof

    # ---- end to end through the public API with host buffers. Every step
    # copies its inputs (W, act RMS) from pinned host memory and reads back its
    # results (decoded bf16 matrix, packed stream, r, s, sigma). Steps are
    # pipelined over two buffer slots and three streams (host-to-device copy,
    # compute, device-to-host copy), so step i+1's upload and step i-1's
    # read-back overlap step i's kernels, as a stream of matrices would run.
    e2e = None
    if not args.no_e2e:
        Wh = Wt.pin_memory()
        acth = torch.from_numpy(act).pin_memory()
        outh = torch.empty((M, K), dtype=torch.bfloat16).pin_memory()
        pkh = torch.empty((M, wpr), dtype=torch.int32).pin_memory()
        rh = torch.empty(M, dtype=torch.float32).pin_memory()
        sh = torch.empty(K, dtype=torch.float32).pin_memory()
        sgh = torch.empty(K // 2, dtype=torch.float32).pin_memory()
        slots = []
        for _ in range(2):
            slots.append(dict(
                W=torch.empty_like(Wd), act=torch.empty_like(actd), ws=torch.empty_like(ws),
                sigma=torch.empty_like(sigma), packed=torch.empty_like(packed), r=torch.empty_like(rnorm),
                s=torch.empty_like(cscale), out=torch.empty_like(out),
                h2d=torch.cuda.Event(), comp=torch.cuda.Event(), d2h=torch.cuda.Event()))
        s_h2d, s_comp, s_d2h = (torch.cuda.Stream(dev) for _ in range(3))

        def e2e_step(i):
            sl = slots[i % 2]
            with torch.cuda.stream(s_h2d):
                s_h2d.wait_event(sl["comp"])            # step i-2 has finished reading this slot's inputs
                sl["W"].copy_(Wh, non_blocking=True)
                sl["act"].copy_(acth, non_blocking=True)
                sl["h2d"].record(s_h2d)
            with torch.cuda.stream(s_comp):
                s_comp.wait_event(sl["h2d"])
                s_comp.wait_event(sl["d2h"])            # step i-2's results have been read back
                enc = q.calibrate_encode(sl["W"], sl["act"], spec.alpha, spec.block, spec.seed, Cd, spec.bits,
                                         status=status, out=(sl["packed"], sl["r"], sl["s"], sl["sigma"]),
                                         search_table=table, workspace=sl["ws"], stream=s_comp)
                q.decode(enc, Cd, out_dtype=torch.bfloat16, status=status, out=sl["out"], stream=s_comp)
                sl["comp"].record(s_comp)
            with torch.cuda.stream(s_d2h):
                s_d2h.wait_event(sl["comp"])
                outh.copy_(sl["out"], non_blocking=True)
                pkh.copy_(sl["packed"], non_blocking=True)
                rh.copy_(sl["r"], non_blocking=True)
                sh.copy_(sl["s"], non_blocking=True)
                sgh.copy_(sl["sigma"], non_blocking=True)
                sl["d2h"].record(s_d2h)

        for i in range(max(2, args.warmup)):
            e2e_step(i)
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for st in (s_h2d, s_comp, s_d2h):
            st.wait_event(e0)
        for i in range(args.steps):
            e2e_step(i)
        stream.wait_stream(s_d2h)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        e2e_s = max_over_ranks(e0.elapsed_time(e1) / 1e3, dev)
        if status.item() != 0:
            raise SystemExit(f"device status {status.item()} in the end-to-end steps")
        if not torch.equal(pkh, packed.cpu()):
            raise SystemExit("end-to-end packed stream differs from the device-resident run")
        e2e = {"value": aggregate_throughput(weights * args.steps, e2e_s, world) / 1e9, "unit": "Gweights/s",
               "h2d_bytes_per_step": Wh.numel() * 2 + acth.numel() * 4,
               "d2h_bytes_per_step": outh.numel() * 2 + pkh.numel() * 4 + 4 * M + 4 * K + 2 * K,
               "pipelining": "2 buffer slots; H2D, compute and D2H on three streams"}

    # ---- the oracle on the host cores (rank 0, N = 1 only): its speed on a
    # row sample over every core, and, in the same leg, the index parity of
    # the whole matrix against the GPU encoding of the timed steps
    cpu, parity = None, None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rows = args.cpu_rows or auto_rows(spec)
        pool = OraclePool()
        try:
            nrows, walls = time_oracle_parallel(pool, W32, act, spec, C, rows, 3)
        finally:
            pool.close()
        cpu = {"value": nrows * K / statistics.median(walls) / 1e9, "unit": "Gweights/s", "cores": pool.workers,
               "kind": "oracle",
               "sample": f"{pool.workers} worker processes x {rows} rows of {M} per step (calibrate + encode + decode "
                         f"of its rows, fp64 numpy, one thread each); median of 3 steps"}
        parity = oracle_parity(W32, act, spec, C, sigma.cpu().numpy(), rnorm.cpu().numpy(), cscale.cpu().numpy(),
                               packed.cpu().numpy().view(np.uint32))

    if world > 1:
        dist.barrier()
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "Gweights/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1e3 * total_s / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic (seeded; no checkpoint)",
            "config": {"workload": wname, "M": M, "K": K, "weight_dtype": spec.dtype, "block": spec.block,
                       "N": spec.N, "bits": spec.bits, "alpha": spec.alpha,
                       "search": "exact pruned (grid table)" if args.search == "pruned" else "brute force",
                       "l2": "flushed by a 256 MiB write before every timed step",
                       "parallelism": f"{world} independent replica(s)"},
            "roofline": enc_roof,
            "rooflines": rooflines,
            "ms": {"calibrate": cal_ms, "encode": enc_ms, "decode": dec_ms,
                   "calibrate_encode": statistics.mean(t_calenc),
                   "note": ("calibrate, encode and decode: the three separate calls (each computes s and r); "
                            "calibrate_encode: the step's fused call (s and r once)")},
            "cpu_baseline": cpu, "parity": parity, "e2e": e2e, "gpu_launches": 6 * args.steps, "clocks": clk,
            "timing": ("each step replays a CUDA graph of the 6 kernels (captured once from the C-ABI calls); "
                       "'eager' is the same step launched call by call" if args.graph else
                       "each step launched call by call"),
            "eager": eager,
            "dtype_detail": "rotation fp64, search and decode fp32, decode output bf16",
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
