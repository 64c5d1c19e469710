#!/usr/bin/env python
"""Throughput of reciprocal nearest-neighbour matching (MASt3R) on B200.

Default workload (the headline): one step = one ``fastnn_reciprocal`` call on
one 512x384 image pair with d = 24 int8 descriptors, seeds on an 8-px grid
(3,072 seeds), max_iter = 10 -- every round's forward and backward
nearest-neighbour passes, the reciprocal check and the frontier compaction.
Inputs are synthetic (``synth``: a smooth warp of map 1 with 30% outliers and
+-2 noise). Printed value: reciprocal matches per second (unique pairs kept /
device time of the call), whole job over all ranks.

Other workloads (``--workload``): ``pair_512x384_d24_bf16`` (float
descriptors), ``batch16_512x288_d32_i8`` (16 pairs per call) and
``dense_512x384_d24_i8`` (``fastnn_mutual_dense`` over all 196,608 pixels;
value = mutual pairs per second).

Each rank processes its own independent pair(s) (pair-level data parallelism,
no collective on the data path); rank r > 0 draws its inputs from the
workload's seed + 7919 r.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME]
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "reciprocal matches/sec and pairs/sec at 512×384 d=24; tensor-pipe % of peak"
# FP32 fused multiply-add peak of one B200: 148 SMs x 128 lanes x 2 flop x 1.965 GHz.
FP32_FMA_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12
UNIT = "matches/s"
DEFAULT_WORKLOAD = "pair_512x384_d24_i8"
L2_FLUSH_BYTES = 256 << 20  # > 126 MB L2


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=4000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(synth.CONFIGS))
    ap.add_argument("--cpu-baseline", type=int, default=1,
                    help="time the CPU oracle on a bounded sample (rank 0, N=1)")
    return ap.parse_args()


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def metric_for(name, dense):
    if name == DEFAULT_WORKLOAD:
        return METRIC
    if name == "dense_512x384_d24_i8":
        return "dense mutual nearest-neighbour pairs/sec at 512×384 d=24 (all 196,608 pixels)"
    if dense:
        return f"dense mutual nearest-neighbour pairs/sec, workload {name}"
    return f"reciprocal matches/sec, workload {name}"


def load_workload(name, rank):
    """The named workload; rank r > 0 gets its own independent inputs."""
    w = synth.make_workload(name)
    if rank == 0:
        return w
    seed = synth.CONFIGS[name]["seed"] + 7919 * rank
    if name.startswith("batch16"):
        w.pairs = [synth.warped_pair_int8(seed + 1000 * b, H=288, W=512, d=32) for b in range(16)]
    elif name.endswith("pts3_f32"):
        w.pairs = [synth.pointmap_pair(seed)]
    elif name.endswith("bf16") or name.endswith("f16"):
        w.pairs = [synth.warped_pair_bf16(seed, storage=w.pairs[0].dtype)]
    elif name.startswith("tiny"):
        w.pairs = [synth.tiny_permuted_pair(seed)]
    else:
        w.pairs = [synth.warped_pair_int8(seed, d=w.pairs[0].d)]
    return w


def config_dict(w, extra=None):
    p = w.pairs[0]
    c = {"workload": w.name, "image": f"{p.W1}x{p.H1}", "d": p.d,
         "descriptor": {"bf16": "bf16 unit-norm", "f16": "IEEE half unit-norm",
                        "l2": "float32 3D pointmap, Euclidean distance"}.get(p.dtype, "int8"),
         "pairs_per_rank_per_step": w.batch,
         "parallelism": "pair-parallel replicas, no collective",
         "l2": "flushed between timed steps (256 MiB write)"}
    if w.dense:
        c["method"] = "dense mutual nearest neighbours (fastnn_mutual_dense)"
    else:
        c.update({"method": "fast reciprocal matching (fastnn_reciprocal)",
                  "subsample": w.subsample, "max_iter": w.max_iter,
                  "seeds_per_pair": (p.H1 + w.subsample - 1) // w.subsample
                  * ((p.W1 + w.subsample - 1) // w.subsample)})
    if "conf1" in w.extra:
        c.update({"method": "confidence-masked fast reciprocal matching "
                            "(fastnn_reciprocal_masked)",
                  "conf_threshold": w.extra["threshold"]})
    if extra:
        c.update(extra)
    return c


def to_pinned(arr, torch, storage="i8"):
    if arr.dtype == np.uint16:
        half = torch.float16 if storage == "f16" else torch.bfloat16
        return torch.from_numpy(arr.view(np.int16)).view(half).pin_memory()
    return torch.from_numpy(arr).pin_memory()


# ---------------------------------------------------------------------------
# CPU oracle samples (the reference arm and the cpu_baseline key)
# ---------------------------------------------------------------------------

def oracle_sample(w, n_seeds, dense_rows=None):
    """Time the CPU oracle on a bounded sample of workload ``w``.

    Fast workloads: the fast scheme on pair 0 from the first ``n_seeds`` seeds
    of its grid (row-major). Dense: nearest neighbours of the first
    ``dense_rows`` (default ``n_seeds``) image-1 pixels and of their matches,
    i.e. the mutual pairs among those pixels.
    Returns (matches found, seconds, threads, description).
    """
    import oracle
    p = w.pairs[0]
    threads = oracle.default_threads()
    if w.dense:
        D1 = p.desc1.reshape(-1, p.d)
        D2 = p.desc2.reshape(-1, p.d)
        dense_rows = min(n_seeds if dense_rows is None else dense_rows, D1.shape[0])
        t0 = time.perf_counter()
        r12 = oracle.nn(D1[:dense_rows], D2, p.dtype, threads)
        r21 = oracle.nn(D2[r12.idx], D1, p.dtype, threads)
        found = int(np.sum(r21.idx == np.arange(dense_rows)))
        dt = time.perf_counter() - t0
        return found, dt, threads, (f"mutual pairs among the first {dense_rows} image-1 pixels "
                                    f"(nearest neighbours over all {D2.shape[0]} pixels each way)")
    if "conf1" in w.extra:
        thr = w.extra["threshold"]
        k1 = oracle.confident(w.extra["conf1"][0], p.H1 * p.W1, thr)
        k2 = oracle.confident(w.extra["conf2"][0], p.H2 * p.W2, thr)
        t0 = time.perf_counter()
        r = oracle.fast_reciprocal_masked(p.desc1, p.H1, p.W1, k1, p.desc2, p.H2, p.W2, k2,
                                          p.dtype, w.subsample, w.max_iter, nthreads=threads,
                                          max_seeds=n_seeds)
        dt = time.perf_counter() - t0
        return len(r.pairs), dt, threads, (f"confidence-masked fast reciprocal matching of pair 0 "
                                           f"from its first {n_seeds} kept grid seeds, "
                                           f"max_iter {w.max_iter}")
    seeds = oracle.grid_seeds(p.H1, p.W1, w.subsample)[:n_seeds]
    t0 = time.perf_counter()
    r = oracle.fast_reciprocal(p.desc1, p.H1, p.W1, p.desc2, p.H2, p.W2, p.dtype, w.subsample,
                               w.max_iter, nthreads=threads, seeds=seeds)
    dt = time.perf_counter() - t0
    return len(r.pairs), dt, threads, (f"fast reciprocal matching of pair 0 from the first "
                                       f"{len(seeds)} of its grid seeds, max_iter {w.max_iter}")


def run_reference(args, rank, world):
    """The oracle as it stands, on this machine's host cores (rank 0 only)."""
    if rank != 0:
        return 0
    w = synth.make_workload(args.workload)
    # Size each step's sample so that warm-up plus timed steps take about two
    # minutes of host time: calibrate on 64 seeds (or pixels), then scale.
    _, t64, _, _ = oracle_sample(w, 64)
    budget = 120.0 / max(1, args.steps + args.warmup)
    n = int(max(1, min(4096, 64 * budget / max(t64, 1e-6))))
    for _ in range(args.warmup):
        oracle_sample(w, n)
    tot_m, tot_t = 0, 0.0
    threads, desc = 0, ""
    for _ in range(args.steps):
        m, dt, threads, desc = oracle_sample(w, n)
        tot_m += m
        tot_t += dt
    value = tot_m / tot_t
    line = {
        "impl": "reference", "metric": metric_for(args.workload, w.dense), "value": value, "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * tot_t / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "int64" if w.pairs[0].dtype == "i8" else "f64",
        "data": "synthetic", "config": config_dict(w, {"reference": "CPU oracle (oracle/)"}),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": desc + ", per step"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# clocks
# ---------------------------------------------------------------------------

class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""

    FIELDS = ("uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid):
        self.uuid = uuid
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        self.p = None
        try:
            self.p = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}",
                                       "--format=csv,noheader,nounits", "-lms", "100"],
                                      stdout=self.f, stderr=subprocess.DEVNULL)
        except (FileNotFoundError, OSError):
            self.p = None

    def stop(self):
        if self.p is not None:
            time.sleep(0.25)
            self.p.terminate()
            self.p.wait(timeout=10)
        self.f.flush()
        self.f.seek(0)
        rows = [ln.strip().split(", ") for ln in self.f if ln.strip()]
        self.f.close()
        os.unlink(self.f.name)
        if self.p is None:
            return None
        mine = [r for r in rows if len(r) >= 9 and (self.uuid is None or r[0] in self.uuid
                                                     or self.uuid in r[0])]
        if not mine:
            mine = [r for r in rows if len(r) >= 9]
        if not mine:
            return None
        try:
            sm = [float(r[1]) for r in mine]
            smax = max(float(r[2]) for r in mine)
        except ValueError:
            return None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in mine for n, v in zip(names, r[5:9]) if v.strip() == "Active"})
        loaded = [x for x in sm if x > 0.5 * smax] or sm
        power = []
        for r in mine:
            try:
                power.append(float(r[3]))
            except ValueError:
                pass
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": smax, "reasons": reasons,
                "samples": len(mine), "power_w_max": max(power) if power else None}


# DRAM traffic per launch of the dominant kernel, from one ncu capture
# (dram__bytes_read.sum + dram__bytes_write.sum; profiles/*.md), keyed by
# workload and by a hash of the kernel sources it was taken on. A changed
# kernel reports null until it is captured again.
TRAFFIC = {
    "pair_512x384_d24_i8": (12.716e6, "172ee1fa511b4f34"),
    "pair_512x384_pts3_f32": (6.441e6, "172ee1fa511b4f34"),
    # Dense: the two launches of one step (forward 14.21 MB + backward 13.59 MB).
    "dense_512x384_d24_i8": (27.80e6, "172ee1fa511b4f34"),
}
KERNEL_SOURCES = ["reciprocal_nearest_neighbours_b200/csrc/nn_tc.cu",
                  "reciprocal_nearest_neighbours_b200/csrc/l2_nn.cu",
                  "reciprocal_nearest_neighbours_b200/csrc/frontier_dev.cuh",
                  "reciprocal_nearest_neighbours_b200/csrc/frontier.cuh",
                  "reciprocal_nearest_neighbours_b200/csrc/common.cuh",
                  "reciprocal_nearest_neighbours_b200/csrc/ptx.cuh"]


def kernel_source_hash():
    import hashlib
    h = hashlib.sha256()
    for f in KERNEL_SOURCES:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def traffic_for(name):
    rec = TRAFFIC.get(name)
    if rec is None or rec[1] != kernel_source_hash():
        return None
    return rec[0]


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return json.load(f), "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}, "fallback"


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------

def run_ours(args, rank, world, local):
    import torch
    import torch.distributed as dist
    import reciprocal_nearest_neighbours_b200 as fnn

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)

    w = load_workload(args.workload, rank)
    p0 = w.pairs[0]
    B = w.batch
    H1, W1, d = p0.desc1.shape
    H2, W2, _ = p0.desc2.shape
    N1, N2 = H1 * W1, H2 * W2
    i8 = p0.dtype == "i8"
    code = {"i8": fnn.FASTNN_I8, "bf16": fnn.FASTNN_BF16, "f16": fnn.FASTNN_F16,
            "l2": fnn.FASTNN_F32_L2}[p0.dtype]
    sdt = torch.int32 if i8 else torch.float32
    l2 = p0.dtype == "l2"
    masked = "conf1" in w.extra
    esize = 1 if i8 else 4 if l2 else 2
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    if w.dense:
        h1 = to_pinned(np.ascontiguousarray(p0.desc1.reshape(-1, d)), torch, p0.dtype)
        h2 = to_pinned(np.ascontiguousarray(p0.desc2.reshape(-1, d)), torch, p0.dtype)
        cap = min(N1, N2)
        out_pairs = torch.empty((cap, 2), dtype=torch.int32, device=dev)
        out_score = torch.empty(cap, dtype=sdt, device=dev)
        out_count = torch.empty(1, dtype=torch.int32, device=dev)
        nbytes = fnn.fastnn_workspace_size(fnn.FASTNN_OP_MUTUAL_DENSE, N1, N2, d, code)
        hp_pairs = torch.empty((cap, 2), dtype=torch.int32).pin_memory()
        hp_score = torch.empty(cap, dtype=sdt).pin_memory()
    else:
        d1n, d2n = w.stacked()
        h1, h2 = to_pinned(d1n, torch, p0.dtype), to_pinned(d2n, torch, p0.dtype)
        S = fnn.seed_count(H1, W1, w.subsample)
        out_pairs = torch.empty((B, S, 2), dtype=torch.int32, device=dev)
        out_score = torch.empty((B, S), dtype=sdt, device=dev)
        out_count = torch.empty(B, dtype=torch.int32, device=dev)
        out_iters = torch.empty(B, dtype=torch.int32, device=dev)
        out_front = torch.empty((B, w.max_iter), dtype=torch.int32, device=dev)
        op = fnn.FASTNN_OP_RECIPROCAL_MASKED if masked else fnn.FASTNN_OP_RECIPROCAL
        nbytes = fnn.fastnn_workspace_size(op, N1, N2, d, code, B, S)
        hp_pairs = torch.empty((B, S, 2), dtype=torch.int32).pin_memory()
        hp_score = torch.empty((B, S), dtype=sdt).pin_memory()
    hp_count = torch.empty(out_count.shape, dtype=torch.int32).pin_memory()
    d1 = h1.to(dev)
    d2 = h2.to(dev)
    ws = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    hc1 = hc2 = c1 = c2 = None
    if masked:
        hc1 = torch.from_numpy(np.ascontiguousarray(np.stack(w.extra["conf1"]))).pin_memory()
        hc2 = torch.from_numpy(np.ascontiguousarray(np.stack(w.extra["conf2"]))).pin_memory()
        c1, c2 = hc1.to(dev), hc2.to(dev)

    if w.dense:
        def call():
            fnn.fastnn_mutual_dense(d1, d2, out_pairs=out_pairs, out_score=out_score,
                                    out_count=out_count, workspace=ws, stream=stream)
        # 2 repack, forward pass, image list (mark/count/scan/emit), pointmaps:
        # chunk boxes of image 1, backward pass, mutual count/scan/emit
        launches_per_step = 2 + 1 + 4 + (1 if l2 else 0) + 1 + 3
        kernels_per_step = 2
    elif masked:
        def call():
            fnn.fastnn_reciprocal_masked(d1, d2, w.subsample, w.max_iter, conf1=c1, conf2=c2,
                                         threshold=w.extra["threshold"], out_pairs=out_pairs,
                                         out_score=out_score, out_count=out_count,
                                         out_iters=out_iters, out_frontier=out_front,
                                         workspace=ws, stream=stream)
        # 2 x (count, scan, emit) mask compaction, seeds, 1 persistent matching kernel
        launches_per_step = 8
        kernels_per_step = 1
    else:
        def call():
            fnn.fastnn_reciprocal(d1, d2, w.subsample, w.max_iter, out_pairs=out_pairs,
                                  out_score=out_score, out_count=out_count, out_iters=out_iters,
                                  out_frontier=out_front, workspace=ws, stream=stream)
        launches_per_step = 3  # 2 repack kernels + 1 persistent matching kernel (all rounds)
        kernels_per_step = 1

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)

    for _ in range(max(args.warmup, 3)):
        flush.zero_()
        call()
    torch.cuda.synchronize(dev)
    assert fnn.fastnn_device_status(ws) == 0
    matches = int(out_count.cpu().sum())
    image = None
    if w.dense:
        # The backward pass runs on the image of NN12 only (the rows that can
        # be in a mutual pair): count them for the useful-work figure.
        idx12, _ = fnn.fastnn_nn(d1, d2)
        image = int(torch.unique(idx12[(idx12 >= 0) & (idx12 < N2)]).numel())
        pairs_per_step = N1 * N2 + image * N1
    else:
        pairs_per_step = int(out_front.cpu().sum()) * (N1 + N2)
    macs_per_step = pairs_per_step * d

    # ---- device-timed region ------------------------------------------------
    uuid = None
    try:
        uuid = str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:  # noqa: BLE001
        pass
    sampler = ClockSampler(uuid) if rank == 0 else None
    if sampler:
        time.sleep(0.5)
    K = args.steps
    fnn.fastnn_kernel_timer_enable(K * kernels_per_step + 8)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(K)]
    barrier()
    for i in range(K):
        flush.zero_()
        evs[i][0].record(stream)
        call()
        evs[i][1].record(stream)
    barrier()
    clocks = sampler.stop() if sampler else None
    total_ms = sum(s.elapsed_time(e) for s, e in evs)
    nn_launches, nn_ms = fnn.fastnn_kernel_timer_read()
    fnn.fastnn_kernel_timer_enable(0)
    assert fnn.fastnn_device_status(ws) == 0
    assert int(out_count.cpu().sum()) == matches

    # ---- end to end through the C ABI with host buffers --------------------
    Ke = max(1, min(K, 1000))
    evs2 = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            for _ in range(Ke)]
    barrier()
    for i in range(Ke):
        flush.zero_()
        evs2[i][0].record(stream)
        d1.copy_(h1, non_blocking=True)
        d2.copy_(h2, non_blocking=True)
        if masked:
            c1.copy_(hc1, non_blocking=True)
            c2.copy_(hc2, non_blocking=True)
        call()
        hp_count.copy_(out_count, non_blocking=True)
        hp_pairs.copy_(out_pairs, non_blocking=True)
        hp_score.copy_(out_score, non_blocking=True)
        evs2[i][1].record(stream)
    barrier()
    e2e_ms = sum(s.elapsed_time(e) for s, e in evs2)
    assert int(hp_count.sum()) == matches

    # ---- reduce over ranks ----------------------------------------------------
    vals = torch.tensor([total_ms, e2e_ms, nn_ms], dtype=torch.float64, device=dev)
    m = torch.tensor([matches], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(vals, op=dist.ReduceOp.MAX)
        dist.all_reduce(m, op=dist.ReduceOp.SUM)
    total_ms, e2e_ms, _ = vals.tolist()
    all_matches = float(m.item())

    if rank == 0:
        value = all_matches * K / (total_ms / 1e3)
        e2e_value = all_matches * Ke / (e2e_ms / 1e3)
        pairs_per_s = world * B * K / (total_ms / 1e3)
        peaks, src = measured_peaks()
        bf16_peak = float(peaks["bf16_tflops"])
        if l2:
            # Pointmaps: 3 fused multiply-adds per (query, point) pair on the
            # FP32 pipe; peak = 148 SMs x 128 FMA lanes x 2 flop x 1.965 GHz.
            peak = FP32_FMA_TFLOPS
            achieved = 6.0 * pairs_per_step * K / (nn_ms / 1e3) / 1e12 if nn_ms > 0 else None
        else:
            peak = 2.0 * bf16_peak if i8 else bf16_peak  # dense int8 = 2 x bf16 (nominal ratio)
            achieved = 2.0 * macs_per_step * K / (nn_ms / 1e3) / 1e12 if nn_ms > 0 else None
        bytes_in = (N1 + N2) * d * esize * B + ((N1 + N2) * 4 * B if masked else 0)
        bytes_out = int(hp_count.numel() * 4 + hp_pairs.numel() * 4 + hp_score.numel() * 4)
        if l2:
            kname = ("nn_l2_kernel (FP32 FMA nearest point: forward pass over every image-1 "
                     "point, backward pass over the image of the forward matches)"
                     if w.dense else
                     "reciprocal_l2_kernel (persistent: seeds, FP32 FMA forward and backward "
                     "passes, per-pair compaction)")
        else:
            kname = ("nn_tc_kernel (tcgen05 argmax-GEMM: forward pass over every image-1 row, "
                     "backward pass over the image of the forward matches)" if w.dense else
                     "reciprocal_kernel (persistent: seeds, tcgen05 forward and backward passes, "
                     "per-pair compaction)")
        if l2:
            peak_source = ("derived: FP32 FMA pipe, 148 SMs x 128 lanes x 2 flop x 1.965 GHz "
                           "(clocks.max.sm)")
            ops = (f"3 FMA = 6 flop per (query, point) pair: {pairs_per_step:.4g} pairs "
                   f"per step")
            if image is not None:
                ops += f" ({N1} x {N2} forward + {image} x {N1} backward)"
        else:
            peak_source = (f"{src}: bf16_tflops {bf16_peak}" +
                           (" x 2 (int8 = 2 x bf16, nominal ratio)" if i8 else ""))
            ops = f"2 x useful MACs (d = {d}) per step: {macs_per_step:.4g} MAC"
            if image is not None:
                ops += f" ({N1} x {N2} forward + {image} x {N1} backward)"
        line = {
            "metric": metric_for(w.name, w.dense), "value": value, "unit": UNIT, "n_gpus": world,
            "steps": K, "warmup": args.warmup, "ms_per_step": total_ms / K,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": {"i8": "int8", "bf16": "bf16", "f16": "f16", "l2": "f32"}[p0.dtype],
            "data": "synthetic",
            "config": config_dict(w),
            "pairs_per_s": pairs_per_s,
            "matches_per_step_rank0": matches,
            "roofline": {
                "bound": "alu" if l2 else "tensor", "kernel": kname,
                "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": (achieved / peak) if achieved else None,
                "traffic": traffic_for(w.name),
                "traffic_unit": ("bytes per step: forward + backward launch (ncu dram read + write)"
                                 if w.dense else "bytes per launch (ncu dram read + write)"),
                "peak_source": peak_source,
                "ops": ops,
                "kernel_ms_per_step": nn_ms / K, "kernel_launches": nn_launches,
                "kernel_share_of_step": nn_ms / total_ms if total_ms else None,
            },
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": bytes_in,
                    "d2h_bytes_per_step": bytes_out, "steps": Ke},
            "gpu_launches": launches_per_step * K,
            "clocks": clocks,
        }
        if not w.dense:
            line["frontier_per_round_pair0"] = out_front[0].cpu().tolist()
        if args.cpu_baseline and world == 1:
            try:
                cm, cdt, cthreads, cdesc = oracle_sample(w, 256, dense_rows=1024)
                line["cpu_baseline"] = {"value": cm / cdt, "unit": UNIT, "cores": cthreads,
                                        "kind": "oracle",
                                        "sample": f"{cdesc}, one oracle call, {cdt:.2f} s"}
            except Exception as e:  # noqa: BLE001
                line["cpu_baseline"] = {"value": None, "unit": UNIT, "cores": None,
                                        "kind": "oracle", "sample": f"failed: {e}"}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main():
    args = parse_args()
    rank, world, local = dist_env()
    if args.impl == "reference":
        return run_reference(args, rank, world)
    return run_ours(args, rank, world, local)


if __name__ == "__main__":
    sys.exit(main())
