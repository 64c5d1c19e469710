#!/usr/bin/env python
"""Throughput of MASt3R fast reciprocal matching on B200.

One step = one call of ``fastnn_reciprocal`` on one 512x384 image pair with
d = 24 int8 descriptors, seeds on an 8-px grid (3,072 seeds), max_iter = 10:
every round's forward and backward nearest-neighbour passes, the reciprocal
check and the frontier compaction. Inputs are synthetic (``synth``: a smooth
warp of map 1 with 30% outliers and +-2 noise).

Printed value: reciprocal matches per second (unique pairs kept / device time
of the call), whole job over all ranks. Each rank processes its own
independent pair (pair-level data parallelism, no collective on the data
path); rank r > 0 draws its pair from seed + 7919 r.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
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
UNIT = "matches/s"
WORKLOAD = "pair_512x384_d24_i8"
L2_FLUSH_BYTES = 256 << 20  # > 126 MB L2


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=4000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-baseline", type=int, default=1,
                    help="time the CPU oracle on a bounded sample (rank 0, N=1)")
    return ap.parse_args()


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def config_dict(w, extra=None):
    c = {"workload": WORKLOAD, "image": "512x384", "d": 24, "descriptor": "int8 uniform [-16,16]",
         "subsample": w.subsample, "max_iter": w.max_iter, "seeds_per_pair": 3072,
         "pairs_per_rank_per_step": 1, "parallelism": "pair-parallel replicas, no collective",
         "l2": "flushed between timed steps (256 MiB write)"}
    if extra:
        c.update(extra)
    return c


def oracle_sample(pair, w, n_seed_rows):
    """Time the CPU oracle on the first ``n_seed_rows`` rows of the seed grid."""
    import oracle
    seeds = oracle.grid_seeds(pair.H1, pair.W1, w.subsample)
    per_row = (pair.W1 + w.subsample - 1) // w.subsample
    seeds = seeds[: n_seed_rows * per_row]
    threads = oracle.default_threads()
    t0 = time.perf_counter()
    r = oracle.fast_reciprocal(pair.desc1, pair.H1, pair.W1, pair.desc2, pair.H2, pair.W2, "i8",
                               w.subsample, w.max_iter, nthreads=threads, seeds=seeds)
    dt = time.perf_counter() - t0
    return len(r.pairs), dt, threads, len(seeds)


def run_reference(args, rank, world):
    """The oracle as it stands, on this machine's host cores (rank 0 only)."""
    if rank != 0:
        return 0
    w = synth.make_workload(WORKLOAD)
    pair = w.pairs[0]
    rows = 2  # 2 seed rows x 64 = 128 of the 3,072 seeds per step
    for _ in range(args.warmup):
        oracle_sample(pair, w, rows)
    tot_m, tot_t = 0, 0.0
    threads = seeds = 0
    for _ in range(args.steps):
        m, dt, threads, seeds = oracle_sample(pair, w, rows)
        tot_m += m
        tot_t += dt
    value = tot_m / tot_t
    sample = (f"fast reciprocal matching of the {WORKLOAD} pair from the first {seeds} of its "
              f"3,072 grid seeds (2 seed rows), max_iter {w.max_iter}, per step")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot_t / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int64",
        "data": "synthetic", "config": config_dict(w, {"reference": "CPU oracle (oracle/)"}),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


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
        self.t_start = self.t_stop = None

    def mark_start(self):
        self.t_start = time.time()

    def stop(self):
        self.t_stop = time.time()
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
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": smax, "reasons": reasons,
                "samples": len(mine), "power_w_max": max(float(r[3]) for r in mine
                                                         if r[3].replace(".", "").isdigit())
                if any(r[3].replace(".", "").isdigit() for r in mine) else None}


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return json.load(f), "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}, "fallback"


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

    w = synth.make_workload(WORKLOAD)
    if rank == 0:
        pair = w.pairs[0]
    else:
        pair = synth.warped_pair_int8(synth.CONFIGS[WORKLOAD]["seed"] + 7919 * rank)
    H1, W1, d = pair.desc1.shape
    H2, W2, _ = pair.desc2.shape
    N1, N2 = H1 * W1, H2 * W2

    h1 = torch.from_numpy(pair.desc1).pin_memory()
    h2 = torch.from_numpy(pair.desc2).pin_memory()
    d1 = h1.to(dev)
    d2 = h2.to(dev)
    S = fnn.seed_count(H1, W1, w.subsample)
    out_pairs = torch.empty((1, S, 2), dtype=torch.int32, device=dev)
    out_score = torch.empty((1, S), dtype=torch.int32, device=dev)
    out_count = torch.empty(1, dtype=torch.int32, device=dev)
    out_iters = torch.empty(1, dtype=torch.int32, device=dev)
    out_front = torch.empty((1, w.max_iter), dtype=torch.int32, device=dev)
    nbytes = fnn.fastnn_workspace_size(fnn.FASTNN_OP_RECIPROCAL, N1, N2, d, fnn.FASTNN_I8, 1, S)
    ws = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    hp_pairs = torch.empty((1, S, 2), dtype=torch.int32).pin_memory()
    hp_score = torch.empty((1, S), dtype=torch.int32).pin_memory()
    hp_count = torch.empty(1, dtype=torch.int32).pin_memory()
    stream = torch.cuda.current_stream(dev)

    def call():
        fnn.fastnn_reciprocal(d1, d2, w.subsample, w.max_iter, out_pairs=out_pairs,
                              out_score=out_score, out_count=out_count, out_iters=out_iters,
                              out_frontier=out_front, workspace=ws, stream=stream)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)

    for _ in range(max(args.warmup, 3)):
        flush.zero_()
        call()
    torch.cuda.synchronize(dev)
    assert fnn.fastnn_device_status(ws) == 0
    matches = int(out_count[0])
    frontier = out_front[0].cpu().tolist()
    launches_per_step = 3  # 2 repack kernels + 1 persistent matching kernel (all rounds)

    # ---- device-timed region ------------------------------------------------
    uuid = None
    try:
        uuid = str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        pass
    sampler = ClockSampler(uuid) if rank == 0 else None
    if sampler:
        time.sleep(0.5)
        sampler.mark_start()
    K = args.steps
    fnn.fastnn_kernel_timer_enable(K + 8)
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
    assert int(out_count[0]) == matches

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
        call()
        hp_count.copy_(out_count, non_blocking=True)
        hp_pairs.copy_(out_pairs, non_blocking=True)
        hp_score.copy_(out_score, non_blocking=True)
        evs2[i][1].record(stream)
    barrier()
    e2e_ms = sum(s.elapsed_time(e) for s, e in evs2)
    assert int(hp_count[0]) == matches

    # ---- reduce over ranks ----------------------------------------------------
    vals = torch.tensor([total_ms, e2e_ms, nn_ms], dtype=torch.float64, device=dev)
    m = torch.tensor([matches], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(vals, op=dist.ReduceOp.MAX)
        dist.all_reduce(m, op=dist.ReduceOp.SUM)
    total_ms, e2e_ms, nn_ms_max = vals.tolist()
    all_matches = float(m.item())

    if rank == 0:
        value = all_matches * K / (total_ms / 1e3)
        e2e_value = all_matches * Ke / (e2e_ms / 1e3)
        pairs_per_s = world * K / (total_ms / 1e3)
        peaks, src = measured_peaks()
        int8_peak = 2.0 * float(peaks["bf16_tflops"])  # dense int8 = 2 x bf16 (nominal ratio)
        macs_per_step = sum(f * (N1 + N2) * d for f in frontier)
        achieved = 2.0 * macs_per_step * K / (nn_ms / 1e3) / 1e12 if nn_ms > 0 else None
        bytes_in = (N1 + N2) * d  # int8 descriptors of both maps
        bytes_out = 4 + S * 8 + S * 4
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": total_ms / K, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "int8", "data": "synthetic",
            "config": config_dict(w),
            "pairs_per_s": pairs_per_s,
            "matches_per_pair": matches,
            "frontier_per_round": frontier,
            "roofline": {
                "bound": "tensor",
                "kernel": "reciprocal_kernel<int8> (persistent: seeds, tcgen05 kind::i8 forward and "
                          "backward passes, per-pair compaction)",
                "achieved": achieved, "peak": int8_peak, "unit": "TFLOP/s",
                "frac": (achieved / int8_peak) if achieved else None,
                "traffic": None,
                "peak_source": f"{src}: bf16_tflops {peaks['bf16_tflops']} x 2 (int8/bf16 nominal)",
                "ops": "2 x useful MACs (d = 24) over all rounds' frontiers",
                "kernel_ms_per_step": nn_ms / K, "kernel_launches": nn_launches,
                "kernel_share_of_step": nn_ms / total_ms if total_ms else None,
            },
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": bytes_in,
                    "d2h_bytes_per_step": bytes_out, "steps": Ke},
            "gpu_launches": launches_per_step * K,
            "clocks": clocks,
        }
        if args.cpu_baseline and world == 1:
            try:
                cm, cdt, cthreads, cseeds = oracle_sample(pair, w, 4)
                line["cpu_baseline"] = {
                    "value": cm / cdt, "unit": UNIT, "cores": cthreads, "kind": "oracle",
                    "sample": f"fast reciprocal matching from the first {cseeds} of the 3,072 "
                              f"grid seeds (4 seed rows) of the same pair, one oracle call, "
                              f"{cdt:.2f} s"}
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
