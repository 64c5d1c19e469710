#!/usr/bin/env python
"""Throughput of reciprocal nearest-neighbour matching (MASt3R) on B200.

Default workload (the headline): one step = one ``fastnn_reciprocal`` call on
one 512x384 image pair with d = 24 int8 descriptors, seeds on an 8-px grid
(3,072 seeds), max_iter = 10 -- every round's forward and backward
nearest-neighbour passes, the reciprocal check and the frontier compaction.
Inputs are synthetic (``synth``: a smooth warp of map 1 with 30% outliers and
+-2 noise). Printed value: reciprocal matches per second (unique pairs kept /
device time of the call), whole job over all ranks.

After the headline, the dense 196,608-pixel mutual set
(``dense_512x384_d24_i8``), the bf16 pair (``pair_512x384_d24_bf16``) and the
16-pair batch (``batch16_512x288_d32_i8``) are measured the same way and
nested in the same JSON line under ``workloads`` (``--also`` changes the
list). Every workload reports the mean and the 10th / 50th / 90th percentile
of the per-step device time, its dominant kernel's roofline and the SM clocks
sampled during its timed region. ``--workload`` makes any other
configuration the main one.

Each rank processes its own independent pair(s) (pair-level data parallelism,
no collective on the data path); rank r > 0 draws its inputs from the
workload's seed + 7919 r. ``--gpus N`` outside a launcher starts the N ranks
itself (torch.distributed.run, rendezvous on 127.0.0.1).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--also NAME,NAME] [--also-steps K2]
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
# Workloads nested in the headline's JSON line by default.
NESTED_DEFAULT = ["dense_512x384_d24_i8", "pair_512x384_d24_bf16", "batch16_512x288_d32_i8"]


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(synth.CONFIGS))
    ap.add_argument("--cpu-baseline", type=int, default=1,
                    help="time the CPU oracle on a bounded sample (rank 0, N=1)")
    ap.add_argument("--also", default=None,
                    help="comma-separated workloads measured after the main one and nested "
                         "in its JSON line (default with the headline workload: the dense, "
                         "bf16 and 16-pair workloads; 'none' for none)")
    ap.add_argument("--also-steps", type=int, default=100)
    ap.add_argument("--stream-steps", type=int, default=None,
                    help="steps of the 64M-row memory-bound kernel suite nested in the line "
                         "(default 10 with the headline workload, else 0)")
    ap.add_argument("--selftest-launcher", action="store_true", help=argparse.SUPPRESS)
    a = ap.parse_args()
    if a.also is None:
        a.also = ",".join(NESTED_DEFAULT) if a.workload == DEFAULT_WORKLOAD else ""
    if a.stream_steps is None:
        a.stream_steps = 10 if a.workload == DEFAULT_WORKLOAD else 0
    return a


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
    "pair_512x384_d24_i8": (9.605e6, "6c88e67c0142acfe"),
    "pair_512x384_pts3_f32": (6.463e6, "6c88e67c0142acfe"),
    # Dense: the two launches of one step (forward 14.23 MB + backward 13.65 MB).
    "dense_512x384_d24_i8": (27.88e6, "6c88e67c0142acfe"),
    # 16 pairs: 151 MB of repacked rows exceed the 126 MB L2, so tiles are re-read.
    "batch16_512x288_d32_i8": (939.2e6, "6c88e67c0142acfe"),
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
# ranks
# ---------------------------------------------------------------------------

def free_port():
    import socket
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def launch_ranks(args):
    """``--gpus N`` with N > 1 outside a launcher: start N ranks of this script
    (one process per GPU, local rendezvous on 127.0.0.1) and return their exit
    status. Under torchrun (RANK set) the ranks already exist: returns None."""
    if args.gpus <= 1 or "RANK" in os.environ:
        return None
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
           f"--nproc-per-node={args.gpus}", "--master-addr", "127.0.0.1",
           f"--master-port={free_port()}", os.path.abspath(__file__)] + sys.argv[1:]
    return subprocess.run(cmd).returncode


class Ranks:
    """Process-group plumbing shared by the measurement and its CPU self-test:
    barrier, and max / sum reductions of host values over ranks."""

    def __init__(self, world, backend, device):
        import datetime
        import torch
        import torch.distributed as dist
        self.torch, self.dist, self.world, self.device = torch, dist, world, device
        if world > 1:
            kw = {"device_id": device} if backend == "nccl" else {}
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120), **kw)

    def barrier(self):
        if self.world > 1:
            self.dist.barrier()
        if self.device is not None and self.device.type == "cuda":
            self.torch.cuda.synchronize(self.device)

    def _reduce(self, values, op):
        t = self.torch.tensor(values, dtype=self.torch.float64, device=self.device)
        if self.world > 1:
            self.dist.all_reduce(t, op=op)
        return t.tolist()

    def max(self, values):
        return self._reduce(values, self.dist.ReduceOp.MAX)

    def sum(self, values):
        return self._reduce(values, self.dist.ReduceOp.SUM)

    def close(self):
        if self.world > 1:
            self.dist.barrier()
            self.dist.destroy_process_group()


def selftest_launcher(rank, world):
    """The rank launch and reductions without a GPU (gloo): each rank reports
    rank + 1 and its rank; rank 0 prints the sum and the maximum."""
    r = Ranks(world, "gloo", None)
    s = r.sum([float(rank + 1)])[0]
    m = r.max([float(rank)])[0]
    if rank == 0:
        print(json.dumps({"selftest": "launcher", "n_gpus": world, "rank_sum": s,
                          "rank_max": m}), flush=True)
    r.close()
    return 0


def percentiles(ms):
    a = sorted(ms)
    pick = lambda q: a[min(len(a) - 1, int(q * len(a)))]  # noqa: E731
    return {"p10": pick(0.10), "p50": pick(0.50), "p90": pick(0.90)}


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------

class Runner:
    """One workload on this rank's GPU: device inputs, outputs and workspace,
    the library call of one step, and its host copies for the end-to-end leg."""

    def __init__(self, name, rank, dev, stream):
        import torch
        import reciprocal_nearest_neighbours_b200 as fnn
        self.torch, self.fnn, self.dev, self.stream = torch, fnn, dev, stream
        w = self.w = load_workload(name, rank)
        p0 = w.pairs[0]
        self.B = w.batch
        H1, W1, d = p0.desc1.shape
        H2, W2, _ = p0.desc2.shape
        self.N1, self.N2, self.d = H1 * W1, H2 * W2, d
        self.i8 = p0.dtype == "i8"
        self.l2 = p0.dtype == "l2"
        code = {"i8": fnn.FASTNN_I8, "bf16": fnn.FASTNN_BF16, "f16": fnn.FASTNN_F16,
                "l2": fnn.FASTNN_F32_L2}[p0.dtype]
        sdt = torch.int32 if self.i8 else torch.float32
        self.masked = masked = "conf1" in w.extra
        self.esize = 1 if self.i8 else 4 if self.l2 else 2
        N1, N2, B = self.N1, self.N2, self.B
        if w.dense:
            h1 = to_pinned(np.ascontiguousarray(p0.desc1.reshape(-1, d)), torch, p0.dtype)
            h2 = to_pinned(np.ascontiguousarray(p0.desc2.reshape(-1, d)), torch, p0.dtype)
            cap = min(N1, N2)
            self.out_pairs = torch.empty((cap, 2), dtype=torch.int32, device=dev)
            self.out_score = torch.empty(cap, dtype=sdt, device=dev)
            self.out_count = torch.empty(1, dtype=torch.int32, device=dev)
            nbytes = fnn.fastnn_workspace_size(fnn.FASTNN_OP_MUTUAL_DENSE, N1, N2, d, code)
            self.hp_pairs = torch.empty((cap, 2), dtype=torch.int32).pin_memory()
            self.hp_score = torch.empty(cap, dtype=sdt).pin_memory()
        else:
            d1n, d2n = w.stacked()
            h1, h2 = to_pinned(d1n, torch, p0.dtype), to_pinned(d2n, torch, p0.dtype)
            S = fnn.seed_count(H1, W1, w.subsample)
            self.out_pairs = torch.empty((B, S, 2), dtype=torch.int32, device=dev)
            self.out_score = torch.empty((B, S), dtype=sdt, device=dev)
            self.out_count = torch.empty(B, dtype=torch.int32, device=dev)
            self.out_iters = torch.empty(B, dtype=torch.int32, device=dev)
            self.out_front = torch.empty((B, w.max_iter), dtype=torch.int32, device=dev)
            op = fnn.FASTNN_OP_RECIPROCAL_MASKED if masked else fnn.FASTNN_OP_RECIPROCAL
            nbytes = fnn.fastnn_workspace_size(op, N1, N2, d, code, B, S)
            self.hp_pairs = torch.empty((B, S, 2), dtype=torch.int32).pin_memory()
            self.hp_score = torch.empty((B, S), dtype=sdt).pin_memory()
        self.hp_count = torch.empty(self.out_count.shape, dtype=torch.int32).pin_memory()
        self.h1, self.h2 = h1, h2
        self.d1, self.d2 = h1.to(dev), h2.to(dev)
        self.ws = torch.empty(nbytes, dtype=torch.uint8, device=dev)
        self.hc1 = self.hc2 = self.c1 = self.c2 = None
        if masked:
            self.hc1 = torch.from_numpy(np.ascontiguousarray(np.stack(w.extra["conf1"]))).pin_memory()
            self.hc2 = torch.from_numpy(np.ascontiguousarray(np.stack(w.extra["conf2"]))).pin_memory()
            self.c1, self.c2 = self.hc1.to(dev), self.hc2.to(dev)
        if w.dense:
            # 2 repack, forward pass, image list (mark/count/scan/emit), pointmaps:
            # chunk boxes of image 1, backward pass, mutual count/scan/emit
            self.launches_per_step = 2 + 1 + 4 + (1 if self.l2 else 0) + 1 + 3
            self.kernels_per_step = 2
        elif masked:
            # 2 x (count, scan, emit) mask compaction, seeds, 1 persistent matching kernel
            self.launches_per_step = 8
            self.kernels_per_step = 1
        else:
            # The persistent matching kernel repacks both maps itself when their
            # rows are whole 8-byte words (int8 d = 8, 16, 24, 32, ...; 16-bit
            # d = 4, 8, ...); otherwise two repack kernels run before it.
            in_kernel = not self.l2 and (d * self.esize) % 8 == 0
            self.launches_per_step = 1 if in_kernel else 3
            self.kernels_per_step = 1

    def buffers(self):
        """The device inputs and outputs of one call."""
        return {k: getattr(self, k, None) for k in
                ("d1", "d2", "c1", "c2", "out_pairs", "out_score", "out_count", "out_iters",
                 "out_front")}

    def second_buffers(self):
        """A second set of device inputs and outputs (the end-to-end pipeline's
        double buffer)."""
        return {k: (v.clone() if v is not None else None) for k, v in self.buffers().items()}

    def call(self, buf=None, stream=None):
        fnn, w = self.fnn, self.w
        b = buf or self.buffers()
        st = stream or self.stream
        if w.dense:
            fnn.fastnn_mutual_dense(b["d1"], b["d2"], out_pairs=b["out_pairs"],
                                    out_score=b["out_score"], out_count=b["out_count"],
                                    workspace=self.ws, stream=st)
        elif self.masked:
            fnn.fastnn_reciprocal_masked(b["d1"], b["d2"], w.subsample, w.max_iter,
                                         conf1=b["c1"], conf2=b["c2"],
                                         threshold=w.extra["threshold"],
                                         out_pairs=b["out_pairs"], out_score=b["out_score"],
                                         out_count=b["out_count"], out_iters=b["out_iters"],
                                         out_frontier=b["out_front"], workspace=self.ws,
                                         stream=st)
        else:
            fnn.fastnn_reciprocal(b["d1"], b["d2"], w.subsample, w.max_iter,
                                  out_pairs=b["out_pairs"], out_score=b["out_score"],
                                  out_count=b["out_count"], out_iters=b["out_iters"],
                                  out_frontier=b["out_front"], workspace=self.ws, stream=st)

    def copy_in(self, b):
        b["d1"].copy_(self.h1, non_blocking=True)
        b["d2"].copy_(self.h2, non_blocking=True)
        if self.masked:
            b["c1"].copy_(self.hc1, non_blocking=True)
            b["c2"].copy_(self.hc2, non_blocking=True)

    def copy_out(self, b):
        self.hp_count.copy_(b["out_count"], non_blocking=True)
        self.hp_pairs.copy_(b["out_pairs"], non_blocking=True)
        self.hp_score.copy_(b["out_score"], non_blocking=True)

    def bytes_per_step(self):
        bin_ = (self.N1 + self.N2) * self.d * self.esize * self.B + \
            ((self.N1 + self.N2) * 4 * self.B if self.masked else 0)
        bout = int(self.hp_count.numel() * 4 + self.hp_pairs.numel() * 4 +
                   self.hp_score.numel() * 4)
        return bin_, bout

    def matches(self):
        return int(self.out_count.cpu().sum())

    def work_per_step(self):
        """(score elements per step, row count of the dense backward pass or None)."""
        if self.w.dense:
            # The backward pass runs on the image of NN12 only (the rows that
            # can be in a mutual pair): count them for the useful-work figure.
            idx12, _ = self.fnn.fastnn_nn(self.d1, self.d2)
            image = int(self.torch.unique(idx12[(idx12 >= 0) & (idx12 < self.N2)]).numel())
            return self.N1 * self.N2 + image * self.N1, image
        return int(self.out_front.cpu().sum()) * (self.N1 + self.N2), None


def time_steps(run, K, flush, ranks):
    """K steps, L2 flushed before each; CUDA events on the launching stream
    around each step. Returns per-step ms (max over ranks) and this rank's
    (timed kernel launches, kernel ms)."""
    torch, fnn = run.torch, run.fnn
    fnn.fastnn_kernel_timer_enable(K * run.kernels_per_step + 8)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(K)]
    ranks.barrier()
    for i in range(K):
        flush.zero_()
        evs[i][0].record(run.stream)
        run.call()
        evs[i][1].record(run.stream)
    ranks.barrier()
    ms = [s.elapsed_time(e) for s, e in evs]
    nn = fnn.fastnn_kernel_timer_read()
    fnn.fastnn_kernel_timer_enable(0)
    return ranks.max(ms), nn


def time_end_to_end(run, K, ranks):
    """K steps through the public API with host buffers, as a stream of pairs
    is matched: every step copies its inputs in from pinned host memory, runs
    the call and copies every output back. Two device buffer sets and two copy
    streams (inputs, outputs) let step i + 1's inputs and step i - 1's outputs
    cross the bus while step i runs; the events bracket the first copy in and
    the last copy out. Returns the total ms (max over ranks)."""
    torch = run.torch
    bufs = [run.buffers(), run.second_buffers()]
    cin, cout = torch.cuda.Stream(device=run.dev), torch.cuda.Stream(device=run.dev)
    ev = lambda: torch.cuda.Event()  # noqa: E731
    done = [ev(), ev()]      # compute of the last step on buffer set s finished
    copied = [ev(), ev()]    # outputs of the last step on set s copied out
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for s in range(2):
        done[s].record(run.stream)
        copied[s].record(cout)
    ranks.barrier()
    start.record(cin)
    for i in range(K):
        s = i & 1
        b = bufs[s]
        inp = ev()
        with torch.cuda.stream(cin):
            cin.wait_event(done[s])  # step i - 2 no longer reads set s
            run.copy_in(b)
            inp.record(cin)
        run.stream.wait_event(inp)
        run.stream.wait_event(copied[s])  # step i - 2's outputs are out of set s
        run.call(b)
        done[s].record(run.stream)
        with torch.cuda.stream(cout):
            cout.wait_event(done[s])
            run.copy_out(b)
            copied[s].record(cout)
    cout.wait_stream(cin)
    end.record(cout)
    ranks.barrier()
    end.synchronize()
    return ranks.max([start.elapsed_time(end)])[0]


def roofline_for(run, work, image, K, nn_launches, nn_ms, total_ms):
    d, w, l2 = run.d, run.w, run.l2
    peaks, src = measured_peaks()
    bf16_peak = float(peaks["bf16_tflops"])
    if l2:
        # Pointmaps: 3 fused multiply-adds per (query, point) pair on the FP32
        # pipe; peak = 148 SMs x 128 FMA lanes x 2 flop x 1.965 GHz.
        peak = FP32_FMA_TFLOPS
        achieved = 6.0 * work * K / (nn_ms / 1e3) / 1e12 if nn_ms > 0 else None
        kname = ("nn_l2_kernel (FP32 FMA nearest point: forward pass over every image-1 "
                 "point, backward pass over the image of the forward matches)" if w.dense else
                 "reciprocal_l2_kernel (persistent: seeds, FP32 FMA forward and backward "
                 "passes, per-pair compaction)")
        peak_source = ("derived: FP32 FMA pipe, 148 SMs x 128 lanes x 2 flop x 1.965 GHz "
                       "(clocks.max.sm)")
        ops = f"3 FMA = 6 flop per (query, point) pair: {work:.4g} pairs per step"
    else:
        peak = 2.0 * bf16_peak if run.i8 else bf16_peak  # dense int8 = 2 x bf16 (nominal ratio)
        achieved = 2.0 * work * d * K / (nn_ms / 1e3) / 1e12 if nn_ms > 0 else None
        kname = ("nn_tc_kernel (tcgen05 argmax-GEMM: forward pass over every image-1 row, "
                 "backward pass over the image of the forward matches)" if w.dense else
                 "reciprocal_kernel (persistent: seeds, tcgen05 forward and backward passes, "
                 "per-pair compaction)")
        peak_source = (f"{src}: bf16_tflops {bf16_peak}" +
                       (" x 2 (int8 = 2 x bf16, nominal ratio)" if run.i8 else ""))
        ops = f"2 x useful MACs (d = {d}) per step: {work * d:.4g} MAC"
    if image is not None:
        ops += f" ({run.N1} x {run.N2} forward + {image} x {run.N1} backward)"
    return {
        "bound": "alu" if l2 else "tensor", "kernel": kname,
        "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
        "frac": (achieved / peak) if achieved else None,
        "traffic": traffic_for(w.name),
        "traffic_unit": ("bytes per step: forward + backward launch (ncu dram read + write)"
                         if w.dense else "bytes per launch (ncu dram read + write)"),
        "peak_source": peak_source, "ops": ops,
        "kernel_ms_per_step": nn_ms / K, "kernel_launches": nn_launches,
        "kernel_share_of_step": nn_ms / total_ms if total_ms else None,
    }


def measure(name, K, W, rank, ranks, dev, stream, flush, sample_clocks, e2e_steps=0):
    """Warm up, time K steps (and optionally an end-to-end leg) of one workload.
    Returns this workload's result dict (meaningful on rank 0)."""
    import torch
    run = Runner(name, rank, dev, stream)
    fnn = run.fnn
    for _ in range(max(W, 3)):
        flush.zero_()
        run.call()
    torch.cuda.synchronize(dev)
    assert fnn.fastnn_device_status(run.ws) == 0
    matches = run.matches()
    work, image = run.work_per_step()
    sampler = None
    if sample_clocks:
        uuid = None
        try:
            uuid = str(torch.cuda.get_device_properties(dev).uuid)
        except Exception:  # noqa: BLE001
            pass
        sampler = ClockSampler(uuid)
        time.sleep(0.5)
    step_ms, (nn_launches, nn_ms) = time_steps(run, K, flush, ranks)
    clocks = sampler.stop() if sampler else None
    assert fnn.fastnn_device_status(run.ws) == 0
    assert run.matches() == matches
    e2e_ms = None
    if e2e_steps:
        e2e_ms = time_end_to_end(run, e2e_steps, ranks)
        assert int(run.hp_count.sum()) == matches
    total_ms = sum(step_ms)
    nn_ms = ranks.max([nn_ms])[0]
    all_matches = ranks.sum([float(matches)])[0]
    world = ranks.world
    res = {
        "metric": metric_for(name, run.w.dense), "value": all_matches * K / (total_ms / 1e3),
        "unit": UNIT, "n_gpus": world, "steps": K, "warmup": W, "ms_per_step": total_ms / K,
        "ms_per_step_percentiles": percentiles(step_ms),
        "dtype": {"i8": "int8", "bf16": "bf16", "f16": "f16", "l2": "f32"}[run.w.pairs[0].dtype],
        "config": config_dict(run.w),
        "pairs_per_s": world * run.B * K / (total_ms / 1e3),
        "matches_per_step_rank0": matches,
        "roofline": roofline_for(run, work, image, K, nn_launches, nn_ms, total_ms),
        "gpu_launches": run.launches_per_step * K,
        "clocks": clocks,
    }
    if not run.w.dense:
        res["frontier_per_round_pair0"] = run.out_front[0].cpu().tolist()
    if e2e_ms is not None:
        bin_, bout = run.bytes_per_step()
        res["e2e"] = {"value": all_matches * e2e_steps / (e2e_ms / 1e3), "unit": UNIT,
                      "h2d_bytes_per_step": bin_, "d2h_bytes_per_step": bout,
                      "steps": e2e_steps, "ms_per_step": e2e_ms / e2e_steps,
                      "pipeline": "step i+1's inputs and step i-1's outputs are copied on two "
                                  "copy streams while step i runs (two device buffer sets)"}
    res["_workload"] = run.w
    return res


# ---------------------------------------------------------------------------
# the memory-bound kernels at a scale where HBM bandwidth bounds them
# ---------------------------------------------------------------------------

STREAM_ROWS = 64 << 20  # 67,108,864 rows: inputs far larger than L2


def measure_stream(K, ranks, dev, stream, flush, sample_clocks):
    """Achieved HBM bandwidth of the repack, dense mutual test/emit, image-row
    list and confidence-mask compaction kernels on a 64M-row int8 map (d = 24; a few
    GB on the device). Each kind is timed with the library's launch timer
    restricted to that kind, inside an ordinary call:
      repack  -- fastnn_nn of the 64M-row map against a 256-row database
                 (its query map's repack: N x 24 B read, N x 32 B written);
      mutual  -- fastnn_mutual_from_nn on 64M-row index arrays of a smooth
                 synthetic correspondence (test and ordered emit in one pass:
                 NN12 and the partner's NN21 read, 2 x 4 B per row; per kept
                 pair its score read and the pair and score written, 16 B);
      image   -- fastnn_image_rows of the same 64M-row NN12 (the list the
                 sharded dense backward pass runs on: 4 B read per row,
                 4 B written per listed image-2 row);
      mask    -- fastnn_mutual_dense_masked of the 64M-row map (confidences
                 uniform in [0, 1), threshold 0.5) against a 256-row map
                 without confidences (map 1's compaction: 4 B of confidence
                 and the 24 B row read per pixel, 32 B repacked row + 4 B
                 pixel index written per kept pixel; map 2's: every pixel's
                 row read and written the same way).
    Inputs are drawn on the device from a seeded generator."""
    import torch
    import reciprocal_nearest_neighbours_b200 as fnn
    N, d = STREAM_ROWS, 24
    g = torch.Generator(device=dev)
    g.manual_seed(synth.BASE_SEED + 60 + 7919 * ranks_rank(ranks))
    peaks, src = measured_peaks()
    hbm = float(peaks["hbm_gbs"])
    out = {"workload": f"stream_{N >> 20}M_d{d}_i8", "rows": N, "steps": K,
           "peak": hbm, "peak_source": f"{src}: hbm_gbs", "kernels": []}

    def timed(kind, call, nbytes_fn):
        for _ in range(3):
            call()
        torch.cuda.synchronize(dev)
        prev = fnn.fastnn_kernel_timer_select(kind)
        fnn.fastnn_kernel_timer_enable(4 * K + 8)
        sampler = ClockSampler(None) if sample_clocks else None
        ranks.barrier()
        for _ in range(K):
            flush.zero_()
            call()
        ranks.barrier()
        clocks = sampler.stop() if sampler else None
        n, ms = fnn.fastnn_kernel_timer_read()
        fnn.fastnn_kernel_timer_enable(0)
        fnn.fastnn_kernel_timer_select(prev)
        ms = ranks.max([ms])[0]
        nbytes = nbytes_fn()
        gbs = nbytes * K / (ms / 1e3) / 1e9
        return {"launch_brackets": n, "ms_per_step": ms / K, "bytes_per_step": nbytes,
                "achieved_gbs": gbs, "frac": gbs / hbm, "clocks": clocks}

    A = torch.randint(-16, 17, (N, d), dtype=torch.int8, device=dev, generator=g)
    db = torch.randint(-16, 17, (256, d), dtype=torch.int8, device=dev, generator=g)
    ws = torch.empty(fnn.fastnn_workspace_size(fnn.FASTNN_OP_NN, N, 256, d, fnn.FASTNN_I8),
                     dtype=torch.uint8, device=dev)
    idx = torch.empty(N, dtype=torch.int32, device=dev)
    r = timed(fnn.FASTNN_TIME_REPACK, lambda: fnn.fastnn_nn(A, db, out_idx=idx, workspace=ws),
              lambda: N * d + N * 32 + 256 * d + 512 * 32)
    r["kind"] = "repack (repack_staged_kernel: 64M x 24 B rows into 32 B rows)"
    out["kernels"].append(r)
    del ws, idx

    # A smooth correspondence: row i's partner is i + a small signed offset,
    # and a partner points back to i for about 70% of rows.
    off = torch.randint(-3, 4, (N,), dtype=torch.int32, device=dev, generator=g)
    ar = torch.arange(N, dtype=torch.int32, device=dev)
    nn12 = (ar + off).clamp_(0, N - 1)
    nn21 = ar.clone()
    nn21[nn12] = ar
    miss = torch.rand(N, device=dev, generator=g) < 0.3
    nn21[miss] = (nn21[miss] + 1).clamp_(max=N - 1)
    score = torch.randint(0, 1000, (N,), dtype=torch.int32, device=dev, generator=g)
    mws = torch.empty(fnn.fastnn_workspace_size(fnn.FASTNN_OP_MUTUAL_FROM_NN, N, N, 1,
                                                fnn.FASTNN_I8), dtype=torch.uint8, device=dev)
    pairs = torch.empty((N, 2), dtype=torch.int32, device=dev)
    pscore = torch.empty(N, dtype=torch.int32, device=dev)
    cnt = torch.empty(1, dtype=torch.int32, device=dev)
    r = timed(fnn.FASTNN_TIME_MUTUAL,
              lambda: fnn.fastnn_mutual_from_nn(nn12, score, 0, nn21, N, out_pairs=pairs,
                                                out_score=pscore, out_count=cnt, workspace=mws),
              lambda: 8 * N + 16 * int(cnt.item()))
    r["kind"] = "mutual test and ordered emit in one pass (mutual_select)"
    r["kept"] = int(cnt.item())
    out["kernels"].append(r)
    del nn21, miss, score, pairs, pscore
    rows = torch.empty(N, dtype=torch.int32, device=dev)
    iws = torch.empty(fnn.fastnn_workspace_size(fnn.FASTNN_OP_IMAGE_ROWS, N, N, 1, fnn.FASTNN_I8),
                      dtype=torch.uint8, device=dev)
    r = timed(fnn.FASTNN_TIME_MUTUAL,
              lambda: fnn.fastnn_image_rows(nn12, N, out_rows=rows, out_count=cnt, workspace=iws),
              lambda: 4 * N + 4 * int(cnt.item()))
    r["kind"] = ("image-2 rows of an NN12 (image_flag, image_rows_count, scan, "
                 "image_rows_emit: 4 B read per image-1 row, 4 B written per listed row)")
    r["listed"] = int(cnt.item())
    out["kernels"].append(r)
    del off, ar, nn12, mws, iws, rows

    conf = torch.rand(N, device=dev, generator=g)
    kept1 = int((conf >= 0.5).sum().item())
    wsm = torch.empty(fnn.fastnn_workspace_size(fnn.FASTNN_OP_MUTUAL_DENSE_MASKED, N, 256, d,
                                                fnn.FASTNN_I8), dtype=torch.uint8, device=dev)
    mp = torch.empty((256, 2), dtype=torch.int32, device=dev)
    ms_ = torch.empty(256, dtype=torch.int32, device=dev)
    r = timed(fnn.FASTNN_TIME_MASK,
              lambda: fnn.fastnn_mutual_dense_masked(A, db, conf1=conf, threshold=0.5,
                                                     out_pairs=mp, out_score=ms_, out_count=cnt,
                                                     workspace=wsm),
              lambda: 4 * N + N * d + kept1 * 36 + 256 * (d + 36))
    r["kind"] = ("confidence-mask compaction (mask_count, scan, mask_emit) of the 64M-row map "
                 "and of the 256-row map")
    r["kept"] = kept1
    out["kernels"].append(r)
    return out


def ranks_rank(ranks):
    return ranks.dist.get_rank() if ranks.world > 1 else 0


def run_ours(args, rank, world, local):
    import torch

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    ranks = Ranks(world, "nccl", dev)
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    head = measure(args.workload, args.steps, args.warmup, rank, ranks, dev, stream, flush,
                   sample_clocks=rank == 0, e2e_steps=max(1, min(args.steps, 1000)))
    also = [x for x in (args.also.split(",") if args.also and args.also != "none" else [])
            if x and x != args.workload]
    nested = []
    for name in also:
        r = measure(name, args.also_steps, args.warmup, rank, ranks, dev, stream, flush,
                    sample_clocks=rank == 0)
        r.pop("_workload")
        nested.append({k: r[k] for k in ("metric", "value", "unit", "steps", "ms_per_step",
                                         "ms_per_step_percentiles", "dtype", "config",
                                         "pairs_per_s", "roofline", "clocks", "gpu_launches")})
    streams = None
    if args.stream_steps > 0:
        streams = measure_stream(args.stream_steps, ranks, dev, stream, flush,
                                 sample_clocks=rank == 0)
    if rank == 0:
        w = head.pop("_workload")
        line = {
            "metric": head["metric"], "value": head["value"], "unit": UNIT, "n_gpus": world,
            "steps": head["steps"], "warmup": args.warmup, "ms_per_step": head["ms_per_step"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": head["dtype"], "data": "synthetic", "config": head["config"],
        }
        line.update({k: v for k, v in head.items() if k not in line})
        line["gpu_launches"] = head["gpu_launches"] + sum(n["gpu_launches"] for n in nested)
        line["gpu_launches_headline"] = head["gpu_launches"]
        if nested:
            line["workloads"] = nested
        if streams:
            line["stream_kernels"] = streams
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
    ranks.close()
    return 0


def main():
    args = parse_args()
    rc = launch_ranks(args)
    if rc is not None:
        return rc
    rank, world, local = dist_env()
    if args.selftest_launcher:
        return selftest_launcher(rank, world)
    if args.impl == "reference":
        return run_reference(args, rank, world)
    return run_ours(args, rank, world, local)


if __name__ == "__main__":
    sys.exit(main())
