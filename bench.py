#!/usr/bin/env python
"""Benchmark of the N:M sparse path on B200: useful TFLOP/s and roofline fraction.

One step is one pass of the whole hot path over the LLaMA-7B-shaped 2:4
workload with the learned-permutation stand-in: for each of the three linear
shapes (4096x4096, 11008x4096, 4096x11008; T = 2048 tokens) the weights are
magnitude-pruned and compressed to 2:4 (nm_prune_compress), then
Y = (W' Pi) X runs with Pi applied as an index map on the input read
(nm_spmm_permuted).  `value` is useful (non-zero) GEMM FLOPs per second of the
whole step, inputs resident in HBM.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Under torchrun (N > 1) every rank runs its own replica of the workload (the
path has no exchange step); timing is the max over ranks.  `--impl reference`
times the fp64 CPU oracle on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import dataclasses
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as wl  # noqa: E402

METRIC = "N:M sparse GEMM useful TFLOP/s & % of sparse-TC/HBM roofline (1×B200)"
WORKLOAD = "llama7b"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--cpu-seconds", type=float, default=10.0, help="target length of the oracle baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the pass over the other configurations (decode, ViT, PATCH, RL-MLP, tiny)")
    ap.add_argument("--workload", default=WORKLOAD, choices=wl.ALL_WORKLOADS,
                    help="llama7b (default, the headline), decode, vit, patch_p25/p50/p75, tiny, rl_mlp_*")
    ap.add_argument("--layers", default=None, help="comma-separated subset of the workload's layers")
    ap.add_argument("--algo", choices=["auto", "sparse", "dense"], default="auto",
                    help="kernel design for 1:4 / 1:8 (nm_spmm_algo)")
    ap.add_argument("--plain", action="store_true", help="ignore the workload's index map (y = W x)")
    ap.add_argument("--pattern", default=None,
                    help="N:M to use instead of the workload's own pattern (e.g. --workload decode --pattern 1:8)")
    ap.add_argument("--diag", action="store_true",
                    help="diagonal pattern at 90 %% sparsity (D = K/10 kept diagonals) on the workload's shapes: "
                         "nm_diag_prune_compress, then nm_diag_spmm with the index map, per layer")
    ap.add_argument("--dtype", choices=["bf16", "i8", "tf32"], default="bf16",
                    help="i8: INT8 2:4 weights and int8 inputs on the workload's shapes (nm_prune_compress_i8, then "
                         "nm_spmm_i8; no index map), useful TOP/s against the int8 dense peak; tf32: 1:2 float32 "
                         "weights and float32 inputs (nm_prune_compress_tf32, then nm_spmm_tf32 with fp32 output), "
                         "useful TFLOP/s against the tf32 dense peak")
    ap.add_argument("--step", choices=["one-call", "two-calls"], default="one-call",
                    help="one-call: nm_prune_spmm per layer (prune + compress + GEMM in one library call, the "
                         "compressed form written too); two-calls: nm_prune_compress, then the GEMM call.  The "
                         "hybrid workloads and --algo other than auto always use two calls")
    ap.add_argument("--quick", action="store_true",
                    help="timed region only: no clock sampling, end-to-end pass, oracle baseline or extras")
    return ap.parse_args(argv)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ----------------------------------------------------------------------------
# Clock sampling during the timed region
# ----------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid: str, period_ms: int = 100):
        self.uuid = uuid
        self.period_ms = period_ms
        self.rows = []
        self.proc = None
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 f"-lms", str(self.period_ms)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()
        time.sleep(0.3)

    def _read(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 9:
                self.rows.append(parts)

    def stop(self):
        if self.proc is None:
            return
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=5)

    def summary(self):
        mine = [r for r in self.rows if self.uuid and self.uuid in r[0]] or self.rows
        if not mine:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = [num(r[1]) for r in mine if num(r[1]) is not None]
        mx = [num(r[2]) for r in mine if num(r[2]) is not None]
        load = [s for s in sm if s > 0] or sm
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in mine:
            for name, v in zip(names, r[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(load) if load else None,
                "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(mine)}


# ----------------------------------------------------------------------------
# Oracle baseline (CPU): the oracle as it stands, its rows spread over threads
# ----------------------------------------------------------------------------
def host_threads() -> int:
    """Host cores this process may run on."""
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def oracle_sample(d, r0: int, r1: int, cols: int):
    """Oracle compress of weight rows r0..r1-1 and their permuted GEMM over the first `cols` tokens."""
    import oracle
    L = d.layer
    Xs = np.ascontiguousarray(d.X[:, :cols])
    vals, meta = oracle.compress(np.ascontiguousarray(d.W[r0:r1]), 2, 4)
    oracle.spmm(vals, meta, 2, 4, L.K, Xs, d.idx)
    return 2.0 * (r1 - r0) * cols * (L.K // 2)


def oracle_parallel(d, rows: int, cols: int, threads: int):
    """Rows 0..rows-1 split into `threads` contiguous blocks, one oracle call pair per thread (the
    oracle's C functions run without the GIL).  Returns (useful FLOPs, seconds)."""
    from concurrent.futures import ThreadPoolExecutor
    bounds = np.linspace(0, rows, threads + 1).astype(int)
    blocks = [(int(a), int(b)) for a, b in zip(bounds[:-1], bounds[1:]) if b > a]
    t0 = time.perf_counter()
    with ThreadPoolExecutor(max_workers=len(blocks)) as ex:
        flops = sum(ex.map(lambda ab: oracle_sample(d, ab[0], ab[1], cols), blocks))
    return flops, time.perf_counter() - t0


def cpu_baseline(data, target_s: float):
    """The oracle on all of this host's cores, on a sample of the first layer sized for ~target_s seconds."""
    d = data[0]
    L = d.layer
    threads = host_threads()
    f0, t0 = oracle_parallel(d, 16, 16, 1)
    rate = f0 / max(t0, 1e-9)                      # one thread
    want = target_s * rate * threads               # FLOPs for about target_s seconds on every core
    cols = int(min(L.T, 512))
    rows = int(min(L.R, max(threads, want / (2.0 * cols * (L.K // 2)))))
    if rows == L.R:
        cols = int(min(L.T, max(cols, want / (2.0 * rows * (L.K // 2)))))
    flops, dt = oracle_parallel(d, rows, cols, threads)
    return {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
            "cpu_model": cpu_model(),
            "sample": f"{L.name}: oracle compress of {rows} weight rows + permuted spmm of those rows over "
                      f"{cols} of {L.T} tokens ({flops / 1e9:.2f} useful GFLOP, {dt:.1f} s wall, rows split "
                      f"over {threads} threads)"}


# ----------------------------------------------------------------------------
# Multi-rank plumbing (one process per GPU; replicas, no data-path collective)
# ----------------------------------------------------------------------------
def rank_barrier(dist) -> None:
    if dist is not None:
        dist.barrier()


def max_over_ranks_on(ms: float, dist, device) -> float:
    """The slowest rank's time: all-reduce MAX of one float64 (NCCL on the GPU, gloo on the CPU)."""
    if dist is None:
        return ms
    import torch
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def layer_mode(L, step_mode: str, algo: str, permuted: bool) -> str:
    """How a layer of the step runs (mirrors the library's dispatch for nm_prune_spmm), and what the
    kernel-timing pass brackets: "fused" the whole call (prune_spmm_skinny_kernel + reduction);
    "combined" the pair GEMM on the gathered input, the launch the call makes after its compress-and-gather
    grid; "split" the GEMM call after a separate compress."""
    one_call = step_mode == "one-call" and L.tile_p is None and algo == "auto"
    if one_call and L.n == 2 and L.m == 4 and L.K % 128 == 0:
        if 1 <= L.T <= 64:
            return "fused"
        if permuted and L.T >= 192 and L.T % 8 == 0:
            return "combined"
    return "split"


def reencoded_bound_s(bufs, tc_peak: float, hbm_peak: float) -> float:
    """Lower bound (seconds) on the GEMM launches of a 1:8 step run as re-encoded 2:4.

    Each group of eight weights becomes two 2:4 groups, so the sparse tensor cores multiply four stored
    values (one survivor, three zeros) where the pattern keeps one: 4x the useful products.  Stored
    2:4 values are multiplied at the dense product rate (the sparse MMA's 2x is over the logical K it
    covers), so the tensor term is the executed products over the dense peak.  The other term is the
    algorithmic bytes at the HBM rate."""
    executed = sum(4.0 * b["flops"] for b in bufs)
    return max(executed / (tc_peak * 1e12), sum(b["gemm_bytes"] for b in bufs) / (hbm_peak * 1e9))


def step_config(workload: str, layers, step_mode: str, algo: str, plain: bool, world: int) -> dict:
    """The `config` object of a bench line (the same for both arms)."""
    permuted = [L.permuted and not plain for L in layers]
    one_call = step_mode == "one-call" and all(L.tile_p is None for L in layers) and algo == "auto"
    ws = sum(2 * L.R * L.K + 2 * L.K * L.T + 2 * L.R * L.T for L in layers)
    return {"workload": workload, "shapes": [[L.R, L.K] for L in layers], "T": [L.T for L in layers],
            "pattern": [f"{L.n}:{L.m}" if L.tile_p is None else f"dense/2:4 tiles p={L.tile_p}" for L in layers],
            "permuted": any(permuted), "algo": algo,
            "step": ("one nm_prune_spmm call per layer: prune + compress (the compressed form written) + the sparse "
                     "GEMM" if one_call else "nm_prune_compress, then the sparse GEMM call, for every layer"),
            "layer_paths": {L.name: layer_mode(L, step_mode, algo, p) for L, p in zip(layers, permuted)},
            "kernel_timing": ("CUDA events in a second pass of K steps: per layer the compress and the GEMM launch "
                              "(\"combined\": the pair GEMM on the gathered input, the launch nm_prune_spmm makes "
                              "after its compress-and-gather grid; \"fused\": the whole call)"),
            "l2": ("inputs larger than L2 (126 MB) per step" if ws > 126e6
                   else "working set below L2 size (small config)"),
            "parallelism": f"replicas x{world}"}


def run_reference(args, rank: int, world: int):
    """The oracle on the host's cores: each step a bounded sample of the workload's first layer."""
    if rank != 0:
        return
    layers = wl.workload(args.workload)
    if args.layers:
        layers = [layers[int(i)] for i in args.layers.split(",")]
    d = wl.make_layer(layers[0])
    threads = host_threads()
    rows, cols = int(min(d.layer.R, 8 * threads)), 64  # bounded sample per step
    for _ in range(args.warmup):
        oracle_parallel(d, rows, cols, threads)
    t = 0.0
    flops = 0.0
    for _ in range(args.steps):
        f, dt = oracle_parallel(d, rows, cols, threads)
        t += dt
        flops += f
    value = flops / t / 1e12
    cfg = step_config(args.workload, layers, args.step, args.algo, args.plain, world)
    sample = (f"per step {rows} weight rows x {cols} tokens of {d.layer.name}: oracle compress + permuted spmm, "
              f"rows split over {threads} threads")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * t / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded numpy PCG64 draws rounded to bf16; shapes and distributions of the workload)",
            "config": cfg,
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                             "cpu_model": cpu_model(), "sample": sample},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------
# Our CUDA path
# ----------------------------------------------------------------------------
def gemm_bytes(L, d) -> float:
    """Algorithmic HBM bytes of one GEMM launch: values + metadata + X + Y (+ index map, + dense tiles)."""
    b = 2.0 * L.R * (L.K // L.m * L.n) + 4.0 * L.R * -(-(L.K // L.m * L.n) // (32 // {2: 1, 4: 2, 8: 3, 16: 4}[L.m]))
    b += 2.0 * L.K * L.T + 2.0 * L.R * L.T
    if d.idx is not None:
        b += 4.0 * L.K
    if d.tmap is not None:  # dense tiles are read from W instead of the compressed form
        dense = float((d.tmap == 0).sum()) * L.tile * L.tile
        b += 2.0 * dense - 1.125 * dense + d.tmap.size
    return b


class Runner:
    """Device buffers and library calls (through the C ABI) of one workload's step."""

    def __init__(self, workload, dev, stream, nm, algo="auto", layers=None, plain=False, step_mode="one-call",
                 pattern=None):
        import torch
        self.torch, self.nm, self.L_ = torch, nm, nm.lib()
        self.dev, self.stream, self.sp = dev, stream, stream.cuda_stream
        self.algo_name = algo
        self.algo = {"auto": nm.NM_ALGO_AUTO, "sparse": nm.NM_ALGO_SPARSE_TC, "dense": nm.NM_ALGO_DENSE_TC}[algo]
        lay = wl.workload(workload)
        if layers:
            lay = [lay[int(i)] for i in layers.split(",")]
        if pattern:
            n, m = (int(x) for x in pattern.split(":"))
            lay = [dataclasses.replace(L, n=n, m=m) for L in lay]
        self.layers = lay
        self.data = [wl.make_layer(L) for L in lay]
        self.one_call = step_mode == "one-call" and all(d.tmap is None for d in self.data) and algo == "auto"
        self.bufs = []
        for d in self.data:
            L = d.layer
            b = {"L": L, "d": d, "W": self.up(d.W), "X": self.up(d.X),
                 "idx": torch.from_numpy(d.idx).to(dev) if d.idx is not None and not plain else None,
                 "tmap": torch.from_numpy(d.tmap).to(dev) if d.tmap is not None else None,
                 "vals": torch.empty((L.R, max(nm.nm_value_cols(L.K, L.n, L.m), 0)), dtype=torch.bfloat16,
                                     device=dev),
                 "meta": torch.empty((max(nm.nm_meta_words(L.R, L.K, L.n, L.m), 0),), dtype=torch.int32, device=dev),
                 "Y": torch.empty((L.R, L.T), dtype=torch.bfloat16, device=dev)}
            b["flops"] = float(wl.hybrid_useful_flops(d) if d.tmap is not None else L.useful_flops)
            b["comp_bytes"] = 2.0 * L.R * L.K + 2.0 * b["vals"].numel() + 4.0 * b["meta"].numel()
            b["mode"] = layer_mode(L, step_mode, algo, b["idx"] is not None)
            if b["mode"] == "combined":
                b["Xp"] = b["X"][b["idx"].long()].contiguous()  # input of the timed GEMM launch (setup only)
            if b["mode"] == "fused":  # W read once, compressed form written, X read, Y written
                b["gemm_bytes"] = b["comp_bytes"] + 2.0 * L.K * L.T + 2.0 * L.R * L.T
            elif b["mode"] == "combined":  # the GEMM reads the gathered input: no index map
                b["gemm_bytes"] = gemm_bytes(L, d) - 4.0 * L.K
            else:
                b["gemm_bytes"] = gemm_bytes(L, d)
            self.bufs.append(b)
        torch.cuda.synchronize()
        self.useful = sum(b["flops"] for b in self.bufs)

    def up(self, bits):
        return self.torch.from_numpy(bits.view(np.int16)).to(self.dev).view(self.torch.bfloat16)

    def check(self, st, what):
        if st != 0:
            raise RuntimeError(f"{what}: {self.L_.nm_last_error().decode()}")

    def launch_compress(self, b):
        L = b["L"]
        self.check(self.L_.nm_prune_compress(b["W"].data_ptr(), L.R, L.K, L.K, L.n, L.m, b["vals"].data_ptr(),
                                             b["meta"].data_ptr(), self.sp), "nm_prune_compress")

    def launch_gemm(self, b, permuted=True):
        L, L_, sp = b["L"], self.L_, self.sp
        if b["tmap"] is not None:
            self.check(L_.nm_hybrid_spmm(b["W"].data_ptr(), L.K, b["vals"].data_ptr(), b["meta"].data_ptr(),
                                         b["tmap"].data_ptr(), L.tile, L.R, L.K, b["X"].data_ptr(), L.T, L.T,
                                         b["Y"].data_ptr(), L.T, 0, sp), "nm_hybrid_spmm")
        elif b["idx"] is not None and permuted:
            self.check(L_.nm_spmm_permuted(b["vals"].data_ptr(), b["meta"].data_ptr(), L.n, L.m, L.R, L.K,
                                           b["idx"].data_ptr(), b["X"].data_ptr(), L.T, L.T, b["Y"].data_ptr(), L.T,
                                           0, sp), "nm_spmm_permuted")
        elif self.algo != self.nm.NM_ALGO_AUTO:
            self.check(L_.nm_spmm_algo(b["vals"].data_ptr(), b["meta"].data_ptr(), L.n, L.m, L.R, L.K, None,
                                       b["X"].data_ptr(), L.T, L.T, b["Y"].data_ptr(), L.T, 0, self.algo, sp),
                       "nm_spmm_algo")
        else:
            self.check(L_.nm_spmm(b["vals"].data_ptr(), b["meta"].data_ptr(), L.n, L.m, L.R, L.K, b["X"].data_ptr(),
                                  L.T, L.T, b["Y"].data_ptr(), L.T, 0, sp), "nm_spmm")

    def launch_fused(self, b, permuted=True):
        L = b["L"]
        idx = b["idx"].data_ptr() if b["idx"] is not None and permuted else None
        self.check(self.L_.nm_prune_spmm(b["W"].data_ptr(), L.K, L.n, L.m, L.R, L.K, idx, b["X"].data_ptr(), L.T,
                                         L.T, b["Y"].data_ptr(), L.T, 0, b["vals"].data_ptr(), b["meta"].data_ptr(),
                                         self.sp), "nm_prune_spmm")

    def launch_gemm_xp(self, b):
        L = b["L"]
        self.check(self.L_.nm_spmm(b["vals"].data_ptr(), b["meta"].data_ptr(), 2, 4, L.R, L.K, b["Xp"].data_ptr(),
                                   L.T, L.T, b["Y"].data_ptr(), L.T, 0, self.sp), "nm_spmm")

    def launch_layer(self, b):  # one layer of the timed step
        if self.one_call:
            self.launch_fused(b)
        else:
            self.launch_compress(b)
            self.launch_gemm(b)

    def step(self, evs=None):
        """The step; with events, the kernel-timing form of it (see layer_mode)."""
        for i, b in enumerate(self.bufs):
            if evs is None:
                self.launch_layer(b)
                continue
            evs[2 * i].record(self.stream)
            if b["mode"] == "fused":  # the whole call; the compress slot stays empty
                evs[2 * i + 1].record(self.stream)
                self.launch_fused(b)
                continue
            self.launch_compress(b)
            evs[2 * i + 1].record(self.stream)
            if b["mode"] == "combined":
                self.launch_gemm_xp(b)
            else:
                self.launch_gemm(b)
        if evs is not None:
            evs[2 * len(self.bufs)].record(self.stream)

    def gemm_only(self):
        """The step's GEMM launches alone (the dominant kernel of every workload)."""
        for b in self.bufs:
            if b["mode"] == "fused":
                self.launch_fused(b)
            elif b["mode"] == "combined":
                self.launch_gemm_xp(b)
            else:
                self.launch_gemm(b)

    def compress_only(self):
        for b in self.bufs:
            self.launch_compress(b)

    def timed(self, fn, reps, warm=2):
        """Milliseconds per call of fn(), CUDA events on the launching stream around `reps` back-to-back calls."""
        torch = self.torch
        for _ in range(warm):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(self.stream)
        for _ in range(reps):
            fn()
        e1.record(self.stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / reps

    def timed_graph(self, fn, calls, replays):
        """Milliseconds per call of fn() from replays of a CUDA graph that holds `calls` of them (launches,
        staging allocations and all), timed with CUDA events around the replays: no host work in the timed
        region.  None when the calls do not capture."""
        torch = self.torch
        fn()
        torch.cuda.synchronize()
        side = torch.cuda.Stream(device=self.dev)
        sp0, g = self.sp, torch.cuda.CUDAGraph()
        try:
            self.sp = side.cuda_stream
            with torch.cuda.graph(g, stream=side):
                for _ in range(calls):
                    fn()
        except Exception:  # noqa: BLE001 - a call that does not capture: the caller times it eagerly
            return None
        finally:
            self.sp = sp0
        with torch.cuda.stream(self.stream):
            g.replay()
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(self.stream)
            for _ in range(replays):
                g.replay()
            e1.record(self.stream)
            torch.cuda.synchronize()
        del g
        return e0.elapsed_time(e1) / (replays * calls)

    def kernels(self, comp_ms, gemm_ms, tc_peak, hbm_peak):
        out = {}
        for i, b in enumerate(self.bufs):
            L = b["L"]
            t_tc = b["flops"] / (tc_peak * 1e12)
            t_hbm = b["gemm_bytes"] / (hbm_peak * 1e9)
            k = {"gemm_us": 1e3 * gemm_ms[i],
                 "gemm_tflops": b["flops"] / (gemm_ms[i] * 1e-3) / 1e12,
                 "gemm_gbs": b["gemm_bytes"] / (gemm_ms[i] * 1e-3) / 1e9,
                 "gemm_bound": "tensor" if t_tc >= t_hbm else "hbm",
                 "gemm_frac": max(t_tc, t_hbm) / (gemm_ms[i] * 1e-3),
                 "timed": {"fused": "the nm_prune_spmm call", "combined": "spmm_pair_kernel on the gathered input",
                           "split": "the GEMM call"}[b["mode"]]}
            if comp_ms is not None:
                k["compress_us"] = 1e3 * comp_ms[i]
                if b["mode"] != "fused":
                    k["compress_gbs"] = b["comp_bytes"] / (comp_ms[i] * 1e-3) / 1e9
                    k["compress_frac"] = k["compress_gbs"] / hbm_peak
            out[L.name] = k
        return out

    def roofline(self, gemm_step_ms, tc_peak, hbm_peak, peak_note):
        """Roofline of the step's GEMM launches together: useful FLOPs against the dense bf16 peak (2:4 useful
        FLOPs run at half the sparse-MMA rate, i.e. at most at the dense rate) or algorithmic bytes against the
        HBM copy bandwidth, whichever bound is slower."""
        flops_all = sum(b["flops"] for b in self.bufs)
        bytes_all = sum(b["gemm_bytes"] for b in self.bufs)
        gsec = gemm_step_ms * 1e-3
        tensor_bound = flops_all / (tc_peak * 1e12) >= bytes_all / (hbm_peak * 1e9)
        if tensor_bound:
            achieved, peak, unit = flops_all / gsec / 1e12, tc_peak, "TFLOP/s"
        else:
            achieved, peak, unit = bytes_all / gsec / 1e9, hbm_peak, "GB/s"
        modes = {b["mode"] for b in self.bufs}
        kernel = ("nm_prune_spmm call: prune_spmm_skinny_kernel + split-K reduction" if modes == {"fused"} else
                  "spmm_pair_kernel (tcgen05 2-SM GEMM) on the gathered input, as launched by nm_prune_spmm"
                  if modes == {"combined"} else
                  "the GEMM call (nm_spmm_permuted: gather_rows_kernel + spmm_pair_kernel, or nm_spmm / "
                  "nm_hybrid_spmm)")
        return {"bound": "tensor" if tensor_bound else "hbm", "achieved": achieved, "peak": peak, "unit": unit,
                "frac": achieved / peak, "traffic": None, "kernel": kernel,
                "peak_source": peak_note if tensor_bound else "measured HBM copy bandwidth",
                "algorithmic_per_launch": [b["flops"] if tensor_bound else b["gemm_bytes"] for b in self.bufs],
                "gemm_step_us": 1e3 * gemm_step_ms}


EXTRA_CONFIGS = ["decode", "vit", "patch_p25", "patch_p50", "patch_p75", "rl_mlp_2of4", "rl_mlp_1of4",
                 "rl_mlp_1of8", "tiny"]


def measure_config(name, args, dev, stream, nm, peaks, world, loaded_ms=0.0):
    """One further configuration of the pages' workloads: the step timed back to back (CUDA events around
    enough steps for >= 20 ms), the GEMM launches alone for `roofline`, the compress calls alone, and the
    per-layer event pass.  Inputs stay resident in HBM.  `loaded_ms`: the unbroken load that ran just before
    (the headline's); past a second of it the power cap sets the clocks, so the sustained peak applies."""
    torch = __import__("torch")
    r = Runner(name, dev, stream, nm)
    sustained = loaded_ms > 1000.0
    tc_peak, hbm_peak = peaks["bf16_tflops_sustained" if sustained else "bf16_tflops"], peaks["hbm_gbs"]
    peak_note = (f"measured bf16 sustained dense peak (measured right after {loaded_ms:.0f} ms of the headline's "
                 "unbroken load)" if sustained else "measured bf16 burst dense peak")
    est = r.timed(r.step, 3, warm=3)
    reps = int(min(2000, max(args.steps, 20.0 / max(est, 1e-4))))
    launches0 = nm.nm_launch_count()
    ms = r.timed(r.step, reps, warm=0)
    launches = (nm.nm_launch_count() - launches0) / reps
    greps = int(min(2000, max(args.steps, 20.0 / max(r.timed(r.gemm_only, 3), 1e-4))))
    gemm_step_ms = r.timed(r.gemm_only, greps)
    comp_ms_step = None if r.one_call and all(b["mode"] == "fused" for b in r.bufs) else \
        r.timed(r.compress_only, greps)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2 * len(r.bufs) + 1)] for _ in range(20)]
    for e in evs:
        r.step(e)
    torch.cuda.synchronize()
    comp_ms = np.zeros(len(r.bufs))
    gemm_ms = np.zeros(len(r.bufs))
    for e in evs:
        for i in range(len(r.bufs)):
            comp_ms[i] += e[2 * i].elapsed_time(e[2 * i + 1]) / len(evs)
            gemm_ms[i] += e[2 * i + 1].elapsed_time(e[2 * i + 2]) / len(evs)
    nm.nm_device_status(r.sp)
    roof = r.roofline(gemm_step_ms, tc_peak, hbm_peak, peak_note)
    roof["timing"] = f"CUDA events around {greps} back-to-back repetitions of the step's GEMM launches"
    out = {"value": world * r.useful / (ms * 1e-3) / 1e12, "unit": "TFLOP/s", "ms_per_step": ms,
           "steps": reps, "gpu_launches_per_step": launches,
           "config": step_config(name, r.layers, "one-call", "auto", False, world),
           "roofline": roof, "kernels": r.kernels(comp_ms if comp_ms_step is not None else None, gemm_ms,
                                                  tc_peak, hbm_peak)}
    if comp_ms_step is not None:
        cb = sum(b["comp_bytes"] for b in r.bufs)
        out["compress_roofline"] = {"bound": "hbm", "achieved": cb / (comp_ms_step * 1e-3) / 1e9, "peak": hbm_peak,
                                    "unit": "GB/s", "frac": cb / (comp_ms_step * 1e-3) / 1e9 / hbm_peak,
                                    "compress_step_us": 1e3 * comp_ms_step}
    if name in ("tiny",) or name.startswith("rl_mlp"):
        out["latency_us"] = 1e3 * ms
        out["note"] = ("launch-latency-bound: the roofline bound is well under a microsecond; the step time is "
                       "host call overhead and launch latency")
    if any(b["mode"] == "fused" for b in r.bufs):
        # the two-call design's GEMM (nm_spmm on the compressed operand, the split-K skinny kernel): the
        # decode-batch GEMM whose HBM fraction the pages' shape targets
        two = r.timed(lambda: [r.launch_gemm(b) for b in r.bufs], greps)
        gb = sum(gemm_bytes(b["L"], b["d"]) for b in r.bufs)
        out["gemm_call_roofline"] = {"bound": "hbm", "achieved": gb / (two * 1e-3) / 1e9, "peak": hbm_peak,
                                     "unit": "GB/s", "frac": gb / (two * 1e-3) / 1e9 / hbm_peak,
                                     "kernel": "nm_spmm: spmm_skinny_kernel + split-K reduction",
                                     "call_us": 1e3 * two}
    if name == "vit":
        t_exec = reencoded_bound_s(r.bufs, tc_peak, hbm_peak)
        out["roofline_reencoded"] = {"t_bound_us": 1e6 * t_exec, "frac": t_exec / (gemm_step_ms * 1e-3),
                                     "bound": "tensor" if t_exec * hbm_peak * 1e9 > sum(
                                         b["gemm_bytes"] for b in r.bufs) * (1 + 1e-9) else "hbm",
                                     "note": "max(the re-encoded 2:4 form's executed products (4x the useful "
                                             "ones) at the dense product rate, algorithmic bytes at the HBM "
                                             "rate) over the step's GEMM launches"}
    del r
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return out


def run_ours(args, rank: int, world: int, dist):
    import torch
    import sparse_gemm_nm_b200 as nm

    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream(dev)
    r = Runner(args.workload, dev, stream, nm, algo=args.algo, layers=args.layers, plain=args.plain,
               step_mode=args.step, pattern=args.pattern)
    bufs, sp = r.bufs, r.sp

    def barrier():
        rank_barrier(dist)

    def max_over_ranks(ms):
        return max_over_ranks_on(ms, dist, dev)

    useful = r.useful
    for _ in range(args.warmup):
        r.step()
    torch.cuda.synchronize()
    nm.nm_device_status(sp)

    props = torch.cuda.get_device_properties(dev)
    sampler = None
    if not args.quick:
        sampler = ClockSampler(f"GPU-{props.uuid}" if getattr(props, "uuid", None) else "")
        sampler.start()

    # Timed region: exactly K steps between two events.  An event recorded
    # between every pair of kernels would break the programmatic-dependent
    # launch overlap and slow the step by 3-5 %, so the per-kernel events run in
    # a second timed pass of the same K steps right after (same clocks sampler).
    nev = 2 * len(bufs) + 1
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(nev)] for _ in range(args.steps)]
    launches0 = nm.nm_launch_count()
    barrier()
    torch.cuda.synchronize()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for k in range(args.steps):
        r.step()
    t_end.record(stream)
    torch.cuda.synchronize()
    barrier()
    launches = nm.nm_launch_count() - launches0
    for k in range(args.steps):  # second pass: per-kernel events
        r.step(evs[k])
    torch.cuda.synchronize()
    barrier()

    # Third pass, for `roofline`: the GEMM launches of the step alone, back to back, no events between them
    # (the step's layers together exceed L2, so every launch reads its operands from HBM).
    greps = max(10, min(args.steps, 200))
    for _ in range(2):
        r.gemm_only()
    torch.cuda.synchronize()
    barrier()
    g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    g0.record(stream)
    for _ in range(greps):
        r.gemm_only()
    g1.record(stream)
    torch.cuda.synchronize()
    barrier()
    gemm_only_ms = max_over_ranks(g0.elapsed_time(g1)) / greps

    # Fourth pass, for `compress_roofline`: the step's compress calls (nm_prune_compress) alone, back to back.
    for _ in range(2):
        r.compress_only()
    torch.cuda.synchronize()
    barrier()
    c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    c0.record(stream)
    for _ in range(greps):
        r.compress_only()
    c1.record(stream)
    torch.cuda.synchronize()
    barrier()
    compress_only_ms = max_over_ranks(c0.elapsed_time(c1)) / greps
    nm.nm_device_status(sp)

    elapsed_ms = max_over_ranks(t_start.elapsed_time(t_end))
    ms_per_step = elapsed_ms / args.steps

    # per-kernel durations over the timed region (same stream as the launches)
    comp_ms = np.zeros(len(bufs))
    gemm_ms = np.zeros(len(bufs))
    for k in range(args.steps):
        e = evs[k]
        for i in range(len(bufs)):
            comp_ms[i] += e[2 * i].elapsed_time(e[2 * i + 1])
            gemm_ms[i] += e[2 * i + 1].elapsed_time(e[2 * i + 2])
    comp_ms /= args.steps
    gemm_ms /= args.steps

    peaks, peak_src = load_peaks()
    # The roofline pass runs at the end of an unbroken stretch of load (timed steps, the event pass, then the
    # GEMM-only pass); past a second of it the 1 kW power cap sets the clocks, so the sustained peak applies.
    loaded_ms = t_start.elapsed_time(g1)
    sustained = loaded_ms > 1000.0
    tc_peak = peaks["bf16_tflops_sustained" if sustained else "bf16_tflops"]
    hbm_peak = peaks["hbm_gbs"]
    kernels = r.kernels(comp_ms, gemm_ms, tc_peak, hbm_peak)
    roofline = r.roofline(gemm_only_ms, tc_peak, hbm_peak,
                          f"{peak_src} bf16 {'sustained' if sustained else 'burst'} dense peak ({loaded_ms:.0f} ms "
                          "of unbroken load up to the end of the roofline pass); useful 2:4 FLOPs run at half the "
                          "sparse-MMA rate, i.e. at the dense rate")
    roofline["timing"] = (f"CUDA events around {greps} back-to-back repetitions of the step's GEMM launches "
                          "(one per layer, no events between them); per-layer event-bracketed times are in `kernels`")
    if roofline["bound"] == "hbm":
        roofline["peak_source"] = f"{peak_src} HBM copy bandwidth"
    # DRAM bytes (read + write) of the GEMM call's kernels per layer, from one ncu capture
    # (profiles/<workload>_gemm_traffic.json); summed over the step like `achieved`.
    tfile = os.path.join(ROOT, "profiles", f"{args.workload}_gemm_traffic.json")
    if os.path.exists(tfile) and args.algo == "auto" and all(b["mode"] != "fused" for b in bufs):
        with open(tfile) as f:
            per = json.load(f).get("bytes_per_launch", {})
        names = [f"{b['L'].R}x{b['L'].K}" for b in bufs]
        kinds = [("spmm_pair_kernel",) if b["mode"] == "combined" else ("spmm_pair_kernel", "gather_rows_kernel")
                 for b in bufs]
        if all(n in per and all(k in per[n] for k in ks) for n, ks in zip(names, kinds)):
            roofline["traffic"] = sum(sum(per[n][k] for k in ks) for n, ks in zip(names, kinds))

    cfg = step_config(args.workload, r.layers, args.step, args.algo, args.plain, world)
    comp_bytes_all = sum(b["comp_bytes"] for b in bufs)
    comp_gbs = comp_bytes_all / (compress_only_ms * 1e-3) / 1e9
    compress_roofline = {"bound": "hbm", "achieved": comp_gbs, "peak": hbm_peak, "unit": "GB/s",
                         "frac": comp_gbs / hbm_peak, "kernel": "nm_prune_compress on the step's weights",
                         "algorithmic_per_launch": [b["comp_bytes"] for b in bufs],
                         "timing": f"CUDA events around {greps} back-to-back repetitions of the step's compress calls",
                         "compress_step_us": 1e3 * compress_only_ms}
    line = {"metric": METRIC, "value": world * useful / (ms_per_step * 1e-3) / 1e12, "unit": "TFLOP/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded numpy PCG64 draws rounded to bf16; shapes and distributions of the workload)",
            "config": cfg, "roofline": roofline, "compress_roofline": compress_roofline, "kernels": kernels,
            "gpu_launches": launches}

    if not args.quick and any(b["idx"] is not None for b in bufs) and all(b["tmap"] is None for b in bufs):
        # cost of the index-map read: per layer the GEMM call with the map (nm_spmm_permuted: gather pass +
        # GEMM) and without it (nm_spmm) on the compressed operand, each timed from replays of a CUDA graph
        # of 20 calls (an eager loop of a 30 us call can be bound by the host's call overhead instead)
        reps = max(10, min(200, args.steps))
        over = {}
        how = set()
        for b in bufs:
            L = b["L"]
            res = {}
            for name, permuted in (("permuted", True), ("plain", False)):
                fn = (lambda b=b, permuted=permuted: r.launch_gemm(b, permuted))
                t = r.timed_graph(fn, 20, max(1, reps // 20))
                how.add("graph" if t is not None else "eager")
                res[name] = t if t is not None else r.timed(fn, reps, warm=3)
            t_bound = max(b["flops"] / (tc_peak * 1e12), gemm_bytes(L, b["d"]) / (hbm_peak * 1e9))
            over[L.name] = {"plain_us": 1e3 * res["plain"], "permuted_us": 1e3 * res["permuted"],
                            "overhead": res["permuted"] / res["plain"] - 1.0,
                            "plain_tflops": b["flops"] / (res["plain"] * 1e-3) / 1e12,
                            "plain_frac": t_bound / (res["plain"] * 1e-3)}
        nm.nm_device_status(sp)
        over["timing"] = ("CUDA events around replays of a CUDA graph of 20 calls per layer and form" if how == {"graph"}
                          else "event-bracketed loops of calls (some calls did not capture into a CUDA graph)")
        line["permutation_overhead"] = over

    if not args.quick and all(b["tmap"] is None for b in bufs) and all(
            b["L"].n == 2 and b["L"].m == 4 for b in bufs):
        # backward products of each layer (training): dX = (W' Pi)^T dY and the value gradient dV,
        # timed in event-free loops of the same calls; dense tensor-core FLOPs 2 R K T per call
        reps = max(10, min(50, args.steps))
        back = {}
        L_ = r.L_
        for i, b in enumerate(bufs):
            L = b["L"]
            dY = r.up(wl.normal_bf16((L.R, L.T), 1.0, seed=100 + i))
            dX = torch.empty((L.K, L.T), dtype=torch.bfloat16, device=dev)
            dV = torch.empty((L.R, L.K // 2), dtype=torch.bfloat16, device=dev)
            idx = b["idx"].data_ptr() if b["idx"] is not None else None
            calls = {
                "spmm_t": lambda: r.check(L_.nm_spmm_t(b["vals"].data_ptr(), b["meta"].data_ptr(), 2, 4, L.R, L.K,
                                                       idx, dY.data_ptr(), L.T, L.T, dX.data_ptr(), L.T, 0, sp),
                                          "nm_spmm_t"),
                "sddmm": lambda: r.check(L_.nm_sddmm(b["meta"].data_ptr(), 2, 4, L.R, L.K, idx, dY.data_ptr(), L.T,
                                                     b["X"].data_ptr(), L.T, L.T, dV.data_ptr(), 0, sp), "nm_sddmm")}
            res = {}
            for name, fn in calls.items():
                us = r.timed(fn, reps, warm=3) * 1e3
                tflops = 2.0 * L.R * L.K * L.T / (us * 1e-6) / 1e12
                res[name] = {"us": us, "dense_tflops": tflops, "frac": tflops / tc_peak}
            back[L.name] = res
        nm.nm_device_status(sp)
        line["backward"] = {"calls": back, "timing": f"event-free loops of {reps} calls per product",
                            "roofline": "dense tcgen05 FLOPs 2*R*K*T per call against the same dense bf16 peak "
                                        "as `roofline` (the useful, survivor-only FLOPs are half of these)",
                            "spmm_t": "includes the decompression of W' into the staged dense operand",
                            "permuted": any(b["idx"] is not None for b in bufs)}

    # end-to-end through the public API with host buffers
    if not args.quick and not args.no_e2e:
        hW = [torch.from_numpy(b["d"].W.view(np.int16)).pin_memory() for b in bufs]
        hX = [torch.from_numpy(b["d"].X.view(np.int16)).pin_memory() for b in bufs]
        hI = [torch.from_numpy(b["d"].idx).pin_memory() if b["idx"] is not None else None for b in bufs]
        hY = [torch.empty((b["L"].R, b["L"].T), dtype=torch.int16).pin_memory() for b in bufs]
        h2d = sum(a.numel() * a.element_size() for a in hW + hX + [h for h in hI if h is not None])
        d2h = sum(a.numel() * a.element_size() for a in hY)

        # Per layer: host-to-device copies on one stream, the API calls on the
        # compute stream, the device-to-host read on a third, chained by events:
        # layer i+1's inputs cross PCIe while layer i computes and layer i-1's
        # result comes back.  A buffer is overwritten only after its last reader.
        s_h2d, s_d2h = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
        nl = len(bufs)
        ev = lambda: torch.cuda.Event()
        copied, computed, returned = [ev() for _ in range(nl)], [ev() for _ in range(nl)], [ev() for _ in range(nl)]
        started = [False] * nl

        def e2e_step():
            for i, b in enumerate(bufs):
                with torch.cuda.stream(s_h2d):
                    if started[i]:
                        s_h2d.wait_event(computed[i])  # compress/GEMM of the previous step have read W, X, idx
                    b["W"].view(torch.int16).copy_(hW[i], non_blocking=True)
                    b["X"].view(torch.int16).copy_(hX[i], non_blocking=True)
                    if hI[i] is not None:
                        b["idx"].copy_(hI[i], non_blocking=True)
                    copied[i].record(s_h2d)
                stream.wait_event(copied[i])
                if started[i]:
                    stream.wait_event(returned[i])  # Y of the previous step has been read back
                r.launch_layer(b)
                computed[i].record(stream)
                with torch.cuda.stream(s_d2h):
                    s_d2h.wait_event(computed[i])
                    hY[i].copy_(b["Y"].view(torch.int16), non_blocking=True)
                    returned[i].record(s_d2h)
                started[i] = True

        e2e_step()
        torch.cuda.synchronize()
        barrier()
        a = torch.cuda.Event(enable_timing=True)
        z = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        s_h2d.wait_event(a)
        s_d2h.wait_event(a)
        for _ in range(args.e2e_steps):
            e2e_step()
        for i in range(nl):
            stream.wait_event(returned[i])
        z.record(stream)
        torch.cuda.synchronize()
        e_ms = max_over_ranks(a.elapsed_time(z))
        line["e2e"] = {"value": world * useful * args.e2e_steps / (e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                       "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                       "ms_per_step": e_ms / args.e2e_steps,
                       "overlap": "per-layer H2D / compute / D2H on three streams, chained by events"}

    # The pages' other configurations, each measured on its own (same clocks sampler), each with its
    # own roofline.  Every rank measures them (identical collective-free work); rank 0 reports.
    if not args.quick and not args.no_configs and args.workload == WORKLOAD and args.algo == "auto" \
            and not args.layers and not args.plain and args.step == "one-call" and not args.pattern:
        data_host = r.data
        del r, bufs
        torch.cuda.empty_cache()
        configs = {}
        for name in EXTRA_CONFIGS:
            barrier()
            configs[name] = measure_config(name, args, dev, stream, nm, peaks, world, loaded_ms)
        line["configs"] = configs
    else:
        data_host = r.data
    if sampler:
        sampler.stop()
    line["clocks"] = sampler.summary() if sampler else None
    if rank == 0 and world == 1 and not args.quick and not args.no_cpu_baseline and args.workload == "llama7b" \
            and not args.pattern:
        line["cpu_baseline"] = cpu_baseline(data_host, args.cpu_seconds)
    elif rank == 0:
        line["cpu_baseline"] = None
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_i8(args, rank: int, world: int, dist):
    """INT8 2:4 step on the workload's shapes: per layer nm_prune_compress_i8 then nm_spmm_i8 (exact int32)."""
    import torch
    import sparse_gemm_nm_b200 as nm

    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream(dev)
    sp = stream.cuda_stream
    L_ = nm.lib()
    layers = wl.workload(args.workload)
    if args.layers:
        layers = [layers[int(i)] for i in args.layers.split(",")]
    if any(L.n != 2 or L.m != 4 or L.K % 16 for L in layers):
        raise SystemExit("--dtype i8 needs 2:4 layers with K % 16 == 0")
    bufs = []
    for i, L in enumerate(layers):
        T16 = (L.T + 15) // 16 * 16
        Xb = np.zeros((L.K, T16), np.int8)
        Xb[:, :L.T] = wl.integer_i8((L.K, L.T), -128, 127, seed=10 * i + 2)
        b = {"L": L, "W": torch.from_numpy(wl.normal_i8((L.R, L.K), 32.0, seed=10 * i + 1)).to(dev),
             "X": torch.from_numpy(Xb).to(dev), "ldx": T16,
             "vals": torch.empty((L.R, L.K // 2), dtype=torch.int8, device=dev),
             "meta": torch.empty((nm.nm_meta_words(L.R, L.K, 2, 4),), dtype=torch.int32, device=dev),
             "Y": torch.empty((L.R, (L.T + 3) // 4 * 4), dtype=torch.int32, device=dev)}
        b["ops"] = 2.0 * L.R * L.T * L.K / 2  # useful: survivors only
        bufs.append(b)
    torch.cuda.synchronize()

    def check(st, what):
        if st != 0:
            raise RuntimeError(f"{what}: {L_.nm_last_error().decode()}")

    def compress(b):
        L = b["L"]
        check(L_.nm_prune_compress_i8(b["W"].data_ptr(), L.R, L.K, L.K, b["vals"].data_ptr(), b["meta"].data_ptr(),
                                      sp), "nm_prune_compress_i8")

    def gemm(b):
        L = b["L"]
        check(L_.nm_spmm_i8(b["vals"].data_ptr(), b["meta"].data_ptr(), L.R, L.K, b["X"].data_ptr(), b["ldx"], L.T,
                            b["Y"].data_ptr(), b["Y"].shape[1], sp), "nm_spmm_i8")

    def step():
        for b in bufs:
            compress(b)
            gemm(b)

    def timed(fn, reps):
        rank_barrier(dist)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        rank_barrier(dist)
        return max_over_ranks_on(e0.elapsed_time(e1), dist, dev) / reps

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    props = torch.cuda.get_device_properties(dev)
    sampler = None if args.quick else ClockSampler(f"GPU-{props.uuid}" if getattr(props, "uuid", None) else "")
    if sampler:
        sampler.start()
    launches0 = nm.nm_launch_count()
    ms_per_step = timed(step, args.steps)
    launches = nm.nm_launch_count() - launches0
    gemm_ms = timed(lambda: [gemm(b) for b in bufs], max(10, min(args.steps, 200)))
    if sampler:
        sampler.stop()
    nm.nm_device_status(sp)
    peaks, peak_src = load_peaks()
    i8_peak = 2.0 * peaks["bf16_tflops"]
    useful = sum(b["ops"] for b in bufs)
    achieved = useful / (gemm_ms * 1e-3) / 1e12
    line = {"metric": METRIC, "value": world * useful / (ms_per_step * 1e-3) / 1e12, "unit": "TOP/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "s8",
            "data": "synthetic int8: W rounded N(0, 32^2) clipped to [-128, 127], X uniform int8",
            "config": {"workload": args.workload + " (INT8 2:4)", "shapes": [[b["L"].R, b["L"].K] for b in bufs],
                       "T": [b["L"].T for b in bufs], "step": "nm_prune_compress_i8, then nm_spmm_i8, per layer",
                       "parallelism": f"replicas x{world}"},
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": i8_peak, "unit": "TOP/s",
                         "frac": achieved / i8_peak, "traffic": None,
                         "kernel": "nm_spmm_i8 calls: relayout_meta_i8_kernel + spmm_pair_kernel (sparse kind::i8)",
                         "peak_source": f"{peak_src} bf16 burst dense peak x 2 (the nominal int8 / bf16 dense ratio); "
                                        "useful (survivor) operations: the sparse MMA multiplies the stored values "
                                        "at the dense rate (its 2x is over the logical K), so they reach this peak "
                                        "at most",
                         "timing": "CUDA events around back-to-back repetitions of the step's GEMM calls"},
            "gpu_launches": launches, "clocks": sampler.summary() if sampler else None, "cpu_baseline": None}
    if rank == 0:
        print(json.dumps(line))


def run_tf32(args, rank: int, world: int, dist):
    """TF32 1:2 step on the workload's shapes: per layer nm_prune_compress_tf32 then nm_spmm_tf32 (fp32 out)."""
    import torch
    import sparse_gemm_nm_b200 as nm

    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream(dev)
    sp = stream.cuda_stream
    L_ = nm.lib()
    layers = wl.workload(args.workload)
    if args.layers:
        layers = [layers[int(i)] for i in args.layers.split(",")]
    if any(L.K % 2 for L in layers):
        raise SystemExit("--dtype tf32 needs even K")
    bufs = []
    for i, L in enumerate(layers):
        T4 = (L.T + 3) // 4 * 4
        Xb = np.zeros((L.K, T4), np.float32)
        Xb[:, :L.T] = wl.normal_f32((L.K, L.T), 1.0, seed=10 * i + 2)
        b = {"L": L, "W": torch.from_numpy(wl.normal_f32((L.R, L.K), 0.02, seed=10 * i + 1)).to(dev),
             "X": torch.from_numpy(Xb).to(dev), "ldx": T4,
             "vals": torch.empty((L.R, L.K // 2), dtype=torch.float32, device=dev),
             "meta": torch.empty((nm.nm_meta_words(L.R, L.K, 1, 2),), dtype=torch.int32, device=dev),
             "Y": torch.empty((L.R, T4), dtype=torch.float32, device=dev)}
        b["flops"] = 2.0 * L.R * L.T * L.K / 2  # useful: survivors only
        bufs.append(b)
    torch.cuda.synchronize()

    def check(st, what):
        if st != 0:
            raise RuntimeError(f"{what}: {L_.nm_last_error().decode()}")

    def compress(b):
        L = b["L"]
        check(L_.nm_prune_compress_tf32(b["W"].data_ptr(), L.R, L.K, L.K, b["vals"].data_ptr(),
                                        b["meta"].data_ptr(), sp), "nm_prune_compress_tf32")

    def gemm(b):
        L = b["L"]
        check(L_.nm_spmm_tf32(b["vals"].data_ptr(), b["meta"].data_ptr(), L.R, L.K, b["X"].data_ptr(), b["ldx"],
                              L.T, b["Y"].data_ptr(), b["Y"].shape[1], 1, sp), "nm_spmm_tf32")

    def step():
        for b in bufs:
            compress(b)
            gemm(b)

    def timed(fn, reps):
        rank_barrier(dist)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        rank_barrier(dist)
        return max_over_ranks_on(e0.elapsed_time(e1), dist, dev) / reps

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    props = torch.cuda.get_device_properties(dev)
    sampler = None if args.quick else ClockSampler(f"GPU-{props.uuid}" if getattr(props, "uuid", None) else "")
    if sampler:
        sampler.start()
    launches0 = nm.nm_launch_count()
    ms_per_step = timed(step, args.steps)
    launches = nm.nm_launch_count() - launches0
    gemm_ms = timed(lambda: [gemm(b) for b in bufs], max(10, min(args.steps, 200)))
    if sampler:
        sampler.stop()
    nm.nm_device_status(sp)
    peaks, peak_src = load_peaks()
    tf32_peak = 0.5 * peaks["bf16_tflops"]
    useful = sum(b["flops"] for b in bufs)
    achieved = useful / (gemm_ms * 1e-3) / 1e12
    line = {"metric": METRIC, "value": world * useful / (ms_per_step * 1e-3) / 1e12, "unit": "TFLOP/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "tf32",
            "data": "synthetic float32: W ~ N(0, 0.02^2), X ~ N(0, 1) (seeded PCG64)",
            "config": {"workload": args.workload + " (TF32 1:2)", "shapes": [[b["L"].R, b["L"].K] for b in bufs],
                       "T": [b["L"].T for b in bufs],
                       "step": "nm_prune_compress_tf32, then nm_spmm_tf32 (fp32 out), per layer",
                       "parallelism": f"replicas x{world}"},
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": tf32_peak, "unit": "TFLOP/s",
                         "frac": achieved / tf32_peak, "traffic": None,
                         "kernel": "nm_spmm_tf32 calls: relayout_meta_tf32_kernel + spmm_pair_kernel (sparse kind::tf32)",
                         "peak_source": f"{peak_src} bf16 burst dense peak x 0.5 (the nominal tf32 / bf16 dense "
                                        "ratio); useful (survivor) FLOPs: the sparse MMA multiplies the stored "
                                        "values at the dense rate (its 2x is over the logical K), so they reach "
                                        "this peak at most",
                         "timing": "CUDA events around back-to-back repetitions of the step's GEMM calls"},
            "gpu_launches": launches, "clocks": sampler.summary() if sampler else None, "cpu_baseline": None}
    if rank == 0:
        print(json.dumps(line))


def run_diag(args, rank: int, world: int, dist):
    """Diagonal-pattern step: per layer nm_diag_prune_compress (D = K/10) then nm_diag_spmm with the index map."""
    import torch
    import sparse_gemm_nm_b200 as nm

    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream(dev)
    sp = stream.cuda_stream
    L_ = nm.lib()
    layers = wl.workload(args.workload)
    if args.layers:
        layers = [layers[int(i)] for i in args.layers.split(",")]
    up = lambda bits: torch.from_numpy(bits.view(np.int16)).to(dev).view(torch.bfloat16)
    bufs = []
    for i, L in enumerate(layers):
        d = wl.make_layer(L)
        D = max(1, round(L.K / 10))
        T8 = (L.T + 7) // 8 * 8
        Xb = np.zeros((L.K, T8), np.uint16)
        Xb[:, :L.T] = d.X
        idx = d.idx if d.idx is not None else wl.permutation(L.K, 100 + i)
        b = {"L": L, "D": D, "W": up(d.W), "X": up(Xb), "ldx": T8, "idx": torch.from_numpy(idx).to(dev),
             "offs": torch.empty((D,), dtype=torch.int32, device=dev),
             "V": torch.empty((D, L.R), dtype=torch.bfloat16, device=dev),
             "Y": torch.empty((L.R, T8), dtype=torch.bfloat16, device=dev)}
        b["flops"] = 2.0 * L.R * D * L.T  # useful: kept entries only
        bufs.append(b)
    torch.cuda.synchronize()

    def check(st, what):
        if st != 0:
            raise RuntimeError(f"{what}: {L_.nm_last_error().decode()}")

    def select(b):
        L = b["L"]
        check(L_.nm_diag_prune_compress(b["W"].data_ptr(), L.R, L.K, L.K, b["D"], b["offs"].data_ptr(),
                                        b["V"].data_ptr(), sp), "nm_diag_prune_compress")

    def gemm(b):
        L = b["L"]
        check(L_.nm_diag_spmm(b["V"].data_ptr(), b["offs"].data_ptr(), b["D"], L.R, L.K, b["idx"].data_ptr(),
                              b["X"].data_ptr(), b["ldx"], L.T, b["Y"].data_ptr(), b["ldx"], 0, sp), "nm_diag_spmm")

    def step():
        for b in bufs:
            select(b)
            gemm(b)

    def timed(fn, reps):
        rank_barrier(dist)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        rank_barrier(dist)
        return max_over_ranks_on(e0.elapsed_time(e1), dist, dev) / reps

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    props = torch.cuda.get_device_properties(dev)
    sampler = None if args.quick else ClockSampler(f"GPU-{props.uuid}" if getattr(props, "uuid", None) else "")
    if sampler:
        sampler.start()
    launches0 = nm.nm_launch_count()
    ms_per_step = timed(step, args.steps)
    launches = nm.nm_launch_count() - launches0
    gemm_ms = timed(lambda: [gemm(b) for b in bufs], max(10, min(args.steps, 200)))
    if sampler:
        sampler.stop()
    nm.nm_device_status(sp)
    peaks, peak_src = load_peaks()
    useful = sum(b["flops"] for b in bufs)
    dense = sum(2.0 * b["L"].R * b["L"].K * b["L"].T for b in bufs)
    line = {"metric": METRIC, "value": world * useful / (ms_per_step * 1e-3) / 1e12, "unit": "TFLOP/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded numpy PCG64 draws rounded to bf16; the workload's shapes)",
            "config": {"workload": args.workload + " (diagonal, 90 % sparse)",
                       "shapes": [[b["L"].R, b["L"].K] for b in bufs], "T": [b["L"].T for b in bufs],
                       "kept_diagonals": [b["D"] for b in bufs], "permuted": True,
                       "step": "nm_diag_prune_compress, then nm_diag_spmm with the index map, per layer",
                       "parallelism": f"replicas x{world}"},
            "roofline": {"bound": "tensor", "achieved": dense / (gemm_ms * 1e-3) / 1e12,
                         "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                         "frac": dense / (gemm_ms * 1e-3) / 1e12 / peaks["bf16_tflops"], "traffic": None,
                         "kernel": "nm_diag_spmm calls: dense copy + gather pass + dense_pair_kernel",
                         "peak_source": f"{peak_src} bf16 burst dense peak; executed dense FLOPs 2 R K T (the "
                                        "useful ones, 2 R D T, are what `value` counts)",
                         "useful_tflops_in_gemm": useful / (gemm_ms * 1e-3) / 1e12,
                         "timing": "CUDA events around back-to-back repetitions of the step's GEMM calls"},
            "gpu_launches": launches, "clocks": sampler.summary() if sampler else None, "cpu_baseline": None}
    if rank == 0:
        print(json.dumps(line))


def main(argv=None):
    args = parse_args(argv)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return 0
    dist = None
    if world > 1:
        import datetime

        import torch
        import torch.distributed as tdist
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
        dist = tdist
    try:
        (run_i8 if args.dtype == "i8" else run_tf32 if args.dtype == "tf32" else run_diag if args.diag else run_ours)(args, rank, world, dist)
    finally:
        if dist is not None:
            dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
