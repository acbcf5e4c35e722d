"""Benchmark of the ELSAA attention operator (forward + backward) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl elsaa|reference]

A step is one forward and one backward pass of the whole operator (selection,
RACE features and chunk statistics, RACE read-out, sparse forward with the fusion,
row scalars, suffix statistics, selection inverse, the RACE backward and the
sparse dQ and dK/dV kernels) over one batch of synthetic input that is resident
in HBM.  Default workload: B=1, H=32,
N=16384, d=128, bf16, causal, r=128, 128-key blocks, top-16 blocks per tile.
Each rank runs its own batch (independent problems, no collective on the data
path), so multi-GPU runs scale weakly; rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import csv
import hashlib
import io
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402
import torch.distributed as dist  # noqa: E402

from sparse_rank_approximation_b200.workloads import HEADLINE, WORKLOADS, make_inputs  # noqa: E402

METRIC = "ELSAA fwd+bwd tokens/sec and % of roofline at N=16K, 1×B200"
UNIT = "tokens/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return json.load(f), "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# --------------------------------------------------------------------------
# Algorithmic work per kernel (the method's own counts, not what a kernel
# happens to move): used for the roofline numbers.
# --------------------------------------------------------------------------

def selected_blocks_per_head(w):
    """sum over tiles of the number of selected key blocks (causal tiles near the
    start have fewer eligible blocks)."""
    n_t = w.n_tiles
    if w.topk == 0:
        return 0
    if not w.causal:
        return n_t * w.topk
    return sum(min(w.topk, t + 1) for t in range(n_t))


def work_model(w):
    BH, N, d, T, r = w.B * w.H, w.N, w.d, w.block_size, w.rank_r
    sel = selected_blocks_per_head(w) * BH          # (tile, block) pairs
    pair_mma = 2 * T * T * d                        # one T x T x d product
    L = w.n_tables
    m = {}
    # sparse branch forward: QK^T and PV per selected (tile, block) pair (the useful work; with
    # blocks of 64 keys the kernels stage two tiles' blocks side by side and mask half of it)
    f_sparse = 2 * pair_mma * sel
    tiles = w.n_tiles * BH
    m["attn_fwd_tc"] = dict(flops=f_sparse, bytes=sel * 2 * T * d * 2 + tiles * T * d * 2 * 5)   # K,V + Q,O,O_lr + O_s fp32
    m["dq_tc"] = dict(flops=3 * pair_mma * sel, bytes=sel * 2 * T * d * 2 + tiles * T * d * 2 * 3)
    m["dkdv_tc"] = dict(flops=4 * pair_mma * sel, bytes=sel * 2 * T * d * 2 + tiles * T * d * 2 * 4)
    # RACE on the tensor cores, per launch: chunks of C = 128 rows, one launch per group of 128
    # features (8 tables; G = ceil(r / 128) groups, the last zero-padded)
    C, R = 128, 128
    chunks = -(-N // C) * BH
    G = max(1, -(-r // R))
    NH = 4 * min(L, 8)                                          # projections of one group
    cz = 1 if w.causal else 0
    state_b = R * d * 2 * 2 + R * 4                             # per-chunk statistics (bf16 hi + lo, mass)
    # read-out: Phi_Q Phi_K^T, kappa V, Phi_Q P
    m["race_readout_tc"] = dict(flops=chunks * 2 * C * (cz * C * R + cz * C * d + R * d),
                                bytes=chunks * (C * R * 2 * (1 + cz) + cz * C * d * 2 + state_b + C * d * 2 + C * 4))
    # query side: dO V^T, dO P^T, dkappa Phi_K, dh W^T;  key side: Phi_K Phi_Q^T, V dO^T, Phi_K R,
    # V R^T, kappa^T dO, dkappa^T Phi_Q, dh W^T
    m["race_q_bwd_tc"] = dict(flops=chunks * 2 * C * (cz * C * d + d * R + cz * C * R + NH * d),
                              bytes=chunks * (C * d * 2 * (2 + cz) + cz * C * R * 2 + state_b + C * NH * 4 + C * 12
                                              + C * d * 4))
    m["race_k_bwd_tc"] = dict(flops=chunks * 2 * C * (2 * cz * C * R + 2 * cz * C * d + 2 * R * d + NH * d),
                              bytes=chunks * (C * R * 2 * (1 + cz) + C * d * 2 * (2 + cz) + state_b + C * NH * 4
                                              + C * 12 + 2 * C * d * 4))
    # statistics of one group: the totals pass reads Phi and Y once; the emit pass reads them
    # again (causal) and writes every chunk's statistics
    f_stats = chunks * 2 * C * R * d
    rd = chunks * C * (R + d) * 2
    for side in ("fwd", "bwd"):
        m[f"race_stats_{side}_totals"] = dict(flops=f_stats, bytes=rd)
        m[f"race_stats_{side}_emit"] = dict(flops=f_stats * cz, bytes=rd * cz + chunks * state_b)
    rp = 128 * G
    m["race_features_tc"] = dict(flops=2 * 2 * BH * N * d * 4 * L * 2,
                                 bytes=2 * BH * N * (d * 2 + rp * 2 + 4 * L * 4 + 4))
    if w.selector == "sortlsh":
        esz = 2 if w.dtype == "bf16" else 4
        mat = BH * N * d * esz
        m["sortlsh_order"] = dict(flops=0, bytes=2 * mat + 2 * BH * N * 4)   # Q, K read; orders written
        m["sortlsh_gather"] = dict(flops=0, bytes=2 * mat)                   # per launch: one matrix in, one out
        m["sortlsh_scatter"] = dict(flops=0, bytes=2 * mat)
    unique_fwd = 4 * BH * N * d * 2                # Q, K, V read, O written
    f_read = G * m["race_readout_tc"]["flops"]
    return m, dict(sel_pairs=sel, tiles=tiles, f_sparse_fwd=f_sparse, f_lr_fwd=f_read + G * f_stats,
                   gathered_fwd=sel * 2 * T * d * 2, unique_fwd=unique_fwd)


def whole_step_roofline(w, peaks, t_step_ms):
    """T_roof = max(F / P_bf16, gathered bytes / BW), forward + backward, counted as
    sparse F_bwd = 2.5 F_fwd, low-rank F_bwd = 2 F_fwd, backward bytes = 2x gathered
    plus 8 N d bf16 rows per head."""
    _, tot = work_model(w)
    F = tot["f_sparse_fwd"] * 3.5 + tot["f_lr_fwd"] * 3.0
    BH = w.B * w.H
    bytes_ = tot["gathered_fwd"] * 3 + 8 * BH * w.N * w.d * 2 + tot["unique_fwd"]
    t_f = F / (peaks["bf16_tflops"] * 1e12)
    t_b = bytes_ / (peaks["hbm_gbs"] * 1e9)
    t_roof = max(t_f, t_b)
    return dict(t_roof_ms=t_roof * 1e3, frac=t_roof * 1e3 / t_step_ms, flops=F, bytes=bytes_,
                bound="tensor" if t_f >= t_b else "hbm",
                compute_only_frac=t_f * 1e3 / t_step_ms)


# --------------------------------------------------------------------------
# Multi-rank plumbing: each rank runs its own batch; the only collectives are a
# barrier around the timed region and the max-reduce of the elapsed time.
# --------------------------------------------------------------------------

def max_over_ranks(value: float, device=None) -> float:
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_seed(rank: int) -> int:
    """Seed of the batch a rank processes (independent problems per rank)."""
    return rank


# --------------------------------------------------------------------------

class NvmlClockSampler:
    """SM clock and throttle reasons read through NVML every 5 ms on a host thread while the
    timed region runs (reading only; a short timed region still gets dozens of samples)."""
    REASONS = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def __init__(self, dev):
        import threading
        import pynvml
        self.nv = pynvml
        pynvml.nvmlInit()
        props = torch.cuda.get_device_properties(dev)
        bus = f"{props.pci_domain_id:08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0"
        self.h = pynvml.nvmlDeviceGetHandleByPciBusId(bus.encode())
        self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        self.bits = [pynvml.nvmlClocksEventReasonHwSlowdown, pynvml.nvmlClocksEventReasonHwThermalSlowdown,
                     pynvml.nvmlClocksEventReasonSwThermalSlowdown, pynvml.nvmlClocksEventReasonSwPowerCap]
        self.rows, self.on = [], False
        self.stop = threading.Event()
        self.thread = threading.Thread(target=self._loop, daemon=True)

    def _loop(self):
        nv = self.nv
        while not self.stop.is_set():
            if self.on:
                try:
                    mhz = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                    rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                    self.rows.append((mhz, [n for n, b in zip(self.REASONS, self.bits) if rs & b]))
                except nv.NVMLError:
                    pass
            self.stop.wait(0.005)

    def __enter__(self):
        self.thread.start()
        return self

    def mark(self, begin: bool):
        self.on = begin

    def __exit__(self, *exc):
        self.stop.set()
        self.thread.join(timeout=2)

    def summary(self):
        if not self.rows:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0, "source": "nvml"}
        return {"sm_mhz": statistics.median(r[0] for r in self.rows), "sm_max_mhz": self.max_mhz,
                "reasons": sorted({n for r in self.rows for n in r[1]}), "samples": len(self.rows),
                "in_window": True, "source": "nvml, every 5 ms"}


def clock_sampler(dev, index):
    try:
        return NvmlClockSampler(dev)
    except Exception:
        return ClockSampler(index)


def bf16_peak(peaks, clocks):
    """The measured bf16 rate that matches the run's clocks: the burst figure (measured at
    full clock) when the timed region's median SM clock is within 5 % of its maximum, else
    the sustained one (measured under the power cap)."""
    mhz, mx = clocks.get("sm_mhz"), clocks.get("sm_max_mhz")
    if "bf16_tflops_sustained" in peaks and not (mhz and mx and mhz >= 0.95 * mx):
        return peaks["bf16_tflops_sustained"], "sustained"
    return peaks["bf16_tflops"], "burst"


class ClockSampler:
    """nvidia-smi sampling (every 100 ms) while the timed region runs."""
    QUERY = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASONS = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.out = ""
        self.window = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.QUERY}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def mark(self, begin: bool):
        import datetime
        now = datetime.datetime.now()
        self.window = (now, None) if begin else (self.window[0], now)

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.out, _ = self.proc.communicate()

    def summary(self):
        import datetime
        rows = []
        for r in csv.reader(io.StringIO(self.out)):
            if len(r) < 10:
                continue
            try:
                ts = datetime.datetime.strptime(r[0].strip(), "%Y/%m/%d %H:%M:%S.%f")
                rows.append((ts, float(r[2]), float(r[3]), [x.strip().lower() for x in r[6:10]]))
            except ValueError:
                continue
        inside = [x for x in rows if self.window and self.window[1] and self.window[0] <= x[0] <= self.window[1]]
        use = inside or rows
        if not use:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        reasons = sorted({n for x in use for n, v in zip(self.REASONS, x[3]) if v == "active"})
        return {"sm_mhz": statistics.median(x[1] for x in use), "sm_max_mhz": max(x[2] for x in use),
                "reasons": reasons, "samples": len(use), "in_window": bool(inside)}


# the sources each profiled kernel is compiled from (its file and the headers it includes)
KERNEL_SOURCES = {
    "dkdv_tc": ("bwd_tc.cu", "tc_common.cuh", "common.cuh", "kernels.h"),
    "dq_tc": ("bwd_tc.cu", "tc_common.cuh", "common.cuh", "kernels.h"),
    "attn_fwd_tc": ("attn_fwd_tc.cu", "tc_common.cuh", "common.cuh", "kernels.h"),
    "race_k_bwd_tc": ("race_tc.cu", "tc_common.cuh", "common.cuh", "kernels.h"),
}


def kernel_sources_hash(kernel: str):
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "sparse_rank_approximation_b200", "csrc")
    for f in KERNEL_SOURCES.get(kernel, sorted(os.listdir(csrc))):
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def dram_traffic(kernel: str, workload: str):
    """Per-launch DRAM bytes of `kernel` from the committed ncu summary, if it was
    taken on the current kernel sources; else None."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    if not os.path.exists(path):
        return None
    src = kernel_sources_hash(kernel)
    for line in open(path):
        parts = line.split()
        if len(parts) >= 4 and not line.startswith("#") and parts[0] == kernel and parts[1] == workload \
                and parts[3] == src:
            return float(parts[2])
    return None


# --------------------------------------------------------------------------

class OracleSample:
    """The float64 oracle (forward + backward) on a bounded sample of the workload:
    one head, and of its query tiles an evenly spaced subset (the backward is a
    sum of per-tile contributions, so a subset is that share of the work)."""

    def __init__(self, w):
        from oracle import elsaa_oracle as orc
        self.orc, self.w = orc, w
        inp = make_inputs(w, 0, heads=range(1))
        self.p = orc.Params(N=w.N, d=w.d, block_size=w.block_size, topk=w.topk, rank_r=w.rank_r,
                            causal=w.causal, scale=w.scale)
        if w.selector == "sortlsh":
            self.p.selector = "sortlsh"
            self.p.lsh_planes = inp["R"].double().numpy()
        self.W = inp["W"].double().numpy()
        self.x = {n: inp[n][0, 0].double().numpy() for n in ("Q", "K", "V", "dO")}

    def run(self, n_tiles):
        """Returns (equivalent tokens of the full batch, seconds)."""
        w, x = self.w, self.x
        nt = w.n_tiles
        n_tiles = max(1, min(nt, n_tiles))
        tiles = sorted({int(round(i * (nt - 1) / max(1, n_tiles - 1))) for i in range(n_tiles)})
        t0 = time.perf_counter()
        fw = self.orc.forward_head(x["Q"], x["K"], x["V"], self.W, self.p, tiles=tiles)
        self.orc.backward_head(x["Q"], x["K"], x["V"], self.W, x["dO"], fw, self.p, tiles=tiles)
        dt = time.perf_counter() - t0
        return w.B * w.N * (len(tiles) / nt) / w.H, dt

    def calibrate(self, seconds):
        """Number of query tiles whose fwd+bwd takes about `seconds`."""
        _, t1 = self.run(1)
        _, t4 = self.run(4)
        per_tile = max((t4 - t1) / 3, 1e-3)
        fixed = max(t1 - per_tile, 0.0)
        return max(1, min(self.w.n_tiles, int((seconds - fixed) / per_tile)))


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return max(n)
    except Exception:
        pass
    return len(os.sched_getaffinity(0))


def run_reference(args, w, rank, world):
    if rank != 0:
        return 0
    budget = 150.0                      # seconds for the whole warm-up + timed run
    smp = OracleSample(w)
    n_tiles = smp.calibrate(budget / (args.steps + args.warmup))
    for _ in range(args.warmup):
        smp.run(n_tiles)
    tokens, secs = 0.0, 0.0
    for _ in range(args.steps):
        tk, dt = smp.run(n_tiles)
        tokens += tk
        secs += dt
    value = tokens / secs
    sample = (f"float64 oracle fwd+bwd, per step {n_tiles} of {w.n_tiles} query tiles of 1 of {w.H} heads, "
              f"scaled to the full batch")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": secs / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": w.name, "shape": w.describe(), "sample": sample},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=HEADLINE, choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="elsaa", choices=["elsaa", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-graph", action="store_true", help="skip the CUDA-graph replay timing")
    ap.add_argument("--heads", type=int, default=0,
                    help="run the workload with this many heads (a smaller case for ncu captures)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    w = WORKLOADS[args.workload]
    if args.heads:
        import dataclasses
        w = dataclasses.replace(w, H=args.heads, name=f"{w.name}_h{args.heads}")
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        return run_reference(args, w, rank, world)

    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (no CPU fallback)")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", device_id=dev, timeout=datetime.timedelta(seconds=120))

    from sparse_rank_approximation_b200 import binding as bd
    peaks, peak_kind = load_peaks()
    inp = make_inputs(w, seed=rank_seed(rank))
    key = "16" if w.dtype == "bf16" else ""
    q, k, v, dO = (inp[n + key].to(dev) for n in ("Q", "K", "V", "dO"))
    W = inp["W"].to(dev)
    lsh = w.selector == "sortlsh"
    R = inp["R"].to(dev) if lsh else None
    op = bd.Elsaa(bd.make_params(w.B, w.H, w.N, w.d,
                                 dtype=bd.ELSAA_DTYPE_BF16 if w.dtype == "bf16" else bd.ELSAA_DTYPE_F32,
                                 causal=w.causal, rank_r=w.rank_r, block_size=w.block_size, topk=w.topk,
                                 selector=bd.ELSAA_SEL_SORTLSH if lsh else bd.ELSAA_SEL_TOPK_BLOCKS,
                                 lsh_bits=w.lsh_bits), dev, lsh_planes=R)
    O = op._empty_like_io()
    grads = (op._empty_like_io(), op._empty_like_io(), op._empty_like_io())
    stream = torch.cuda.current_stream(dev)

    def step():
        op.forward(q, k, v, W, out=O)
        op.backward(q, k, v, W, dO, grads=grads)

    def barrier():
        if world > 1:
            dist.barrier(device_ids=[local])
        torch.cuda.synchronize(dev)

    for _ in range(args.warmup):
        step()
    barrier()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with clock_sampler(dev, local) as clk:
        time.sleep(0.3)
        barrier()
        bd.profile_begin()
        clk.mark(True)
        ev0.record(stream)
        for _ in range(args.steps):
            step()
        ev1.record(stream)
        # wait without holding the interpreter lock, so the clock sampler keeps sampling
        while not ev1.query():
            time.sleep(0.0005)
        barrier()
        clk.mark(False)
        prof = bd.profile_end()
    ms_total = max_over_ranks(ev0.elapsed_time(ev1), dev)
    ms_step = ms_total / args.steps
    tokens_step = w.B * w.N * world
    value = tokens_step / (ms_step * 1e-3)
    launches = sum(c for _, c in prof.values())

    # the same step captured once in a CUDA graph and replayed K times: what is left when
    # the host launch path is taken out (reported beside the eager `value`)
    graph_line = None
    if not args.no_graph:
        side = torch.cuda.Stream(dev)
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            step()
        stream.wait_stream(side)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            step()
        for _ in range(3):
            graph.replay()
        barrier()
        g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        g0.record(stream)
        for _ in range(args.steps):
            graph.replay()
        g1.record(stream)
        barrier()
        tg = max_over_ranks(g0.elapsed_time(g1) / args.steps, dev)
        graph_line = {"ms_per_step": tg, "value": tokens_step / (tg * 1e-3), "unit": UNIT}
        del graph

    # end to end, through the library's host-buffer entry (elsaa_step_host): pinned host
    # inputs in, results (O and the three gradients) out, every step.  Two sets of device
    # inputs and outputs: step i copies its inputs in on an H2D stream, computes on the compute
    # stream and copies its results out on a D2H stream, so step i+1's inputs and step i-1's
    # results cross PCIe (full duplex) while step i computes.  The library orders each set's
    # reuse with the set's three events.
    e2e = None
    if not args.no_e2e:
        names = ("Q", "K", "V", "dO")
        host = {n: inp[n + key].pin_memory() for n in names}
        host_W = inp["W"].pin_memory()
        host_R = inp["R"].pin_memory() if lsh else None
        outs = [[torch.empty(O.shape, dtype=O.dtype).pin_memory() for _ in range(4)] for _ in range(2)]
        h2d = (sum(x.numel() * x.element_size() for x in host.values()) + host_W.numel() * 4
               + (host_R.numel() * 4 if lsh else 0))
        d2h = sum(x.numel() * x.element_size() for x in outs[0])
        dsets = [dict(Q=q, K=k, V=v, dO=dO, W=W),
                 {n: torch.empty_like(t) for n, t in dict(Q=q, K=k, V=v, dO=dO, W=W).items()}]
        osets = [(O,) + grads, tuple(torch.empty_like(O) for _ in range(4))]
        s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        in_ready = [torch.cuda.Event() for _ in range(2)]
        comp_done = [torch.cuda.Event() for _ in range(2)]
        out_done = [torch.cuda.Event() for _ in range(2)]
        for e in in_ready + comp_done + out_done:     # create the events before the first wait
            e.record(stream)
        host_in = [host[n] for n in names] + [host_W] + ([host_R] if lsh else [])

        def e2e_step(i):
            j = i % 2
            d, o = dsets[j], osets[j]
            op.step_host(host_in, outs[j], [d[n] for n in names] + [d["W"]], list(o),
                         (in_ready[j], comp_done[j], out_done[j]), stream, s_in, s_out)

        for i in range(4):
            e2e_step(i)
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        n_e2e = max(4, args.steps // 4)
        e0.record(stream)
        s_in.wait_event(e0)
        for i in range(n_e2e):
            e2e_step(i)
        stream.wait_event(out_done[(n_e2e - 1) % 2])
        stream.wait_event(out_done[n_e2e % 2])
        e1.record(stream)
        barrier()
        te = max_over_ranks(e0.elapsed_time(e1) / n_e2e, dev)
        e2e = {"value": tokens_step / (te * 1e-3), "unit": UNIT,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": te,
               "api": "elsaa_step_host (pinned host buffers, two device sets)",
               "pipelined": "double-buffered: step i+1's H2D and step i-1's D2H overlap step i's compute"}

    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return 0

    model, _ = work_model(w)
    clocks = clk.summary()
    peak_f, peak_f_kind = bf16_peak(peaks, clocks)
    dom = max(prof.items(), key=lambda kv: kv[1][0])[0]
    dom_ms = prof[dom][0] / prof[dom][1]
    wm = model.get(dom)
    roof = None
    if wm is not None:
        # the bound is whichever of the kernel's flops and algorithmic bytes takes longer at peak
        tensor_kernel = wm["flops"] / (peak_f * 1e12) >= wm["bytes"] / (peaks["hbm_gbs"] * 1e9)
        if tensor_kernel:
            ach = wm["flops"] / (dom_ms * 1e-3) / 1e12
            roof = {"bound": "tensor", "achieved": ach, "peak": peak_f, "unit": "TFLOP/s", "frac": ach / peak_f}
            src = f"bf16 {peak_f_kind}"
        else:
            ach = wm["bytes"] / (dom_ms * 1e-3) / 1e9
            roof = {"bound": "hbm", "achieved": ach, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                    "frac": ach / peaks["hbm_gbs"]}
            src = "copy bandwidth"
        roof.update({"kernel": dom, "ms_per_launch": dom_ms,
                     "peak_source": f"{src}, of measured (MEASURED_PEAKS.json)" if peak_kind == "measured"
                     else f"{src}, of fallback",
                     "traffic": dram_traffic(dom, w.name)})
    kernels = {n: {"ms_per_launch": ms / c, "launches": c, "share": ms / sum(x for x, _ in prof.values())}
               for n, (ms, c) in sorted(prof.items(), key=lambda kv: -kv[1][0])}
    for n, kd in kernels.items():
        if n in model:
            kd["tflops"] = model[n]["flops"] / (kd["ms_per_launch"] * 1e-3) / 1e12
            kd["alg_gbs"] = model[n]["bytes"] / (kd["ms_per_launch"] * 1e-3) / 1e9

    cpu = None
    if not args.no_cpu_baseline and world == 1:
        smp = OracleSample(w)
        n_tiles = smp.calibrate(15.0)
        tk, dt = smp.run(n_tiles)
        cpu = {"value": tk / dt, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
               "sample": f"float64 oracle fwd+bwd on {n_tiles} of {w.n_tiles} query tiles of 1 of {w.H} heads "
                         f"({dt:.1f} s), scaled to the full batch"}

    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
            "config": {"workload": w.name, "shape": w.describe(), "global_batch": w.B * world,
                       "seq_len": w.N, "parallelism": f"replicas{world}" if world > 1 else "single",
                       "l2": "inputs larger than L2 (Q, K, V, dO: 4 x %.0f MB)" % (q.numel() * 2 / 1e6)},
            "roofline": roof, "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": launches, "graph": graph_line,
            "clocks": clocks,
            "whole_step_roofline": whole_step_roofline(w, dict(peaks, bf16_tflops=peak_f), ms_step),
            "kernels": kernels}
    print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
