"""Benchmark of the RT-Lynx fused activation-sparse + LoRA linear layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload video] [--impl ours|reference]
    python bench.py --workload dit_mlp   (the feed-forward block of two layers, one GPU)
    python bench.py --workload lora_fit  (the closed-form LoRA fit and the error it removes, one GPU)

One step = one call of the whole layer (sparsify prologue with the LoRA
down-projection, then the sparse GEMM with the LoRA up-projection accumulated
in the same tensor-memory accumulator) on one batch of tokens resident in HBM.
L2 is flushed (a 256 MB write) before every timed step; each step is timed
with CUDA events on the launching stream and the mean over K steps is
reported; under torchrun the max over ranks is taken.  Every rank processes
its own token block with the same weights (tokens are independent, so there
is no data-path collective): scaling is weak.

Prints ONE JSON line (rank 0).  value = dense-equivalent TFLOP/s of the whole
job: (2*M*D_in*D_out + 2*M*R*(D_in+D_out)) * ranks / time.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "fused 2:4 act-sparse+LoRA linear: µs/call, TFLOP/s, speedup vs dense bf16"
FLUSH_BYTES = 256 << 20


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    # the headline: the largest single-GPU configuration (32760 tokens, 5120 -> 13824)
    ap.add_argument("--workload", default="video")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--fp8", action="store_true", help="the layer's FP8 (E4M3) form on the workload's shape")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="target CPU time of the oracle sample")
    return ap.parse_args()


def workload_desc(wl):
    return {"workload": f"{wl.name}: M={wl.M} D_in={wl.D_in} D_out={wl.D_out} R={wl.R}",
            "M": wl.M, "D_in": wl.D_in, "D_out": wl.D_out, "R": wl.R, "p_out": wl.p_out,
            "seed": wl.seed, "x_dist": "GELU(N(0,1)*c)" if wl.gelu else "N(0,1)*c, c~LogNormal(0,1), outliers x10"}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


# ------------------------------------------------------------------ oracle (CPU) timing
def oracle_sample(wl, X, W, L_A, L_B, target_s, min_rows=32):
    """Times the CPU oracle on the first n token rows, n chosen for ~target_s of work."""
    import oracle
    n = min(min_rows, wl.M)
    t0 = time.perf_counter()
    oracle.linear(X, W, L_A, L_B, rows=list(range(n)))
    dt = max(time.perf_counter() - t0, 1e-6)
    n = int(max(min_rows, min(wl.M, n * target_s / dt)))
    t0 = time.perf_counter()
    oracle.linear(X, W, L_A, L_B, rows=list(range(n)))
    dt = time.perf_counter() - t0
    flop = 2 * n * wl.D_in * wl.D_out + 2 * n * wl.R * (wl.D_in + wl.D_out)
    return {"value": flop / dt / 1e12, "unit": "TFLOP/s", "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"first {n} of {wl.M} tokens of the {wl.name} workload (all D_out outputs), "
                      f"{dt:.1f} s wall, fp64 triple loop, OpenMP over tokens"}


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while running."""

    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4, "hw_slowdown": 0x8,
        "sync_boost": 0x10, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
        "hw_power_brake_slowdown": 0x80, "display_clock_setting": 0x100,
    }

    def __init__(self, torch_device):
        self.samples = []
        self.ok = False
        self._stop = threading.Event()
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            uuid = "GPU-" + str(torch.cuda.get_device_properties(torch_device).uuid)
            self.h = pynvml.nvmlDeviceGetHandleByUUID(uuid.encode())
            self.nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # noqa: BLE001
            self.err = repr(e)

    def sample(self):
        if not self.ok:
            return
        try:
            mhz = self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM)
            get = getattr(self.nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                self.nv.nvmlDeviceGetCurrentClocksThrottleReasons
            reasons = get(self.h)
            self.samples.append((mhz, reasons))
        except Exception:  # noqa: BLE001
            pass

    def _run(self):
        while not self._stop.is_set():
            self.sample()
            time.sleep(0.005)

    def start(self):
        self.sample()
        self._t = threading.Thread(target=self._run, daemon=True)
        self._t.start()

    def stop(self):
        self._stop.set()
        self._t.join()
        self.sample()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "note": getattr(self, "err", "no samples")}
        mhz = [m for m, _ in self.samples]
        active = 0
        for _, r in self.samples:
            active |= r
        names = [k for k, v in self.REASONS.items() if active & v and k != "gpu_idle"]
        return {"sm_mhz": statistics.median(mhz), "sm_max_mhz": self.max_mhz, "reasons": names,
                "samples": len(mhz), "sm_mhz_min": min(mhz)}


# ------------------------------------------------------------------ reference arm
def run_reference(args, wl):
    from activation_sparse_gemm_b200.inputs import make_inputs
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    X, W, L_A, L_B = make_inputs(wl)
    import oracle
    oracle.build()
    # rows per step sized so warm-up + K steps stay within a few minutes
    t0 = time.perf_counter()
    oracle.linear(X, W, L_A, L_B, rows=[0, 1])
    per_row = (time.perf_counter() - t0) / 2
    budget = 150.0 / max(1, args.steps + args.warmup)
    n = int(max(1, min(wl.M, budget / max(per_row, 1e-9))))
    rows = list(range(n))
    for _ in range(args.warmup):
        oracle.linear(X, W, L_A, L_B, rows=rows[:1])
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        oracle.linear(X, W, L_A, L_B, rows=rows)
        times.append(time.perf_counter() - t0)
    ms = statistics.mean(times) * 1e3
    flop = 2 * n * wl.D_in * wl.D_out + 2 * n * wl.R * (wl.D_in + wl.D_out)
    value = flop / (ms / 1e3) / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_desc(wl),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": oracle.num_threads(), "kind": "oracle",
                         "sample": f"first {n} of {wl.M} tokens per step (all D_out outputs)"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ our arm
def run_ours(args, wl):
    import numpy as np
    import torch

    import activation_sparse_gemm_b200 as rl
    from activation_sparse_gemm_b200.inputs import make_inputs

    from activation_sparse_gemm_b200 import dist as rdist
    world, rank, local = rdist.env_ranks()
    torch.cuda.set_device(local if world > 1 else 0)
    rdist.init("nccl", timeout_s=120)
    device = torch.device("cuda", torch.cuda.current_device())
    rl.lib()

    X, W, L_A, L_B = make_inputs(wl)

    def dev(a):
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(device)

    Xd, Wd, Ad, Bd = dev(X), dev(W), dev(L_A), dev(L_B)
    M, K, N, R = wl.M, wl.D_in, wl.D_out, wl.R
    Y = torch.empty((M, N), dtype=torch.bfloat16, device=device)
    ws_bytes = rl.rtlynx_workspace_size(M, K, N, R, rl.MODE_SPARSE)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=device)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream()

    barrier = rdist.barrier

    def ev():
        e = torch.cuda.Event(enable_timing=True)
        e.record(stream)
        return e

    def sparse_step(e0=None, e1=None, e2=None, mode=rl.MODE_SPARSE):
        rl.rtlynx_linear_ws_events(Xd, Wd, Ad, Bd, Y, M, K, N, R, mode, ws, ws_bytes, e0, e1, e2, stream)

    # warm-up (also checks the device error word once)
    for _ in range(max(args.warmup, 3)):
        sparse_step()
    if rl.rtlynx_stream_status(stream) != rl.OK:
        raise RuntimeError("device-side error during warm-up")

    def timed(fn, steps, n_events=2):
        """Runs fn(events) steps times with an L2 flush before each; returns per-step event lists."""
        evs = []
        for _ in range(steps):
            flush.fill_(1)
            es = [ev() for _ in range(n_events)]
            evs.append(es)
            fn(es)
        return evs

    clocks = ClockSampler(device)
    barrier()
    torch.cuda.synchronize()
    clocks.start()
    # the headline: whole calls, nothing recorded between the kernels (the
    # kernels launch as programmatic dependents of one another)
    evs = timed(lambda es: sparse_step(es[0], None, es[1]), args.steps, 2)
    torch.cuda.synchronize()
    clocks.stop()
    barrier()
    step_ms = [a.elapsed_time(b) for a, b in evs]
    ms = rdist.max_over_ranks(statistics.mean(step_ms), device)
    # the phase split (an event between prologue and GEMM keeps them apart);
    # a problem on the small path is one kernel, timed whole
    small = rl.rtlynx_schedule_info(M, K, N, R, torch.cuda.get_device_properties(device).multi_processor_count
                                    ).small_path == 1
    if small:
        pro_ms, gemm_ms = [0.0], list(step_ms)
    else:
        pevs = timed(lambda es: sparse_step(es[0], es[1], es[2]), args.steps, 3)
        torch.cuda.synchronize()
        pro_ms = [a.elapsed_time(b) for a, b, c in pevs]
        gemm_ms = [b.elapsed_time(c) for a, b, c in pevs]

    # same-run comparisons (not part of the headline value), each with its own
    # clock record: long dense loops can run into the power cap
    for _ in range(3):
        torch.matmul(Xd, Wd.t(), out=Y)
    cublas_clocks = ClockSampler(device)
    cublas_clocks.start()
    # cuBLAS and our sparse call alternate, each after an L2 flush, so that both
    # run in the same power and clock state: the speedup comes from this loop
    cublas_pairs, ours_pairs = [], []
    for _ in range(args.steps):
        flush.fill_(1)
        a = ev()
        torch.matmul(Xd, Wd.t(), out=Y)
        b = ev()
        cublas_pairs.append((a, b))
        flush.fill_(1)
        es = [ev(), ev()]
        sparse_step(es[0], None, es[1])
        ours_pairs.append(es)
    torch.cuda.synchronize()
    cublas_clocks.stop()
    cublas_ms = statistics.mean(a.elapsed_time(b) for a, b in cublas_pairs)
    ours_alt_ms = statistics.mean(a.elapsed_time(b) for a, b in ours_pairs)
    ours_dense_pairs = []
    for _ in range(max(3, args.warmup)):
        sparse_step(mode=rl.MODE_DENSE_SKIP)
    dense_clocks = ClockSampler(device)
    dense_clocks.start()
    for _ in range(args.steps):
        flush.fill_(1)
        a = ev()
        sparse_step(mode=rl.MODE_DENSE_SKIP)
        b = ev()
        ours_dense_pairs.append((a, b))
    torch.cuda.synchronize()
    dense_clocks.stop()
    ours_dense_ms = statistics.mean(a.elapsed_time(b) for a, b in ours_dense_pairs)

    # end to end through the host-buffer entry point
    Xh = torch.from_numpy(X.view(np.int16)).view(torch.bfloat16).pin_memory()
    Yh = torch.empty((M, N), dtype=torch.bfloat16).pin_memory()
    for _ in range(2):
        rl.rtlynx_linear_host(Xh, Wd, Ad, Bd, Yh, M, K, N, R, rl.MODE_SPARSE, Xd, Y, stream)
    e2e_pairs = []
    for _ in range(args.steps):
        flush.fill_(1)
        a = ev()
        rl.rtlynx_linear_host(Xh, Wd, Ad, Bd, Yh, M, K, N, R, rl.MODE_SPARSE, Xd, Y, stream)
        b = ev()
        e2e_pairs.append((a, b))
    torch.cuda.synchronize()
    e2e_ms = statistics.mean(a.elapsed_time(b) for a, b in e2e_pairs)
    status = rl.rtlynx_stream_status(stream)
    if status != rl.OK:
        raise RuntimeError(f"device-side error: {rl.rtlynx_status_string(status)}")
    e2e_ms = rdist.max_over_ranks(e2e_ms, device)

    flop = wl.dense_equiv_flop
    value = flop * world / (ms / 1e3) / 1e12
    gemm_mean = statistics.mean(gemm_ms)
    gemm_flop = 2 * M * N * K + 2 * M * R * N
    peaks, peaks_kind = load_peaks()
    clock_summary = clocks.summary()
    # A GEMM that runs under the power cap during the timed loop is a kernel
    # timed inside a long step: its denominator is the sustained dense rate.
    sustained = "sw_power_cap" in clock_summary.get("reasons", [])
    dense_peak = peaks["bf16_tflops_sustained"] if sustained else peaks["bf16_tflops"]
    sparse_peak = 2.0 * dense_peak
    achieved = gemm_flop / (gemm_mean / 1e3) / 1e12
    traffic = profiled_traffic(wl.name)
    pro_bytes = 2 * M * K + M * K + M * K // 8 + 4 * M + 2 * M * R + 2 * R * K

    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "us_per_call": ms * 1e3,
        "speedup_vs_dense_bf16": cublas_ms / ours_alt_ms, "dense_bf16_cublas_us": cublas_ms * 1e3,
        "us_per_call_alternating": ours_alt_ms * 1e3,
        "ours_dense_skip_us": ours_dense_ms * 1e3,
        "phases_us": ({"one_kernel": gemm_mean * 1e3} if small else
                      {"sparsify_prologue": statistics.mean(pro_ms) * 1e3, "sparse_gemm_lora": gemm_mean * 1e3}),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded, DiT-shaped; random-init weights)",
        "config": {**workload_desc(wl), "global_batch": M * world,
                   "parallelism": f"token blocks, {world} rank(s), no collective",
                   "l2": "flushed before every timed step (256 MB write)"},
        "e2e": {"value": flop * world / (e2e_ms / 1e3) / 1e12, "unit": "TFLOP/s",
                "h2d_bytes_per_step": M * K * 2, "d2h_bytes_per_step": M * N * 2,
                "us_per_call": e2e_ms * 1e3},
        "gpu_launches": rl.rtlynx_kernel_launches(M, K, N, R, rl.MODE_SPARSE) * args.steps,
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": sparse_peak, "unit": "TFLOP/s",
                     "frac": achieved / sparse_peak, "traffic": traffic,
                     "kernel": "rtlynx_small_kernel" if small else "rtlynx_gemm_pair_kernel<sparse, 240>",
                     "peak_note": f"2 x {peaks_kind} dense bf16 {'sustained' if sustained else 'burst'} "
                                  f"({dense_peak} TFLOP/s; sustained when the timed loop ran under the power cap): "
                                  "2:4 sparse nominal ratio",
                     "frac_of_burst": achieved / (2.0 * peaks["bf16_tflops"])},
        "clocks": clock_summary,
        "comparison_clocks": {"cublas_and_ours_alternating": _clock_brief(cublas_clocks.summary()),
                              "ours_dense_skip": _clock_brief(dense_clocks.summary())},
    }
    if not small:
        # the prologue (both passes) against the HBM roofline: algorithmic bytes
        # are X read, kept values + metadata + s + T written, L_B read once
        pro_gbs = pro_bytes / (statistics.mean(pro_ms) / 1e3) / 1e9
        line["prologue_roofline"] = {
            "bound": "hbm", "bytes": pro_bytes, "achieved": pro_gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": pro_gbs / peaks["hbm_gbs"],
            "note": "phase time from the split loop (an event between prologue and GEMM)"}
    else:
        # one kernel: sparsify, both GEMMs and the epilogue; its bytes (X, W,
        # L_A, L_B read; Y and the workspace copy written) over the call time
        # show how far a problem this small is from any bandwidth roofline
        one_bytes = 2 * M * K + 2 * N * K + 2 * (N * R + R * K) + 2 * M * N + pro_bytes - 2 * M * K - 2 * R * K
        line["small_path"] = {"kernel": "rtlynx_small_kernel", "launches_per_call": 1, "bytes": one_bytes,
                              "achieved_gbs": one_bytes / (ms / 1e3) / 1e9, "peak_gbs": peaks["hbm_gbs"],
                              "frac": one_bytes / (ms / 1e3) / 1e9 / peaks["hbm_gbs"]}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        oracle.build()
        line["cpu_baseline"] = oracle_sample(wl, X, W, L_A, L_B, args.cpu_seconds)
    if rank == 0:
        print(json.dumps(line), flush=True)
    rdist.shutdown()
    return 0


def _clock_brief(summary):
    """Median SM MHz and the throttle reasons seen, from a ClockSampler summary."""
    return {"sm_mhz": summary.get("sm_mhz"), "reasons": summary.get("reasons", [])}


def profiled_traffic(workload):
    """DRAM bytes per GEMM launch from the committed ncu counters of this
    workload (profiles/gemm_sparse_<workload>.json: traffic_bytes_per_launch,
    kernel_rev), or None when there are none or the kernel source changed since."""
    path = os.path.join(ROOT, "profiles", f"gemm_sparse_{workload}.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        fields = json.load(f)
    if fields.get("kernel_rev") != kernel_rev():
        return None
    try:
        return int(fields["traffic_bytes_per_launch"])
    except (KeyError, TypeError, ValueError):
        return None


def run_block(args):
    """The DiT feed-forward block (rtlynx_mlp_block): up-projection with GELU in
    its epilogue, then the down-projection, at the MLP workloads' shape; one
    JSON line.  cuBLAS matmul + torch GELU + matmul on the same tensors is
    timed in the same run."""
    import numpy as np
    import torch

    import activation_sparse_gemm_b200 as rl
    from activation_sparse_gemm_b200.inputs import make_block_inputs

    torch.cuda.set_device(0)
    device = torch.device("cuda", 0)
    rl.lib()
    M, D, D_ff, R = 4608, 3072, 12288, 64
    host = make_block_inputs(M, D, D_ff, R, seed=2)

    def dev(a):
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(device)

    X, W_up, LA_up, LB_up, W_down, LA_down, LB_down = [dev(a) for a in host]
    H = torch.empty((M, D_ff), dtype=torch.bfloat16, device=device)
    Y = torch.empty((M, D), dtype=torch.bfloat16, device=device)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream()

    def ev():
        e = torch.cuda.Event(enable_timing=True)
        e.record(stream)
        return e

    def timed(fn):
        for _ in range(max(args.warmup, 3)):
            fn()
        pairs = []
        for _ in range(args.steps):
            flush.fill_(1)
            a = ev()
            fn()
            b = ev()
            pairs.append((a, b))
        torch.cuda.synchronize()
        return statistics.mean(a.elapsed_time(b) for a, b in pairs)

    def block(mu, md):
        return lambda: rl.rtlynx_mlp_block(X, W_up, LA_up, LB_up, W_down, LA_down, LB_down, H, Y, M, D, D_ff, R,
                                           mu, md, stream)

    clocks = ClockSampler(device)
    clocks.start()
    ms = timed(block(rl.MODE_SPARSE, rl.MODE_SPARSE))
    clocks.stop()
    status = rl.rtlynx_stream_status(stream)
    if status != rl.OK:
        raise RuntimeError(f"device-side error: {rl.rtlynx_status_string(status)}")
    skip_down_ms = timed(block(rl.MODE_SPARSE, rl.MODE_DENSE_SKIP))
    gelu = torch.nn.GELU()

    def cublas_chain():
        torch.matmul(gelu(torch.matmul(X, W_up.t())), W_down.t(), out=Y)

    cublas_ms = timed(cublas_chain)
    flop = 2 * 2 * M * D * D_ff + 2 * 2 * M * R * (D + D_ff)
    launches = (rl.rtlynx_kernel_launches(M, D, D_ff, R, rl.MODE_SPARSE) +
                rl.rtlynx_kernel_launches(M, D_ff, D, R, rl.MODE_SPARSE))
    line = {
        "metric": "DiT feed-forward block (up + GELU + down, both RT-Lynx sparse): us/call, TFLOP/s, "
                  "speedup vs cuBLAS dense chain",
        "value": flop / (ms / 1e3) / 1e12, "unit": "TFLOP/s", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "us_per_call": ms * 1e3, "higher_is_better": True,
        "dense_chain_cublas_us": cublas_ms * 1e3, "speedup_vs_dense_chain": cublas_ms / ms,
        "down_skipped_us": skip_down_ms * 1e3, "dtype": "bf16", "vs_baseline": None,
        "data": "synthetic (seeded, DiT-shaped; random-init weights)",
        "config": {"workload": f"dit_mlp: M={M} D={D} D_ff={D_ff} R={R}", "M": M, "D": D, "D_ff": D_ff, "R": R,
                   "l2": "flushed before every timed step (256 MB write)"},
        "gpu_launches": launches * args.steps, "clocks": clocks.summary(),
    }
    print(json.dumps(line), flush=True)
    return 0


def run_fp8(args, wl):
    """The FP8 (E4M3) form of the layer on a workload's shape: weights prepared
    once (rtlynx_quantize_weight_fp8, outside the timed region, as a model
    would at load time), then rtlynx_linear_fp8 per step; one JSON line.  The
    bf16 sparse layer and cuBLAS's dense FP8 GEMM (torch._scaled_mm, one scale
    per tensor) on the same shape are timed in the same run."""
    import numpy as np
    import torch

    import activation_sparse_gemm_b200 as rl
    from activation_sparse_gemm_b200.inputs import make_inputs

    from activation_sparse_gemm_b200 import dist as rdist
    world, rank, local = rdist.env_ranks()
    if rank != 0:  # a one-GPU measurement: under torchrun only rank 0 runs it
        return 0
    torch.cuda.set_device(local if world > 1 else 0)
    device = torch.device("cuda", torch.cuda.current_device())
    rl.lib()
    X, W, L_A, L_B = make_inputs(wl)
    M, K, N, R = wl.M, wl.D_in, wl.D_out, wl.R

    def dev(a):
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(device)

    Xd, Wd, Ad, Bd = dev(X), dev(W), dev(L_A), dev(L_B)
    W8 = torch.empty((N, K), dtype=torch.uint8, device=device)
    qw = torch.empty((N,), dtype=torch.float32, device=device)
    A8 = torch.empty((N, R), dtype=torch.bfloat16, device=device)
    stream = torch.cuda.current_stream()
    rl.rtlynx_quantize_weight_fp8(Wd, Ad, W8, qw, A8, N, K, R, stream)
    Y = torch.empty((M, N), dtype=torch.bfloat16, device=device)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=device)

    def ev():
        e = torch.cuda.Event(enable_timing=True)
        e.record(stream)
        return e

    def step(e0=None, e1=None, e2=None):
        rl.rtlynx_linear_fp8_events(Xd, W8, qw, A8, Bd, Y, M, K, N, R, e0, e1, e2, stream)

    def timed(fn, n_events=2):
        """fn(events) must record the events itself (the library entry points do)."""
        for _ in range(max(args.warmup, 3)):
            fn([None] * n_events)
        evs = []
        for _ in range(args.steps):
            flush.fill_(1)
            es = [ev() for _ in range(n_events)]
            evs.append(es)
            fn(es)
        torch.cuda.synchronize()
        return evs

    clocks = ClockSampler(device)
    clocks.start()
    evs = timed(lambda es: step(es[0], None, es[1]))
    clocks.stop()
    status = rl.rtlynx_stream_status(stream)
    if status != rl.OK:
        raise RuntimeError(f"device-side error: {rl.rtlynx_status_string(status)}")
    ms = statistics.mean(a.elapsed_time(b) for a, b in evs)
    pevs = timed(lambda es: step(*es), 3)
    pro_ms = statistics.mean(a.elapsed_time(b) for a, b, c in pevs)
    gemm_ms = statistics.mean(b.elapsed_time(c) for a, b, c in pevs)
    ws_bytes = rl.rtlynx_workspace_size(M, K, N, R, rl.MODE_SPARSE)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=device)
    bevs = timed(lambda es: rl.rtlynx_linear_ws_events(Xd, Wd, Ad, Bd, Y, M, K, N, R, rl.MODE_SPARSE, ws, ws_bytes,
                                                       es[0], None, es[1], stream))
    bf16_ms = statistics.mean(a.elapsed_time(b) for a, b in bevs)
    cublas_fp8_us = None
    try:
        xa = Xd.to(torch.float8_e4m3fn)
        wb = Wd.to(torch.float8_e4m3fn)
        one = torch.ones((), dtype=torch.float32, device=device)
        for _ in range(max(args.warmup, 3)):
            torch._scaled_mm(xa, wb.t(), scale_a=one, scale_b=one, out_dtype=torch.bfloat16)
        cpairs = []
        for _ in range(args.steps):
            flush.fill_(1)
            a = ev()
            torch._scaled_mm(xa, wb.t(), scale_a=one, scale_b=one, out_dtype=torch.bfloat16)
            cpairs.append((a, ev()))
        torch.cuda.synchronize()
        cublas_fp8_us = statistics.mean(a.elapsed_time(b) for a, b in cpairs) * 1e3
    except Exception as e:  # the baseline is context only
        cublas_fp8_us = f"unavailable: {type(e).__name__}"
    flop = wl.dense_equiv_flop
    gemm_flop = 2 * M * N * K + 2 * M * R * N
    peaks, peaks_kind = load_peaks()
    peak = 4.0 * peaks["bf16_tflops"]
    achieved = gemm_flop / (gemm_ms / 1e3) / 1e12
    line = {
        "metric": "fused 2:4 act-sparse+LoRA linear, FP8 (E4M3) operands: us/call, TFLOP/s",
        "value": flop / (ms / 1e3) / 1e12, "unit": "TFLOP/s", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "us_per_call": ms * 1e3, "higher_is_better": True,
        "phases_us": {"sparsify_prologue": pro_ms * 1e3, "sparse_gemm_lora": gemm_ms * 1e3},
        "bf16_sparse_layer_us": bf16_ms * 1e3, "speedup_vs_bf16_sparse_layer": bf16_ms / ms,
        "dense_fp8_cublas_us": cublas_fp8_us, "dtype": "e4m3", "vs_baseline": None,
        "data": "synthetic (seeded, DiT-shaped; random-init weights)",
        "config": {**workload_desc(wl), "form": "fp8", "l2": "flushed before every timed step (256 MB write)"},
        "gpu_launches": rl.rtlynx_kernel_launches(M, K, N, R, rl.MODE_SPARSE) * args.steps,
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak, "traffic": None, "kernel": "rtlynx_gemm_pair_kernel<sparse, 224, fp8>",
                     "peak_note": f"4 x {peaks_kind} dense bf16 burst ({peaks['bf16_tflops']} TFLOP/s): "
                                  "fp8 and 2:4 sparse nominal ratios"},
        "clocks": clocks.summary(),
    }
    print(json.dumps(line), flush=True)
    return 0


def run_lora_fit(args):
    """The closed-form LoRA fit at the qkv shape: 4096 calibration tokens of the
    qkv workload, R = 64; seconds per fit (CUDA events) and the relative error
    of the sparse layer against the dense layer (both through the library) on
    the calibration tokens and on 1024 further tokens of the same recipe."""
    import numpy as np
    import torch

    import activation_sparse_gemm_b200 as rl
    from activation_sparse_gemm_b200.inputs import WORKLOADS, make_inputs
    from activation_sparse_gemm_b200.lora_fit import fit_lora

    torch.cuda.set_device(0)
    wl = WORKLOADS["qkv"]
    M_cal, M_test = wl.M, 1024
    X, W, L_A, L_B = make_inputs(wl, M=M_cal + M_test)

    def dev(a):
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda()

    Xd, Wd, Ad, Bd = dev(X), dev(W), dev(L_A), dev(L_B)
    K, N, R = wl.D_in, wl.D_out, wl.R
    Xc, Xt = Xd[:M_cal].contiguous(), Xd[M_cal:].contiguous()
    fit_lora(Xc, Wd, R)  # warm-up (library handles, workspaces)
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record()
    FA, FB = fit_lora(Xc, Wd, R)
    b.record()
    torch.cuda.synchronize()
    fit_s = a.elapsed_time(b) / 1e3

    def rel(Xs, LA, LB):
        M = Xs.shape[0]
        Yd = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        Ys = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        rl.rtlynx_linear(Xs, Wd, None, None, Yd, M, K, N, 0, rl.MODE_DENSE_SKIP)
        rl.rtlynx_linear(Xs, Wd, LA, LB, Ys, M, K, N, R if LA is not None else 0, rl.MODE_SPARSE)
        torch.cuda.synchronize()
        d = Yd.double()
        return float((Ys.double() - d).norm() / d.norm())

    errs = {name: {"no_lora": rel(Xs, None, None), "random_lora": rel(Xs, Ad, Bd), "fitted_lora": rel(Xs, FA, FB)}
            for name, Xs in (("calibration", Xc), ("held_out", Xt))}
    line = {
        "metric": "closed-form LoRA fit (reduced-rank regression on the sparsification residual): "
                  "seconds per fit; relative error of the sparse layer against the dense layer",
        "value": fit_s, "unit": "s", "higher_is_better": False, "n_gpus": 1, "steps": 1, "warmup": 1,
        "rel_err_vs_dense": errs, "dtype": "bf16 layer, f64 fit", "vs_baseline": None,
        "data": "synthetic (seeded qkv recipe: independent tokens, lognormal channel scales, outlier channels)",
        "config": {"workload": f"lora_fit: calibration M={M_cal} held-out M={M_test} D_in={K} D_out={N} R={R}"},
    }
    print(json.dumps(line), flush=True)
    return 0


def kernel_rev():
    """Hash of the GEMM kernel source, to tell whether stored ncu counters still apply."""
    import hashlib
    with open(os.path.join(ROOT, "activation_sparse_gemm_b200", "csrc", "gemm.cu"), "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def main():
    args = parse()
    from activation_sparse_gemm_b200.inputs import WORKLOADS
    if args.workload == "dit_mlp" and args.impl == "ours":
        return run_block(args)
    if args.workload == "lora_fit" and args.impl == "ours":
        return run_lora_fit(args)
    wl = WORKLOADS[args.workload]
    if args.fp8 and args.impl == "ours":
        return run_fp8(args, wl)
    if args.impl == "reference":
        return run_reference(args, wl)
    return run_ours(args, wl)


if __name__ == "__main__":
    sys.exit(main())
