#!/usr/bin/env python
"""Benchmark of the NVFP4 W4A4 matmul on B200 (one JSON line on rank 0).

Workload: the FFN down projection, Y[4096,5376] = A[4096,14336] . W[5376,14336]^T
in NVFP4 (two-level quantisation of N(0,1) activations and N(0,0.02) weights,
seeded).  A step packs the activations' scales into the MMA's layout
(nvfp4_pack_scales) and runs gemm_nvfp4_w4a4_packed on device-resident inputs,
with its last waves of tiles balanced over the SM pairs (stream-K workspace);
the weights' scales are packed once, as at model load.
L2 is flushed (a 256 MiB write) between timed steps, outside the timed events.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

With N > 1 (launched by torchrun, one process per GPU) every rank runs its own
batch of the same shape (data parallel, weak scaling, no collective on the
data path); the per-step device time is the max over ranks.

`--impl reference` times the FP64 CPU oracle instead (rank 0 only; each step is
a bounded sample of rows of the same workload), for the driver's ratio.
`--workload` picks another path for profiling runs only; its line is not the
headline.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "NVFP4 W4A4 GEMM TFLOPS at M4096 N5376 K14336; % of B200 dense FP4 peak"
FP4_PER_BF16 = 9.0 / 2.25          # nominal dense FP4 : BF16 tensor ratio
FP8_PER_BF16 = 4.5 / 2.25          # nominal dense FP8 : BF16 tensor ratio
FALLBACK_BF16_TFLOPS = 1590.0      # used only if MEASURED_PEAKS.json is absent
FALLBACK_HBM_GBS = 6650.0
L2_FLUSH_BYTES = 256 << 20


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=200)
    p.add_argument("--warmup", type=int, default=10)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--workload", choices=list(WORKLOADS), default="ffn_down")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-graph", action="store_true", help="time the eager launches only")
    p.add_argument("--no-other-paths", action="store_true",
                   help="on one GPU, the default FFN-down line also times the other paths "
                        "(short runs, summarised under other_paths); this skips them")
    return p.parse_args()


# the paths the default one-GPU line also times, each in its own short run
OTHER_PATHS = ["grouped", "moe", "w4a8", "via_fp8", "w4a16", "quantize"]


def other_paths(args):
    """{workload: summary} of a short run of each other path (errors recorded, not raised)."""
    out = {}
    for w in OTHER_PATHS:
        sub = argparse.Namespace(**vars(args))
        sub.workload, sub.steps, sub.warmup = w, max(1, min(args.steps, 30)), 3
        sub.no_e2e = sub.no_cpu_baseline = sub.no_other_paths = True
        try:
            d = run_ours(sub, emit=False)
            r = d.get("roofline", {})
            out[w] = {"metric": d["metric"], "value": d["value"], "unit": d["unit"],
                      "ms_per_step": d["ms_per_step"], "steps": d["steps"],
                      "roofline": {k: r.get(k) for k in ("bound", "achieved", "peak", "unit", "frac",
                                                         "traffic", "kernel", "kernel_ms")},
                      "gpu_launches": d.get("gpu_launches"), "clocks": d.get("clocks")}
        except Exception as exc:  # keep the headline line; report what failed
            out[w] = {"error": f"{type(exc).__name__}: {str(exc)[:200]}"}
    return out


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["bf16_tflops"]), float(d.get("hbm_gbs", FALLBACK_HBM_GBS)), "measured"
    except Exception:
        return FALLBACK_BF16_TFLOPS, FALLBACK_HBM_GBS, "fallback"


# Each workload: how to build it, which entry point a step calls, its algorithmic
# work (flops) and bytes, and the roofline that bounds it.
WORKLOADS = {
    "ffn_down": dict(path="w4a4", bound="tensor", desc="FFN down W4A4 4096x5376x14336"),
    "via_fp8": dict(path="via_fp8", bound="alu", desc="FFN down through the exact FP8 path"),
    "w4a8": dict(path="w4a8", bound="tensor_fp8",
                 desc="FFN down W4A8 (E4M3 activations) 4096x5376x14336"),
    "w4a16": dict(path="w4a16", bound="hbm", desc="W4A16 decode 16x5376x14336"),
    "grouped": dict(path="grouped", bound="tensor", desc="grouped MoE W4A4, 8 experts"),
    "tiny": dict(path="w4a4", bound="tensor", desc="tiny W4A4 128x256x256"),
    "quantize": dict(path="quantize", bound="hbm",
                     desc="NVFP4 quantiser of the FFN-down activations, BF16 4096x14336"),
    "moe": dict(path="moe", bound="tensor",
                desc="MoE layer from BF16 tokens (route, quantise into the experts' row order, "
                     "grouped W4A4, combine), 8 experts [14336,4096], 8192 tokens"),
}


def make_workload(name):
    from block_scaled_precision_nvfp4_b200 import workloads as wl
    if name == "tiny":
        return wl.tiny_w4a4(0)
    if name == "w4a16":
        return wl.w4a16_decode()
    if name == "grouped":
        return wl.grouped_w4a4()
    if name == "quantize":
        return wl.activations_bf16()
    if name == "moe":
        return wl.moe_layer()
    if name == "w4a8":
        return wl.w4a8_ffn_down()
    return wl.ffn_down_w4a4()


def algorithmic(wl_, path):
    """(flops, bytes) of one step: 2*M*N*K and every input byte read once plus Y written."""
    M, N, K = wl_.M, wl_.N, wl_.K
    flops = 2.0 * M * N * K
    ybytes = M * N * 2
    if path == "quantize":
        # X read once; codes, packed scales and g written (the two-pass amax reads X twice)
        return 0.0, M * K * 2 + M * K // 2 + M * K // 16 + 4
    if path == "w4a16":
        return flops, N * K // 2 + N * K // 16 + M * K * 2 + ybytes
    if path == "w4a8":
        return flops, N * K // 2 + N * K // 16 + M * K + ybytes
    if path == "grouped":
        return flops, wl_.E * (N * K // 2 + N * K // 16) + M * (K // 2 + K // 16) + ybytes
    if path == "moe":
        # BF16 tokens in, every expert's weights once, Y out
        return flops, M * K * 2 + wl_.E * (N * K // 2 + N * K // 16) + ybytes
    return flops, (M + N) * (K // 2 + K // 16) + ybytes


# --- clock sampling during the timed region (NVML reads only) -------------------------

class ClockSampler:
    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
        0x8: "hw_slowdown", 0x20: "sync_boost", 0x40: "sw_thermal_slowdown",
        0x80: "hw_thermal_slowdown", 0x100: "hw_power_brake_slowdown",
        0x200: "display_clock_setting"}

    def __init__(self, torch_dev):
        self.samples, self.reasons, self.ok = [], 0, False
        self.max_mhz = None
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(torch_dev).uuid)
            self.h = None
            for i in range(pynvml.nvmlDeviceGetCount()):
                h = pynvml.nvmlDeviceGetHandleByIndex(i)
                u = pynvml.nvmlDeviceGetUUID(h)
                u = u.decode() if isinstance(u, bytes) else u
                if u.replace("GPU-", "") == uuid.replace("GPU-", ""):
                    self.h = h
            if self.h is None:
                self.h = pynvml.nvmlDeviceGetHandleByIndex(torch_dev)
            self.nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # pragma: no cover - no NVML
            self.err = str(e)
        self._stop = threading.Event()

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                self.reasons |= int(nv.nvmlDeviceGetCurrentClocksEventReasons(self.h))
            except Exception:
                pass
            time.sleep(0.002)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [],
                    "samples": len(self.samples)}
        names = [n for bit, n in self.REASONS.items() if self.reasons & bit and bit != 0x1]
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": names, "samples": len(self.samples)}


# --- the reference arm: the FP64 oracle on the host cores ------------------------------

def _oracle_rows(wl_, rows):
    """The FP64 oracle on the first `rows` output rows of the workload."""
    import oracle
    if wl_.N == 0:
        from oracle import quantize as oq
        oq.quantize_nvfp4_bf16(wl_.A_bf16[:rows])
        return
    if wl_.expert_ids is not None:
        # the MoE layer on the first `rows` tokens: the quantiser (with the whole tensor's
        # amax), each token through its expert, weight 1 (top-1)
        from oracle import quantize as oq
        amax = float(np.max(np.abs(oq.bf16_to_f32(wl_.A_bf16))))
        codes, scales, g = oq.quantize_nvfp4_bf16(wl_.A_bf16[:rows], amax=amax)
        ids = wl_.expert_ids[:rows, 0]
        for e in range(wl_.E):
            sel = np.nonzero(ids == e)[0]
            if sel.size:
                W = wl_.W_e[e]
                oracle.gemm_w4a4(codes[sel], scales[sel], float(g), W.codes, W.scales, W.g,
                                 sel.size, wl_.N, wl_.K)
        return
    if wl_.A_fp8 is not None:
        oracle.gemm_w4a8(wl_.A_fp8[:rows], wl_.gA, wl_.W.codes, wl_.W.scales, wl_.W.g, rows,
                         wl_.N, wl_.K)
    elif wl_.A_bf16 is not None:
        oracle.gemm_w4a16(wl_.A_bf16[:rows], wl_.W.codes, wl_.W.scales, wl_.W.g, rows, wl_.N,
                          wl_.K)
    elif wl_.E:
        from block_scaled_precision_nvfp4_b200 import workloads as wlm
        Wc, Ws, gW = wlm.stack_experts(wl_)
        r = np.repeat(np.arange(rows), wl_.N)
        c = np.tile(np.arange(wl_.N), rows)
        oracle.gemm_grouped_w4a4(wl_.A.codes, wl_.A.scales, wl_.A.g, Wc, Ws,
                                 gW.astype(np.float64), wl_.offsets, wl_.N, wl_.K, rows=r, cols=c)
    else:
        oracle.gemm_w4a4(wl_.A.codes[:rows], wl_.A.scales[:rows], wl_.A.g, wl_.W.codes,
                         wl_.W.scales, wl_.W.g, rows, wl_.N, wl_.K)


def oracle_rows_for(seconds, wl_, rate_probe_rows=2):
    t0 = time.perf_counter()
    _oracle_rows(wl_, rate_probe_rows)
    rate = rate_probe_rows / max(time.perf_counter() - t0, 1e-6)  # rows per second
    return int(max(1, min(wl_.M, round(rate * seconds))))


def time_oracle(wl_, rows):
    """(throughput in the workload's unit, seconds) of the oracle on `rows` rows."""
    t0 = time.perf_counter()
    _oracle_rows(wl_, rows)
    dt = time.perf_counter() - t0
    if wl_.N == 0:  # the quantiser: GB/s of its algorithmic bytes
        return rows * wl_.K * (2 + 0.5 + 1 / 16) / dt / 1e9, dt
    return 2.0 * rows * wl_.N * wl_.K / dt / 1e12, dt


def cpu_baseline(wl_, seconds=12.0):
    import oracle
    rows = oracle_rows_for(seconds, wl_)
    tflops, dt = time_oracle(wl_, rows)
    return {"value": tflops, "unit": "GB/s" if wl_.N == 0 else "TFLOP/s",
            "cores": oracle.default_threads(),
            "kind": "oracle",
            "sample": (f"first {rows} of {wl_.M} rows of X ({rows}x{wl_.K}), {dt:.1f} s" if wl_.N == 0 else
                       f"first {rows} of {wl_.M} rows of Y ({rows}x{wl_.N}x{wl_.K}), {dt:.1f} s")}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import oracle
    wl_ = make_workload(args.workload)
    rows = oracle_rows_for(1.0, wl_)
    for _ in range(args.warmup):
        time_oracle(wl_, rows)
    times = []
    for _ in range(args.steps):
        _, dt = time_oracle(wl_, rows)
        times.append(dt)
    t = sum(times) / len(times)
    value = 2.0 * rows * wl_.N * wl_.K / t / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": t * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": wl_.name, "M": wl_.M, "N": wl_.N, "K": wl_.K,
                   "sample_rows_per_step": rows},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "kind": "oracle",
                         "cores": oracle.default_threads(),
                         "sample": f"first {rows} of {wl_.M} rows of Y per step"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# --- our arm ---------------------------------------------------------------------------

# the sources that define each workload's dominant kernel (the stored ncu traffic
# of a kernel is used only while these are unchanged)
KERNEL_SOURCES = {
    "w4a4": ["w4a4_pair_kernel.cuh", "w4a4_kernel.cuh", "ptx.cuh"],
    "via_fp8": ["via_fp8_kernel.cuh", "ptx.cuh"],
    "w4a8": ["w4a8_kernel.cuh", "via_fp8_kernel.cuh", "ptx.cuh"],
    "w4a16": ["w4a16_kernel.cuh"],
    "grouped": ["grouped_pair_kernel.cuh", "w4a4_pair_kernel.cuh", "w4a4_kernel.cuh", "ptx.cuh"],
    "moe": ["grouped_pair_kernel.cuh", "w4a4_pair_kernel.cuh", "w4a4_kernel.cuh", "ptx.cuh",
            "moe_kernel.cuh", "quantize_kernel.cuh"],
    "quantize": ["quantize_kernel.cuh", "ptx.cuh"],
}


# The per-update FP32 work of the exact paths' scale-apply, measured on the device
# itself: a kernel of independent chains, each step one scale product and one FMA
# into an accumulator (no loop-invariant operand a compiler could hoist), written
# once with scalar FP32 instructions and once with packed f32x2 ones.  The larger
# rate is the roofline's peak.
APPLY_PEAK_SRC = r"""
#include <cstdio>
#include <cstdint>
#include <cuda_runtime.h>
template <int PACKED>
__global__ void __launch_bounds__(256, 1) apply_peak(float* out, int iters, long long* cyc) {
    uint64_t a[16], sc[16];
    const uint64_t p = 0x3f8000013f800001ull;
    const uint64_t c = 0x3f8000003f800000ull ^ (uint64_t)(threadIdx.x & 1);
    for (int j = 0; j < 16; ++j) { a[j] = (uint64_t)(threadIdx.x + j) * 0x0000000100000001ull; sc[j] = 0x3f0000003f000000ull + j; }
    const long long t0 = clock64();
    for (int i = 0; i < iters; ++i) {
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            if (PACKED) {
                asm volatile("mul.rn.f32x2 %0, %0, %1;" : "+l"(sc[j]) : "l"(c));
                asm volatile("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(a[j]) : "l"(p), "l"(sc[j]));
            } else {
                float s0 = __uint_as_float((uint32_t)sc[j]), s1 = __uint_as_float((uint32_t)(sc[j] >> 32));
                float x0 = __uint_as_float((uint32_t)a[j]), x1 = __uint_as_float((uint32_t)(a[j] >> 32));
                asm volatile("mul.rn.f32 %0, %0, %1;" : "+f"(s0) : "f"(__uint_as_float((uint32_t)c)));
                asm volatile("mul.rn.f32 %0, %0, %1;" : "+f"(s1) : "f"(__uint_as_float((uint32_t)c)));
                asm volatile("fma.rn.f32 %0, %1, %2, %0;" : "+f"(x0) : "f"(1.0000001f), "f"(s0));
                asm volatile("fma.rn.f32 %0, %1, %2, %0;" : "+f"(x1) : "f"(1.0000001f), "f"(s1));
                sc[j] = (uint64_t)__float_as_uint(s0) | ((uint64_t)__float_as_uint(s1) << 32);
                a[j] = (uint64_t)__float_as_uint(x0) | ((uint64_t)__float_as_uint(x1) << 32);
            }
        }
    }
    const long long t1 = clock64();
    uint64_t x = 0;
    for (int j = 0; j < 16; ++j) x ^= a[j] ^ sc[j];
    out[blockIdx.x * blockDim.x + threadIdx.x] = (float)(x & 0xffff);
    if (threadIdx.x == 0) cyc[blockIdx.x] = t1 - t0;
}
template <int PACKED> double rate(int sms, float* out, long long* cyc) {
    const int iters = 4096, threads = 256;
    apply_peak<PACKED><<<sms, threads>>>(out, 2, cyc);
    apply_peak<PACKED><<<sms, threads>>>(out, iters, cyc);
    if (cudaDeviceSynchronize() != cudaSuccess) return -1.0;
    long long h[1024];
    cudaMemcpy(h, cyc, sizeof(long long) * sms, cudaMemcpyDeviceToHost);
    double mx = 0;
    for (int b = 0; b < sms; ++b) mx = h[b] > mx ? (double)h[b] : mx;
    return 32.0 * threads * iters / mx;  // updates per clock per SM (two per j per thread)
}
int main() {
    int sms = 0;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, 0);
    float* out; long long* cyc;
    if (cudaMalloc(&out, sizeof(float) * sms * 256) != cudaSuccess || cudaMalloc(&cyc, 8 * 1024) != cudaSuccess) return 1;
    printf("scalar %.2f\npacked %.2f\n", rate<0>(sms, out, cyc), rate<1>(sms, out, cyc));
    return 0;
}
"""


def measure_apply_peak():
    """Scale-apply updates per clock per SM (scalar, packed), from APPLY_PEAK_SRC compiled
    with nvcc into _build/ (cached by source hash) and run on the current device."""
    import subprocess
    h = hashlib.sha256(APPLY_PEAK_SRC.encode()).hexdigest()[:16]
    d = os.path.join(ROOT, "_build")
    os.makedirs(d, exist_ok=True)
    exe = os.path.join(d, f"apply_peak_{h}")
    if not os.path.exists(exe):
        src = exe + ".cu"
        with open(src, "w") as f:
            f.write(APPLY_PEAK_SRC)
        nvcc = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
        subprocess.check_call([nvcc if os.path.exists(nvcc) else "nvcc", "-gencode",
                               "arch=compute_100a,code=sm_100a", "-O3", "-o", exe, src])
    out = subprocess.run([exe], capture_output=True, text=True, timeout=120, check=True).stdout
    vals = dict(line.split() for line in out.strip().splitlines())
    return float(vals["scalar"]), float(vals["packed"])


def kernel_source_hash(path):
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "block_scaled_precision_nvfp4_b200", "csrc")
    for n in KERNEL_SOURCES[path]:
        with open(os.path.join(csrc, n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(workload_name, path):
    """DRAM bytes per launch from the committed ncu summary, if it matches this source."""
    fn = os.path.join(ROOT, "profiles", f"traffic_{path}_{workload_name}.txt")
    if not os.path.exists(fn):
        fn = os.path.join(ROOT, "profiles", f"traffic_{workload_name}.txt")
    try:
        kv = {}
        with open(fn) as f:
            for ln in f:
                if ":" in ln:
                    k, v = ln.split(":", 1)
                    kv[k.strip()] = v.strip()
        if kv.get("source_hash") == kernel_source_hash(path):
            return float(kv["dram_bytes_per_launch"])
    except Exception:
        pass
    return None


def run_ours(args, emit=True):
    import torch
    import torch.distributed as dist
    import block_scaled_precision_nvfp4_b200 as nv
    from block_scaled_precision_nvfp4_b200 import workloads as wlm

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        torch.cuda.set_device(local)
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local if world > 1 else torch.cuda.current_device())
    torch.cuda.set_device(dev)
    nv.load_library(build_if_missing=False)

    spec = WORKLOADS[args.workload]
    path = spec["path"]
    wl_ = make_workload(args.workload)
    M, N, K = wl_.M, wl_.N, wl_.K
    flops, alg_bytes = algorithmic(wl_, path)

    def dev_(x):
        return torch.from_numpy(np.ascontiguousarray(x)).to(dev)

    # host copies of the inputs (pinned) and their device twins
    if path == "quantize":
        host = [wl_.A_bf16.view(np.int16)]
    elif path == "w4a16":
        host = [wl_.A_bf16.view(np.int16), wl_.W.codes, wl_.W.scales]
    elif path == "w4a8":
        host = [wl_.A_fp8, wl_.W.codes, wl_.W.scales]
    elif path == "moe":
        host = [wl_.A_bf16.view(np.int16), wl_.expert_ids]     # per-step inputs only
    elif path == "grouped":
        Wc, Ws, gW = wlm.stack_experts(wl_)
        host = [wl_.A.codes, wl_.A.scales, Wc, Ws]
    else:
        host = [wl_.A.codes, wl_.A.scales, wl_.W.codes, wl_.W.scales]
    dv = [dev_(h) for h in host]
    Y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    if path == "quantize":
        xq = dv[0].view(torch.bfloat16)
        q_ws = torch.empty(16, dtype=torch.uint8, device=dev)
        # codes, scales in the product's packed layout, and g (what the product consumes)
        Y = torch.empty((M, K // 2), dtype=torch.uint8, device=dev)
        q_out = (Y, None, torch.empty(nv.nvfp4_scale_layout_bytes(M, K), dtype=torch.uint8,
                                      device=dev), torch.empty(4, dtype=torch.float32, device=dev))

        def step():
            nv.nvfp4_quantize_bf16(xq, plain=False, packed=True, workspace=q_ws, stream=stream,
                                   out=q_out)
    elif path == "w4a16":
        a16 = dv[0].view(torch.bfloat16)
        def step():
            nv.gemm_w4a16(a16, dv[1], dv[2], wl_.W.g, out=Y, stream=stream)
    elif path == "grouped":
        # weight scales packed once per expert (model load); each step packs the routed
        # tokens' scales per expert and runs the grouped product on pairs of SMs
        gw_list = [float(x) for x in gW]
        offs = [int(x) for x in wl_.offsets]
        E = len(gw_list)
        sw_packed = nv.nvfp4_pack_scales_grouped(dv[3].view(E * N, K // 16),
                                                 [e * N for e in range(E + 1)], K, stream=stream)
        sa_packed = torch.empty(nv.nvfp4_grouped_scale_layout_bytes(offs, K), dtype=torch.uint8,
                                device=dev)

        def step(mid=None, s=None):
            s = s or stream
            nv.nvfp4_pack_scales_grouped(dv[1], offs, K, out=sa_packed, stream=s)
            if mid is not None:
                mid.record(s)
            nv.gemm_nvfp4_w4a4_grouped_packed(dv[0], sa_packed, wl_.A.g, dv[2], sw_packed,
                                              gw_list, offs, out=Y, stream=s)

        def plain_step():
            nv.gemm_nvfp4_w4a4_grouped(dv[0], dv[1], wl_.A.g, dv[2], dv[3], gw_list, offs,
                                       out=Y, stream=stream)
    elif path == "moe":
        # expert weights resident, their scales packed once (model load)
        Wc_h, Ws_h, gW_h = wlm.stack_experts(wl_)
        E = wl_.E
        Wc_d, Ws_d = dev_(Wc_h), dev_(Ws_h)
        gws = [float(x) for x in gW_h]
        sw_packed = nv.nvfp4_pack_scales_grouped(Ws_d.view(E * N, K // 16),
                                                 [e * N for e in range(E + 1)], K, stream=stream)
        q_ws = torch.empty(16, dtype=torch.uint8, device=dev)
        g_b = torch.empty(4, dtype=torch.float32, device=dev)
        route_ws = torch.empty(nv.load_library().nvfp4_moe_route_workspace_bytes(M, E),
                               dtype=torch.uint8, device=dev)
        gc_b = torch.empty((M, K // 2), dtype=torch.uint8, device=dev)    # codes, experts' order
        gs_b = torch.empty((M, K // 16), dtype=torch.uint8, device=dev)   # scales, experts' order
        ones = torch.ones((M, 1), dtype=torch.float32, device=dev)

        sa_b = torch.empty(nv.load_library().nvfp4_grouped_scale_layout_bytes_bound(M, E, K),
                           dtype=torch.uint8, device=dev)

        def step(stages=None, s=None):
            # the whole layer on the device: the grouped product is planned from the
            # route's device offsets and the quantiser's device gA, so no host round trip
            s = s or stream

            def mark(i):
                if stages is not None:
                    stages[i].record(s)
            mark(0)
            off, dest, src = nv.moe_route(dv[1], E, workspace=route_ws, stream=s)
            mark(1)
            # the quantiser writes each token's codes and scales straight to its row in
            # the experts' order (the dispatch permutation, fused)
            nv.nvfp4_quantize_bf16_routed(dv[0].view(torch.bfloat16), dest, 1, workspace=q_ws,
                                          stream=s, out=(gc_b, gs_b, g_b))
            mark(2)
            sched = nv.GroupedSchedule(off, E, M, N, K, gws, gA=g_b[:1], stream=s)
            sched.pack(gs_b, out=sa_b, stream=s)
            mark(3)
            # top-1: the combine (weight, then each row to its token) is fused into the
            # grouped product's epilogue, so the expert-order rows never reach memory
            sched.gemm_combine(gc_b, sa_b, Wc_d, sw_packed, src, M, weights=ones, out=Y, stream=s)
            mark(4)
    elif path == "w4a8":
        def step():
            nv.gemm_nvfp4_w4a8(dv[0], wl_.gA, dv[1], dv[2], wl_.W.g, out=Y, stream=stream)
    elif path == "via_fp8":
        def step():
            nv.gemm_nvfp4_via_fp8(dv[0], dv[1], wl_.A.g, dv[2], dv[3], wl_.W.g, out=Y, stream=stream)
    else:
        # W4A4: the weights' scales are packed once (model load); each step packs the
        # activations' scales and runs the product on pairs of SMs.
        # With a workspace, the product balances its last waves of tiles over the SM
        # pairs (stream-K); the workspace is allocated and zeroed once.
        sw_packed = nv.nvfp4_pack_scales(dv[3], K, stream=stream)
        sa_packed = torch.empty(nv.nvfp4_scale_layout_bytes(M, K), dtype=torch.uint8, device=dev)
        pair_ws = nv.w4a4_packed_workspace(M, N, K, device=dev)
        mid_events = []

        def step(mid=None, s=None):
            s = s or stream
            nv.nvfp4_pack_scales(dv[1], K, out=sa_packed, stream=s)
            if mid is not None:
                mid.record(s)
            nv.gemm_nvfp4_w4a4_packed(dv[0], sa_packed, wl_.A.g, dv[2], sw_packed, wl_.W.g,
                                      out=Y, stream=s, workspace=pair_ws)

        def plain_step():
            nv.gemm_nvfp4_w4a4(dv[0], dv[1], wl_.A.g, dv[2], dv[3], wl_.W.g, out=Y, stream=stream)
    launches_per_step = {"w4a16": (M + 15) // 16, "w4a4": 2, "grouped": 2, "quantize": 2,
                         "moe": 6}.get(path, 1)

    for _ in range(max(3, args.warmup)):
        flush.zero_()
        step()
    torch.cuda.synchronize(dev)
    nv.nvfp4_check_device_error(stream)

    # The multi-launch steps (pack the activations' scales, then the product; the whole
    # MoE layer) are also captured once in a CUDA graph; its replay times the same
    # kernels without the host launch gaps between them, and gives `value`.  The eager
    # loop below still times the product (and the MoE stages) between events.
    graph, launch = None, "eager"
    # (the two-kernel steps launch the product with programmatic dependent launch,
    # which overlaps its set-up with the scale packing; replayed from a graph they
    # measured slower than launched eagerly, so only the MoE layer replays a graph)
    if path in ("moe",) and not args.no_graph:
        try:
            gstream = torch.cuda.Stream(dev)
            gstream.wait_stream(stream)
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph, stream=gstream):
                step(s=gstream)
            torch.cuda.synchronize(dev)
            for _ in range(3):
                flush.zero_()
                graph.replay()
            torch.cuda.synchronize(dev)
            nv.nvfp4_check_device_error(stream)
            launch = "cuda_graph"
        except Exception as exc:  # report it and time the eager steps
            graph, launch = None, f"eager (graph capture failed: {str(exc)[:80]})"

    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    mids = ([torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
            if path in ("w4a4", "grouped") else None)
    stage_ev = ([[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(args.steps)]
                if path == "moe" else None)
    gstarts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    gends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    with ClockSampler(dev.index) as clk:
        # `value` times whole steps with nothing between their kernels (an event recorded
        # between the scale packing and the product would stop the product's launch from
        # overlapping the packing), or the graph replay.  Those steps alternate with the
        # steps that carry the per-kernel events, so that both see the same clocks and
        # temperature over a long run.
        for i in range(args.steps):
            flush.zero_()
            starts[i].record(stream)
            if mids is not None:
                step(mids[i])
            elif stage_ev is not None:
                step(stage_ev[i])
            else:
                step()
            ends[i].record(stream)
            if graph is not None or mids is not None:
                flush.zero_()
                gstarts[i].record(stream)
                if graph is not None:
                    graph.replay()
                else:
                    step()
                gends[i].record(stream)
        torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    nv.nvfp4_check_device_error(stream)
    per_step = [s.elapsed_time(e) for s, e in zip(starts, ends)]  # ms
    eager_ms = sum(per_step) / len(per_step)   # with the stage events (MoE, W4A4, grouped)
    if graph is not None or mids is not None:
        per_step = [s.elapsed_time(e) for s, e in zip(gstarts, gends)]
    t_ms = sum(per_step) / len(per_step)
    if world > 1:
        tt = torch.tensor([t_ms], dtype=torch.float64, device=dev)
        dist.all_reduce(tt, op=dist.ReduceOp.MAX)
        t_ms = float(tt.item())
    value = world * flops / (t_ms * 1e-3) / 1e12
    if path == "quantize":  # no flops: whole-job GB/s of the algorithmic bytes
        value = world * alg_bytes / (t_ms * 1e-3) / 1e9

    # End to end through the public API, as a serving loop runs it: the weights are
    # resident (loaded once, like model weights); every step copies its activations in
    # from pinned host memory, runs, and copies its output back.  Two buffer sets and two
    # copy streams let step i+1's input copy and step i-1's output copy overlap step i.
    e2e = None
    if not args.no_e2e:
        n_act = {"quantize": 1, "w4a16": 1, "w4a8": 1}.get(path, 2)   # activations lead `host`
        hp = [torch.from_numpy(np.ascontiguousarray(h)).pin_memory() for h in host[:n_act]]
        dsets = [list(dv[:n_act]), [torch.empty_like(d) for d in dv[:n_act]]]
        Ysets = [Y, torch.empty_like(Y)]
        hYs = [torch.empty(tuple(Y.shape), dtype=Y.dtype).pin_memory() for _ in range(2)]
        qsets = None
        if path == "quantize":
            qsets = [q_out, (Ysets[1], None, torch.empty_like(q_out[2]), torch.empty_like(q_out[3]))]
        copy_in, copy_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        in_ready = [torch.cuda.Event() for _ in range(2)]
        comp_done = [torch.cuda.Event() for _ in range(2)]
        out_done = [torch.cuda.Event() for _ in range(2)]
        e_steps = max(2, min(args.steps, 20))

        def e2e_step(i):
            nonlocal Y, xq, q_out, a16
            b = i % 2
            copy_in.wait_event(comp_done[b])          # step i-2 has finished reading set b
            with torch.cuda.stream(copy_in):
                for d, h in zip(dsets[b], hp):
                    d.copy_(h, non_blocking=True)
                in_ready[b].record(copy_in)
            stream.wait_event(in_ready[b])
            stream.wait_event(out_done[b])            # step i-2's output has left set b
            dv[:n_act] = dsets[b]
            Y = Ysets[b]
            if path == "quantize":
                xq, q_out = dsets[b][0].view(torch.bfloat16), qsets[b]
            if path == "w4a16":
                a16 = dsets[b][0].view(torch.bfloat16)
            step()
            comp_done[b].record(stream)
            copy_out.wait_event(comp_done[b])
            with torch.cuda.stream(copy_out):
                hYs[b].copy_(Ysets[b], non_blocking=True)
                out_done[b].record(copy_out)

        for i in range(2):
            e2e_step(i)
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        e0 = torch.cuda.Event(enable_timing=True); e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        copy_in.wait_event(e0)
        for i in range(e_steps):
            e2e_step(i)
        for b in range(2):
            stream.wait_event(out_done[b])            # the last outputs are on the host
        e1.record(stream)
        torch.cuda.synchronize(dev)
        te = e0.elapsed_time(e1) / e_steps
        if world > 1:
            tt = torch.tensor([te], dtype=torch.float64, device=dev)
            dist.all_reduce(tt, op=dist.ReduceOp.MAX)
            te = float(tt.item())
        dv[:n_act] = dsets[0]
        Y = Ysets[0]
        h2d = sum(x.numel() * x.element_size() for x in hp)
        e2e = {"value": (world * alg_bytes / (te * 1e-3) / 1e9 if path == "quantize"
                         else world * flops / (te * 1e-3) / 1e12),
               "unit": "GB/s" if path == "quantize" else "TFLOP/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": hYs[0].numel() * hYs[0].element_size(),
               "ms_per_step": te,
               "note": "weights resident; activations in and output out every step, "
                       "two buffer sets, copies on two streams overlapping compute"}

    bf16_peak, hbm_peak, peak_src = peaks()
    kern_s = t_ms * 1e-3
    extra = {}
    if mids is not None:
        # the dominant kernel alone (the product), and the plain-scale entry point for context
        gemm_ms = [m.elapsed_time(e) for m, e in zip(mids, ends)]
        kern_s = (sum(gemm_ms) / len(gemm_ms)) * 1e-3
        pack_ms = [s_.elapsed_time(m) for s_, m in zip(starts, mids)]
        p0 = torch.cuda.Event(enable_timing=True); p1 = torch.cuda.Event(enable_timing=True)
        plain = []
        for _ in range(10):
            flush.zero_()
            p0.record(stream)
            plain_step()
            p1.record(stream)
            torch.cuda.synchronize(dev)
            plain.append(p0.elapsed_time(p1))
        extra = {"pack_activation_scales_ms": statistics.median(pack_ms),
                 "gemm_packed_ms": statistics.median(gemm_ms),
                 "plain_scale_entry_ms": statistics.median(plain),
                 "plain_scale_entry_tflops": flops / (statistics.median(plain) * 1e-3) / 1e12}
    if stage_ev is not None:
        names = ["route", "quantize_dispatched", "schedule_and_pack", "grouped_gemm_and_combine"]
        med = {n: statistics.median(ev[j].elapsed_time(ev[j + 1]) for ev in stage_ev) * 1e3
               for j, n in enumerate(names)}
        kern_s = med["grouped_gemm_and_combine"] * 1e-6
        extra = {"stage_us": med}
    kernel_name = {"w4a4": "w4a4_pair_kernel", "via_fp8": "via_fp8_kernel", "w4a8": "w4a8_kernel",
                   "moe": "grouped_pair_kernel",
                   "w4a16": "w4a16_ldg_kernel", "grouped": "grouped_pair_kernel",
                   "quantize": "quantize_bf16_kernel (+ amax_bf16_kernel)"}[path]
    if spec["bound"] == "tensor_fp8":
        # the W4A8 kernel runs three E4M3 x E5M2 MMAs per K step (one per signed digit of
        # the weight group scale): algorithmic work 2MNK against the FP8 dense peak, and
        # the tensor work actually issued (x3) for context
        fp8_peak = bf16_peak * FP8_PER_BF16
        achieved = flops / kern_s / 1e12
        roof = {"bound": "tensor", "achieved": achieved, "peak": fp8_peak, "unit": "TFLOP/s",
                "frac": achieved / fp8_peak,
                "peak_note": f"{peak_src} bf16 {bf16_peak:.1f} TFLOP/s x nominal fp8/bf16 2",
                "issued_tflops": 3 * achieved, "issued_frac": 3 * achieved / fp8_peak}
    elif spec["bound"] == "tensor":
        fp4_peak = bf16_peak * FP4_PER_BF16
        achieved = flops / kern_s / 1e12
        roof = {"bound": "tensor", "achieved": achieved, "peak": fp4_peak, "unit": "TFLOP/s",
                "frac": achieved / fp4_peak,
                "peak_note": f"{peak_src} bf16 {bf16_peak:.1f} TFLOP/s x nominal fp4/bf16 4"}
    elif spec["bound"] == "hbm":
        achieved = alg_bytes / kern_s / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                "frac": achieved / hbm_peak, "peak_note": f"{peak_src} copy bandwidth",
                "algorithmic_bytes": alg_bytes}
        # context: a plain library copy of the same bytes (the input of the path's main
        # stream) under the same L2 flush, counted as read + write like the measured copy
        # peak: the 256 MiB flush write leaves L2 dirty, and the misses of a short kernel
        # must write those lines back, so this is the practical ceiling of the regime
        wsrc = dv[0] if path == "quantize" else dv[1]
        wdst = torch.empty_like(wsrc)
        r0 = torch.cuda.Event(enable_timing=True); r1 = torch.cuda.Event(enable_timing=True)
        reads = []
        for _ in range(10):
            flush.zero_()
            r0.record(stream)
            wdst.copy_(wsrc)
            r1.record(stream)
            torch.cuda.synchronize(dev)
            reads.append(r0.elapsed_time(r1))
        rd = statistics.median(reads)
        nbytes = wsrc.numel() * wsrc.element_size()
        extra = {"copy_same_bytes_same_flush_us": rd * 1e3,
                 "copy_same_bytes_same_flush_gbs": 2 * nbytes / (rd * 1e-3) / 1e9,
                 "copy_note": ("torch copy of the " + ("input activations" if path == "quantize"
                                                       else "weight codes")
                               + " after the same flush; GB/s counts read + write")}
    else:
        # The W4A4 exact path does two FP32 operations per (row, column, group) update:
        # the scale product and the FMA into the accumulator; its peak is the measured
        # rate of that pair on this device, scalar or packed, whichever is higher, at the
        # maximum SM clock.  The W4A8 path's FP32 work is one FMA per update; its peak is
        # SMs x 128 FP32 lanes x max clock.
        sms = torch.cuda.get_device_properties(dev).multi_processor_count
        clk_mhz = clk.summary().get("sm_max_mhz") or 1965
        if path == "w4a8":
            per_clk, note = 128.0, "one FMA per update: SMs x 128 FP32 lanes x max clock"
        else:
            scalar, packed = measure_apply_peak()
            per_clk = max(scalar, packed)
            note = (f"measured scale product + FMA per update on this device: {scalar:.1f} "
                    f"(scalar FP32) / {packed:.1f} (packed f32x2) updates per clock per SM; "
                    f"peak = SMs x the larger x max clock")
        peak_upd = sms * per_clk * clk_mhz * 1e6 / 1e12  # T updates / s
        achieved = (M * N * K / 16) / kern_s / 1e12
        roof = {"bound": "alu", "achieved": achieved, "peak": peak_upd,
                "unit": "Tupdate/s", "frac": achieved / peak_upd, "peak_note": note}
    roof.update({"traffic": profiled_traffic(wl_.name, path), "kernel": kernel_name,
                 "kernel_ms": kern_s * 1e3})
    roof.update(extra)
    line = {
        "metric": (METRIC if args.workload == "ffn_down" else
                   f"{spec['desc']} " + ("GB/s" if path == "quantize" else "TFLOP/s")),
        "value": value, "unit": "GB/s" if path == "quantize" else "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": t_ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "step_ms_stats": {"median": statistics.median(per_step), "min": min(per_step),
                          "p90": sorted(per_step)[min(len(per_step) - 1, int(0.9 * len(per_step)))]},
        "dtype": ("bf16 -> nvfp4 (fp32 scale arithmetic)" if path == "quantize" else
                  "bf16 x nvfp4(e2m1, e4m3 group scales) -> f32 accumulate -> bf16"
                  if path == "w4a16" else
                  "e4m3 x nvfp4(e2m1, e4m3 group scales) -> f32 accumulate -> bf16"
                  if path == "w4a8" else
                  "bf16 -> nvfp4 -> grouped nvfp4 x nvfp4 -> f32 -> x routing weight -> bf16 "
                  "(top-1 combine fused)"
                  if path == "moe" else
                  "nvfp4(e2m1 x e2m1, e4m3 group scales) -> f32 accumulate -> bf16"),
        "data": "synthetic",
        "config": {"workload": wl_.name, "M": M, "N": N, "K": K, "global_batch": world * M,
                   "parallelism": f"dp{world}", "l2": "flushed between timed steps (256 MiB write)",
                   "launch": launch, "eager_ms_per_step": eager_ms,
                   "inputs": wl_.notes, "algorithmic_bytes": alg_bytes,
                   **({"tile_balance": "stream-K over the last waves" if pair_ws is not None
                       else "whole tiles"} if path == "w4a4" else {})},
        "roofline": roof,
        "gpu_launches": args.steps * launches_per_step,
        "clocks": clk.summary(),
        "e2e": e2e,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(wl_)
    graph = None  # release the captured step before the process group goes
    if (emit and world == 1 and args.workload == "ffn_down"
            and not getattr(args, "no_other_paths", False)):
        line["other_paths"] = other_paths(args)
    if rank == 0 and emit:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return line


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    run_ours(args)
    return 0


if __name__ == "__main__":
    sys.exit(main())
