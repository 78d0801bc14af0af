"""Benchmark of the NVFP4 W4A4 hot path on B200.

One step = dynamic NVFP4 quantization of the activations (amax pass +
quantize/pack) followed by the block-scaled W4A4 GEMM against statically
max-quantized weights, on the dense transformer MLP workload
X[4096 x 5120] (Student-t df=3 * 0.5) x W_up[17408 x 5120]^T -> BF16.
Metric: quant+GEMM TFLOP/s (2*M*N*K per step). Every other hot-path row
(four_over_six calibration, fake-quant, lm_head decode GEMM, routed-expert
MoE) is measured on its own workload in the "rows" object of the same line.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
For N > 1 launch with torch.distributed.run; each rank runs an independent
replica on its own GPU (weak scaling, no data-path collective).
"""
from __future__ import annotations

import argparse
import glob
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "W4A4 NVFP4 quant+GEMM TFLOPS & % of FP4 tensor peak; quantize GB/s vs HBM"
UNIT = "TFLOP/s"
DENSE = dict(M=4096, N=17408, K=5120)
L2_FLUSH_BYTES = 512 << 20  # 256 MiB written + 256 MiB read (flush_l2)
FP4_OVER_BF16 = 4.0          # nominal dense ratio (9 PF FP4 / 2.25 PF BF16)
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0


# ----------------------------------------------------------------------------- helpers

def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return dict(hbm=float(p["hbm_gbs"]), bf16=float(p["bf16_tflops"]),
                    bf16_sustained=float(p.get("bf16_tflops_sustained", p["bf16_tflops"])), source="measured")
    return dict(hbm=FALLBACK_HBM_GBS, bf16=FALLBACK_BF16_TFLOPS, bf16_sustained=1400.0, source="fallback")


KERNEL_SOURCES = {
    "gemm_dense_mlp": ["common.cuh", "gemm_kernel.cuh", "gemm.cu"],
    "quantize_dense_mlp": ["common.cuh", "block_math.cuh", "kernels.h", "quantize.cu"],
}


def kernel_sources_digest(kernel_key: str):
    """Digest of the sources a kernel is built from (its traffic figure is
    stale once any of them changes)."""
    h = hashlib.sha256()
    for name in KERNEL_SOURCES[kernel_key]:
        with open(os.path.join(ROOT, "qad_nvfp4_quantize_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel_key: str):
    """DRAM bytes per launch recorded from an ncu capture under profiles/, valid
    only while the kernel sources are unchanged since the capture."""
    digest = kernel_sources_digest(kernel_key)
    for path in glob.glob(os.path.join(ROOT, "profiles", "*.md")):
        with open(path) as f:
            for line in f:
                m = re.match(r"^traffic\s+(\S+)\s+bytes_per_launch=(\d+)\s+sources=(\w+)", line.strip())
                if m and m.group(1) == kernel_key and m.group(3) == digest:
                    return int(m.group(2))
    return None


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the timed region runs."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def wait_first(self, timeout_s: float):
        """Block until the first sample has arrived (nvidia-smi takes a moment to start)."""
        t_end = time.time() + timeout_s
        while self.proc is not None and not self.lines and time.time() < t_end:
            time.sleep(0.01)
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        return self

    def summary(self, t0: float, t1: float):
        rows = []
        for ts, line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((ts, float(parts[1]), float(parts[2]), parts[5:9]))
            except ValueError:
                continue
        inside = [r for r in rows if t0 - 0.05 <= r[0] <= t1 + 0.05]
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in inside for i, v in enumerate(r[3]) if v.lower() == "active"})
        loaded = [r[1] for r in inside]
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": max(r[2] for r in inside),
                "reasons": reasons, "samples": len(inside)}


def flush_l2(buf: torch.Tensor):
    """Evict L2 between timed steps: write a buffer twice the size of L2, then
    read a second one, so that the timed kernels start on a cold L2 holding
    no dirty lines (the write alone leaves ~L2-sized dirty data whose
    write-back would land inside the next timed kernel). buf holds both
    halves: the first is written, the second read."""
    half = buf.numel() // 2
    buf[:half].zero_()
    buf[half:].max()


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if world == 1:
        return 0, 1, 0
    import datetime
    import torch.distributed as dist
    rank = int(os.environ["RANK"])
    local = int(os.environ.get("LOCAL_RANK", rank))
    backend = "nccl" if torch.cuda.is_available() else "gloo"
    if torch.cuda.is_available():
        torch.cuda.set_device(local)
    dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return rank, world, local


def dist_max(v: float, world: int) -> float:
    if world == 1:
        return v
    import torch.distributed as dist
    dev = torch.device("cuda", torch.cuda.current_device()) if torch.cuda.is_available() else torch.device("cpu")
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ----------------------------------------------------------------------------- oracle arm

def oracle_sample_step(x_rows: np.ndarray, wq: dict):
    """Oracle quant+GEMM of a row sample against the statically quantized W."""
    from oracle import nvfp4_oracle as o
    q = o.quantize(x_rows, "max")
    C, _S = o.gemm_reference(q["codes"], q["scales"], q["g"], wq["codes"], wq["scales"], wq["g"])
    return C


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return 1


def host_cpu():
    """CPU model and logical core count of the host the oracle runs on."""
    model = "unknown"
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"cpu_model": model, "nproc": os.cpu_count()}


def oracle_setup(seed: int, rows: int):
    from oracle import nvfp4_oracle as o
    from qad_nvfp4_quantize_b200 import inputs
    d = inputs.dense_mlp(seed)
    w = inputs.bf16_to_f32(d["w"])
    wq = o.quantize(w, "max")
    x = inputs.bf16_to_f32(d["x"][:rows])
    return x, wq


def cpu_baseline(seed: int, rows: int = 96):
    x, wq = oracle_setup(seed, rows)
    t0 = time.perf_counter()
    oracle_sample_step(x, wq)
    dt = time.perf_counter() - t0
    flops = 2.0 * rows * DENSE["N"] * DENSE["K"]
    return {"value": flops / dt / 1e12, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
            "sample": f"{rows} of 4096 activation rows: oracle quantize + FP64 GEMM against all 17408 "
                      f"statically quantized weight rows ({dt:.1f} s)",
            "cores_note": "cores = threads of the BLAS pool the FP64 GEMM runs on; the quantize steps are "
                          "single-threaded numpy", **host_cpu()}


def run_reference(args, rank, world):
    if rank != 0:
        return 0
    rows = 32
    x, wq = oracle_setup(0, rows)
    for _ in range(args.warmup):
        oracle_sample_step(x, wq)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_sample_step(x, wq)
    dt = time.perf_counter() - t0
    flops = 2.0 * rows * DENSE["N"] * DENSE["K"] * args.steps
    val = flops / dt / 1e12
    line = {"metric": METRIC, "value": val, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": {"workload": "dense_mlp", "M": DENSE["M"], "N": DENSE["N"], "K": DENSE["K"],
                       "step_sample_rows": rows},
            "cpu_baseline": {"value": val, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                             "sample": f"{rows} activation rows per step (oracle quantize + FP64 GEMM)",
                             **host_cpu()},
            "e2e": {"value": val, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------- GPU arm

def measure_fp4_peak(nv, stream, sampler, iters=20000, bursts=5):
    """Best-of-`bursts` rate of the FP4 MMA probe (TFLOP/s), with the SM clock
    the sampler saw while it ran."""
    nv.probe_mma_peak(200)                                  # warm-up
    torch.cuda.synchronize()
    best = 0.0
    t0 = time.time()
    for _ in range(bursts):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        fl = nv.probe_mma_peak(iters)
        e1.record(stream)
        torch.cuda.synchronize()
        best = max(best, fl / (e0.elapsed_time(e1) * 1e-3) / 1e12)
    t1 = time.time()
    if nv.device_status() != 0:
        raise RuntimeError("the FP4 MMA probe reported a device error")
    c = sampler.summary(t0, t1)
    return best, {"tflops": best, "iters": iters, "bursts": bursts, "ms_total": (t1 - t0) * 1e3,
                  "sm_mhz": c["sm_mhz"], "samples": c["samples"], "reasons": c["reasons"]}


def parity_gate(nv, x_dev, xq, wq, w_cpu_rows=None):
    """Verify before timing: quantized activations of sampled rows bit-exact,
    GEMM of sampled rows within tolerance (oracle on the same inputs)."""
    from oracle import nvfp4_oracle as o
    rows = np.array([0, 1, 1000, 2047, 4095])
    M, K = x_dev.shape
    x = x_dev.float().cpu().numpy()
    ref = o.quantize(x, "max")          # full tensor: the global scale depends on every row
    codes = o.unpack_codes(xq.codes[rows].cpu().numpy())
    if not np.array_equal(codes, ref["codes"][rows]):
        return "activation codes differ from the oracle"
    if xq.g.item() != ref["g"]:
        return "global scale differs from the oracle"
    C = nv.gemm(xq, wq)[rows].float().cpu().numpy()
    wc = o.unpack_codes(wq.codes.cpu().numpy())
    ws = o.scales_from_tiled(wq.scales.cpu().numpy(), wq.rows, K)
    C_ref, S = o.gemm_reference(ref["codes"][rows], ref["scales"][rows], ref["g"], wc, ws, wq.g.item())
    if np.any(np.abs(C - C_ref) > o.gemm_tolerance(C_ref, S)):
        return "GEMM outside tolerance"
    return None


def time_loop(fn, steps, warmup, flush_buf, stream, marks=0, launches=None):
    """Run warmup, then `steps` timed steps with the L2 flushed before each;
    per-step CUDA events on `stream` exclude the flush. fn(evs) records its own
    intermediate events into evs (list of `marks` events). With `launches` (a
    dict), launches["timed"] receives the library's kernel launches issued by
    the timed steps."""
    import qad_nvfp4_quantize_b200 as nv
    for _ in range(warmup):
        flush_l2(flush_buf)
        fn([torch.cuda.Event(enable_timing=True) for _ in range(marks)])
    torch.cuda.synchronize()
    n0 = nv.kernel_launches()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    mids = [[torch.cuda.Event(enable_timing=True) for _ in range(marks)] for _ in range(steps)]
    for i in range(steps):
        flush_l2(flush_buf)
        starts[i].record(stream)
        fn(mids[i])
        ends[i].record(stream)
    torch.cuda.synchronize()
    if launches is not None:
        launches["timed"] = nv.kernel_launches() - n0
    total = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    seg = []
    for i in range(steps):
        pts = [starts[i]] + mids[i] + [ends[i]]
        seg.append([pts[j].elapsed_time(pts[j + 1]) for j in range(len(pts) - 1)])
    return total, seg


ROW_MIN_S = 0.25   # wall time per row (--row-min-s)


def row_loop(fn, flush_buf, stream, spans, name, min_s=None, min_iters=10, max_iters=3000, marks=0):
    """time_loop for one row, run long enough (about min_s of wall time) for
    the clock sampler to see it; the row's wall span goes to spans[name]."""
    min_s = ROW_MIN_S if min_s is None else min_s
    tot, _ = time_loop(fn, 2, 2, flush_buf, stream, marks=marks)
    per = max(statistics.median(tot) * 1e-3 + 90e-6, 1e-6)      # + the L2 flush between steps
    n = int(min(max_iters, max(min_iters, min_s / per)))
    t0 = time.time()
    tot, seg = time_loop(fn, n, 1, flush_buf, stream, marks=marks)
    spans[name] = (t0, time.time(), n)
    return tot, seg


def measure_rows(nv, peaks, flush_buf, stream, spans, iters=10):
    """Each other hot-path row on its own workload (device time, L2 flushed)."""
    from qad_nvfp4_quantize_b200 import inputs
    rows = {}
    hbm = peaks["hbm"]
    fp4_peak = peaks["fp4"]

    def time_loop(fn, steps, warmup, flush_buf, stream, name=None, marks=0):  # noqa: F811 (per-row form)
        return row_loop(fn, flush_buf, stream, spans, name, marks=marks)

    # four_over_six static calibration + QAD fake-quant + W4A4 GEMM (W 14336x4096, X 16384x4096)
    d = inputs.four_over_six_linear(0)
    w = d["w"].cuda()
    x = d["x"].cuda()
    del d
    wq = nv.quantize(w, "four_over_six", want_choice=True)
    tot, _ = time_loop(lambda ev: nv.quantize(w, "four_over_six", want_choice=True, out=wq), iters, 2, flush_buf, stream, name='four_over_six_calibration')
    t = statistics.median(tot) * 1e-3
    n = w.numel()
    alg = n * (2 + 0.5 + 1 / 16 + 1 / 16)     # read W, write codes, scales, choice
    rows["four_over_six_calibration"] = {"workload": "W 14336x4096 BF16, 0.1% entries x20", "ms": t * 1e3,
                                         "GB/s": alg / t / 1e9, "frac_hbm": alg / t / 1e9 / hbm,
                                         "algorithmic_bytes": alg}
    wq_mse = nv.quantize(w, "mse")
    tot, _ = time_loop(lambda ev: nv.quantize(w, "mse", out=wq_mse), 3, 1, flush_buf, stream, name='mse_calibration')
    t = statistics.median(tot) * 1e-3
    alg = n * (2 + 0.5 + 1 / 16)
    rows["mse_calibration"] = {"workload": "W 14336x4096 BF16, 0.1% entries x20; all 126 E4M3 scales per block "
                                           "(pruned by the clipping bound)",
                               "ms": t * 1e3, "GB/s": alg / t / 1e9, "frac_hbm": alg / t / 1e9 / hbm,
                               "blocks_per_s": n / 16 / t, "algorithmic_bytes": alg}
    del wq_mse
    y = torch.empty_like(x)
    tot, _ = time_loop(lambda ev: nv.fake_quant(x, "max", out=y), iters, 2, flush_buf, stream, name='fake_quant_dynamic')
    t = statistics.median(tot) * 1e-3
    alg = x.numel() * 4.0
    rows["fake_quant_dynamic"] = {"workload": "X 16384x4096 BF16 -> BF16", "ms": t * 1e3, "GB/s": alg / t / 1e9,
                                  "frac_hbm": alg / t / 1e9 / hbm, "algorithmic_bytes": alg}
    gy = torch.randn_like(x)
    gx = torch.empty_like(x)
    tot, _ = time_loop(lambda ev: nv.fake_quant_backward(x, gy, "max", out=gx), iters, 2, flush_buf, stream, name='qad_backward_ste_dynamic')
    t = statistics.median(tot) * 1e-3
    alg = x.numel() * 6.0
    rows["qad_backward_ste_dynamic"] = {"workload": "X 16384x4096 BF16 and dL/dy BF16 -> dL/dx BF16 (clipped STE, "
                                                    "dynamic max scales)", "ms": t * 1e3, "GB/s": alg / t / 1e9,
                                        "frac_hbm": alg / t / 1e9 / hbm, "algorithmic_bytes": alg}
    # the same ops with scales fixed beforehand (a static global scale, or the
    # frozen scales of a calibration): one streaming pass each
    qf = nv.quantize(x)
    xq_s = nv.quantize(x, "max", g=qf.g)
    tot, _ = time_loop(lambda ev: nv.quantize(x, "max", g=qf.g, out=xq_s), iters, 2, flush_buf, stream,
                       name='quantize_static_g_cfg5_x')
    t = statistics.median(tot) * 1e-3
    alg = x.numel() * 2.5625
    rows["quantize_static_g_cfg5_x"] = {"workload": "X 16384x4096 BF16, given global scale", "ms": t * 1e3,
                                        "GB/s": alg / t / 1e9, "frac_hbm": alg / t / 1e9 / hbm,
                                        "algorithmic_bytes": alg}
    tot, _ = time_loop(lambda ev: nv.fake_quant(x, g=qf.g, scales=qf.scales, out=y), iters, 2, flush_buf, stream,
                       name='fake_quant_frozen')
    t = statistics.median(tot) * 1e-3
    alg = x.numel() * (4.0 + 1 / 16)
    rows["fake_quant_frozen"] = {"workload": "X 16384x4096 BF16 -> BF16 with frozen global and block scales",
                                 "ms": t * 1e3, "GB/s": alg / t / 1e9, "frac_hbm": alg / t / 1e9 / hbm,
                                 "algorithmic_bytes": alg}
    tot, _ = time_loop(lambda ev: nv.fake_quant_backward(x, gy, g=qf.g, scales=qf.scales, out=gx), iters, 2,
                       flush_buf, stream, name='qad_backward_ste_frozen')
    t = statistics.median(tot) * 1e-3
    alg = x.numel() * (6.0 + 1 / 16)
    rows["qad_backward_ste_frozen"] = {"workload": "as qad_backward_ste_dynamic with frozen global and block scales",
                                       "ms": t * 1e3, "GB/s": alg / t / 1e9, "frac_hbm": alg / t / 1e9 / hbm,
                                       "algorithmic_bytes": alg}
    del gy, gx, qf, xq_s
    xq = nv.quantize(x)
    tot, _ = time_loop(lambda ev: nv.quantize(x, out=xq), iters, 2, flush_buf, stream, name='quantize_dynamic_cfg5_x')
    t = statistics.median(tot) * 1e-3
    alg = x.numel() * 2.5625
    rows["quantize_dynamic_cfg5_x"] = {"workload": "X 16384x4096 BF16 (larger than L2)", "ms": t * 1e3,
                                       "GB/s": alg / t / 1e9, "frac_hbm": alg / t / 1e9 / hbm,
                                       "algorithmic_bytes": alg}
    C = torch.empty((x.shape[0], w.shape[0]), dtype=torch.bfloat16, device="cuda")
    tot, _ = time_loop(lambda ev: nv.gemm(xq, wq, out=C), iters, 2, flush_buf, stream, name='gemm_fos_16384x14336x4096')
    t = statistics.median(tot) * 1e-3
    fl = 2.0 * x.shape[0] * w.shape[0] * x.shape[1]
    rows["gemm_fos_16384x14336x4096"] = {"ms": t * 1e3, "TFLOP/s": fl / t / 1e12, "frac_fp4_peak": fl / t / 1e12 / fp4_peak}

    # the same linear as one quant+GEMM step (dynamic X quantize, then the
    # GEMM as its programmatic dependent), timed like the dense_mlp headline
    def fos_step(ev):
        nv.quantize(x, out=xq)
        ev[0].record(stream)
        nv.gemm(xq, wq, out=C)
    tot, seg = time_loop(fos_step, iters, 2, flush_buf, stream, name="step_four_over_six_linear", marks=1)
    t = statistics.median(tot) * 1e-3
    tq = statistics.median([sg[0] for sg in seg]) * 1e-3
    tg = statistics.median([sg[1] for sg in seg]) * 1e-3
    rows["step_four_over_six_linear"] = {
        "workload": "X 16384x4096 N(0,1) dynamic NVFP4 quantize + GEMM against W 14336x4096 four_over_six",
        "ms": t * 1e3, "TFLOP/s": fl / t / 1e12, "frac_fp4_peak": fl / t / 1e12 / fp4_peak,
        "quantize_ms": tq * 1e3, "quantize_frac_hbm": x.numel() * 2.5625 / tq / 1e9 / hbm,
        "gemm_ms": tg * 1e3, "gemm_frac_fp4_peak": fl / tg / 1e12 / fp4_peak}
    del w, x, y, xq, wq, C
    torch.cuda.empty_cache()

    # NVFP4 KV cache: K and V of 32768 tokens x 8 heads x 128, four_over_six on
    # write, BF16 on read (dequantize is the per-step read side)
    kv = torch.randn((2 * 32768, 1024), device="cuda").to(torch.bfloat16)
    kvq = nv.quantize(kv, "four_over_six")
    kvy = torch.empty_like(kv)
    tot, _ = time_loop(lambda ev: nv.dequantize(kvq, out=kvy), iters, 2, flush_buf, stream, name='kv_cache_dequantize')
    t = statistics.median(tot) * 1e-3
    alg = kv.numel() * (0.5 + 1 / 16 + 2)
    rows["kv_cache_dequantize"] = {"workload": "K,V 2x32768x1024 NVFP4 -> BF16", "ms": t * 1e3, "GB/s": alg / t / 1e9,
                                   "frac_hbm": alg / t / 1e9 / hbm, "algorithmic_bytes": alg}
    tot, _ = time_loop(lambda ev: nv.quantize(kv, "four_over_six", out=kvq), iters, 2, flush_buf, stream, name='kv_cache_quantize_fos')
    t = statistics.median(tot) * 1e-3
    alg = kv.numel() * (2 + 0.5 + 1 / 16)
    rows["kv_cache_quantize_fos"] = {"workload": "K,V 2x32768x1024 BF16 -> NVFP4 four_over_six", "ms": t * 1e3,
                                     "GB/s": alg / t / 1e9, "frac_hbm": alg / t / 1e9 / hbm, "algorithmic_bytes": alg}
    del kv, kvq, kvy
    torch.cuda.empty_cache()

    # top-k logit KL: 2048 positions x 248,320-entry vocabulary, teacher top-4096
    gen = torch.Generator(device="cuda").manual_seed(7)
    R, V = 2048, 248320
    tl = torch.randn((R, V), device="cuda", generator=gen) * 2.0
    tl.scatter_add_(1, torch.randint(0, V, (R, 64), device="cuda", generator=gen),
                    torch.full((R, 64), 8.0, device="cuda"))
    sl = (tl + torch.randn((R, V), device="cuda", generator=gen) * 0.5).to(torch.bfloat16)
    tl = tl.to(torch.bfloat16)
    kl = torch.empty(R, dtype=torch.float32, device="cuda")
    tot, _ = time_loop(lambda ev: nv.topk_kl(tl, sl, 4096, loss_out=kl), iters, 2, flush_buf, stream, name='kd_topk_kl')
    t = statistics.median(tot) * 1e-3
    alg = 2.0 * R * V + 2.0 * R * 4096  # teacher rows read once; student logits needed only on the set
    rows["kd_topk_kl"] = {"workload": "2048 x 248320 BF16 teacher/student logits, top-4096 KL per row",
                          "ms": t * 1e3, "GB/s": alg / t / 1e9, "frac_hbm": alg / t / 1e9 / hbm,
                          "algorithmic_bytes": alg}
    # the training form: loss, the set (idx) and d loss / d student logits on it
    kidx = torch.empty((R, 4096), dtype=torch.int32, device="cuda")
    kgrad = torch.empty((R, 4096), dtype=torch.float32, device="cuda")
    tot, _ = time_loop(lambda ev: nv.topk_kl(tl, sl, 4096, loss_out=kl, idx_out=kidx, grad_out=kgrad),
                       iters, 2, flush_buf, stream, name='kd_topk_kl_loss_grad')
    t = statistics.median(tot) * 1e-3
    alg = 2.0 * R * V + 2.0 * R * 4096 + 8.0 * R * 4096  # + idx and grad written
    rows["kd_topk_kl_loss_grad"] = {"workload": "as kd_topk_kl, plus idx [2048x4096] int32 and grad FP32",
                                    "ms": t * 1e3, "GB/s": alg / t / 1e9, "frac_hbm": alg / t / 1e9 / hbm,
                                    "algorithmic_bytes": alg}
    del tl, sl, kl, kidx, kgrad
    torch.cuda.empty_cache()

    # lm_head decode: X 128x2048, W 151936x2048 (HBM-bound weight streaming)
    d = inputs.lm_head(0)
    w = d["w"].cuda()
    x = d["x"].cuda()
    wq = nv.quantize(w)
    xq = nv.quantize(x)
    C = torch.empty((128, w.shape[0]), dtype=torch.bfloat16, device="cuda")
    tot, _ = time_loop(lambda ev: nv.gemm(xq, wq, out=C), iters, 2, flush_buf, stream, name='lm_head_gemm')
    t = statistics.median(tot) * 1e-3
    M, N, K = 128, w.shape[0], 2048
    alg = N * K * 0.5625 + M * K * 0.5625 + M * N * 2
    rows["lm_head_gemm"] = {"workload": "128x151936x2048", "ms": t * 1e3, "TFLOP/s": 2.0 * M * N * K / t / 1e12,
                            "GB/s": alg / t / 1e9, "frac_hbm": alg / t / 1e9 / hbm, "algorithmic_bytes": alg}
    del w, x, wq, xq, C, d
    torch.cuda.empty_cache()

    # routed experts: T=8192, H=2048, E=256, top-8, I=512
    d = inputs.moe_experts(0)
    x = d["x"].cuda()
    ids = d["topk_ids"].cuda()
    tw = d["topk_w"].cuda()
    w13, g13 = nv.quantize_experts(d["w13"].cuda())
    w2, g2 = nv.quantize_experts(d["w2"].cuda())
    del d
    out, ws = nv.moe_grouped_gemm(x, ids, tw, 512, w13, g13, w2, g2)
    tot, _ = time_loop(lambda ev: nv.moe_grouped_gemm(x, ids, tw, 512, w13, g13, w2, g2, out=out, workspace=ws),
                       iters, 2, flush_buf, stream, name='moe_routed_experts')
    t = statistics.median(tot) * 1e-3
    T, H, E, I = 8192, 2048, 256, 512
    alg = T * H * 2 + E * (2 * I * H + H * I) * 0.5625 + T * H * 4
    fl = 2.0 * T * 8 * (2 * I * H + H * I)
    rows["moe_routed_experts"] = {"workload": "T8192 H2048 E256 top8 I512", "ms": t * 1e3,
                                  "TFLOP/s": fl / t / 1e12, "GB/s": alg / t / 1e9, "frac_hbm": alg / t / 1e9 / hbm,
                                  "algorithmic_bytes": alg}
    return rows


def run_gpu(args, rank, world, local):
    import qad_nvfp4_quantize_b200 as nv
    from qad_nvfp4_quantize_b200 import inputs
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    nv.check_device()
    peaks = load_peaks()
    stream = torch.cuda.current_stream(dev)
    M, N, K = DENSE["M"], DENSE["N"], DENSE["K"]

    d = inputs.dense_mlp(seed=rank)
    x_host = d["x"].pin_memory()
    x = d["x"].to(dev)
    w = d["w"].to(dev)
    del d
    wq = nv.quantize(w, "max")                    # static weights, quantized offline
    del w
    xq = nv.quantize(x, "max")
    C = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    err = parity_gate(nv, x, xq, wq)
    if err is not None:
        print(json.dumps({"metric": METRIC, "error": f"parity check failed before timing: {err}"}), flush=True)
        return 1
    flush_buf = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def step(ev):
        nv.quantize(x, "max", out=xq)
        if ev:
            ev[0].record(stream)  # split steps only: an event between the two kernels stops their overlap
        nv.gemm(xq, wq, out=C)

    sampler = ClockSampler(local).start()
    sampler.wait_first(3.0)
    # the dense FP4 tensor peak, measured: the MMA rate probe (no memory traffic)
    peaks["fp4"], peaks["fp4_probe"] = measure_fp4_peak(nv, stream, sampler)
    barrier(world)
    torch.cuda.synchronize()
    t_wall0 = time.time()
    launches = {}
    # the timed steps run as in production: the GEMM is a programmatic
    # dependent of the quantize, nothing recorded between them
    total, _ = time_loop(step, args.steps, args.warmup, flush_buf, stream, marks=0, launches=launches)
    t_wall1 = time.time()
    barrier(world)
    torch.cuda.synchronize()
    step_ms = dist_max(float(np.mean(total)), world)
    clocks = sampler.summary(t_wall0, t_wall1)
    # quantize / GEMM split from separate steps with an event between the kernels
    split_steps = max(10, min(args.steps, 500))
    _, seg = time_loop(step, split_steps, 3, flush_buf, stream, marks=1)
    quant_ms = float(np.mean([s[0] for s in seg]))
    gemm_ms = float(np.mean([s[1] for s in seg]))
    flops = 2.0 * M * N * K
    value = flops * world / (step_ms * 1e-3) / 1e12

    # e2e through the public API with host buffers: every step copies its X
    # from pinned host memory, quantizes it, runs the GEMM and copies C back.
    # Consecutive steps are pipelined on three streams (H2D, compute, D2H)
    # with double buffers, so step i+1's H2D and step i's D2H overlap.
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    xs = [torch.empty_like(x) for _ in range(2)]
    xqs = [nv.quantize(x, "max") for _ in range(2)]
    Cs = [C, torch.empty_like(C)]
    C_hosts = [torch.empty((M, N), dtype=torch.bfloat16, pin_memory=True) for _ in range(2)]
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_c = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def e2e_run(n):
        for i in range(n):
            b = i % 2
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(ev_c[b])          # xs[b] consumed by step i-2
                xs[b].copy_(x_host, non_blocking=True)
                ev_in[b].record(s_in)
            stream.wait_event(ev_in[b])
            if i >= 2:
                stream.wait_event(ev_out[b])          # Cs[b] copied out by step i-2
            nv.quantize(xs[b], "max", out=xqs[b])
            nv.gemm(xqs[b], wq, out=Cs[b])
            ev_c[b].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_c[b])
                C_hosts[b].copy_(Cs[b], non_blocking=True)
                ev_out[b].record(s_out)
        stream.wait_stream(s_in)
        stream.wait_stream(s_out)

    e2e_steps = max(3, min(args.steps, 50))
    e2e_run(max(3, min(args.warmup, 5)))
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    e2e_run(e2e_steps)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = dist_max(e0.elapsed_time(e1) / e2e_steps, world)
    e2e_val = flops * world / (e2e_ms * 1e-3) / 1e12
    del xs, xqs, C_hosts, Cs

    fp4_peak = peaks["fp4"]
    achieved = flops / (gemm_ms * 1e-3) / 1e12
    roofline = {"bound": "tensor", "kernel": "nvf4_gemm_kernel<DenseProblem>", "achieved": achieved,
                "peak": fp4_peak, "unit": "TFLOP/s", "frac": achieved / fp4_peak,
                "traffic": recorded_traffic("gemm_dense_mlp"),
                "peak_source": "measured MMA: nvfp4_probe_mma_peak, kind::mxf4nvf4 128x256x64 back to back on "
                               "shared-memory operands, one CTA per SM, best of 5 bursts",
                "peak_probe": peaks["fp4_probe"],
                "peak_bf16_x4": peaks["bf16"] * FP4_OVER_BF16,
                "algorithmic_flops_per_launch": flops}
    quant_bytes = M * K * 2.5625
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "nvfp4 (e2m1 x e2m1, ue4m3 block scales, fp32 accumulate)",
            "data": "synthetic",
            "config": {"workload": "dense_mlp: X 4096x5120 Student-t(3)*0.5 -> NVFP4 dynamic quantize; "
                                   "W_up 17408x5120 N(0,0.02) static max NVFP4; C BF16 4096x17408",
                       "M": M, "N": N, "K": K, "l2": "flushed before every step, outside the step's "
                                                       "events: a 256 MiB write, then a 256 MiB read of "
                                                       "another buffer (cold L2, no dirty lines)", "parallelism": f"replicas x{world}"},
            "roofline": roofline,
            "quantize": {"ms": quant_ms, "GB/s": quant_bytes / (quant_ms * 1e-3) / 1e9,
                         "frac_hbm": quant_bytes / (quant_ms * 1e-3) / 1e9 / peaks["hbm"],
                         "algorithmic_bytes": quant_bytes, "peak_GB/s": peaks["hbm"],
                         "traffic": recorded_traffic("quantize_dense_mlp")},
            "gemm_ms": gemm_ms,
            "split_note": f"quantize / GEMM split from {split_steps} separate steps with a CUDA event between the "
                          "two kernels (the event stops the GEMM's programmatic early start); value and "
                          "ms_per_step come from steps without it",
            "e2e": {"value": e2e_val, "unit": UNIT, "h2d_bytes_per_step": x.numel() * 2,
                    "d2h_bytes_per_step": C.numel() * 2, "ms_per_step": e2e_ms,
                    "pipelining": "2 steps in flight: H2D / compute / D2H streams, double buffers"},
            "gpu_launches": launches["timed"],
            "clocks": {"sm_mhz": clocks["sm_mhz"], "sm_max_mhz": clocks["sm_max_mhz"], "reasons": clocks["reasons"],
                       "samples": clocks["samples"]},
            "wall_s_timed_region": t_wall1 - t_wall0}
    if world == 1 and not args.no_rows:
        del xq, C
        spans = {}
        line["rows"] = measure_rows(nv, peaks, flush_buf, stream, spans)
        for name, (t0, t1, n) in spans.items():
            c = sampler.summary(t0, t1)
            line["rows"][name]["iters"] = n
            line["rows"][name]["clocks"] = {"sm_mhz": c["sm_mhz"], "samples": c["samples"], "reasons": c["reasons"]}
    sampler.stop()
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(0)
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def kernels_once():
    """Every library kernel once, at the workloads' sizes, inside a
    cudaProfilerStart/Stop range (the set-up launches stay outside it): the
    command the per-kernel ncu summaries under profiles/ are captured from,
    with ncu --profile-from-start off."""
    import qad_nvfp4_quantize_b200 as nv
    from qad_nvfp4_quantize_b200 import inputs
    torch.cuda.set_device(0)
    nv.check_device()
    d = inputs.four_over_six_linear(0)
    w5, x5 = d["w"].cuda(), d["x"].cuda()                  # W 14336x4096, X 16384x4096
    del d
    gy = torch.randn_like(x5)
    y5, gx5 = torch.empty_like(x5), torch.empty_like(x5)
    xq5 = nv.quantize(x5)
    wq5 = nv.quantize(w5, "four_over_six", want_choice=True)
    wmse = nv.quantize(w5, "mse")
    kv = torch.randn((2 * 32768, 1024), device="cuda").to(torch.bfloat16)
    kvq = nv.quantize(kv, "four_over_six")
    kvy = torch.empty_like(kv)
    g_static = torch.tensor([0.01], device="cuda")
    d = inputs.dense_mlp(0)
    xd, wd = d["x"].cuda(), nv.quantize(d["w"].cuda())
    del d
    xqd = nv.quantize(xd)
    Cd = torch.empty((xd.shape[0], wd.rows), dtype=torch.bfloat16, device="cuda")
    d = inputs.lm_head(0)
    wl, xl = nv.quantize(d["w"].cuda()), nv.quantize(d["x"].cuda())
    del d
    Cl = torch.empty((128, wl.rows), dtype=torch.bfloat16, device="cuda")
    m = inputs.moe_experts(0)
    mx, mids, mw = m["x"].cuda(), m["topk_ids"].cuda(), m["topk_w"].cuda()
    w13, g13 = nv.quantize_experts(m["w13"].cuda())
    w2, g2 = nv.quantize_experts(m["w2"].cuda())
    del m
    mout, mws = nv.moe_grouped_gemm(mx, mids, mw, 512, w13, g13, w2, g2)
    R, V = 512, 248320                                     # 508 MB of logits: larger than L2
    gen = torch.Generator(device="cuda").manual_seed(7)
    tl = torch.randn((R, V), device="cuda", generator=gen) * 2.0
    sl = (tl + torch.randn((R, V), device="cuda", generator=gen) * 0.5).to(torch.bfloat16)
    tl = tl.to(torch.bfloat16)
    kl = torch.empty(R, dtype=torch.float32, device="cuda")
    nv.probe_mma_peak(100)
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    torch.cuda.profiler.start()
    nv.quantize(xd, "max", out=xqd)                                    # dense_mlp X 4096x5120
    nv.gemm(xqd, wd, out=Cd)                                           # dense_mlp GEMM (programmatic dependent)
    nv.quantize(x5, "max", out=xq5)                                    # X 16384x4096
    nv.quantize(w5, "four_over_six", want_choice=True, out=wq5)        # W 14336x4096 four_over_six
    nv.fake_quant(x5, "max", out=y5)
    nv.fake_quant_backward(x5, gy, "max", out=gx5)
    nv.quantize(w5, "mse", out=wmse)
    nv.dequantize(kvq, out=kvy)
    nv.fake_quant(x5, g=xq5.g, scales=xq5.scales, out=y5)             # frozen scales
    nv.quantize(x5, "max", g=g_static, out=xq5)                        # static global scale
    nv.gemm(xl, wl, out=Cl)                                            # lm_head 128x151936x2048
    nv.moe_grouped_gemm(mx, mids, mw, 512, w13, g13, w2, g2, out=mout, workspace=mws)
    nv.topk_kl(tl, sl, 4096, loss_out=kl)
    nv.probe_mma_peak(2000)
    torch.cuda.synchronize()
    torch.cuda.profiler.stop()
    if nv.device_status() != 0:
        raise RuntimeError("a kernel reported a device error")
    print("kernels-once ok", flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-rows", action="store_true", help="skip the per-row measurements")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--row-min-s", type=float, default=0.25,
                    help="wall time each row is timed for (at least 10 steps)")
    ap.add_argument("--kernels-once", action="store_true",
                    help="run every library kernel once inside a profiler range (for ncu) and exit")
    args = ap.parse_args()
    if args.kernels_once:
        sys.exit(kernels_once())
    global ROW_MIN_S
    ROW_MIN_S = args.row_min_s
    if args.warmup < 3:
        args.warmup = 3
    rank, world, local = dist_setup()
    try:
        if args.impl == "reference":
            rc = run_reference(args, rank, world)
        else:
            rc = run_gpu(args, rank, world, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
    sys.exit(rc)


if __name__ == "__main__":
    main()
