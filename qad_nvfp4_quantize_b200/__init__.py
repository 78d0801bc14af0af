"""NVFP4 W4A4 quantization and block-scaled GEMM on B200 (sm_100a).

Thin ctypes binding over ``libnvfp4.so`` (C ABI declared in include/nvfp4.h).
Every step runs in the library's CUDA kernels; this module only marshals
torch tensors (device memory and the current stream) into the C calls. There
is no CPU fallback: if the library is missing or the device is not sm_100,
the calls raise.
"""
from __future__ import annotations

import ctypes
import os
import threading
from typing import NamedTuple, Optional

import torch

__all__ = [
    "MODE_MAX", "MODE_FOUR_OVER_SIX", "NVFP4Error", "Quantized", "lib", "library_path",
    "check_device", "scale_bytes", "quantize", "fake_quant", "fake_quant_backward", "dequantize", "topk_kl", "gemm", "moe_grouped_gemm",
    "moe_workspace_layout", "convert_e2m1", "convert_e4m3", "device_status", "selftest_timeout",
    "quantize_workspace_bytes", "moe_workspace_bytes", "quantize_experts", "quantize_noalloc",
    "selftest_gemm_timeout", "kernel_launches", "probe_mma_peak",
]

MODE_MAX = 0
MODE_FOUR_OVER_SIX = 1
MODE_MSE = 2
_MODES = {"max": MODE_MAX, "four_over_six": MODE_FOUR_OVER_SIX, "mse": MODE_MSE, MODE_MAX: MODE_MAX,
          MODE_FOUR_OVER_SIX: MODE_FOUR_OVER_SIX, MODE_MSE: MODE_MSE}

_HERE = os.path.dirname(os.path.abspath(__file__))
# NVFP4_LIBRARY=debug selects the bounds-checking build (libnvfp4_debug.so);
# any other value is taken as the path of the library to load.
_choice = os.environ.get("NVFP4_LIBRARY", "")
library_path = (os.path.join(_HERE, "libnvfp4_debug.so") if _choice == "debug"
                else (_choice or os.path.join(_HERE, "libnvfp4.so")))

_STATUS = {0: "ok", 1: "invalid argument", 2: "unsupported device", 3: "CUDA error",
           4: "workspace missing or too small", 5: "non-finite input", 6: "device wait timed out",
           7: "input too large for the no-alloc entry point (M*K > 2^30)",
           8: "index outside its buffer (bounds-checking build)"}


class NVFP4Error(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {_STATUS.get(status, status)} (status {status})")
        self.status = status


class _MoeLayout(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int64) for n in (
        "rows_capacity", "counts", "offsets", "row_pair", "xq_codes", "xq_scales", "xq_g",
        "h", "hq_codes", "hq_scales", "hq_g", "total_bytes")]


_lib = None
_lib_lock = threading.Lock()
P, I64, I32, SZ, U64 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t, ctypes.c_uint64

_SIGS = {
    "nvfp4_version": (I32, []),
    "nvfp4_check_device": (I32, []),
    "nvfp4_status_string": (ctypes.c_char_p, [I32]),
    "nvfp4_scale_bytes": (SZ, [I64, I64]),
    "nvfp4_quantize_workspace_bytes": (SZ, [I64, I64]),
    "nvfp4_quantize": (I32, [P, I64, I64, I32, P, P, P, P, P, P, SZ, P]),
    "nvfp4_fake_quant": (I32, [P, I64, I64, I32, P, P, P, P, SZ, P]),
    "nvfp4_fake_quant_backward": (I32, [P, P, I64, I64, I32, P, P, P, P, SZ, P]),
    "nvfp4_dequantize": (I32, [P, P, P, I64, I64, P, P]),
    "nvfp4_topk_kl": (I32, [P, P, I64, I64, I32, P, P, P, P]),
    "nvfp4_quantize_noalloc": (I32, [P, I64, I64, I32, P, P, P, P, P, P]),
    "nvfp4_gemm": (I32, [P, P, P, P, P, P, I64, I64, I64, P, P]),
    "nvfp4_moe_workspace_bytes": (SZ, [I64, I64, I64, I32, I32]),
    "nvfp4_moe_grouped_gemm": (I32, [P, I64, I64, P, P, I32, I32, I64, P, P, P, P, P, P, P, P, SZ, P]),
    "nvfp4_moe_workspace_layout": (I32, [I64, I64, I64, I32, I32, ctypes.POINTER(_MoeLayout)]),
    "nvfp4_convert_e2m1": (I32, [P, I64, P, P]),
    "nvfp4_convert_e4m3": (I32, [P, I64, P, P]),
    "nvfp4_get_device_status": (I32, [P, I32, ctypes.POINTER(ctypes.c_int)]),
    "nvfp4_selftest_timeout": (I32, [U64, P]),
    "nvfp4_selftest_gemm_timeout": (I32, [P, P, P, P, P, P, I64, I64, I64, P, U64, P]),
    "nvfp4_kernel_launches": (U64, []),
    "nvfp4_probe_mma_peak": (I32, [I32, ctypes.POINTER(ctypes.c_double), P]),
}


def lib() -> ctypes.CDLL:
    """The loaded C library (raises if it has not been built)."""
    global _lib
    with _lib_lock:
        if _lib is None:
            if not os.path.exists(library_path):
                raise NVFP4Error(3, f"{library_path} is missing; build it with "
                                    "`python -m qad_nvfp4_quantize_b200.build`")
            handle = ctypes.CDLL(library_path)
            for name, (res, args) in _SIGS.items():
                fn = getattr(handle, name, None)
                if fn is None:
                    continue  # reported by the symbol-export test; calling it raises AttributeError
                fn.restype = res
                fn.argtypes = args
            _lib = handle
    return _lib


def _check(st: int, what: str) -> None:
    if st != 0:
        raise NVFP4Error(st, what)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device: torch.device):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _cuda(t: torch.Tensor, name: str, dtype=None) -> torch.Tensor:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


def check_device(device=None) -> None:
    with torch.cuda.device(device or torch.cuda.current_device()):
        _check(lib().nvfp4_check_device(), "nvfp4_check_device")


def scale_bytes(rows: int, K: int) -> int:
    return int(lib().nvfp4_scale_bytes(rows, K))


def quantize_workspace_bytes(M: int, K: int) -> int:
    return int(lib().nvfp4_quantize_workspace_bytes(M, K))


def moe_workspace_bytes(T: int, H: int, I: int, E: int, topk: int) -> int:
    return int(lib().nvfp4_moe_workspace_bytes(T, H, I, E, topk))


# Scratch for the dynamic global scale (the library itself never allocates).
# It holds a grid-wide barrier, so it must start zero-filled and two calls
# that use it must never overlap on the GPU: one workspace per (device,
# stream), so calls issued on different streams never share one. After a
# call reports a timed-out wait the barrier state is stale; device_status()
# zero-fills every workspace of that device again when it reads that status.
_ws_cache: dict = {}
_ws_lock = threading.Lock()


def _workspace(device: torch.device, nbytes: int) -> torch.Tensor:
    stream = torch.cuda.current_stream(device)
    key = (device.index, stream.cuda_stream)
    with _ws_lock:
        entry = _ws_cache.get(key)
        if entry is None or entry[1].numel() < nbytes:
            entry = (stream, torch.zeros(nbytes, dtype=torch.uint8, device=device))
            _ws_cache[key] = entry
    return entry[1]


def _reset_workspaces(device_index: int) -> None:
    """Zero-fill every cached workspace of one device (after a timed-out wait).
    Each is cleared on the stream that uses it, after the work queued there."""
    with _ws_lock:
        items = [entry for key, entry in _ws_cache.items() if key[0] == device_index]
    for stream, ws in items:
        with torch.cuda.stream(stream):
            ws.zero_()


class Quantized(NamedTuple):
    """An NVFP4 tensor: packed codes [rows, K/2] uint8, tiled E4M3 scales,
    FP32 global scale (1-element device tensor) and the optional
    four_over_six choice map [rows, K/16] uint8."""
    codes: torch.Tensor
    scales: torch.Tensor
    g: torch.Tensor
    choice: Optional[torch.Tensor]
    rows: int
    K: int


def quantize(x: torch.Tensor, mode="max", g: Optional[torch.Tensor] = None, want_choice: bool = False,
             out: Optional[Quantized] = None) -> Quantized:
    """NVFP4-quantize a BF16 [M, K] CUDA tensor along K (nvfp4_quantize)."""
    x = _cuda(x, "x", torch.bfloat16)
    if x.dim() != 2:
        raise ValueError("x must be 2-D [M, K]")
    M, K = x.shape
    dev = x.device
    if out is None:
        codes = torch.empty((M, K // 2), dtype=torch.uint8, device=dev)
        scales = torch.empty(max(scale_bytes(M, K), 16), dtype=torch.uint8, device=dev)
        g_out = torch.empty(1, dtype=torch.float32, device=dev)
        choice = torch.empty((M, K // 16), dtype=torch.uint8, device=dev) if want_choice else None
        out = Quantized(codes, scales, g_out, choice, M, K)
    ws = None
    ws_bytes = 0
    if g is None:
        ws_bytes = quantize_workspace_bytes(M, K)
        ws = _workspace(dev, ws_bytes)
    else:
        g = _cuda(g, "g", torch.float32)
    st = lib().nvfp4_quantize(_ptr(x), M, K, _MODES[mode], _ptr(g), _ptr(out.codes), _ptr(out.scales),
                              _ptr(out.g), _ptr(out.choice), _ptr(ws), ws_bytes, _stream(dev))
    _check(st, "nvfp4_quantize")
    return out


def quantize_noalloc(x: torch.Tensor, mode="max", g: Optional[torch.Tensor] = None,
                     want_choice: bool = False, out: Optional[Quantized] = None) -> Quantized:
    """nvfp4_quantize_noalloc: like quantize(), but the library reduces the
    global scale through its own static device scratch instead of a caller
    workspace (for callers that cannot allocate; M*K <= 2^30). Pass ``out`` to
    make the call itself allocation-free."""
    x = _cuda(x, "x", torch.bfloat16)
    M, K = x.shape
    dev = x.device
    if out is None:
        out = Quantized(torch.empty((M, K // 2), dtype=torch.uint8, device=dev),
                        torch.empty(max(scale_bytes(M, K), 16), dtype=torch.uint8, device=dev),
                        torch.empty(1, dtype=torch.float32, device=dev),
                        torch.empty((M, K // 16), dtype=torch.uint8, device=dev) if want_choice else None, M, K)
    st = lib().nvfp4_quantize_noalloc(_ptr(x), M, K, _MODES[mode], _ptr(g), _ptr(out.codes), _ptr(out.scales),
                                      _ptr(out.g), _ptr(out.choice), _stream(dev))
    _check(st, "nvfp4_quantize_noalloc")
    return out


def fake_quant(x: torch.Tensor, mode="max", g: Optional[torch.Tensor] = None,
               scales: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """QAD fake-quant forward y = BF16(g*s*q) (nvfp4_fake_quant). ``g`` alone:
    static global scale; ``g`` and ``scales``: frozen scales."""
    x = _cuda(x, "x", torch.bfloat16)
    M, K = x.shape
    dev = x.device
    y = torch.empty_like(x) if out is None else out
    ws = None
    ws_bytes = 0
    if g is None:
        ws_bytes = quantize_workspace_bytes(M, K)
        ws = _workspace(dev, ws_bytes)
    st = lib().nvfp4_fake_quant(_ptr(x), M, K, _MODES[mode], _ptr(g), _ptr(scales), _ptr(y), _ptr(ws),
                                ws_bytes, _stream(dev))
    _check(st, "nvfp4_fake_quant")
    return y


def topk_kl(teacher: torch.Tensor, student: torch.Tensor, k: int, want_idx: bool = False,
            want_grad: bool = False, loss_out: Optional[torch.Tensor] = None,
            idx_out: Optional[torch.Tensor] = None, grad_out: Optional[torch.Tensor] = None):
    """Top-k logit KL distillation loss per row (nvfp4_topk_kl). Returns
    (loss [rows] FP32, idx [rows, k] int32 or None, grad [rows, k] FP32 or None).
    loss_out / idx_out / grad_out: optional preallocated outputs (idx_out or
    grad_out given implies want_idx / want_grad)."""
    teacher = _cuda(teacher, "teacher", torch.bfloat16)
    student = _cuda(student, "student", torch.bfloat16)
    if teacher.shape != student.shape or teacher.dim() != 2:
        raise ValueError("teacher and student must be equal [rows, V]")
    rows, V = teacher.shape
    dev = teacher.device
    loss = torch.empty(rows, dtype=torch.float32, device=dev) if loss_out is None else loss_out
    want_grad = want_grad or grad_out is not None
    want_idx = want_idx or want_grad or idx_out is not None
    idx = (torch.empty((rows, k), dtype=torch.int32, device=dev) if idx_out is None else idx_out) if want_idx else None
    grad = (torch.empty((rows, k), dtype=torch.float32, device=dev) if grad_out is None else grad_out) \
        if want_grad else None
    for name, t_, dt in (("idx_out", idx, torch.int32), ("grad_out", grad, torch.float32)):
        if t_ is not None and (t_.shape != (rows, k) or t_.dtype != dt or not t_.is_contiguous() or t_.device != dev):
            raise ValueError(f"{name} must be a contiguous [rows, k] {dt} tensor on {dev}")
    _check(lib().nvfp4_topk_kl(_ptr(teacher), _ptr(student), rows, V, k, _ptr(loss), _ptr(idx), _ptr(grad),
                               _stream(dev)), "nvfp4_topk_kl")
    return loss, idx, grad


def dequantize(q: Quantized, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """BF16 values g*s*q of an NVFP4 tensor (nvfp4_dequantize)."""
    dev = q.codes.device
    y = torch.empty((q.rows, q.K), dtype=torch.bfloat16, device=dev) if out is None else out
    _check(lib().nvfp4_dequantize(_ptr(q.codes), _ptr(q.scales), _ptr(q.g), q.rows, q.K, _ptr(y), _stream(dev)),
           "nvfp4_dequantize")
    return y


def fake_quant_backward(x: torch.Tensor, grad_y: torch.Tensor, mode="max", g: Optional[torch.Tensor] = None,
                        scales: Optional[torch.Tensor] = None,
                        out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Gradient of fake_quant w.r.t. x, clipped straight-through
    (nvfp4_fake_quant_backward); scales as fake_quant with the same arguments."""
    x = _cuda(x, "x", torch.bfloat16)
    grad_y = _cuda(grad_y, "grad_y", torch.bfloat16)
    if grad_y.shape != x.shape:
        raise ValueError("grad_y must have x's shape")
    M, K = x.shape
    dev = x.device
    gx = torch.empty_like(x) if out is None else out
    ws = None
    ws_bytes = 0
    if g is None:
        ws_bytes = quantize_workspace_bytes(M, K)
        ws = _workspace(dev, ws_bytes)
    st = lib().nvfp4_fake_quant_backward(_ptr(x), _ptr(grad_y), M, K, _MODES[mode], _ptr(g), _ptr(scales),
                                         _ptr(gx), _ptr(ws), ws_bytes, _stream(dev))
    _check(st, "nvfp4_fake_quant_backward")
    return gx


def gemm(a: Quantized, b: Quantized, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """C = (ga*gb) * A_deq @ B_deq^T in BF16 [a.rows, b.rows] (nvfp4_gemm)."""
    if a.K != b.K:
        raise ValueError("K mismatch")
    dev = b.codes.device
    C = torch.empty((a.rows, b.rows), dtype=torch.bfloat16, device=dev) if out is None else out
    st = lib().nvfp4_gemm(_ptr(a.codes), _ptr(a.scales), _ptr(a.g), _ptr(b.codes), _ptr(b.scales), _ptr(b.g),
                          a.rows, b.rows, a.K, _ptr(C), _stream(dev))
    _check(st, "nvfp4_gemm")
    return C


def quantize_experts(w: torch.Tensor, mode="max") -> tuple:
    """Static per-expert weight quantization of w [E, N, K] (BF16, CUDA): one
    global scale per expert. Returns (Quantized over the E*N rows with the E
    tiled scale buffers concatenated, g [E] FP32)."""
    w = _cuda(w, "w", torch.bfloat16)
    E, N, K = w.shape
    dev = w.device
    sb = scale_bytes(N, K)
    codes = torch.empty((E * N, K // 2), dtype=torch.uint8, device=dev)
    scales = torch.empty(E * sb, dtype=torch.uint8, device=dev)
    g = torch.empty(E, dtype=torch.float32, device=dev)
    for e in range(E):
        quantize(w[e], mode, out=Quantized(codes[e * N:(e + 1) * N], scales[e * sb:(e + 1) * sb],
                                           g[e:e + 1], None, N, K))
    return Quantized(codes, scales, g, None, E * N, K), g


def moe_workspace_layout(T: int, H: int, I: int, E: int, topk: int) -> dict:
    lay = _MoeLayout()
    _check(lib().nvfp4_moe_workspace_layout(T, H, I, E, topk, ctypes.byref(lay)), "nvfp4_moe_workspace_layout")
    return {n: int(getattr(lay, n)) for n, _ in _MoeLayout._fields_}


def moe_grouped_gemm(x: torch.Tensor, topk_ids: torch.Tensor, topk_w: torch.Tensor, I: int,
                     w13: Quantized, w13_g: torch.Tensor, w2: Quantized, w2_g: torch.Tensor,
                     out: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None):
    """Routed-expert layer (nvfp4_moe_grouped_gemm). ``w13`` / ``w2`` hold the
    E experts' codes [E*2I, H/2] / [E*H, I/2] and concatenated per-expert
    tiled scales; ``w13_g`` / ``w2_g`` are the [E] FP32 global scales.
    Returns (out [T, H] FP32, workspace)."""
    x = _cuda(x, "x", torch.bfloat16)
    topk_ids = _cuda(topk_ids, "topk_ids", torch.int32)
    topk_w = _cuda(topk_w, "topk_w", torch.float32)
    T, H = x.shape
    topk = topk_ids.shape[1]
    E = w13_g.numel()
    dev = x.device
    if out is None:
        out = torch.empty((T, H), dtype=torch.float32, device=dev)
    nbytes = moe_workspace_bytes(T, H, I, E, topk)
    if workspace is None or workspace.numel() < nbytes:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    st = lib().nvfp4_moe_grouped_gemm(_ptr(x), T, H, _ptr(topk_ids), _ptr(topk_w), topk, E, I,
                                      _ptr(w13.codes), _ptr(w13.scales), _ptr(w13_g), _ptr(w2.codes),
                                      _ptr(w2.scales), _ptr(w2_g), _ptr(out), _ptr(workspace), nbytes,
                                      _stream(dev))
    _check(st, "nvfp4_moe_grouped_gemm")
    return out, workspace


def convert_e2m1(v: torch.Tensor) -> torch.Tensor:
    v = _cuda(v, "v", torch.float32)
    out = torch.empty(v.shape, dtype=torch.uint8, device=v.device)
    _check(lib().nvfp4_convert_e2m1(_ptr(v), v.numel(), _ptr(out), _stream(v.device)), "nvfp4_convert_e2m1")
    return out


def convert_e4m3(v: torch.Tensor) -> torch.Tensor:
    v = _cuda(v, "v", torch.float32)
    out = torch.empty(v.shape, dtype=torch.uint8, device=v.device)
    _check(lib().nvfp4_convert_e4m3(_ptr(v), v.numel(), _ptr(out), _stream(v.device)), "nvfp4_convert_e4m3")
    return out


def device_status(clear: bool = True, device=None) -> int:
    """Synchronize the current stream and return (and reset) the device status word.
    A timed-out wait (status 6) also zero-fills this device's cached
    quantize workspaces, whose grid-barrier counters it left stale."""
    dev = torch.device("cuda", torch.cuda.current_device() if device is None else device)
    v = ctypes.c_int(0)
    _check(lib().nvfp4_get_device_status(_stream(dev), int(clear), ctypes.byref(v)), "nvfp4_get_device_status")
    if v.value == 6:
        _reset_workspaces(dev.index)
    return v.value


def kernel_launches() -> int:
    """Kernels this library has launched in the process so far (nvfp4_kernel_launches)."""
    return int(lib().nvfp4_kernel_launches())


def probe_mma_peak(iters: int, device=None) -> float:
    """Launch the FP4 MMA rate probe (nvfp4_probe_mma_peak) on the current
    stream; returns the launch's FLOP count (time it with CUDA events)."""
    dev = torch.device("cuda", torch.cuda.current_device() if device is None else device)
    f = ctypes.c_double(0.0)
    _check(lib().nvfp4_probe_mma_peak(iters, ctypes.byref(f), _stream(dev)), "nvfp4_probe_mma_peak")
    return f.value


def selftest_gemm_timeout(a: Quantized, b: Quantized, timeout_ns: int, out: Optional[torch.Tensor] = None):
    """nvfp4_selftest_gemm_timeout: the GEMM with its first stage left unissued
    in one CTA, so that its bounded wait runs out (device status 6)."""
    dev = b.codes.device
    C = torch.empty((a.rows, b.rows), dtype=torch.bfloat16, device=dev) if out is None else out
    _check(lib().nvfp4_selftest_gemm_timeout(_ptr(a.codes), _ptr(a.scales), _ptr(a.g), _ptr(b.codes),
                                             _ptr(b.scales), _ptr(b.g), a.rows, b.rows, a.K, _ptr(C), timeout_ns,
                                             _stream(dev)), "nvfp4_selftest_gemm_timeout")
    return C


def selftest_timeout(timeout_ns: int, device=None) -> None:
    dev = torch.device("cuda", torch.cuda.current_device() if device is None else device)
    _check(lib().nvfp4_selftest_timeout(timeout_ns, _stream(dev)), "nvfp4_selftest_timeout")
