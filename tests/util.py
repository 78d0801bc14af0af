"""Shared helpers of the GPU parity tests: run the oracle on the same seeded
inputs and compare outputs of the CUDA path with it."""
import numpy as np
import pytest
import torch

from oracle import nvfp4_oracle as o


def require_gpu():
    if not torch.cuda.is_available():
        pytest.fail("GPU test run without a CUDA device")
    import qad_nvfp4_quantize_b200 as nv
    nv.check_device()
    return nv


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().numpy()


def bf16_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().to(torch.float32).numpy()


def oracle_quantized(x_f32: np.ndarray, mode="max", g=None):
    """Oracle quantization in the library's storage format."""
    q = o.quantize(x_f32, mode, g)
    return dict(codes=o.pack_codes(q["codes"]), scales=tiled(q["scales"]),
                g=q["g"], choice=q["choice"], raw=q)


def tiled(scales: np.ndarray) -> np.ndarray:
    """Vectorised placement into the tiled layout (same rule as the oracle's
    scales_to_tiled, which loops element by element)."""
    rows, nb = scales.shape
    kt = (nb + 3) // 4
    out = np.zeros(((rows + 127) // 128) * kt * 512, dtype=np.uint8)
    r = np.arange(rows)[:, None]
    c = np.arange(nb)[None, :]
    off = ((r // 128) * kt + c // 4) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + c % 4
    out[off] = scales
    return out


def assert_quantized_equal(gpu, ref, rows, K, check_choice=False):
    assert to_np(gpu.g)[0] == np.float32(ref["g"]), ("global scale", to_np(gpu.g)[0], ref["g"])
    codes = to_np(gpu.codes)
    mism = np.nonzero(codes != ref["codes"])
    assert mism[0].size == 0, f"{mism[0].size} code bytes differ, first at {mism[0][0]},{mism[1][0]}: " \
                              f"gpu {codes[mism][0]:#x} oracle {ref['codes'][mism][0]:#x}; first scale bytes " \
                              f"gpu {to_np(gpu.scales)[:8].tolist()} oracle {ref['scales'][:8].tolist()}"
    sc = to_np(gpu.scales)[: ref["scales"].size]
    bad = np.nonzero(sc != ref["scales"])[0]
    assert bad.size == 0, f"{bad.size} scale bytes differ, first at byte {bad[0]}"
    if check_choice:
        assert np.array_equal(to_np(gpu.choice), ref["choice"])


def gemm_check(C_gpu: np.ndarray, C_ref: np.ndarray, S: np.ndarray, what=""):
    tol = o.gemm_tolerance(C_ref, S)
    err = np.abs(C_gpu.astype(np.float64) - C_ref)
    bad = err > tol
    assert not bad.any(), (f"{what}: {bad.sum()} of {bad.size} outside tolerance; worst "
                           f"err/tol {np.max(err / np.maximum(tol, 1e-300)):.3g}")
    return float(np.max(err / np.maximum(tol, 1e-300)))
