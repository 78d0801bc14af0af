"""nvfp4_quantize_noalloc: the allocation-free variant of nvfp4_quantize.

Callers such as an inference plugin's enqueue step, which receives only input
and output pointers and may not allocate device memory, cannot pass a
workspace. This entry point reduces the global scale through the library's own
static device array instead. The test calls it through the C ABI twice in a
row (the static array keeps the previous call's contents) and checks each
result against nvfp4_quantize on the same input and against the CPU oracle,
bit for bit, as every quantization test does. This file sorts last so that a
stop-at-first-failure run has already run every other test when it gets here.
"""
import ctypes

import numpy as np
import pytest
import torch

from tests.util import bf16_np, oracle_quantized

pytestmark = pytest.mark.gpu


def _call_noalloc(L, x, q, mode, with_choice, g_in=None):
    M, K = x.shape
    st = L.nvfp4_quantize_noalloc(ctypes.c_void_p(x.data_ptr()), M, K, mode,
                                  None if g_in is None else ctypes.c_void_p(g_in.data_ptr()),
                                  ctypes.c_void_p(q["codes"].data_ptr()), ctypes.c_void_p(q["scales"].data_ptr()),
                                  ctypes.c_void_p(q["g"].data_ptr()),
                                  ctypes.c_void_p(q["choice"].data_ptr()) if with_choice else None,
                                  ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0, st


def _buffers(nv, M, K):
    return dict(codes=torch.empty((M, K // 2), dtype=torch.uint8, device="cuda"),
                scales=torch.empty(nv.scale_bytes(M, K), dtype=torch.uint8, device="cuda"),
                g=torch.empty(1, dtype=torch.float32, device="cuda"),
                choice=torch.empty((M, K // 16), dtype=torch.uint8, device="cuda"))


def test_noalloc_matches_quantize_on_two_calls_in_a_row():
    if not torch.cuda.is_available():
        pytest.fail("GPU test run without a CUDA device")
    import qad_nvfp4_quantize_b200 as nv
    from qad_nvfp4_quantize_b200 import inputs
    nv.check_device()
    L = nv.lib()
    cases = [
        (inputs.dense_mlp(11, M=300, N=16, K=5120)["x"], nv.MODE_MAX),           # 1.5 Mi elements: 6 slots
        (inputs.four_over_six_linear(12, M=8, N=640, K=1024)["w"], nv.MODE_FOUR_OVER_SIX),
    ]
    for x_cpu, mode in cases:
        x = x_cpu.cuda()
        M, K = x.shape
        ref = oracle_quantized(bf16_np(x_cpu), "four_over_six" if mode == nv.MODE_FOUR_OVER_SIX else "max")
        got = _buffers(nv, M, K)
        _call_noalloc(L, x, got, mode, with_choice=True)
        want = nv.quantize(x, mode, want_choice=True)
        torch.cuda.synchronize()
        assert torch.equal(got["codes"], want.codes)
        assert torch.equal(got["scales"], want.scales[: got["scales"].numel()])
        assert torch.equal(got["g"], want.g)
        assert torch.equal(got["choice"], want.choice)
        assert np.array_equal(got["codes"].cpu().numpy(), ref["codes"])
        assert np.array_equal(got["scales"].cpu().numpy()[: ref["scales"].size], ref["scales"])
        assert got["g"].item() == ref["g"]
        assert np.array_equal(got["choice"].cpu().numpy(), ref["choice"])
    assert nv.device_status() == 0


def test_noalloc_static_scale_empty_input_and_modes():
    if not torch.cuda.is_available():
        pytest.fail("GPU test run without a CUDA device")
    import qad_nvfp4_quantize_b200 as nv
    from qad_nvfp4_quantize_b200 import inputs
    nv.check_device()
    L = nv.lib()
    # a static global scale: no amax pass, the scratch array is not touched
    x_cpu = inputs.tiny_linear(13)["x"]
    g = torch.tensor([np.float32(0.0009)], device="cuda")
    got = _buffers(nv, *x_cpu.shape)
    _call_noalloc(L, x_cpu.cuda(), got, nv.MODE_MAX, with_choice=False, g_in=g)
    torch.cuda.synchronize()
    ref = oracle_quantized(bf16_np(x_cpu), "max", np.float32(0.0009))
    assert np.array_equal(got["codes"].cpu().numpy(), ref["codes"])
    assert np.array_equal(got["scales"].cpu().numpy()[: ref["scales"].size], ref["scales"])
    assert got["g"].item() == np.float32(0.0009)
    # M = 0: nothing to quantize, the dynamic global scale is 1
    empty = torch.empty((0, 64), dtype=torch.bfloat16, device="cuda")
    g0 = torch.zeros(1, dtype=torch.float32, device="cuda")
    st = L.nvfp4_quantize_noalloc(ctypes.c_void_p(empty.data_ptr()), 0, 64, nv.MODE_MAX, None, None, None,
                                  ctypes.c_void_p(g0.data_ptr()), None,
                                  ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0
    torch.cuda.synchronize()
    assert g0.item() == 1.0
    # MSE calibration is not offered here (NVFP4_ERR_INVALID_ARG before any launch)
    st = L.nvfp4_quantize_noalloc(ctypes.c_void_p(256), 1, 64, nv.MODE_MSE, None, ctypes.c_void_p(256),
                                  ctypes.c_void_p(256), ctypes.c_void_p(256), None, None)
    assert st == 1
    assert nv.device_status() == 0


def test_noalloc_rejects_inputs_beyond_its_scratch():
    if not torch.cuda.is_available():
        pytest.fail("GPU test run without a CUDA device")
    import qad_nvfp4_quantize_b200 as nv
    L = nv.lib()
    fake = ctypes.c_void_p(256)          # never dereferenced: the size check comes first
    st = L.nvfp4_quantize_noalloc(fake, (1 << 20) + 1, 1024, 0, None, fake, fake, fake, None, None)
    assert st == 7
    assert L.nvfp4_status_string(7).startswith(b"input larger")
