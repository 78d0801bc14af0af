"""nvfp4_quantize_noalloc: the allocation-free variant of nvfp4_quantize.

Callers such as an inference plugin's enqueue step, which receives only input
and output pointers and may not allocate device memory, cannot pass a
workspace. This entry point reduces the global scale through the library's own
static device array instead. The test calls it through the C ABI twice in a
row (the static array keeps the previous call's contents) and checks each
result against nvfp4_quantize on the same input, bit for bit, as every
quantization test does. This file sorts last so that a stop-at-first-failure
run has already run every other test when it gets here.
"""
import ctypes

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


def _call_noalloc(L, x, q, mode, with_choice):
    M, K = x.shape
    st = L.nvfp4_quantize_noalloc(ctypes.c_void_p(x.data_ptr()), M, K, mode, None,
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
        got = _buffers(nv, M, K)
        _call_noalloc(L, x, got, mode, with_choice=True)
        want = nv.quantize(x, mode, want_choice=True)
        torch.cuda.synchronize()
        assert torch.equal(got["codes"], want.codes)
        assert torch.equal(got["scales"], want.scales[: got["scales"].numel()])
        assert torch.equal(got["g"], want.g)
        assert torch.equal(got["choice"], want.choice)
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
