"""GPU parity of the tcgen05 block-scaled W4A4 GEMM against the FP64 oracle,
|C - C_ref| <= 1e-4 * sum|a b| + BF16 rounding, through the C ABI."""
import numpy as np
import pytest
import torch

from oracle import nvfp4_oracle as o
from qad_nvfp4_quantize_b200 import inputs
from tests.util import assert_quantized_equal, bf16_np, gemm_check, oracle_quantized, require_gpu, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nv():
    return require_gpu()


def _operands(q, rows, K):
    return o.unpack_codes(to_np(q.codes)), o.scales_from_tiled(to_np(q.scales), rows, K), to_np(q.g)[0]


def run_gemm(nv, x, w, mode_w="max", rows=None):
    M, K = x.shape
    N = w.shape[0]
    qa = nv.quantize(x.cuda(), "max")
    qb = nv.quantize(w.cuda(), mode_w)
    C = bf16_np(nv.gemm(qa, qb)).astype(np.float64)
    ac, as_, ag = _operands(qa, M, K)
    bc, bs, bg = _operands(qb, N, K)
    C_ref, S = o.gemm_reference(ac, as_, ag, bc, bs, bg, rows=rows)
    return (C if rows is None else C[rows]), C_ref, S, qa, qb


def test_gemm_tiny_linear(nv):
    d = inputs.tiny_linear(0)
    C, C_ref, S, qa, qb = run_gemm(nv, d["x"], d["w"])
    assert_quantized_equal(qa, oracle_quantized(bf16_np(d["x"])), 128, 256)
    assert_quantized_equal(qb, oracle_quantized(bf16_np(d["w"])), 256, 256)
    gemm_check(C, C_ref, S, "tiny")
    # also against numpy float64 matmul of the dequantized operands
    A = o.dequantize_f64(*_operands(qa, 128, 256)[:2]) * float(to_np(qa.g)[0])
    B = o.dequantize_f64(*_operands(qb, 256, 256)[:2]) * float(to_np(qb.g)[0])
    assert np.allclose(A @ B.T, C_ref, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("M,N,K", [(1, 16, 64), (200, 272, 320), (128, 512, 2048), (333, 784, 1088),
                                   (1000, 256, 5120)])
def test_gemm_ragged_shapes(nv, M, N, K):
    rng = np.random.default_rng(M + N + K)
    x = inputs.to_bf16((rng.standard_t(3, (M, K)) * 0.5).astype(np.float32))
    w = inputs.to_bf16((rng.standard_normal((N, K)) * 0.02).astype(np.float32))
    C, C_ref, S, _, _ = run_gemm(nv, x, w, "four_over_six")
    gemm_check(C, C_ref, S, f"{M}x{N}x{K}")


def test_gemm_empty_m(nv):
    w = inputs.to_bf16(np.ones((32, 64), np.float32)).cuda()
    qb = nv.quantize(w)
    qa = nv.quantize(torch.empty((0, 64), dtype=torch.bfloat16, device="cuda"))
    C = nv.gemm(qa, qb)
    assert C.shape == (0, 32)
    assert nv.device_status() == 0


def test_gemm_closed_form(nv):
    # every element 1.0: quantizes exactly (g = 1/448, s = 448, q = 6 ... q*s*g = 1)
    K = 1024
    x = torch.ones((130, K), dtype=torch.bfloat16, device="cuda")
    w = -torch.ones((48, K), dtype=torch.bfloat16, device="cuda")
    C = nv.gemm(nv.quantize(x), nv.quantize(w))
    assert torch.all(C.float() == -K)


def test_gemm_bounded_wait_runs_out_and_context_survives(nv):
    """The first CTA's producer leaves its first stage unissued, so the MMA
    warp's own bounded wait (1 ms here) runs out: the call reports
    NVFP4_ERR_TIMEOUT through the device status word, the other CTAs finish
    their tiles, and the next GEMM on the same context matches the oracle."""
    rng = np.random.default_rng(77)
    M, N, K = 512, 1024, 1024                    # 4 x 4 tiles: CTA 0 times out, 15 finish
    x = inputs.to_bf16((rng.standard_t(3, (M, K)) * 0.5).astype(np.float32))
    w = inputs.to_bf16((rng.standard_normal((N, K)) * 0.02).astype(np.float32))
    qa = nv.quantize(x.cuda(), "max")
    qb = nv.quantize(w.cuda(), "max")
    assert nv.device_status(clear=True) == 0
    nv.selftest_gemm_timeout(qa, qb, 1_000_000)
    assert nv.device_status(clear=True) == 6
    C = bf16_np(nv.gemm(qa, qb)).astype(np.float64)
    assert nv.device_status(clear=True) == 0
    ac, as_, ag = _operands(qa, M, K)
    bc, bs, bg = _operands(qb, N, K)
    C_ref, S = o.gemm_reference(ac, as_, ag, bc, bs, bg)
    gemm_check(C, C_ref, S, "after a timed-out GEMM")


def test_dynamic_quantize_on_two_streams(nv):
    """Two dynamic quantizations issued on two streams with no ordering
    between them: each stream has its own workspace (grid barrier and amax
    partials), so each call's global scale equals the oracle's."""
    rng = np.random.default_rng(78)
    xs = [inputs.to_bf16((rng.standard_t(3, (2048, 2048)) * s).astype(np.float32)) for s in (0.5, 3.0)]
    xd = [x.cuda() for x in xs]
    torch.cuda.synchronize()
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    outs = [None, None]
    for _ in range(3):
        for i in (0, 1):
            with torch.cuda.stream(streams[i]):
                outs[i] = nv.quantize(xd[i], "max")
        torch.cuda.synchronize()
        for i in (0, 1):
            assert to_np(outs[i].g)[0] == o.global_scale(bf16_np(xs[i]))[0], i
    assert nv.device_status(clear=True) == 0
