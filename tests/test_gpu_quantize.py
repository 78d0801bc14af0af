"""GPU parity of conversions, quantize, four_over_six and fake-quant against
the CPU oracle (bit-exact), through the C ABI."""
import numpy as np
import pytest
import torch

from oracle import nvfp4_oracle as o
from qad_nvfp4_quantize_b200 import inputs
from tests.util import assert_quantized_equal, bf16_np, oracle_quantized, require_gpu, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nv():
    return require_gpu()


def _sweep_values():
    rng = np.random.default_rng(21)
    # every finite BF16 bit pattern (as FP32), plus random FP32 values
    bits = np.arange(0, 1 << 16, dtype=np.uint32) << 16
    allbf = bits.view(np.float32)
    allbf = allbf[np.isfinite(allbf)]
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0], np.float32)
    near = np.concatenate([mids, np.nextafter(mids, np.float32(0)), np.nextafter(mids, np.float32(9))])
    return np.concatenate([allbf, near, -near, rng.uniform(-8, 8, 1 << 20).astype(np.float32),
                           (rng.standard_normal(1 << 18) * 1e-3).astype(np.float32)])


def test_e2m1_conversion_matches_oracle(nv):
    v = _sweep_values()
    got = to_np(nv.convert_e2m1(torch.from_numpy(v).cuda()))
    want = o.e2m1_encode(v)
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, f"{bad.size} differ, e.g. v={v[bad[:5]]} gpu={got[bad[:5]]} oracle={want[bad[:5]]}"


def test_e4m3_conversion_matches_oracle(nv):
    v = np.abs(_sweep_values()) * np.float32(64.0)
    v = np.concatenate([v, o.e4m3_decode_table().astype(np.float32), np.array([448, 460, 464, 1e30], np.float32)])
    got = to_np(nv.convert_e4m3(torch.from_numpy(v.astype(np.float32)).cuda()))
    want = o.e4m3_encode(v.astype(np.float32))
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, f"{bad.size} differ, e.g. t={v[bad[:5]]} gpu={got[bad[:5]]} oracle={want[bad[:5]]}"


@pytest.mark.parametrize("which", ["x", "w"])
def test_quantize_tiny_linear(nv, which):
    d = inputs.tiny_linear(0)
    x = d[which]
    q = nv.quantize(x.cuda(), "max")
    assert_quantized_equal(q, oracle_quantized(bf16_np(x)), *x.shape)


@pytest.mark.parametrize("M,K", [(1, 64), (127, 192), (200, 320), (129, 1024), (385, 5120)])
def test_quantize_ragged_shapes(nv, M, K):
    rng = np.random.default_rng(M * 7 + K)
    x = inputs.to_bf16((rng.standard_t(3, (M, K)) * 0.5).astype(np.float32))
    for mode in ("max", "four_over_six"):
        q = nv.quantize(x.cuda(), mode, want_choice=True)
        assert_quantized_equal(q, oracle_quantized(bf16_np(x), mode), M, K, check_choice=True)


def test_quantize_empty(nv):
    x = torch.empty((0, 256), dtype=torch.bfloat16, device="cuda")
    q = nv.quantize(x)
    assert to_np(q.g)[0] == 1.0


def test_quantize_static_global_scale(nv):
    d = inputs.tiny_linear(3)
    x = bf16_np(d["x"])
    g = np.float32(0.0007)
    q = nv.quantize(d["x"].cuda(), "max", g=torch.tensor([g], device="cuda"))
    assert_quantized_equal(q, oracle_quantized(x, "max", g), *x.shape)


def test_quantize_zero_and_tiny_blocks(nv):
    x = np.zeros((128, 256), np.float32)
    x[0, 0] = 3.0
    x[5, 16:32] = 1e-30          # blocks far below the tensor amax: scale floor 2^-9
    x[7, 32:48] = -0.0
    xt = inputs.to_bf16(x)
    for mode in ("max", "four_over_six"):
        q = nv.quantize(xt.cuda(), mode, want_choice=True)
        assert_quantized_equal(q, oracle_quantized(bf16_np(xt), mode), 128, 256, check_choice=True)


def _fma_choice(blocks: np.ndarray, g: np.float32) -> np.ndarray:
    """four_over_six choice as a kernel that fused d*q into the subtraction
    (one rounding of x - d*q) would take it: used only to find blocks whose
    choice depends on the products being rounded separately."""
    bmax = np.max(np.abs(blocks), axis=1)
    errs = []
    for mt in (6.0, 4.0):
        sc = o.block_scale_codes(bmax, g, mt)
        d = (np.float32(g) * o.e4m3_decode(sc).astype(np.float32)).astype(np.float32)
        q = o.e2m1_encode(blocks * (np.float32(1) / d)[:, None])
        # float64 holds x - d*q exactly here; one rounding to FP32 as an FMA does
        df = (blocks.astype(np.float64) - d.astype(np.float64)[:, None] *
              o.e2m1_decode(q).astype(np.float64)).astype(np.float32)
        sq = df * df
        e = np.zeros(len(blocks), np.float32)
        for i in range(16):
            e = e + sq[:, i]
        errs.append(e)
    return (errs[1] < errs[0]).astype(np.uint8)


def test_four_over_six_near_ties_round_each_product(nv):
    # Blocks whose M=4 / M=6 errors agree to the last few ULPs: the choice flips
    # if any product of the error sum is fused with the following subtraction.
    rng = np.random.default_rng(46)
    amax = np.float32(87.5)
    g = np.float32(amax / np.float32(2688.0))
    t = np.clip(rng.standard_t(3, (1 << 19, 16)) * 0.5, -80.0, 80.0).astype(np.float32)
    cand = bf16_np(inputs.to_bf16(t))
    ref = o.quantize(cand, "four_over_six", g)["choice"][:, 0]
    flips = np.nonzero(ref != _fma_choice(cand, g))[0]
    assert flips.size >= 4, flips.size
    picked = cand[flips[: 4 * (flips.size // 4)]]
    top = np.zeros((4, 16), np.float32)
    top[0, 0] = amax  # the tensor's maximum, so the dynamic g equals g
    x = np.ascontiguousarray(np.concatenate([picked, cand[:256], top]).reshape(-1, 64))
    assert o.global_scale(x)[0] == g
    xt = torch.from_numpy(x).to(torch.bfloat16)
    q = nv.quantize(xt.cuda(), "four_over_six", want_choice=True)
    assert_quantized_equal(q, oracle_quantized(x, "four_over_six"), x.shape[0], 64, check_choice=True)
    # the same blocks through fake-quant, whose output follows the choice
    y = to_np(nv.fake_quant(xt.cuda(), "four_over_six").view(torch.int16))
    y_ref = torch.from_numpy(o.fake_quant(x, "four_over_six")).to(torch.bfloat16).view(torch.int16).numpy()
    np.testing.assert_array_equal(y, y_ref)


def test_four_over_six_outlier_weights(nv):
    d = inputs.four_over_six_linear(0, M=16, N=1024, K=2048)
    w = d["w"]
    q = nv.quantize(w.cuda(), "four_over_six", want_choice=True)
    ref = oracle_quantized(bf16_np(w), "four_over_six")
    assert_quantized_equal(q, ref, *w.shape, check_choice=True)
    assert 0 < ref["choice"].mean() < 1          # both candidates occur


@pytest.mark.parametrize("mode", ["max", "four_over_six"])
def test_fake_quant_dynamic(nv, mode):
    d = inputs.four_over_six_linear(1, M=300, N=256, K=1024)
    x = d["w"]
    y = nv.fake_quant(x.cuda(), mode)
    want = o.fake_quant(bf16_np(x), mode)
    assert np.array_equal(bf16_np(y), want)


def test_fake_quant_frozen_and_static(nv):
    rng = np.random.default_rng(5)
    w0 = inputs.to_bf16((rng.standard_normal((256, 512)) * 0.02).astype(np.float32))
    q = nv.quantize(w0.cuda(), "four_over_six")
    ref = o.quantize(bf16_np(w0), "four_over_six")
    drift = inputs.to_bf16(bf16_np(w0) * 1.7 + (rng.standard_normal((256, 512)) * 0.01).astype(np.float32))
    y = nv.fake_quant(drift.cuda(), g=q.g, scales=q.scales)
    want = o.fake_quant(bf16_np(drift), g_frozen=ref["g"], scales_frozen=ref["scales"])
    assert np.array_equal(bf16_np(y), want)
    g = torch.tensor([np.float32(1e-4)], device="cuda")
    y2 = nv.fake_quant(drift.cuda(), "max", g=g)
    q2 = o.quantize(bf16_np(drift), "max", np.float32(1e-4))
    want2 = o.bf16_round(o.dequantize(q2["codes"], q2["scales"], q2["g"]))
    assert np.array_equal(bf16_np(y2), want2)


def test_fake_quant_equals_dequantized_quantize(nv):
    d = inputs.dense_mlp(2, M=64, N=16, K=512)
    x = d["x"].cuda()
    q = nv.quantize(x, "max")
    y = nv.fake_quant(x, "max")
    codes = o.unpack_codes(to_np(q.codes))
    scales = o.scales_from_tiled(to_np(q.scales), 64, 512)
    assert np.array_equal(bf16_np(y), o.bf16_round(o.dequantize(codes, scales, to_np(q.g)[0])))


def test_nonfinite_input_sets_device_status(nv):
    nv.device_status(clear=True)
    x = torch.zeros((128, 256), dtype=torch.bfloat16, device="cuda")
    x[3, 7] = float("inf")
    nv.quantize(x)
    assert nv.device_status(clear=True) == 5
    x[3, 7] = float("nan")
    nv.quantize(x)
    assert nv.device_status(clear=True) == 5
    x[3, 7] = 1.0
    nv.quantize(x)
    assert nv.device_status(clear=True) == 0


def test_bounded_wait_reports_timeout(nv):
    nv.device_status(clear=True)
    nv.selftest_timeout(2_000_000)     # 2 ms on a flag nothing sets
    assert nv.device_status(clear=True) == 6
    x = torch.ones((128, 64), dtype=torch.bfloat16, device="cuda")
    nv.quantize(x)                      # the context is still usable
    assert nv.device_status(clear=True) == 0


@pytest.mark.parametrize("M,K", [(3, 64), (130, 320), (64, 1024)])
def test_mse_calibration_matches_oracle(nv, M, K):
    rng = np.random.default_rng(M + K)
    x = (rng.standard_t(3, (M, K)) * 0.05).astype(np.float32)
    x[0, :16] = 0.0                                             # all-tie block: lowest code
    x[1 % M, 16:32] = rng.choice([-6, -1, 0, 0.5, 3, 6], 16) * 0.01  # exact on some scale grid
    x[2 % M, 40] = 3.0                                          # outlier sets the amax
    xt = inputs.to_bf16(x)
    for g in (None, torch.tensor([np.float32(0.05)])):
        q = nv.quantize(xt.cuda(), "mse", g=None if g is None else g.cuda(), want_choice=True)
        ref = oracle_quantized(bf16_np(xt), "mse", None if g is None else np.float32(0.05))
        assert_quantized_equal(q, ref, M, K)
        assert not to_np(q.choice).any()


def test_mse_calibration_full_weight_sampled_rows(nv):
    # W 14336 x 4096 with 0.1% outliers: quantize on the GPU, check sampled rows
    # against the oracle run with the GPU's global scale
    d = inputs.four_over_six_linear(0, M=16)
    w = d["w"]
    q = nv.quantize(w.cuda(), "mse")
    g = np.float32(to_np(q.g)[0])
    wf = bf16_np(w)
    assert g == o.global_scale(wf)[0]
    rows = np.array([0, 1, 127, 128, 5000, 9999, 14335])
    ref = o.quantize(wf[rows], "mse", g)
    codes = o.unpack_codes(to_np(q.codes)[rows])
    scales = o.scales_from_tiled(to_np(q.scales), w.shape[0], w.shape[1])[rows]
    assert np.array_equal(scales, ref["scales"])
    assert np.array_equal(codes, ref["codes"])


def test_mse_rejected_outside_quantize(nv):
    x = torch.zeros((4, 64), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(nv.NVFP4Error):
        nv.fake_quant(x, "mse")
    with pytest.raises(nv.NVFP4Error):
        nv.quantize_noalloc(x, "mse")


@pytest.mark.parametrize("mode", ["max", "four_over_six"])
def test_ste_backward_dynamic_and_static(nv, mode):
    rng = np.random.default_rng(41)
    M, K = 130, 320
    x = inputs.to_bf16((rng.standard_t(3, (M, K)) * 0.2).astype(np.float32))
    gy = inputs.to_bf16(rng.standard_normal((M, K)).astype(np.float32))
    gx = nv.fake_quant_backward(x.cuda(), gy.cuda(), mode)
    ref = o.fake_quant_backward(bf16_np(x), bf16_np(gy), mode)
    np.testing.assert_array_equal(bf16_np(gx), ref)
    # static g: the scales are recomputed from x under the given g; with g
    # below amax/2688 many blocks saturate at E4M3 448 and clip
    g = np.float32(0.1 / 2688)
    gx = nv.fake_quant_backward(x.cuda(), gy.cuda(), mode, g=torch.tensor([g]).cuda())
    q = o.quantize(bf16_np(x), mode, g)
    ref = o.fake_quant_backward(bf16_np(x), bf16_np(gy), g_frozen=g, scales_frozen=q["scales"])
    np.testing.assert_array_equal(bf16_np(gx), ref)
    assert (ref == 0).any()


@pytest.mark.parametrize("M,K", [(40000, 64), (12000, 1088), (9000, 2048)])
def test_fake_quant_and_ste_refill_freed_slots(nv, M, K):
    # More 512-element chunks per CTA than the 224 it keeps in shared memory,
    # so phase 2 of the fused pass refills freed slots by bulk copies: partial
    # chunks (K = 64, and the 64-element tail of K = 1088) and whole 1 KB
    # chunks (K = 2048), all compared with the oracle bit for bit.
    rng = np.random.default_rng(M + K)
    x = inputs.to_bf16((rng.standard_t(3, (M, K)) * 0.3).astype(np.float32))
    gy = inputs.to_bf16(rng.standard_normal((M, K)).astype(np.float32))
    cpr = -(-K // 512)
    per = -(-(M * cpr) // torch.cuda.get_device_properties(0).multi_processor_count)
    ch = per * 10 + 240  # the 241st chunk of CTA 10's range: not kept
    x[ch // cpr, (ch % cpr) * 512] = 40.0  # the tensor's amax
    xd, gyd = x.cuda(), gy.cuda()
    xf, gf = bf16_np(x), bf16_np(gy)
    for mode in ("max", "four_over_six"):
        np.testing.assert_array_equal(bf16_np(nv.fake_quant(xd, mode)), o.fake_quant(xf, mode))
    np.testing.assert_array_equal(bf16_np(nv.fake_quant_backward(xd, gyd, "max")),
                                  o.fake_quant_backward(xf, gf, "max"))


def test_bf16_outputs_at_16_byte_alignment(nv):
    # BF16 outputs are written 32 bytes per lane when the buffer is 32-byte
    # aligned and 16 bytes at a time otherwise; both layouts give the
    # oracle's values (dynamic and frozen fake-quant, dequantize, STE)
    rng = np.random.default_rng(5)
    M, K = 300, 1024
    x = inputs.to_bf16((rng.standard_t(3, (M, K)) * 0.3).astype(np.float32))
    xd = x.cuda()
    base = torch.empty(M * K + 8, dtype=torch.bfloat16, device="cuda")
    y16 = base[8:].view(M, K)                     # 16 bytes past a 256-byte boundary
    assert y16.data_ptr() % 32 == 16
    want = o.fake_quant(bf16_np(x), "max")
    np.testing.assert_array_equal(bf16_np(nv.fake_quant(xd, "max", out=y16)), want)
    q = nv.quantize(xd, "max")
    np.testing.assert_array_equal(bf16_np(nv.fake_quant(xd, g=q.g, scales=q.scales, out=y16)), want)
    np.testing.assert_array_equal(bf16_np(nv.dequantize(q, out=y16)), want)
    np.testing.assert_array_equal(bf16_np(nv.dequantize(q)), want)
    gy = inputs.to_bf16(rng.standard_normal((M, K)).astype(np.float32))
    want_gx = o.fake_quant_backward(bf16_np(x), bf16_np(gy), "max")
    for out in (y16, None):  # dynamic (fused pass) and frozen scales (streaming pass)
        np.testing.assert_array_equal(bf16_np(nv.fake_quant_backward(xd, gy.cuda(), "max", out=out)), want_gx)
        np.testing.assert_array_equal(
            bf16_np(nv.fake_quant_backward(xd, gy.cuda(), g=q.g, scales=q.scales, out=out)), want_gx)


def test_ste_backward_frozen_scales(nv):
    rng = np.random.default_rng(42)
    M, K = 200, 512
    w0 = inputs.to_bf16((rng.standard_normal((M, K)) * 0.02).astype(np.float32))
    q0 = nv.quantize(w0.cuda(), "four_over_six")                # calibrated once (PTQ)
    w1 = inputs.to_bf16((bf16_np(w0) * 1.3 + rng.standard_normal((M, K)) * 0.004).astype(np.float32))
    gy = inputs.to_bf16(rng.standard_normal((M, K)).astype(np.float32))
    gx = nv.fake_quant_backward(w1.cuda(), gy.cuda(), g=q0.g, scales=q0.scales)
    sc = o.scales_from_tiled(to_np(q0.scales), M, K)
    ref = o.fake_quant_backward(bf16_np(w1), bf16_np(gy), g_frozen=to_np(q0.g)[0], scales_frozen=sc)
    np.testing.assert_array_equal(bf16_np(gx), ref)
    assert (ref == 0).any() and (ref != 0).any()


def test_kv_cache_round_trip(nv):
    # K / V of 8 KV heads x 128 dims per token, NVFP4 (four_over_six) in the
    # cache, BF16 on read: equals the oracle and the GPU fake-quant
    rng = np.random.default_rng(52)
    for T in (1, 300):
        kv = inputs.to_bf16((rng.standard_normal((T, 1024)) * 0.7).astype(np.float32))
        q = nv.quantize(kv.cuda(), "four_over_six")
        y = nv.dequantize(q)
        ref = o.fake_quant(bf16_np(kv), "four_over_six")
        np.testing.assert_array_equal(bf16_np(y), ref)
        np.testing.assert_array_equal(to_np(y.view(torch.int16)),
                                      to_np(nv.fake_quant(kv.cuda(), "four_over_six").view(torch.int16)))


def test_long_rows_take_the_64bit_chunk_path(nv):
    # 4 rows of 2^24 + 64 elements: M * (chunks per row)^2 >= 2^32, so every
    # kernel walks the tensor with 64-bit chunk arithmetic; sampled column
    # windows (the ragged last chunk included) against the oracle with the
    # GPU's global scale, which must equal the oracle's over the whole tensor
    M, K = 4, (1 << 24) + 64
    gen = torch.Generator().manual_seed(61)
    x = (torch.randn((M, K), generator=gen) * 0.3).to(torch.bfloat16)
    x[2, K - 7] = 5.0                                           # amax in the ragged tail
    xf = bf16_np(x)
    g_ref = o.global_scale(xf)[0]
    xd = x.cuda()
    windows = [0, 512 * 1000 + 64, 1 << 23, K - 4096]
    for mode in ("max", "four_over_six"):
        q = nv.quantize(xd, mode)
        assert to_np(q.g)[0] == g_ref
        codes = o.unpack_codes(to_np(q.codes))
        scales = o.scales_from_tiled(to_np(q.scales), M, K)
        y = bf16_np(nv.fake_quant(xd, mode))
        for c0 in windows:
            ref = o.quantize(xf[:, c0:c0 + 4096], mode, g_ref)
            assert np.array_equal(codes[:, c0:c0 + 4096], ref["codes"])
            assert np.array_equal(scales[:, c0 // 16:(c0 + 4096) // 16], ref["scales"])
            fq = o.bf16_round(o.dequantize(ref["codes"], ref["scales"], g_ref))
            np.testing.assert_array_equal(y[:, c0:c0 + 4096], fq)
        if mode == "four_over_six":
            dq = bf16_np(nv.dequantize(q))
            np.testing.assert_array_equal(dq, y)
    qs = nv.quantize(xd, "max", g=torch.tensor([np.float32(0.01)]).cuda())  # static g: streaming kernel
    codes = o.unpack_codes(to_np(qs.codes))
    for c0 in windows:
        ref = o.quantize(xf[:, c0:c0 + 4096], "max", np.float32(0.01))
        assert np.array_equal(codes[:, c0:c0 + 4096], ref["codes"])
