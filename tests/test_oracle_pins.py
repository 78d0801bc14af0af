"""Pins of the CPU oracle to facts outside itself (CPU only).

Each test checks the oracle against something it does not compute itself:
values the pages print (tests/golden/nvfp4_format.json), library conversions
(ml_dtypes float4_e2m1fn / float8_e4m3fn, torch bfloat16 and float8 casts,
numpy stable argsort), closed forms, hand-worked examples and brute force on
tiny inputs.
"""
import json
import os

import ml_dtypes
import numpy as np
import pytest
import torch

from oracle import nvfp4_oracle as o


def lib_e2m1(v):
    """Library E2M1 conversion (RNE, saturating) -> 4-bit codes."""
    return np.asarray(v, np.float32).astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 0xF


def lib_e2m1_value(v):
    return np.asarray(v, np.float32).astype(ml_dtypes.float4_e2m1fn).astype(np.float32)


def lib_e4m3_value(t):
    """Library E4M3 conversion, saturated at 448 (the library itself gives NaN
    above the largest finite value, so clamp first)."""
    t = np.minimum(np.asarray(t, np.float32), np.float32(448.0))
    return t.astype(ml_dtypes.float8_e4m3fn).astype(np.float32)


@pytest.fixture(scope="module")
def fmt(golden_dir):
    with open(os.path.join(golden_dir, "nvfp4_format.json")) as f:
        return json.load(f)


# ---------------------------------------------------------------- formats ----

def test_e2m1_grid_is_the_printed_grid(fmt):
    table = o.e2m1_decode_table()
    assert list(table[:8]) == fmt["e2m1_magnitudes"]
    assert list(-table[8:]) == fmt["e2m1_magnitudes"]
    lib = np.arange(16, dtype=np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    assert np.array_equal(lib, table)
    assert fmt["quantization_recipe"]["num_bits"] == [2, 1]


def test_e2m1_encode_matches_library_sweep():
    rng = np.random.default_rng(1)
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0], np.float32)
    near = np.concatenate([np.nextafter(mids, np.float32(0)), mids, np.nextafter(mids, np.float32(9))])
    vals = np.concatenate([
        near, -near, o.e2m1_decode_table().astype(np.float32),
        rng.uniform(-8, 8, 200000).astype(np.float32),
        rng.standard_normal(100000).astype(np.float32) * 1e-3,
        np.array([0.0, -0.0, 6.0, -6.0, 6.5, 1e30, -1e30, np.inf, -np.inf, 1e-45, -1e-45], np.float32),
    ])
    assert np.array_equal(o.e2m1_encode(vals), lib_e2m1(vals))


def test_e2m1_ties_go_to_the_even_code():
    # midpoint -> expected magnitude, worked from the grid by hand
    table = {0.25: 0.0, 0.75: 1.0, 1.25: 1.0, 1.75: 2.0, 2.5: 2.0, 3.5: 4.0, 5.0: 4.0}
    for v, want in table.items():
        got = o.e2m1_decode(o.e2m1_encode(np.float32(v)))
        assert got == want, (v, got)
    assert o.e2m1_encode(np.float32(-0.1)) == 0x8
    assert o.e2m1_encode(np.float32(100.0)) == 0x7


def test_e4m3_table_matches_library():
    table = o.e4m3_decode_table()
    lib = np.arange(127, dtype=np.uint8).view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    assert np.array_equal(table, lib)
    assert table[0x7E] == 448.0 and table.max() == 448.0
    assert table[1] == 2.0 ** -9
    assert np.all(np.diff(table) > 0)


def test_e4m3_encode_matches_library_and_torch():
    rng = np.random.default_rng(2)
    table = o.e4m3_decode_table().astype(np.float32)
    mids = ((table[1:].astype(np.float64) + table[:-1]) / 2).astype(np.float32)
    vals = np.concatenate([
        table, mids, np.nextafter(mids, np.float32(0)), np.nextafter(mids, np.float32(1e9)),
        rng.uniform(0, 463, 100000).astype(np.float32),
        np.exp(rng.uniform(-30, 6, 100000)).astype(np.float32),
    ])
    vals = vals[vals < 464]
    got = o.e4m3_decode(o.e4m3_encode(vals)).astype(np.float32)
    assert np.array_equal(got, vals.astype(ml_dtypes.float8_e4m3fn).astype(np.float32))
    tor = torch.from_numpy(vals).to(torch.float8_e4m3fn).to(torch.float32).numpy()
    assert np.array_equal(got, tor)
    # satfinite: anything at or above 448 is 448
    big = np.array([448.0, 460.0, 464.0, 1000.0, 1e30], np.float32)
    assert np.all(o.e4m3_encode(big) == 0x7E)


def test_bf16_round_matches_torch():
    rng = np.random.default_rng(3)
    x = np.concatenate([rng.standard_normal(100000).astype(np.float32) * 10.0 ** rng.integers(-20, 20, 100000),
                        np.array([0.0, -0.0, 1.0, 1.00390625, 1.0078125, 3.0e38], np.float32)]).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float32).numpy()
    assert np.array_equal(o.bf16_round(x), ref)


def test_bf16_round_f64_is_nearest():
    rng = np.random.default_rng(4)
    x = rng.standard_normal(20000) * 10.0 ** rng.integers(-5, 5, 20000)
    r = o.bf16_round_f64(x)
    # r is a BF16 value and no BF16 value is closer (brute force over neighbours)
    r32 = r.astype(np.float32)
    assert np.array_equal(o.bf16_round(r32), r32)
    up = (r32.view(np.uint32) + (1 << 16)).view(np.float32).astype(np.float64)
    dn = (r32.view(np.uint32) - (1 << 16)).view(np.float32).astype(np.float64)
    assert np.all(np.abs(x - r) <= np.abs(x - up))
    assert np.all(np.abs(x - r) <= np.abs(x - dn))


# ---------------------------------------------------------- storage / audit ---

def test_storage_is_4_5_bits(fmt):
    b = fmt["bits_per_block"]
    assert (b["elements"] * b["element_bits"] + b["scale_bits"]) / b["elements"] == 4.5
    for K in (16, 64, 256, 2048, 5120):
        assert o.storage_bits_per_element(K) == fmt["quantization_recipe"]["effective_bits"]
    x = np.random.default_rng(5).standard_normal((32, 256)).astype(np.float32)
    q = o.quantize(x)
    packed = o.pack_codes(q["codes"])
    assert 8 * (packed.nbytes + q["scales"].nbytes) / x.size == 4.5
    assert np.array_equal(o.unpack_codes(packed), q["codes"])
    assert fmt["quantization_recipe"]["block_sizes"]["-1"] == o.BLOCK


def test_nibble_order_hand_worked_bytes():
    """Element 2j goes to the low nibble of byte j: codes [1, 2] (+0.5, +1.0)
    pack to 0x21, codes [0xA, 0x7] (-1.0, +6.0) to 0x7A; a row quantized from
    values already on the grid (g*s = 1 exactly) packs the same way."""
    assert o.pack_codes(np.array([[1, 2]], np.uint8)).tolist() == [[0x21]]
    assert o.pack_codes(np.array([[0xA, 0x7, 0x0, 0xF]], np.uint8)).tolist() == [[0x7A, 0xF0]]
    assert o.unpack_codes(np.array([[0x21, 0x7A]], np.uint8)).tolist() == [[1, 2, 0xA, 0x7]]
    # g = 2^-3 and s = 8 (E4M3 exact) give d = 1: a block whose maximum is 6
    # keeps the values as codes. Element 0 = 0.5 (code 1), element 1 = 1.0
    # (code 2), element 2 = -1.0 (code 0xA), element 3 = 6.0 (code 7).
    x = np.zeros((1, 16), np.float32)
    x[0, :4] = [0.5, 1.0, -1.0, 6.0]
    q = o.quantize(x, "max", np.float32(0.125))
    assert q["scales"].tolist() == [[lib_e4m3_code(8.0)]]
    assert o.pack_codes(q["codes"])[0, :2].tolist() == [0x21, 0x7A]


def lib_e4m3_code(t):
    return int(np.float32(t).astype(ml_dtypes.float8_e4m3fn).view(np.uint8))


@pytest.mark.parametrize("dist", ["normal", "student_t", "outliers", "tiny"])
@pytest.mark.parametrize("mode", ["max", "four_over_six"])
def test_scale_audit_invariants(fmt, dist, mode):
    rng = np.random.default_rng(6)
    if dist == "normal":
        x = rng.standard_normal((64, 512)) * 0.02
    elif dist == "student_t":
        x = rng.standard_t(3, (64, 512)) * 0.5
    elif dist == "outliers":
        x = rng.standard_normal((64, 512)) * 0.02
        x.reshape(-1)[rng.choice(x.size, 40, replace=False)] *= 20
    else:
        x = rng.standard_normal((64, 512)) * 1e-6
    x = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).float().numpy()
    q = o.quantize(x, mode)
    s = o.e4m3_decode(q["scales"])
    audit = fmt["scale_audit"]
    assert np.all(np.isfinite(s)) and np.all(s > 0) and s.max() <= audit["max"]
    assert np.isfinite(q["g"]) and q["g"] > 0
    if mode == "max":
        assert s.max() == audit["max"]          # the amax block lands on 448 exactly
    # g is FP32 amax / 2688
    assert q["g"] == np.float32(np.float32(np.abs(x).max()) / np.float32(2688.0))


def test_zero_tensor_edge_case():
    q = o.quantize(np.zeros((4, 32), np.float32))
    assert q["g"] == 1.0
    assert np.all(q["codes"] == 0) and np.all(q["scales"] == 1)


# ------------------------------------------------------------ round trips ----

def _grid_tensor(rng, rows, K):
    """x = 2^-10 * s_b * q_i with s_b from E4M3, q from E2M1, |q| = 6 in every
    block, and the first block scaled 448 so that amax = 2^-10 * 448 * 6."""
    nb = K // 16
    table = o.e4m3_decode_table()
    s = table[rng.integers(1, 127, (rows, nb))]
    s[0, 0] = 448.0
    q = o.e2m1_decode_table()[rng.integers(0, 16, (rows, nb, 16))]
    pos = rng.integers(0, 16, (rows, nb))
    sign = np.where(rng.random((rows, nb)) < 0.5, -1.0, 1.0)
    np.put_along_axis(q, pos[..., None], (6.0 * sign)[..., None], axis=2)
    x = (2.0 ** -10) * s[..., None] * q
    return x.reshape(rows, K).astype(np.float32), s, q


def test_round_trip_on_grid_is_exact():
    rng = np.random.default_rng(7)
    x, s, q = _grid_tensor(rng, 48, 256)
    assert np.array_equal(torch.from_numpy(x).to(torch.bfloat16).float().numpy(), x)
    out = o.quantize(x, "max")
    assert out["g"] == np.float32(2.0 ** -10)
    assert np.array_equal(o.e4m3_decode(out["scales"]), s)
    assert np.array_equal(o.e2m1_decode(out["codes"]).reshape(q.shape), q)
    assert np.array_equal(o.dequantize(out["codes"], out["scales"], out["g"]), x)
    fos = o.quantize(x, "four_over_six")
    assert np.all(fos["choice"] == 0)            # zero error at M=6; ties keep 6
    assert np.array_equal(o.fake_quant(x), x)


def test_every_block_at_amax_is_per_tensor_scaling():
    """When every block holds the tensor amax, every scale is 448 and the codes
    are the E2M1 rounding of x * 6 / amax (per-tensor scaling)."""
    rng = np.random.default_rng(8)
    x = np.clip(rng.standard_normal((16, 256)), -3.4, 3.4).astype(np.float32)
    x = torch.from_numpy(x).to(torch.bfloat16).float().numpy()
    x.reshape(16, 16, 16)[:, :, 0] = 3.5
    out = o.quantize(x, "max")
    assert np.all(out["scales"] == 0x7E)
    v = x.astype(np.float64) * 6.0 / 3.5
    lib = lib_e2m1(v.astype(np.float32))
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])
    far = np.min(np.abs(np.abs(v)[..., None] - mids), axis=-1) > 1e-5
    assert np.array_equal(out["codes"][far], lib[far])


# ---------------------------------------------------------- four_over_six ----

def test_four_over_six_hand_worked_block(golden_dir):
    with open(os.path.join(golden_dir, "four_over_six_worked_block.json")) as f:
        w = json.load(f)
    x = np.array([w["x"]], np.float32)
    out = o.quantize(x, "four_over_six", g=np.float32(w["g"]))
    assert out["choice"][0, 0] == w["choice"]
    assert out["scales"][0, 0] == w["m4"]["scale_code"]
    assert list(out["codes"][0]) == w["m4"]["codes"]
    m6 = o.quantize(x, "max", g=np.float32(w["g"]))
    assert m6["scales"][0, 0] == w["m6"]["scale_code"]
    assert list(m6["codes"][0]) == w["m6"]["codes"]
    assert m6["err"][0, 0] == np.float32(w["m6"]["err"])
    assert out["err"][0, 0] == np.float32(w["m4"]["err"])


def _lib_block_error(xb, g, s):
    """Brute-force block error with library conversions and FP32 arithmetic,
    summed in index order."""
    g = np.float32(g)
    s = np.float32(s)
    d = g * s
    r = np.float32(1.0) / d
    acc = np.float32(0.0)
    for xi in xb:
        qv = lib_e2m1_value(np.float32(xi) * r)
        e = np.float32(xi) - d * np.float32(qv)
        acc = np.float32(acc + np.float32(e * e))
    return acc


def _lib_scale(bmax, g, m):
    t = np.float32(bmax) / (np.float32(m) * np.float32(g))
    return max(lib_e4m3_value(t), np.float32(2.0 ** -9))


def test_four_over_six_brute_force_over_all_scales():
    rng = np.random.default_rng(9)
    rows = []
    for kind in range(6):
        base = rng.standard_normal(16).astype(np.float32) * 0.02
        if kind == 1:
            base[rng.integers(16)] *= 20
        if kind == 2:
            base = rng.uniform(-1, 1, 16).astype(np.float32)
        if kind == 3:
            base = np.sign(base) * np.abs(base) ** 3
        if kind == 4:
            base[:] = 0.01
        if kind == 5:
            base = rng.standard_t(3, 16).astype(np.float32)
        rows.append(base)
    x = torch.from_numpy(np.stack(rows).reshape(3, 32)).to(torch.bfloat16).float().numpy()
    x[0, 0] = 1.0                                       # sets the tensor amax
    out = o.quantize(x, "four_over_six")
    g = out["g"]
    table = o.e4m3_decode_table()[1:]
    for r in range(3):
        for b in range(2):
            xb = x[r, 16 * b:16 * b + 16]
            bmax = np.abs(xb).max()
            e6 = _lib_block_error(xb, g, _lib_scale(bmax, g, 6.0))
            e4 = _lib_block_error(xb, g, _lib_scale(bmax, g, 4.0))
            want_choice = 1 if e4 < e6 else 0
            assert out["choice"][r, b] == want_choice
            assert out["err"][r, b] == min(e4, e6)
            s_kept = o.e4m3_decode(out["scales"][r, b])
            assert s_kept == (_lib_scale(bmax, g, 4.0) if want_choice else _lib_scale(bmax, g, 6.0))
            # exhaustive: the kept candidate is never beaten by the other one,
            # and the global optimum over all 126 scales is at most as large
            best = min(_lib_block_error(xb, g, s) for s in table)
            assert best <= out["err"][r, b]


# --------------------------------------------------------- MSE calibration ---

def _lib_e4m3_scales():
    """(code, value) of every positive finite E4M3 code, decoded by ml_dtypes."""
    codes = np.arange(1, 127, dtype=np.uint8)
    return codes, codes.view(ml_dtypes.float8_e4m3fn).astype(np.float32)


def _mse_blocks(seed):
    rng = np.random.default_rng(seed)
    rows = []
    for kind in range(8):
        base = rng.standard_normal(16).astype(np.float32) * 0.02
        if kind == 1:
            base[rng.integers(16)] *= 20
        if kind == 2:
            base = rng.uniform(-1, 1, 16).astype(np.float32)
        if kind == 3:
            base = np.sign(base) * np.abs(base) ** 3
        if kind == 4:
            base[:] = 0.01
        if kind == 5:
            base = rng.standard_t(3, 16).astype(np.float32)
        if kind == 6:
            base[:] = 0.0
        if kind == 7:
            base = rng.standard_t(2, 16).astype(np.float32) * 1e-3
        rows.append(base)
    x = torch.from_numpy(np.stack(rows).reshape(4, 32)).to(torch.bfloat16).float().numpy()
    x[0, 0] = 1.0                                       # sets the tensor amax
    return x


def test_mse_matches_brute_force_over_all_scales():
    # R10: the kept scale is the lowest code reaching the smallest block error
    # over all 126 scales; errors by library conversions, summed in index order
    codes, values = _lib_e4m3_scales()
    for seed in (3, 4):
        x = _mse_blocks(seed)
        out = o.quantize(x, "mse")
        g = out["g"]
        for r in range(x.shape[0]):
            for b in range(2):
                xb = x[r, 16 * b:16 * b + 16]
                errs = np.array([_lib_block_error(xb, g, v) for v in values], np.float32)
                best = int(np.argmin(errs))                 # first minimum = lowest code
                assert out["err"][r, b] == errs[best], (seed, r, b)
                assert out["scales"][r, b] == codes[best], (seed, r, b)
                s = values[best]
                want = [lib_e2m1(np.float32(v) * (np.float32(1.0) / (np.float32(g) * s))) for v in xb]
                assert list(out["codes"][r, 16 * b:16 * b + 16]) == want


def test_mse_never_worse_than_max_or_four_over_six():
    rng = np.random.default_rng(12)
    x = torch.from_numpy((rng.standard_t(3, (24, 256)) * 0.05).astype(np.float32)).to(torch.bfloat16).float().numpy()
    e_max = o.quantize(x, "max")["err"]
    e_fos = o.quantize(x, "four_over_six")["err"]
    e_mse = o.quantize(x, "mse")["err"]
    assert np.all(e_fos <= e_max)
    assert np.all(e_mse <= e_fos)
    assert np.any(e_mse < e_fos)                            # the wider search does find better scales


def test_mse_finds_exact_representation():
    # a block that is exactly g*s*q for one scale s is reproduced with error 0
    g = np.float32(2.0 ** -8)
    s = np.float32(12.0)                                # E4M3 code 0x52 = 82
    q = np.array([0, .5, 1, 1.5, 2, 3, 4, 6, -0.5, -1, -1.5, -2, -3, -4, -6, 0], np.float32)
    x = (g * s * q).astype(np.float32)[None, :]
    out = o.quantize(x, "mse", g=g)
    assert out["err"][0, 0] == 0.0
    assert np.array_equal(o.dequantize(out["codes"], out["scales"], g), x)


# -------------------------------------------------------------------- GEMM ---

def test_gemm_reference_brute_force_tiny():
    rng = np.random.default_rng(10)
    M, N, K = 3, 4, 48
    a = o.quantize(rng.standard_normal((M, K)).astype(np.float32))
    b = o.quantize((rng.standard_normal((N, K)) * 0.02).astype(np.float32))
    C, S = o.gemm_reference(a["codes"], a["scales"], a["g"], b["codes"], b["scales"], b["g"])
    lib_codes = lambda c: c.astype(np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    lib_scale = lambda c: c.astype(np.uint8).view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    for m in range(M):
        for n in range(N):
            acc = 0.0
            acc_abs = 0.0
            for k in range(K):
                av = float(lib_scale(a["scales"][m, k // 16])) * float(lib_codes(a["codes"][m, k]))
                bv = float(lib_scale(b["scales"][n, k // 16])) * float(lib_codes(b["codes"][n, k]))
                acc += av * bv
                acc_abs += abs(av * bv)
            want = float(a["g"]) * float(b["g"]) * acc
            assert abs(C[m, n] - want) <= 1e-12 * max(1.0, abs(want))
            assert abs(S[m, n] - float(a["g"]) * float(b["g"]) * acc_abs) <= 1e-12 * S[m, n] + 1e-300


def test_gemm_reference_closed_form():
    K = 256
    codes = np.full((2, K), 2, np.uint8)                 # E2M1 code 2 == 1.0
    scales = np.full((2, K // 16), 0x38, np.uint8)       # E4M3 0x38 == 1.0
    C, S = o.gemm_reference(codes, scales, np.float32(0.5), codes, scales, np.float32(0.25))
    assert np.all(C == K * 0.125) and np.all(S == K * 0.125)
    neg = codes | 0x8
    C2, S2 = o.gemm_reference(codes, scales, np.float32(1), neg, scales, np.float32(1))
    assert np.all(C2 == -K) and np.all(S2 == K)


def test_tiled_scale_layout_round_trip_and_offsets():
    rng = np.random.default_rng(11)
    s = rng.integers(0, 127, (200, 20)).astype(np.uint8)
    t = o.scales_to_tiled(s)
    assert t.size == o.scale_tile_bytes(200, 320) == 2 * 5 * 512
    assert np.array_equal(o.scales_from_tiled(t, 200, 320), s)
    # (r=33, c=5): tile 1, byte 16 + 4 + 1
    assert t[512 + 16 + 4 + 1] == s[33, 5]
    # (r=130, c=0): tile (1*5 + 0), byte 2*16
    assert t[5 * 512 + 32] == s[130, 0]


# --------------------------------------------------------------- fake quant --

def test_fake_quant_frozen_saturates():
    rng = np.random.default_rng(12)
    x = torch.from_numpy(rng.standard_normal((8, 64)).astype(np.float32)).to(torch.bfloat16).float().numpy()
    q = o.quantize(x)
    x2 = (x * 4).astype(np.float32)                      # weights drifted past the frozen range
    y = o.fake_quant(x2, g_frozen=q["g"], scales_frozen=q["scales"])
    d = (np.float32(q["g"]) * o.e4m3_decode(q["scales"]).astype(np.float32))
    dd = np.repeat(d, 16, axis=1)
    big = np.abs(x2) >= 6 * dd * 1.0001
    assert big.any()
    assert np.array_equal(y[big], o.bf16_round((np.sign(x2[big]) * 6 * dd[big]).astype(np.float32)))
    # frozen with the tensor's own scales equals the dynamic result
    assert np.array_equal(o.fake_quant(x, g_frozen=q["g"], scales_frozen=q["scales"]), o.fake_quant(x))


# --------------------------------------------------------------------- MoE ---

def test_moe_permutation_is_a_stable_sort():
    rng = np.random.default_rng(13)
    ids = rng.integers(0, 8, (50, 3))
    order, counts, offsets = o.moe_permutation(ids, 8)
    assert np.array_equal(order, np.argsort(ids.reshape(-1), kind="stable"))
    assert np.array_equal(counts, np.bincount(ids.reshape(-1), minlength=8))
    assert np.all(offsets % 128 == 0)


def test_moe_single_expert_is_the_dense_mlp():
    """E = 1, k = 1, weight 1: the MoE layer is the dense gated MLP with
    dynamic activation quantization, computed here with plain loops on
    library conversions."""
    rng = np.random.default_rng(14)
    T, H, I = 6, 32, 16
    x = torch.from_numpy(rng.standard_normal((T, H)).astype(np.float32)).to(torch.bfloat16).float().numpy()
    w13 = (rng.standard_normal((2 * I, H)) * 0.02).astype(np.float32)
    w2 = (rng.standard_normal((H, I)) * 0.02).astype(np.float32)
    q13, q2 = o.quantize(w13), o.quantize(w2)
    ref = o.moe_reference(x, np.zeros((T, 1), np.int32), np.ones((T, 1), np.float32), [q13], [q2])

    def lib_quant(a):
        amax = np.float32(np.abs(a).max())
        g = np.float32(amax / np.float32(2688.0))
        out = np.zeros_like(a, dtype=np.float64)
        for r in range(a.shape[0]):
            for b in range(a.shape[1] // 16):
                blk = a[r, 16 * b:16 * b + 16]
                s = _lib_scale(np.abs(blk).max(), g, 6.0)
                d = g * s
                rr = np.float32(1.0) / d
                out[r, 16 * b:16 * b + 16] = [float(s) * float(lib_e2m1_value(np.float32(v) * rr)) for v in blk]
        return out, float(g)

    def lib_deq(q):
        return o.dequantize_f64(q["codes"], q["scales"]), float(q["g"])

    xa, gx = lib_quant(x)
    wa, gw = lib_deq(q13)
    gu = gx * gw * (xa @ wa.T)
    h = gu[:, :I] / (1 + np.exp(-gu[:, :I])) * gu[:, I:]
    h = torch.from_numpy(h).to(torch.bfloat16).double().numpy()   # FP64 -> BF16 (torch)
    ha, gh = lib_quant(h.astype(np.float32))
    w2a, gw2 = lib_deq(q2)
    y = gh * gw2 * (ha @ w2a.T)
    assert np.allclose(ref["stages"][0]["gate_up"], gu, rtol=1e-12, atol=1e-15)
    assert np.allclose(ref["out"], y, rtol=1e-9, atol=1e-12)


def _loop_expert_mlp(x_rows, q13, q2):
    """Gated MLP of one expert over the rows routed to it (dynamic activation
    quantization over exactly those rows), with plain per-element loops and
    library conversions; returns y [rows, H] in FP64."""
    def lib_quant(a):
        g = np.float32(np.float32(np.abs(a).max()) / np.float32(2688.0))
        out = np.zeros(a.shape, np.float64)
        for r in range(a.shape[0]):
            for b in range(a.shape[1] // 16):
                blk = a[r, 16 * b:16 * b + 16]
                s = _lib_scale(np.abs(blk).max(), g, 6.0)
                rr = np.float32(1.0) / np.float32(g * s)
                out[r, 16 * b:16 * b + 16] = [float(s) * float(lib_e2m1_value(np.float32(v) * rr)) for v in blk]
        return out, float(g)
    xa, gx = lib_quant(x_rows)
    gu = gx * float(q13["g"]) * (xa @ o.dequantize_f64(q13["codes"], q13["scales"]).T)
    inter = gu.shape[1] // 2
    h = gu[:, :inter] / (1 + np.exp(-gu[:, :inter])) * gu[:, inter:]
    h = torch.from_numpy(h).to(torch.bfloat16).double().numpy()
    ha, gh = lib_quant(h.astype(np.float32))
    return gh * float(q2["g"]) * (ha @ o.dequantize_f64(q2["codes"], q2["scales"]).T)


def test_moe_top2_combine_hand_worked():
    """k = 2 with distinct routing weights per (token, slot): out[t] =
    w[t,0] * y_{e0}(t) + w[t,1] * y_{e1}(t), rebuilt token by token from a
    per-expert loop MLP. Indexing the weights by token instead of by
    (token, slot) pair, or swapping the slots, changes the result."""
    rng = np.random.default_rng(15)
    T, H, I, E = 4, 32, 16, 3
    x = torch.from_numpy(rng.standard_normal((T, H)).astype(np.float32)).to(torch.bfloat16).float().numpy()
    ids = np.array([[0, 2], [1, 0], [2, 1], [0, 1]], np.int32)
    w = np.array([[0.9, 0.1], [0.25, 0.75], [0.6, 0.4], [0.3, 0.7]], np.float32)
    q13 = [o.quantize((rng.standard_normal((2 * I, H)) * 0.02).astype(np.float32)) for _ in range(E)]
    q2 = [o.quantize((rng.standard_normal((H, I)) * 0.02).astype(np.float32)) for _ in range(E)]
    ref = o.moe_reference(x, ids, w, q13, q2)
    ys = {}
    for e in range(E):
        toks = [t for t in range(T) for j in range(2) if ids[t, j] == e]   # stable: token order
        ys[e] = dict(zip(toks, _loop_expert_mlp(x[toks], q13[e], q2[e])))
    want = np.zeros((T, H))
    for t in range(T):
        for j in range(2):
            want[t] += float(w[t, j]) * ys[ids[t, j]][t]
    assert np.allclose(ref["out"], want, rtol=1e-9, atol=1e-12)
    # the weights matter: the slot-swapped combine is far from it
    swapped = np.zeros((T, H))
    for t in range(T):
        for j in range(2):
            swapped[t] += float(w[t, 1 - j]) * ys[ids[t, j]][t]
    assert not np.allclose(ref["out"], swapped, rtol=1e-3, atol=1e-6)


# ------------------------------------------------------- QAD backward (STE) ---

def test_ste_backward_closed_form_block():
    # frozen g = 1, s = 1 (E4M3 code 0x38): the range is |x| <= 6
    x = np.zeros((1, 16), np.float32)
    x[0, :8] = [0.5, 6.0, 6.5, -7.0, 5.9375, -6.0, 100.0, -0.0]
    gy = np.arange(1, 17, dtype=np.float32)[None, :]
    gx = o.fake_quant_backward(x, gy, g_frozen=np.float32(1.0), scales_frozen=np.array([[0x38]], np.uint8))
    want = gy.copy()
    want[0, [2, 3, 6]] = 0.0
    assert np.array_equal(gx, want)


def test_ste_backward_matches_autograd_of_clamp():
    # the clipped STE passes the gradient exactly where clamp(x * r, -6, 6)
    # has derivative 1 (rounding passed straight through): torch autograd
    rng = np.random.default_rng(31)
    x = torch.from_numpy((rng.standard_t(3, (8, 64)) * 0.3).astype(np.float32)).to(torch.bfloat16).float().numpy()
    gy = rng.standard_normal((8, 64)).astype(np.float32)
    # frozen scales calibrated on a narrower tensor, so some elements saturate
    q = o.quantize(x * np.float32(0.5), "max")
    g, sc = q["g"], q["scales"]
    gx = o.fake_quant_backward(x, gy, g_frozen=g, scales_frozen=sc)
    d = torch.from_numpy((np.float32(g) * ml_dtypes_values(sc)).astype(np.float32))
    r = (1.0 / d).repeat_interleave(16, dim=1)
    v = (torch.from_numpy(x) * r).requires_grad_(True)     # FP32 products x * r
    torch.clamp(v, -6.0, 6.0).backward(torch.from_numpy(gy))
    assert np.array_equal(gx, v.grad.numpy())
    assert (gx == 0).any() and (gx != 0).any()


def ml_dtypes_values(codes):
    return np.asarray(codes, np.uint8).view(ml_dtypes.float8_e4m3fn).astype(np.float32)


def test_ste_backward_dynamic_passes_unsaturated():
    # dynamic max scales: every element whose forward code is below the E2M1
    # maximum gets its gradient back unchanged
    rng = np.random.default_rng(32)
    x = torch.from_numpy((rng.standard_normal((4, 128))).astype(np.float32)).to(torch.bfloat16).float().numpy()
    gy = np.ones_like(x)
    gx = o.fake_quant_backward(x, gy, "max")
    codes = o.quantize(x, "max")["codes"] & 7
    assert np.all(gx[codes < 7] == 1.0)


# ------------------------------------------------------------- dequantize ---

def test_dequantize_closed_form_and_round_trip():
    # code 7 (6.0) x scale 448 (code 0x7E) x g = 1 -> 2688; code 0xF -> -2688;
    # code 1 (0.5) x scale 2^-9 (code 1) x g = 0.5 -> 2^-11
    codes = np.zeros((1, 16), np.uint8)
    codes[0, :3] = [7, 0xF, 1]
    v = o.dequantize(codes, np.array([[0x7E]], np.uint8), np.float32(1.0))
    assert v[0, 0] == 2688.0 and v[0, 1] == -2688.0 and v[0, 2] == 0.5 * 448.0
    v = o.dequantize(codes, np.array([[1]], np.uint8), np.float32(0.5))
    assert v[0, 2] == np.float32(2.0 ** -11)
    # storing K/V in NVFP4 and reading them back is the fake-quant forward
    rng = np.random.default_rng(51)
    x = torch.from_numpy(rng.standard_normal((8, 128)).astype(np.float32)).to(torch.bfloat16).float().numpy()
    for mode in ("max", "four_over_six"):
        q = o.quantize(x, mode)
        assert np.array_equal(o.bf16_round(o.dequantize(q["codes"], q["scales"], q["g"])), o.fake_quant(x, mode))


# ------------------------------------------------------------- top-k KL ---

def test_topk_kl_full_vocab_equals_library_kl():
    from scipy.special import rel_entr, softmax
    rng = np.random.default_rng(61)
    t = rng.standard_normal((3, 50)) * 2
    s = t + rng.standard_normal((3, 50)) * 0.5
    out = o.topk_kl(t, s, 50)
    want = rel_entr(softmax(t, axis=1), softmax(s, axis=1)).sum(axis=1)
    assert np.allclose(out["loss"], want, rtol=1e-12, atol=1e-14)


def test_topk_kl_set_ties_and_zero_loss():
    t = np.array([[1.0, 3.0, 3.0, 2.0, 3.0]])
    out = o.topk_kl(t, t, 2)
    assert out["idx"].tolist() == [[1, 2]]                 # three 3s: the two lowest indices
    assert out["loss"][0] == 0.0 and np.all(out["grad"] == 0.0)
    out = o.topk_kl(t, t * 0.5, 4)
    assert out["idx"].tolist() == [[1, 2, 3, 4]]


def test_topk_kl_matches_renormalised_library_kl_and_gradient():
    from scipy.special import rel_entr, softmax
    rng = np.random.default_rng(62)
    V, k = 40, 7
    t = np.round(rng.standard_normal((4, V)) * 3) / 2       # many ties
    s = rng.standard_normal((4, V))
    out = o.topk_kl(t, s, k)
    for r in range(4):
        idx = out["idx"][r]
        rest = np.setdiff1d(np.arange(V), idx)
        assert t[r, idx].min() >= t[r, rest].max()          # brute-force set property
        assert np.isclose(out["loss"][r], rel_entr(softmax(t[r, idx]), softmax(s[r, idx])).sum(), rtol=1e-12)
        # gradient by central differences of the loss in each student logit
        for j in range(k):
            h = 1e-6
            sp, sm = s.copy(), s.copy()
            sp[r, idx[j]] += h
            sm[r, idx[j]] -= h
            fd = (o.topk_kl(t[r:r + 1], sp[r:r + 1], k)["loss"][0] - o.topk_kl(t[r:r + 1], sm[r:r + 1], k)["loss"][0]) / (2 * h)
            assert abs(fd - out["grad"][r, j]) < 1e-7
