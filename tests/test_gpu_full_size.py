"""GPU parity at the workloads' full sizes, through the C ABI.

Dense MLP layer (X 4096x5120, W_up 17408x5120), lm_head decode (X 128x2048,
W 151936x2048) and the four_over_six + fake-quant linear (W 14336x4096,
X 16384x4096), each quantized and multiplied in the launch configuration the
benchmark times. The global scales are compared over the whole tensors;
quantized rows are compared bit for bit on a sample of rows (the oracle is
run on those rows with the whole tensor's global scale, which is exactly what
a full-tensor run would give them); the GEMM is compared on every column of
a sample of output rows that touches every 128-row tile, so every output
tile of the persistent kernel's tile walk is checked. A 600-tile GEMM with
ragged M, N and K is compared in full.
"""
import numpy as np
import pytest
import torch

from oracle import nvfp4_oracle as o
from qad_nvfp4_quantize_b200 import inputs
from tests.util import bf16_np, gemm_check, require_gpu, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nv():
    return require_gpu()


def tile_rows(M: int, per_tile: int, seed: int) -> np.ndarray:
    """Rows sampled from every 128-row tile: its first and last row, then
    random rows, plus the tensor's last row."""
    rng = np.random.default_rng(seed)
    rows = []
    for t0 in range(0, M, 128):
        t1 = min(t0 + 128, M)
        pick = {t0, t1 - 1}
        while len(pick) < min(per_tile, t1 - t0):
            pick.add(int(rng.integers(t0, t1)))
        rows.extend(sorted(pick))
    rows.append(M - 1)
    return np.unique(np.array(rows, dtype=np.int64))


def check_quantized_rows(q, x_f32: np.ndarray, mode: str, rows: np.ndarray, K: int):
    """Global scale over the whole tensor, then bit-exact codes, scales (and
    four_over_six choices) of the sampled rows."""
    g_ref = o.global_scale(x_f32)[0]
    assert to_np(q.g)[0] == g_ref, (to_np(q.g)[0], g_ref)
    ref = o.quantize(x_f32[rows], mode, g_ref)
    codes = o.unpack_codes(to_np(q.codes[torch.from_numpy(rows).to(q.codes.device)]))
    assert np.array_equal(codes, ref["codes"]), "codes differ on sampled rows"
    scales = o.scales_from_tiled(to_np(q.scales), q.rows, K)[rows]
    assert np.array_equal(scales, ref["scales"]), "block scales differ on sampled rows"
    if q.choice is not None:
        assert np.array_equal(to_np(q.choice)[rows], ref["choice"]), "four_over_six choices differ"
    return g_ref


def operands(q, K):
    return o.unpack_codes(to_np(q.codes)), o.scales_from_tiled(to_np(q.scales), q.rows, K), to_np(q.g)[0]


def check_gemm_rows(C_gpu: torch.Tensor, qa, qb, rows: np.ndarray, K: int, what: str, n_chunk: int = 8192):
    """Every column of the sampled rows of C against the FP64 oracle; the
    weight side is dequantized in row blocks to bound host memory."""
    ac, as_, ag = operands(qa, K)
    bq_all = to_np(qb.codes)
    bs_all = to_np(qb.scales)
    gb = to_np(qb.g)[0]
    N = qb.rows
    bscales = o.scales_from_tiled(bs_all, N, K)
    C = bf16_np(C_gpu[torch.from_numpy(rows).to(C_gpu.device)]).astype(np.float64)
    worst = 0.0
    for n0 in range(0, N, n_chunk):
        n1 = min(N, n0 + n_chunk)
        C_ref, S = o.gemm_reference(ac[rows], as_[rows], ag, o.unpack_codes(bq_all[n0:n1]), bscales[n0:n1], gb)
        worst = max(worst, gemm_check(C[:, n0:n1], C_ref, S, f"{what} columns {n0}:{n1}"))
    return worst


def test_dense_mlp_full_size(nv):
    """X 4096x5120 Student-t(3)*0.5 dynamic max, W_up 17408x5120 max: 2176
    output tiles over the persistent grid."""
    d = inputs.dense_mlp(0)
    x, w = d["x"], d["w"]
    M, K = x.shape
    wq = nv.quantize(w.cuda(), "max")
    xq = nv.quantize(x.cuda(), "max")
    C = nv.gemm(xq, wq)
    torch.cuda.synchronize()
    assert nv.device_status() == 0
    wf, xf = bf16_np(w), bf16_np(x)
    check_quantized_rows(wq, wf, "max", tile_rows(w.shape[0], 2, 1), K)
    check_quantized_rows(xq, xf, "max", tile_rows(M, 4, 2), K)
    check_gemm_rows(C, xq, wq, tile_rows(M, 2, 3), K, "dense_mlp")


def test_lm_head_full_size(nv):
    """X 128x2048 and W 151936x2048, both dynamic max: one 128-row tile and
    594 column tiles (M = 128, the weight-streaming decode shape)."""
    d = inputs.lm_head(0)
    x, w = d["x"], d["w"]
    M, K = x.shape
    wq = nv.quantize(w.cuda(), "max")
    xq = nv.quantize(x.cuda(), "max")
    C = nv.gemm(xq, wq)
    torch.cuda.synchronize()
    assert nv.device_status() == 0
    check_quantized_rows(wq, bf16_np(w), "max", tile_rows(w.shape[0], 2, 4), K)
    check_quantized_rows(xq, bf16_np(x), "max", np.arange(M), K)
    # every lane quarter of the tile (rows 32 apart) and random rows
    rows = np.unique(np.concatenate([[0, 31, 32, 63, 64, 95, 96, 127],
                                     np.random.default_rng(5).integers(0, M, 24)]))
    check_gemm_rows(C, xq, wq, rows, K, "lm_head")


def test_four_over_six_linear_full_size(nv):
    """W 14336x4096 with 0.1% outliers quantized four_over_six; X 16384x4096
    fake-quantized (dynamic max) and quantized; the 16384x14336x4096 GEMM."""
    d = inputs.four_over_six_linear(0)
    x, w = d["x"], d["w"]
    M, K = x.shape
    xd = x.cuda()
    wq = nv.quantize(w.cuda(), "four_over_six", want_choice=True)
    xq = nv.quantize(xd, "max")
    y = nv.fake_quant(xd, "max")
    C = nv.gemm(xq, wq)
    torch.cuda.synchronize()
    assert nv.device_status() == 0
    wf, xf = bf16_np(w), bf16_np(x)
    check_quantized_rows(wq, wf, "four_over_six", tile_rows(w.shape[0], 2, 6), K)
    assert 0 < to_np(wq.choice).mean() < 1          # both targets occur
    xrows = tile_rows(M, 1, 7)
    g_x = check_quantized_rows(xq, xf, "max", xrows, K)
    # fake-quant of the sampled rows under the whole tensor's g, bit for bit
    ref = o.quantize(xf[xrows], "max", g_x)
    fq = o.bf16_round(o.dequantize(ref["codes"], ref["scales"], g_x))
    got = bf16_np(y[torch.from_numpy(xrows).cuda()])
    np.testing.assert_array_equal(got, fq)
    del y
    check_gemm_rows(C, xq, wq, tile_rows(M, 1, 8)[::2], K, "four_over_six linear")


def test_gemm_600_tiles_in_full(nv):
    """M 1000 (ragged last row tile), N 19088 (ragged last column tile),
    K 576 (a partial last K stage): 8 x 75 = 600 output tiles, about four
    per CTA of the persistent grid, every element checked."""
    rng = np.random.default_rng(600)
    M, N, K = 1000, 19088, 576
    x = inputs.to_bf16((rng.standard_t(3, (M, K)) * 0.5).astype(np.float32))
    w = inputs.to_bf16((rng.standard_normal((N, K)) * 0.02).astype(np.float32))
    xq = nv.quantize(x.cuda(), "max")
    wq = nv.quantize(w.cuda(), "four_over_six")
    C = nv.gemm(xq, wq)
    torch.cuda.synchronize()
    assert nv.device_status() == 0
    check_gemm_rows(C, xq, wq, np.arange(M), K, "600 tiles", n_chunk=4096)
