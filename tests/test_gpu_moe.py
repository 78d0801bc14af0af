"""Stage-wise GPU parity of the routed-expert (MoE) pipeline against the
oracle, through the C ABI. Each stage's oracle is fed the GPU's previous
stage, so quantized tensors compare bit-exactly and GEMM stages within the
GEMM tolerance (the GEMM itself is not bit-exact)."""
import numpy as np
import pytest
import torch

from oracle import nvfp4_oracle as o
from qad_nvfp4_quantize_b200 import inputs
from tests.util import bf16_np, require_gpu, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nv():
    return require_gpu()


def _ws_view(ws, off, count, dtype):
    nbytes = count * torch.tensor([], dtype=dtype).element_size()
    return ws[off:off + nbytes].view(dtype)


def run_moe(nv, d, I):
    x = d["x"].cuda()
    ids = d["topk_ids"].cuda()
    w = d["topk_w"].cuda()
    w13, g13 = nv.quantize_experts(d["w13"].cuda())
    w2, g2 = nv.quantize_experts(d["w2"].cuda())
    out, ws = nv.moe_grouped_gemm(x, ids, w, I, w13, g13, w2, g2)
    torch.cuda.synchronize()
    assert nv.device_status() == 0
    return out, ws, (w13, g13, w2, g2)


def expert_weights(wq, g, E, N, K):
    codes = o.unpack_codes(to_np(wq.codes)).reshape(E, N, K)
    sb = o.scale_tile_bytes(N, K)
    sc = to_np(wq.scales)
    scales = [o.scales_from_tiled(sc[e * sb:(e + 1) * sb], N, K) for e in range(E)]
    return codes, scales, to_np(g)


def check_moe(nv, d, I, experts_checked=None, tokens_checked=None):
    T, H = d["x"].shape
    E, topk = d["w13"].shape[0], d["topk_ids"].shape[1]
    out, ws, (w13, g13, w2, g2) = run_moe(nv, d, I)
    lay = nv.moe_workspace_layout(T, H, I, E, topk)
    R = lay["rows_capacity"]
    ids = d["topk_ids"].numpy()
    tw = d["topk_w"].numpy().astype(np.float64)
    x = bf16_np(d["x"])

    # routing: bit-exact
    order, counts, offs = o.moe_permutation(ids, E)
    g_counts = to_np(_ws_view(ws, lay["counts"], E, torch.int32))
    g_offs = to_np(_ws_view(ws, lay["offsets"], E + 1, torch.int32))
    row_pair = to_np(_ws_view(ws, lay["row_pair"], R, torch.int32))
    assert np.array_equal(g_counts, counts)
    assert np.array_equal(g_offs[:E], offs)
    starts = np.concatenate([[0], np.cumsum(counts)[:-1]])
    for e in range(E):
        seg = row_pair[offs[e]:offs[e] + ((counts[e] + 127) // 128) * 128]
        assert np.array_equal(seg[:counts[e]], order[starts[e]:starts[e] + counts[e]])
        assert np.all(seg[counts[e]:] == -1)

    xq_codes = o.unpack_codes(to_np(_ws_view(ws, lay["xq_codes"], R * H // 2, torch.uint8)).reshape(R, H // 2))
    xq_scales = o.scales_from_tiled(to_np(ws[lay["xq_scales"]:lay["xq_scales"] + o.scale_tile_bytes(R, H)]), R, H)
    xq_g = to_np(_ws_view(ws, lay["xq_g"], E, torch.float32))
    h = _ws_view(ws, lay["h"], R * I, torch.bfloat16).reshape(R, I).float().cpu().numpy()
    hq_codes = o.unpack_codes(to_np(_ws_view(ws, lay["hq_codes"], R * I // 2, torch.uint8)).reshape(R, I // 2))
    hq_scales = o.scales_from_tiled(to_np(ws[lay["hq_scales"]:lay["hq_scales"] + o.scale_tile_bytes(R, I)]), R, I)
    hq_g = to_np(_ws_view(ws, lay["hq_g"], E, torch.float32))

    c13, s13, gg13 = expert_weights(w13, g13, E, 2 * I, H)
    c2, s2, gg2 = expert_weights(w2, g2, E, H, I)

    ys = {}
    for e in (range(E) if experts_checked is None else experts_checked):
        if counts[e] == 0:
            continue
        rows = np.arange(offs[e], offs[e] + counts[e])
        pairs = order[starts[e]:starts[e] + counts[e]]
        # stage 3: gathered per-expert quantization, bit-exact
        ref = o.quantize(x[pairs // topk], "max")
        assert xq_g[e] == ref["g"], e
        assert np.array_equal(xq_codes[rows], ref["codes"]), e
        assert np.array_equal(xq_scales[rows], ref["scales"]), e
        # stage 4: gate_up GEMM + SiLU*up, from the GPU's quantized rows
        gu, gu_S = o.gemm_reference(xq_codes[rows], xq_scales[rows], xq_g[e], c13[e], s13[e], gg13[e])
        tol = o.gemm_tolerance(gu, gu_S)
        gate, up = gu[:, :I], gu[:, I:]
        sig = 1 / (1 + np.exp(-gate))
        silu = gate * sig
        dsilu = np.abs(sig * (1 + gate * (1 - sig)))
        h_ref = silu * up
        h_tol = dsilu * np.abs(up) * tol[:, :I] + np.abs(silu) * tol[:, I:] + 2.0 ** -7 * np.abs(h_ref) + 1e-30
        err = np.abs(h[rows] - h_ref)
        assert np.all(err <= h_tol), (e, float(np.max(err / h_tol)))
        # stage 5: per-expert quantization of the GPU's h, bit-exact
        refh = o.quantize(h[rows], "max")
        assert hq_g[e] == refh["g"], e
        assert np.array_equal(hq_codes[rows], refh["codes"]), e
        assert np.array_equal(hq_scales[rows], refh["scales"]), e
        # pad rows of h are zero
        pad = np.arange(offs[e] + counts[e], offs[e] + ((counts[e] + 127) // 128) * 128)
        assert np.all(h[pad] == 0)

    # stage 6: down GEMM + weighted combine, from the GPU's quantized h
    out_np = to_np(out).astype(np.float64)
    toks = range(T) if tokens_checked is None else tokens_checked
    pos_of_pair = np.empty(T * topk, np.int64)
    for e in range(E):
        pos_of_pair[order[starts[e]:starts[e] + counts[e]]] = np.arange(offs[e], offs[e] + counts[e])
    for t in toks:
        acc = np.zeros(H)
        acc_S = np.zeros(H)
        for j in range(topk):
            pair = t * topk + j
            e = ids[t, j]
            r = pos_of_pair[pair]
            y, yS = o.gemm_reference(hq_codes[r:r + 1], hq_scales[r:r + 1], hq_g[e], c2[e], s2[e], gg2[e])
            acc += tw[t, j] * y[0]
            acc_S += abs(tw[t, j]) * yS[0]
        tol = 1e-4 * acc_S + 1e-5 * np.abs(acc) + 1e-30
        assert np.all(np.abs(out_np[t] - acc) <= tol), (t, float(np.max(np.abs(out_np[t] - acc) / tol)))


@pytest.mark.parametrize("T,H,E,topk,I", [(256, 256, 8, 2, 128), (1000, 512, 16, 4, 256), (64, 256, 32, 8, 384)])
def test_moe_stagewise_small(nv, T, H, E, topk, I):
    d = inputs.moe_experts(seed=T + E, T=T, H=H, E=E, topk=topk, I=I)
    check_moe(nv, d, I, tokens_checked=range(0, T, max(1, T // 64)))


def test_moe_empty_experts_and_skew(nv):
    # few tokens over many experts: most experts get no rows
    d = inputs.moe_experts(seed=3, T=5, H=256, E=64, topk=2, I=128)
    check_moe(nv, d, 128)


def test_moe_full_size_sampled(nv):
    """T=8192, H=2048, E=256, top-8, I=512: routing checked in full, stages on
    a sample of experts, the combined output on a sample of tokens."""
    d = inputs.moe_experts(seed=0)
    check_moe(nv, d, 512, experts_checked=[0, 17, 128, 255], tokens_checked=range(0, 8192, 512))
