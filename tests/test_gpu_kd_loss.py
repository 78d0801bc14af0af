"""GPU parity of the top-k logit KL distillation loss against the CPU oracle
(set bit-exact, loss and gradient within FP32 accumulation tolerance)."""
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


def _check(nv, t, s, k):
    loss, idx, grad = nv.topk_kl(t.cuda(), s.cuda(), k, want_grad=True)
    ref = o.topk_kl(bf16_np(t), bf16_np(s), k)
    assert np.array_equal(to_np(idx), ref["idx"])
    # FP32 exp/log and sums over k terms against FP64
    tol = 4e-5 * (1 + np.abs(ref["lse_t"]) + np.abs(ref["lse_s"])) + 1e-4 * np.abs(ref["loss"])
    err = np.abs(to_np(loss).astype(np.float64) - ref["loss"])
    assert np.all(err <= tol), float(np.max(err / tol))
    tv = bf16_np(t).astype(np.float64)[np.arange(t.shape[0])[:, None], ref["idx"]]
    p_t = np.exp(tv - ref["lse_t"][:, None])
    p_s = ref["grad"] + p_t
    gtol = 1e-5 * (np.abs(p_s) + np.abs(p_t)) + 1e-9
    gerr = np.abs(to_np(grad).astype(np.float64) - ref["grad"])
    assert np.all(gerr <= gtol), float(np.max(gerr / gtol))


# (2, 65536, 8192) has more candidates than the per-row capacity, so it takes
# the full three-pass path; the others take the sampled path
@pytest.mark.parametrize("rows,V,k", [(5, 1024, 64), (3, 64, 64), (4, 256, 1), (2, 8192, 4096), (2, 65536, 8192)])
def test_topk_kl_small(nv, rows, V, k):
    rng = np.random.default_rng(rows * V + k)
    t = np.round(rng.standard_normal((rows, V)) * 4) / 4          # many ties at every threshold
    s = t + rng.standard_normal((rows, V)) * 0.5
    _check(nv, inputs.to_bf16(t.astype(np.float32)), inputs.to_bf16(s.astype(np.float32)), k)


def test_topk_kl_all_equal_and_signed_zero(nv):
    t = np.zeros((2, 512), np.float32)
    t[1, ::2] = -0.0                                                 # -0 and +0 are one value
    s = np.random.default_rng(5).standard_normal((2, 512)).astype(np.float32)
    _check(nv, inputs.to_bf16(t), inputs.to_bf16(s), 100)


def test_topk_kl_vocab_248320_top4096(nv):
    d = inputs.kd_logits(seed=1, rows=6)
    _check(nv, d["teacher"], d["student"], 4096)
