"""Seeded synthetic inputs shaped like the pages' dense, MoE-expert and
lm_head layers.

This module only draws random numbers and casts them to BF16; it holds none of
the quantization arithmetic. Both the CUDA path (tests, bench) and the CPU
oracle are fed from it.

Recipe: ``numpy.random.default_rng`` on one child of
``SeedSequence(seed).spawn(n)`` per tensor, in the order listed by each
function; samples are drawn in FP32 and cast once to BF16 (round to nearest
even, via torch). Routing (top-k and softmax weights) is part of the input.
"""
from __future__ import annotations

import numpy as np
import torch


def _streams(seed: int, n: int):
    return [np.random.default_rng(s) for s in np.random.SeedSequence(seed).spawn(n)]


def to_bf16(a: np.ndarray) -> torch.Tensor:
    """FP32 numpy array -> BF16 torch tensor (CPU), round to nearest even."""
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)


def normal(rng, shape, std=1.0) -> np.ndarray:
    out = rng.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        out *= np.float32(std)
    return out


def tiny_linear(seed: int = 0, M: int = 128, N: int = 256, K: int = 256):
    """X[M x K] ~ N(0,1), W[N x K] ~ N(0, 0.02)."""
    rx, rw = _streams(seed, 2)
    return dict(x=to_bf16(normal(rx, (M, K))), w=to_bf16(normal(rw, (N, K), 0.02)))


def dense_mlp(seed: int = 0, M: int = 4096, N: int = 17408, K: int = 5120):
    """X[M x K] = Student-t(df=3) * 0.5 (heavy-tailed activations),
    W_up[N x K] ~ N(0, 0.02)."""
    rx, rw = _streams(seed, 2)
    x = (rx.standard_t(3, size=(M, K)) * 0.5).astype(np.float32)
    return dict(x=to_bf16(x), w=to_bf16(normal(rw, (N, K), 0.02)))


def lm_head(seed: int = 0, M: int = 128, N: int = 151936, K: int = 2048):
    """X[M x K] ~ N(0,1), W[N x K] ~ N(0, 0.02)."""
    rx, rw = _streams(seed, 2)
    return dict(x=to_bf16(normal(rx, (M, K))), w=to_bf16(normal(rw, (N, K), 0.02)))


def four_over_six_linear(seed: int = 0, M: int = 16384, N: int = 14336, K: int = 4096,
                         outlier_frac: float = 0.001, outlier_gain: float = 20.0):
    """W[N x K] ~ N(0, 0.02) with floor(frac * numel) entries, chosen without
    replacement, multiplied by 20 before the BF16 cast; X[M x K] ~ N(0,1)."""
    rw, ro, rx = _streams(seed, 3)
    w = normal(rw, (N, K), 0.02)
    n_out = int(np.floor(outlier_frac * w.size))
    idx = ro.choice(w.size, size=n_out, replace=False)
    w.reshape(-1)[idx] *= np.float32(outlier_gain)
    return dict(x=to_bf16(normal(rx, (M, K))), w=to_bf16(w))


def moe_experts(seed: int = 0, T: int = 8192, H: int = 2048, E: int = 256, topk: int = 8,
                I: int = 512, weight_std: float = 0.02):
    """Routed-expert layer: x[T x H] ~ N(0,1); router logits [T x E] ~ N(0,1),
    top-k by value (ties -> lower expert id), weights = softmax over the k
    selected logits (FP64, stored FP32); per-expert gate_up [2I x H] and
    down [H x I] ~ N(0, 0.02)."""
    rx, rl, r13, r2 = _streams(seed, 4)
    x = normal(rx, (T, H))
    logits = normal(rl, (T, E))
    order = np.argsort(-logits, axis=1, kind="stable")[:, :topk]
    sel = np.take_along_axis(logits, order, axis=1).astype(np.float64)
    ex = np.exp(sel - sel.max(axis=1, keepdims=True))
    w = (ex / ex.sum(axis=1, keepdims=True)).astype(np.float32)
    w13 = normal(r13, (E, 2 * I, H), weight_std)
    w2 = normal(r2, (E, H, I), weight_std)
    return dict(x=to_bf16(x), topk_ids=torch.from_numpy(order.astype(np.int32)),
                topk_w=torch.from_numpy(w), w13=to_bf16(w13), w2=to_bf16(w2))


def bf16_to_f32(t: torch.Tensor) -> np.ndarray:
    """BF16 torch tensor -> FP32 numpy array with the same values."""
    return t.detach().to("cpu").to(torch.float32).numpy()


def kd_logits(seed: int = 0, rows: int = 2048, V: int = 248320, k_peaked: int = 64):
    """Teacher / student logits for the top-k KL loss ("Model-Optimizer in
    practice: recovering Qwen3.6-35B-A3B W4A4 NVFP4 accuracy with QAD",
    section "QAD": vocabulary of
    248,320 entries): teacher = N(0, 2) with k_peaked entries per row raised
    by 8 (a peaked distribution), student = teacher + N(0, 0.5); both BF16."""
    rt, rp, rs = _streams(seed, 3)
    t = normal(rt, (rows, V), 2.0)
    for r in range(rows):
        t[r, rp.choice(V, size=k_peaked, replace=False)] += np.float32(8.0)
    s = t + normal(rs, (rows, V), 0.5)
    return dict(teacher=to_bf16(t), student=to_bf16(s))
