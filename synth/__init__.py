"""Seeded synthetic inputs shared by the tests, the bench and the oracle checks.

This module holds random-number recipes only: it contains none of the quantization, decode or
matmul arithmetic, so both the CUDA path and the CPU oracle can consume what it produces without
sharing method code.  Every generator takes an explicit integer seed and uses numpy's PCG64.

Seed convention: seed = 1000 * workload_id + tensor_id (+ 100 * layer + expert where relevant).
"""
from __future__ import annotations

import numpy as np
import torch


def rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(int(seed)))


def weights_normal(n: int, k: int, seed: int, std: float = 0.02) -> np.ndarray:
    """fp32 weights [n][k] ~ N(0, std^2)."""
    return (rng(seed).standard_normal((n, k), dtype=np.float32) * np.float32(std)).astype(np.float32)


def bf16_tensor_from_f32(a: np.ndarray) -> torch.Tensor:
    """CPU BF16 tensor holding the fp32 array rounded to BF16 (torch's conversion)."""
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """uint16 bit patterns of a CPU BF16 tensor."""
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def activations(m: int, k: int, seed: int, outlier_frac: float = 0.0, outlier_scale: float = 20.0) -> torch.Tensor:
    """BF16 activations [m][k] ~ N(0,1); a seeded `outlier_frac` of the k channels is scaled by
    `outlier_scale` (the prefill MoE workload uses 1% x20)."""
    g = rng(seed)
    x = g.standard_normal((m, k), dtype=np.float32)
    if outlier_frac > 0.0:
        nout = int(round(outlier_frac * k))
        ch = g.choice(k, size=nout, replace=False)
        x[:, ch] *= np.float32(outlier_scale)
    return bf16_tensor_from_f32(x)


def one_hot_rows(k: int) -> torch.Tensor:
    """BF16 identity [k][k]: row m has a single 1 in column m."""
    return torch.eye(k, dtype=torch.bfloat16)


def _softmax_rows(z: np.ndarray) -> np.ndarray:
    z = z - z.max(axis=1, keepdims=True)
    e = np.exp(z)
    return (e / e.sum(axis=1, keepdims=True)).astype(np.float32)


def routing_uniform(T: int, E: int, topk: int, seed: int):
    """Expert ids [T][topk] (distinct within a token, uniform over E) and routing weights
    [T][topk] = softmax of topk N(0,1) logits."""
    g = rng(seed)
    ids = np.empty((T, topk), dtype=np.int32)
    for t in range(T):
        ids[t] = g.choice(E, size=topk, replace=False)
    w = _softmax_rows(g.standard_normal((T, topk)).astype(np.float64))
    return ids, w


def routing_zipf(T: int, E: int, topk: int, seed: int, s: float = 1.1):
    """Zipf(s)-skewed expert popularity over ranks 1..E with a seeded rank->expert permutation;
    each token draws topk distinct experts by Gumbel-top-k on log p (sampling without
    replacement); routing weights are the softmax of topk N(0,1) logits."""
    g = rng(seed)
    ranks = np.arange(1, E + 1, dtype=np.float64)
    p = ranks ** (-s)
    p /= p.sum()
    perm = g.permutation(E)
    logp = np.empty(E)
    logp[perm] = np.log(p)
    gumbel = -np.log(-np.log(g.random((T, E))))
    ids = np.argsort(-(logp[None, :] + gumbel), axis=1)[:, :topk].astype(np.int32)
    w = _softmax_rows(g.standard_normal((T, topk)).astype(np.float64))
    return ids, w


def w2_format_random(n: int, k: int, seed: int, group: int = 64, scale_std: float = 0.02):
    """Random but well-formed W2 code-cluster parameters, for decode/GEMM parity at sizes the
    encoder would take too long on: codes uniform over 0..255, per-channel code zero-point an
    integer in [0, 12000], code scale uniform so that zero-point + 255 * scale stays below
    2^15, and group scales of the magnitude a N(0, scale_std^2) weight group gives."""
    g = rng(seed)
    codes = g.integers(0, 256, size=(n, k // 4), dtype=np.uint8)
    beta = g.integers(0, 12001, size=n).astype(np.float32)
    hi = (32767.0 - beta.astype(np.float64)) / 255.0
    alpha = (g.random(n) * (hi - 4.0) + 4.0).astype(np.float32)
    scales = (np.abs(g.normal(2.5, 0.4, size=(n, k // group))) * scale_std / 31.0).astype(np.float32)
    return codes, scales, alpha, beta


def w2q4_format_random(n: int, k: int, seed: int, group: int = 64, scale_std: float = 0.02):
    """Random well-formed parameters of the 4-bit-scale W2 format: codes, alpha and beta as
    w2_format_random; 4-bit group scales uniform over 0..15 packed two per byte (even group in
    the low nibble); per-channel super scales of the magnitude a N(0, scale_std^2) row gives."""
    codes, _, alpha, beta = w2_format_random(n, k, seed, group, scale_std)
    g = rng(seed + 7)
    sq = g.integers(0, 256, size=(n, k // (2 * group)), dtype=np.uint8)
    sup = (np.abs(g.normal(3.0, 0.3, size=n)) * scale_std / 31.0 / 15.0).astype(np.float32)
    return codes, sq, sup, alpha, beta


def w4_format_random(n: int, k: int, seed: int, scale_std: float = 0.02):
    """Random W4 per-channel parameters: codes uniform bytes (two signed nibbles), scales of the
    magnitude a N(0, scale_std^2) row gives."""
    g = rng(seed)
    codes = g.integers(0, 256, size=(n, k // 2), dtype=np.uint8)
    scales = (np.abs(g.normal(4.0, 0.3, size=n)) * scale_std / 7.0).astype(np.float32)
    return codes, scales


def std_format_random(n: int, k: int, seed: int, group: int = 64, scale_std: float = 0.02):
    """Random WINT2-Standard parameters: codes uniform bytes (four 2-bit fields), group scales of the
    magnitude max|w|/2 of a N(0, scale_std^2) weight group gives."""
    g = rng(seed)
    codes = g.integers(0, 256, size=(n, k // 4), dtype=np.uint8)
    scales = (np.abs(g.normal(2.5, 0.4, size=(n, k // group))) * scale_std / 2.0).astype(np.float32)
    return codes, scales


def emb_format_random(kind: int, n: int, k: int, seed: int, scale_std: float = 0.02):
    """Random parameters of the formats with the scale in the redundant bits (kind 1: (4,3,2), 22
    bytes per 64 weights; kind 2: hybrid, 20 bytes): uniform code bytes (every byte and 16-bit word
    is a valid code; the scale bits are uniform too) and per-row super scales of the magnitude a
    N(0, scale_std^2) row gives."""
    g = rng(seed)
    gb = 22 if kind == 1 else 20
    codes = g.integers(0, 256, size=(n, k // 64 * gb), dtype=np.uint8)
    levels, qmax = (7.0, 15.0) if kind == 1 else (3.0, 8191.0)
    sup = (np.abs(g.normal(3.0, 0.3, size=n)) * scale_std / levels / qmax).astype(np.float32)
    return codes, sup
