"""CPU oracle for the CCQ WINT2 path (test infrastructure only).

Only tests/, ``__graft_entry__.smoke()`` and bench.py's CPU-baseline leg may import this package.
It shares no code with the CUDA path; the arithmetic lives in ``ccq_oracle.c`` (plain C, fp64),
compiled by :func:`build` with gcc and loaded with ctypes.  The small Python helpers below
(INT4 packing, round-to-nearest) restate the "GPTQ and AWQ" lesson's Part 2 specification.

Sources cited in the docstrings:
  [CCQ]   "CCQ: Convolutional Code for Extreme Low-bit Quantization in LLMs" (arXiv 2507.07145)
  [WINT2] FastDeploy "WINT2 Quantization" documentation page
  [GPTQ]  course lesson "GPTQ and AWQ" (E6.4)

Parity unpinned: the encoder's *quality* (squared error of the chosen codes) has no published
value; its argmin, tie rule, round trip and Eq. 4 properties are pinned instead.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ccq_oracle.c")
_LIB = os.path.join(_HERE, "libccq_oracle.so")

ENC_LITERAL_EQ1 = 1
ENC_REFIT_SCALE = 2


def build(force: bool = False) -> str:
    """Compile ccq_oracle.c into libccq_oracle.so (gcc, OpenMP over independent rows/tokens)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fopenmp", "-fPIC", "-shared",
               "-Wall", "-o", _LIB + ".tmp", _SRC, "-lm"]
        subprocess.check_call(cmd)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        i = ctypes.c_int
        L.oracle_code_bits.argtypes = [i, i, i]
        L.oracle_codebook.argtypes = [i, i, i, P]
        L.oracle_bf16_bits.argtypes = [ctypes.c_float]
        L.oracle_bf16_bits.restype = ctypes.c_uint16
        L.oracle_cluster_code.argtypes = [ctypes.c_uint8, ctypes.c_float, ctypes.c_float]
        L.oracle_cluster_code.restype = ctypes.c_int32
        L.oracle_dequant_w2.argtypes = [P, P, P, P, i, i, i, P]
        L.oracle_dequant_w4.argtypes = [P, P, i, i, P]
        L.oracle_dequant_w2q4.argtypes = [P, P, P, P, P, i, i, i, P]
        L.oracle_dequant_w2std.argtypes = [P, P, i, i, i, P]
        L.oracle_dequant_emb.argtypes = [i, P, P, i, i, P]
        L.oracle_encode_emb.argtypes = [i, P, i, i, P, P]
        L.oracle_quantize_w2std.argtypes = [P, i, i, i, P, P]
        L.oracle_encode_w2q4.argtypes = [P, i, i, i, ctypes.c_uint32, P, P, P, P, P]
        L.oracle_gemm_bf16_f64.argtypes = [P, P, i, i, i, P]
        L.oracle_gemm_bf16_f64.restype = None
        L.oracle_expert_ffn_f64.argtypes = [P, i, i, i, P, P, i, P]
        L.oracle_moe_f64.argtypes = [P, i, i, i, i, P, P, P, P, i, i, P]
        L.oracle_encode_w2.argtypes = [P, i, i, i, ctypes.c_uint32, P, P, P, P]
        L.oracle_w2_sq_error.argtypes = [P, P, P, P, P, i, i, i]
        L.oracle_w2_sq_error.restype = ctypes.c_double
        L.oracle_quantize_w4.argtypes = [P, i, i, P, P]
        _lib = L
    return _lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


# --------------------------------------------------------------------------------------------
# codebook and bit-level helpers ([CCQ] §3.1, Fig. 1)
# --------------------------------------------------------------------------------------------
def code_bits(L: int, N: int, S: int) -> int:
    """T = L + (N-1) S bits per convolutional code ([CCQ] §3.1)."""
    return int(lib().oracle_code_bits(L, N, S))


def codebook(L: int, N: int, S: int) -> np.ndarray:
    """Codebook C in Z^{2^T x N}: row `code` = the N states the code walks through ([CCQ] Fig. 1)."""
    T = code_bits(L, N, S)
    out = np.zeros((1 << T, N), dtype=np.int32)
    rc = lib().oracle_codebook(L, N, S, _p(out))
    if rc != 0:
        raise ValueError(f"codebook({L},{N},{S}) failed: {rc}")
    return out


def bf16_bits(x) -> np.ndarray:
    """BF16 round-to-nearest-even bit patterns of fp32 values."""
    xs = np.asarray(x, dtype=np.float32).ravel()
    out = np.array([lib().oracle_bf16_bits(float(v)) for v in xs], dtype=np.uint16)
    return out.reshape(np.shape(x))


def bf16_to_f64(bits) -> np.ndarray:
    b = np.asarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def cluster_code(q: int, alpha: float, beta: float) -> int:
    """round(q * alpha + beta): fp32 fused multiply-add, ties to even ([CCQ] Eq. 1 / Algorithm 3)."""
    return int(lib().oracle_cluster_code(int(q), float(alpha), float(beta)))


# --------------------------------------------------------------------------------------------
# decode ([CCQ] §3.5 Algorithm 3; [WINT2] W4 per-channel)
# --------------------------------------------------------------------------------------------
def dequant_w2(codes, scales, alpha, beta, group: int = 64) -> np.ndarray:
    """W2 CCQ (6,4,3) code-cluster decode -> BF16 bit patterns [n][k]."""
    codes = _c(codes, np.uint8)
    n, kb = codes.shape
    k = kb * 4
    scales = _c(scales, np.float32).reshape(n, k // group)
    alpha = _c(alpha, np.float32).reshape(n)
    beta = _c(beta, np.float32).reshape(n)
    out = np.zeros((n, k), dtype=np.uint16)
    rc = lib().oracle_dequant_w2(_p(codes), _p(scales), _p(alpha), _p(beta), n, k, group, _p(out))
    if rc != 0:
        raise ValueError("dequant_w2: bad shape")
    return out


def dequant_w2q4(codes, scale_q4, super_scale, alpha, beta, group: int = 64) -> np.ndarray:
    """W2 CCQ decode with 4-bit group scales ([CCQ] §3.4 Scale Compression, Algorithm 3):
    s = q4 * super_scale, two q4 per byte (even group in the low nibble) -> BF16 bits [n][k]."""
    codes = _c(codes, np.uint8)
    n, kb = codes.shape
    k = kb * 4
    nb = (k // group + 1) // 2
    scale_q4 = _c(scale_q4, np.uint8).reshape(n, nb)
    super_scale = _c(super_scale, np.float32).reshape(n)
    alpha = _c(alpha, np.float32).reshape(n)
    beta = _c(beta, np.float32).reshape(n)
    out = np.zeros((n, k), dtype=np.uint16)
    rc = lib().oracle_dequant_w2q4(_p(codes), _p(scale_q4), _p(super_scale), _p(alpha), _p(beta), n, k, group,
                                   _p(out))
    if rc != 0:
        raise ValueError("dequant_w2q4: bad shape")
    return out


def dequant_w2std(codes, scales, group: int = 64) -> np.ndarray:
    """WINT2-Standard decode (plain 2-bit fields, zero-point 2, group scales) -> BF16 bits [n][k]."""
    codes = _c(codes, np.uint8)
    n, kb = codes.shape
    k = kb * 4
    scales = _c(scales, np.float32).reshape(n, k // group)
    out = np.zeros((n, k), dtype=np.uint16)
    if lib().oracle_dequant_w2std(_p(codes), _p(scales), n, k, group, _p(out)) != 0:
        raise ValueError("dequant_w2std: bad shape")
    return out


def quantize_w2std(w, group: int = 64):
    """WINT2-Standard round-to-nearest -> (codes [n][k/4] u8, scales [n][k/g] f32)."""
    w = _c(w, np.float32)
    n, k = w.shape
    codes = np.zeros((n, k // 4), dtype=np.uint8)
    scales = np.zeros((n, k // group), dtype=np.float32)
    if lib().oracle_quantize_w2std(_p(w), n, k, group, _p(codes), _p(scales)) != 0:
        raise ValueError("quantize_w2std: bad shape")
    return codes, scales


# Formats without code cluster, group scale in the redundant bits (CCQ §3.5 Algorithm 2):
# kind 1 = (4,3,2) 2.75 bpw, 22 uint8 codes per 64 weights; kind 2 = hybrid (3,3,2)+(3,4,2) 2.5 bpw,
# 10 uint16 words per 64 weights.  One fp32 super scale per row.
EMB_KINDS = {1: (np.uint8, 22), 2: (np.uint16, 10)}


def dequant_emb(kind: int, codes, super_scale) -> np.ndarray:
    """Algorithm 2 decode -> BF16 bits [n][k]."""
    dt, nw = EMB_KINDS[kind]
    codes = _c(codes, dt)
    n = codes.shape[0]
    k = codes.shape[1] // nw * 64
    sup = _c(super_scale, np.float32).reshape(n)
    out = np.zeros((n, k), dtype=np.uint16)
    if lib().oracle_dequant_emb(kind, _p(codes), _p(sup), n, k, _p(out)) != 0:
        raise ValueError("dequant_emb: bad shape")
    return out


def encode_emb(kind: int, w):
    """Algorithm 2 format encoder -> (codes [n][k/64*words], super_scale [n])."""
    dt, nw = EMB_KINDS[kind]
    w = _c(w, np.float32)
    n, k = w.shape
    codes = np.zeros((n, k // 64 * nw), dtype=dt)
    sup = np.zeros(n, dtype=np.float32)
    if lib().oracle_encode_emb(kind, _p(w), n, k, _p(codes), _p(sup)) != 0:
        raise ValueError("encode_emb: bad shape")
    return codes, sup


def dequant_w4(codes, scales) -> np.ndarray:
    """W4 per-channel decode -> BF16 bit patterns [n][k] (low nibble first)."""
    codes = _c(codes, np.uint8)
    n, kb = codes.shape
    k = kb * 2
    scales = _c(scales, np.float32).reshape(n)
    out = np.zeros((n, k), dtype=np.uint16)
    rc = lib().oracle_dequant_w4(_p(codes), _p(scales), n, k, _p(out))
    if rc != 0:
        raise ValueError("dequant_w4: bad shape")
    return out


# --------------------------------------------------------------------------------------------
# products
# --------------------------------------------------------------------------------------------
def gemm_f64(x_bits, w_bits) -> np.ndarray:
    """y = x W^T over BF16 inputs in fp64 ([WINT2]: BF16 activations times decoded BF16 weights)."""
    x_bits = _c(x_bits, np.uint16)
    w_bits = _c(w_bits, np.uint16)
    m, k = x_bits.shape
    n, k2 = w_bits.shape
    assert k == k2
    y = np.zeros((m, n), dtype=np.float64)
    lib().oracle_gemm_bf16_f64(_p(x_bits), _p(w_bits), m, n, k, _p(y))
    return y


def expert_ffn_f64(x_bits, w13_bits, w2_bits, round_h: bool = False) -> np.ndarray:
    """SiLU(x Wg^T) * (x Wu^T) Wd^T for one expert, fp64; W13 rows [0,I) gate, [I,2I) up."""
    x_bits = _c(x_bits, np.uint16)
    w13_bits = _c(w13_bits, np.uint16)
    w2_bits = _c(w2_bits, np.uint16)
    T, H = x_bits.shape
    I2, H2 = w13_bits.shape
    I = I2 // 2
    assert H2 == H and w2_bits.shape == (H, I)
    out = np.zeros((T, H), dtype=np.float64)
    rc = lib().oracle_expert_ffn_f64(_p(x_bits), T, H, I, _p(w13_bits), _p(w2_bits), int(round_h), _p(out))
    if rc != 0:
        raise MemoryError("expert_ffn_f64")
    return out


def moe_f64(x_bits, w13_bits, w2_bits, ids, rw, round_h: bool = False) -> np.ndarray:
    """Top-k MoE FFN over decoded experts: y_t = sum_j r_tj * FFN_{e_tj}(x_t), fp64."""
    x_bits = _c(x_bits, np.uint16)
    w13_bits = _c(w13_bits, np.uint16)
    w2_bits = _c(w2_bits, np.uint16)
    ids = _c(ids, np.int32)
    rw = _c(rw, np.float32)
    T, H = x_bits.shape
    E, I2, H2 = w13_bits.shape
    I = I2 // 2
    assert H2 == H and w2_bits.shape == (E, H, I)
    topk = ids.shape[1]
    y = np.zeros((T, H), dtype=np.float64)
    rc = lib().oracle_moe_f64(_p(x_bits), T, H, I, E, _p(w13_bits), _p(w2_bits), _p(ids), _p(rw), topk,
                              int(round_h), _p(y))
    if rc != 0:
        raise MemoryError("moe_f64")
    return y


# --------------------------------------------------------------------------------------------
# encoders ([CCQ] Algorithm 1, Eq. 1, Eq. 4; [GPTQ] rtn)
# --------------------------------------------------------------------------------------------
def encode_w2(w, group: int = 64, flags: int = 0):
    """CCQ (6,4,3) code-cluster encode -> (codes [n][k/4] u8, scales [n][k/g] f32, alpha [n], beta [n])."""
    w = _c(w, np.float32)
    n, k = w.shape
    codes = np.zeros((n, k // 4), dtype=np.uint8)
    scales = np.zeros((n, k // group), dtype=np.float32)
    alpha = np.zeros(n, dtype=np.float32)
    beta = np.zeros(n, dtype=np.float32)
    rc = lib().oracle_encode_w2(_p(w), n, k, group, flags, _p(codes), _p(scales), _p(alpha), _p(beta))
    if rc != 0:
        raise ValueError("encode_w2: bad shape")
    return codes, scales, alpha, beta


def encode_w2q4(w, group: int = 64, flags: int = 0):
    """CCQ encode for the 4-bit scale format -> (codes, scale_q4 [n][ceil(k/g/2)] u8, super [n], alpha, beta)."""
    w = _c(w, np.float32)
    n, k = w.shape
    nb = (k // group + 1) // 2
    codes = np.zeros((n, k // 4), dtype=np.uint8)
    sq = np.zeros((n, nb), dtype=np.uint8)
    sup = np.zeros(n, dtype=np.float32)
    alpha = np.zeros(n, dtype=np.float32)
    beta = np.zeros(n, dtype=np.float32)
    rc = lib().oracle_encode_w2q4(_p(w), n, k, group, flags, _p(codes), _p(sq), _p(sup), _p(alpha), _p(beta))
    if rc != 0:
        raise ValueError("encode_w2q4: bad shape or flags")
    return codes, sq, sup, alpha, beta


def q4_unpack(scale_q4, ng: int) -> np.ndarray:
    """The 4-bit group scales as integers [n][ng] (even group in the low nibble)."""
    b = np.asarray(scale_q4, dtype=np.uint8)
    lo, hi = b & 0xF, b >> 4
    return np.stack([lo, hi], axis=-1).reshape(b.shape[0], -1)[:, :ng]


def w2_sq_error(w, codes, scales, alpha, beta, group: int = 64) -> float:
    w = _c(w, np.float32)
    n, k = w.shape
    return float(lib().oracle_w2_sq_error(_p(w), _p(_c(codes, np.uint8)), _p(_c(scales, np.float32)),
                                          _p(_c(alpha, np.float32)), _p(_c(beta, np.float32)), n, k, group))


def quantize_w4(w):
    """W4 per-channel RTN -> (codes [n][k/2] u8, scales [n] f32)."""
    w = _c(w, np.float32)
    n, k = w.shape
    codes = np.zeros((n, k // 2), dtype=np.uint8)
    scales = np.zeros(n, dtype=np.float32)
    rc = lib().oracle_quantize_w4(_p(w), n, k, _p(codes), _p(scales))
    if rc != 0:
        raise ValueError("quantize_w4: bad shape")
    return codes, scales


def pack_int4(codes):
    """[GPTQ] Part 2: two signed 4-bit codes per byte, first of a pair in the low nibble; an odd
    count is padded with 0; a code outside -8..7 raises ValueError."""
    out = []
    cs = list(codes)
    for c in cs:
        if not (-8 <= int(c) <= 7):
            raise ValueError(f"code {c} outside -8..7")
    if len(cs) % 2:
        cs.append(0)
    for i in range(0, len(cs), 2):
        lo, hi = int(cs[i]), int(cs[i + 1])
        out.append((lo & 0xF) | ((hi & 0xF) << 4))
    return out


def unpack_int4(data, n: int):
    """[GPTQ] Part 2: the first n signed codes (each 4-bit field sign-extended)."""
    vals = []
    for b in data:
        b = int(b)
        for nib in (b & 0xF, (b >> 4) & 0xF):
            vals.append(nib - 16 if nib >= 8 else nib)
    return vals[:n]


def packed_size(n_codes: int) -> int:
    """[GPTQ] Part 2: bytes for n 4-bit codes."""
    return (int(n_codes) + 1) // 2


def rtn(w, scale):
    """[GPTQ] Part 2: clip(round(w/scale), -8, 7) * scale with ties to even (np.round)."""
    return np.clip(np.round(np.asarray(w, dtype=np.float64) / scale), -8, 7) * scale


def silu_f64(z):
    """SiLU(z) = z / (1 + e^-z)."""
    z = np.asarray(z, dtype=np.float64)
    return z / (1.0 + np.exp(-z))
