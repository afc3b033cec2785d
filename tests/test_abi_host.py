"""Host-side checks of libccq (no GPU): the library loads and exports every entry point that
include/ccq.h declares, host argument validation, and the host encoders against the oracle."""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle
import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def ccq(built_lib):
    import extreme_bit_weight_b200 as m

    return m


def test_exports_every_declared_symbol(ccq):
    with open(os.path.join(ROOT, "include", "ccq.h")) as f:
        hdr = f.read()
    names = sorted(set(re.findall(r"\b(ccq_[a-z0-9_]+)\s*\(", hdr)))
    assert "ccq_w2a16_gemm" in names and "ccq_moe_w2a16_forward" in names and "ccq_encode_host" in names
    lib = ctypes.CDLL(ccq.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert ccq.exported_symbols() == names


def test_status_strings(ccq):
    for s in range(6):
        assert ccq.ccq_status_string(s)
    assert "sm_100a" in ccq.ccq_build_info()


def test_host_validation_returns_before_launch(ccq):
    lib = ccq._lib
    w = ccq.ccq_weight(ccq.CCQ_FMT_W2_CCQ_G64, 256, 256, 64, None, None, None, None)
    # null weight pointers
    assert lib.ccq_w2a16_gemm(ctypes.byref(w), None, 4, None, None, 0, None) == ccq.CCQ_ERR_INVALID_ARG
    fake = 1 << 40  # never dereferenced: validation fails on other arguments first
    w = ccq.ccq_weight(ccq.CCQ_FMT_W2_CCQ_G64, 256, 200, 64, fake, fake, fake, fake)  # k % 64
    assert lib.ccq_w2a16_gemm(ctypes.byref(w), fake, 4, fake, fake, 1 << 30, None) == ccq.CCQ_ERR_INVALID_ARG
    w = ccq.ccq_weight(ccq.CCQ_FMT_W2_CCQ_G64, 250, 256, 64, fake, fake, fake, fake)  # n % 16
    assert lib.ccq_w2a16_gemm(ctypes.byref(w), fake, 4, fake, fake, 1 << 30, None) == ccq.CCQ_ERR_INVALID_ARG
    w = ccq.ccq_weight(ccq.CCQ_FMT_W2_CCQ_G64, 256, 256, 32, fake, fake, fake, fake)  # group != 64
    assert lib.ccq_w2a16_gemm(ctypes.byref(w), fake, 4, fake, fake, 1 << 30, None) == ccq.CCQ_ERR_UNSUPPORTED
    w = ccq.ccq_weight(7, 256, 256, 64, fake, fake, fake, fake)
    assert lib.ccq_w2a16_gemm(ctypes.byref(w), fake, 4, fake, fake, 1 << 30, None) == ccq.CCQ_ERR_UNSUPPORTED
    w = ccq.ccq_weight(ccq.CCQ_FMT_W2_CCQ_G64, 256, 256, 64, fake + 4, fake, fake, fake)  # misaligned codes
    assert lib.ccq_w2a16_gemm(ctypes.byref(w), fake, 4, fake, fake, 1 << 30, None) == ccq.CCQ_ERR_INVALID_ARG
    w = ccq.ccq_weight(ccq.CCQ_FMT_W2_CCQ_G64, 256, 256, 64, fake, fake, fake, fake)
    assert lib.ccq_w2a16_gemm(ctypes.byref(w), fake, 0, fake, None, 0, None) == ccq.CCQ_OK  # m == 0: no-op
    assert lib.ccq_w2a16_gemm(ctypes.byref(w), fake + 2, 4, fake, fake, 1 << 30, None) == ccq.CCQ_ERR_INVALID_ARG
    need = lib.ccq_gemm_workspace_size(ctypes.byref(w), 4)
    assert need > 0
    assert lib.ccq_w2a16_gemm(ctypes.byref(w), fake, 4, fake, fake, need - 1, None) == ccq.CCQ_ERR_INVALID_ARG
    # MoE: shape mismatch and bad top-k
    w13 = ccq.ccq_weight(ccq.CCQ_FMT_W2_CCQ_G64, 256, 512, 64, fake, fake, fake, fake)
    w2 = ccq.ccq_weight(ccq.CCQ_FMT_W2_CCQ_G64, 512, 64, 64, fake, fake, fake, fake)  # k != I
    assert lib.ccq_moe_w2a16_forward(ctypes.byref(w13), ctypes.byref(w2), 4, fake, 8, fake, fake, 2, fake + 512,
                                     fake, 1 << 30, None) == ccq.CCQ_ERR_INVALID_ARG
    w2 = ccq.ccq_weight(ccq.CCQ_FMT_W2_CCQ_G64, 512, 128, 64, fake, fake, fake, fake)
    assert lib.ccq_moe_w2a16_forward(ctypes.byref(w13), ctypes.byref(w2), 4, fake, 8, fake, fake, 0, fake + 512,
                                     fake, 1 << 30, None) == ccq.CCQ_ERR_INVALID_ARG
    assert lib.ccq_moe_w2a16_forward(ctypes.byref(w13), ctypes.byref(w2), 4, fake, 8, fake, fake, 2, fake,
                                     fake, 1 << 30, None) == ccq.CCQ_ERR_INVALID_ARG  # y aliases x
    assert lib.ccq_moe_w2a16_forward(ctypes.byref(w13), ctypes.byref(w2), 4, fake, 0, fake, fake, 2, fake + 512,
                                     None, 0, None) == ccq.CCQ_OK  # T == 0
    assert lib.ccq_check_device_error(None, None) == ccq.CCQ_ERR_INVALID_ARG
    # WINT2-Standard: no alpha/beta needed (validation passes them and fails on the workspace);
    # group != 64 unsupported; its quantizer checks shapes, pointers and alignment before launching
    w = ccq.ccq_weight(ccq.CCQ_FMT_W2_STD_G64, 256, 256, 64, fake, fake, None, None)
    assert lib.ccq_w2a16_gemm(ctypes.byref(w), fake, 4, fake, fake, 0, None) == ccq.CCQ_ERR_INVALID_ARG
    assert lib.ccq_w2a16_gemm(ctypes.byref(w), fake, 0, fake, None, 0, None) == ccq.CCQ_OK
    w = ccq.ccq_weight(ccq.CCQ_FMT_W2_STD_G64, 256, 256, 32, fake, fake, None, None)
    assert lib.ccq_w2a16_gemm(ctypes.byref(w), fake, 4, fake, fake, 1 << 30, None) == ccq.CCQ_ERR_UNSUPPORTED
    q = lib.ccq_quantize_std_device
    assert q(None, 4, 64, fake, fake, None) == ccq.CCQ_ERR_INVALID_ARG
    assert q(fake, 4, 96, fake, fake, None) == ccq.CCQ_ERR_INVALID_ARG      # k % 64
    assert q(fake, -1, 64, fake, fake, None) == ccq.CCQ_ERR_INVALID_ARG
    assert q(fake + 8, 4, 64, fake, fake, None) == ccq.CCQ_ERR_INVALID_ARG  # misaligned w
    # formats with the scale in the redundant bits: k pitch rules, super scale required, encoder args
    for fmt, kbad in ((ccq.CCQ_FMT_W275_432, 768), (ccq.CCQ_FMT_W25_HYBRID, 320)):
        w = ccq.ccq_weight(fmt, 256, kbad, 64, fake, None, None, None, None, fake)
        assert lib.ccq_w2a16_gemm(ctypes.byref(w), fake, 4, fake, fake, 1 << 30, None) == ccq.CCQ_ERR_INVALID_ARG
        w = ccq.ccq_weight(fmt, 256, 1024, 64, fake, None, None, None, None, None)
        assert lib.ccq_w2a16_gemm(ctypes.byref(w), fake, 4, fake, fake, 1 << 30, None) == ccq.CCQ_ERR_INVALID_ARG
        w = ccq.ccq_weight(fmt, 256, 1024, 64, fake, None, None, None, None, fake)
        assert lib.ccq_w2a16_gemm(ctypes.byref(w), fake, 4, fake, fake, 0, None) == ccq.CCQ_ERR_INVALID_ARG
        assert lib.ccq_gemm_workspace_size(ctypes.byref(w), 1) > 0
        e = lib.ccq_encode_emb_device
        assert e(fmt, None, 4, 64, fake, fake, None) == ccq.CCQ_ERR_INVALID_ARG
        assert e(fmt, fake, 4, 96, fake, fake, None) == ccq.CCQ_ERR_INVALID_ARG
        assert e(fmt, fake + 4, 4, 64, fake, fake, None) == ccq.CCQ_ERR_INVALID_ARG
    assert lib.ccq_encode_emb_device(ccq.CCQ_FMT_W2_CCQ_G64, fake, 4, 64, fake, fake, None) == ccq.CCQ_ERR_UNSUPPORTED
    # failure-detection self-test: argument checks before any launch
    t = lib.ccq_selftest_bounded_wait
    assert t(None, 0, 1000, None) == ccq.CCQ_ERR_INVALID_ARG
    assert t(fake + 4, 0, 1000, None) == ccq.CCQ_ERR_INVALID_ARG
    assert t(fake, 2, 1000, None) == ccq.CCQ_ERR_INVALID_ARG
    assert t(fake, 0, 0, None) == ccq.CCQ_ERR_INVALID_ARG
    assert t(fake, 1, 3000000, None) == ccq.CCQ_ERR_INVALID_ARG


def test_encoder_matches_oracle(ccq):
    # product host encoder (trellis search) vs the oracle's brute-force Algorithm 1
    w = synth.weights_normal(6, 128, 101)
    w[2, 64:] = 0.0  # one all-zero group
    for flags in (0, ccq.CCQ_ENC_LITERAL_EQ1, ccq.CCQ_ENC_REFIT_SCALE):
        c, s, a, b, err = ccq.ccq_encode_host(w, 64, flags, threads=4)
        oc, os_, oa, ob = oracle.encode_w2(w, 64, flags)
        assert np.array_equal(a, oa) and np.array_equal(b, ob)
        assert np.array_equal(s, os_)
        assert np.array_equal(c, oc)
        assert abs(err - oracle.w2_sq_error(w, c, s, a, b)) <= 1e-12 * max(err, 1e-30)


def test_encoder_q4_matches_oracle(ccq):
    # the 4-bit-scale encoder (CCQ §3.4 Scale Compression) vs the oracle's: identical bytes
    w = synth.weights_normal(6, 256, 103)
    w[3, 64:128] = 0.0  # one all-zero group (scale 0)
    for flags in (0, ccq.CCQ_ENC_LITERAL_EQ1):
        c, sq, sup, a, b, err = ccq.ccq_encode_host_q4(w, 64, flags, threads=3)
        oc, osq, osup, oa, ob = oracle.encode_w2q4(w, 64, flags)
        assert np.array_equal(sup, osup) and np.array_equal(sq, osq)
        assert np.array_equal(a, oa) and np.array_equal(b, ob)
        assert np.array_equal(c, oc)
    with pytest.raises(ccq.CcqError):
        ccq.ccq_encode_host_q4(w, 64, ccq.CCQ_ENC_REFIT_SCALE)
    with pytest.raises(ccq.CcqError):
        ccq.ccq_encode_host_q4(np.zeros((2, 192), np.float32), 64)  # k not a multiple of 128


def test_encoder_rejects_bad_args(ccq):
    w = np.zeros((2, 100), np.float32)
    with pytest.raises(ccq.CcqError):
        ccq.ccq_encode_host(w, 64)
    with pytest.raises(ccq.CcqError):
        ccq.ccq_quantize_w4_host(np.zeros((2, 3), np.float32))


def test_w4_quantizer_matches_oracle(ccq):
    w = synth.weights_normal(8, 96, 102)
    c, s = ccq.ccq_quantize_w4_host(w, threads=3)
    oc, os_ = oracle.quantize_w4(w)
    assert np.array_equal(c, oc) and np.array_equal(s, os_)


def test_binding_refuses_host_tensors(ccq):
    # every compute entry point takes device memory; a host tensor is refused before any call
    import torch

    with pytest.raises(ccq.CcqError):
        ccq.CcqWeight(ccq.CCQ_FMT_W2_CCQ_G64, 16, 64, np.zeros((16, 16), np.uint8), np.zeros((16, 1), np.float32),
                      np.zeros(16, np.float32), np.zeros(16, np.float32), device="cpu")
    with pytest.raises(ccq.CcqError):
        ccq.ccq_check_device_error(torch.zeros(256, dtype=torch.uint8))
    with pytest.raises(ccq.CcqError):
        ccq.ccq_selftest_bounded_wait(torch.zeros(256, dtype=torch.uint8), 0)
