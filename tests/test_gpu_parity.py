"""GPU parity of libccq against the CPU oracle (B200, through the C ABI).

Bars: decoded BF16 weights bit-exact; matmul and MoE outputs max|d|/max|ref| <= 1e-2 (the stated
tolerance; fp32 accumulation), with a tighter regression guard where the arithmetic allows.
"""
import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu

TOL = 1e-2


@pytest.fixture(scope="module")
def ccq():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import extreme_bit_weight_b200 as m

    return m


def rel_err(y, ref):
    y = np.asarray(y, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    return float(np.max(np.abs(y - ref)) / max(np.max(np.abs(ref)), 1e-30))


def bits_of(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def w2_weight(ccq, codes, scales, alpha, beta, experts=1):
    n = codes.shape[-2] if codes.ndim == 3 else codes.shape[0] // experts
    k = codes.shape[-1] * 4
    return ccq.CcqWeight(ccq.CCQ_FMT_W2_CCQ_G64, n, k, codes, scales, alpha, beta, experts=experts)


# ----------------------------------------------------------------------------------------------
# decode
# ----------------------------------------------------------------------------------------------
def test_dequant_small_linear_bitexact(ccq):
    # single linear M=4, K=N=256, weights N(0, 0.02) encoded by the oracle
    w = synth.weights_normal(256, 256, 1001)
    codes, scales, alpha, beta = oracle.encode_w2(w, 64)
    W = w2_weight(ccq, codes, scales, alpha, beta)
    got = bits_of(ccq.ccq_dequant_bf16(W))[0]
    assert np.array_equal(got, oracle.dequant_w2(codes, scales, alpha, beta))


@pytest.mark.parametrize("n,k,E", [(16, 64, 1), (48, 192, 3), (272, 576, 2), (1024, 8192, 1)])
def test_dequant_random_format_bitexact(ccq, n, k, E):
    codes, scales, alpha, beta = synth.w2_format_random(n * E, k, 1100 + n + k)
    W = w2_weight(ccq, codes, scales, alpha, beta, experts=E)
    got = bits_of(ccq.ccq_dequant_bf16(W)).reshape(n * E, k)
    assert np.array_equal(got, oracle.dequant_w2(codes, scales, alpha, beta))


def test_dequant_outside_fast_domain_bitexact(ccq):
    # negative, huge and fractional code parameters: the exact decode still matches the definition
    n, k = 64, 128
    g = synth.rng(1200)
    codes = g.integers(0, 256, size=(n, k // 4), dtype=np.uint8)
    alpha = np.concatenate([g.normal(0, 300, 32), g.normal(0, 1e7, 32)]).astype(np.float32)
    beta = np.concatenate([g.normal(0, 1e5, 32), g.normal(0, 3e9, 32)]).astype(np.float32)
    alpha[0], beta[0] = 0.5, 0.5  # exact ties
    scales = (g.random((n, k // 64)) * 2 - 1).astype(np.float32)
    W = w2_weight(ccq, codes, scales, alpha, beta)
    got = bits_of(ccq.ccq_dequant_bf16(W))[0]
    assert np.array_equal(got, oracle.dequant_w2(codes, scales, alpha, beta))


def test_dequant_w4_bitexact(ccq):
    codes, scales = synth.w4_format_random(96, 320, 1300)
    W = ccq.CcqWeight(ccq.CCQ_FMT_W4_PER_CHANNEL, 96, 320, codes, scales)
    got = bits_of(ccq.ccq_dequant_bf16(W))[0]
    assert np.array_equal(got, oracle.dequant_w4(codes, scales))


# ----------------------------------------------------------------------------------------------
# decode-sized matmul
# ----------------------------------------------------------------------------------------------
def test_gemm_one_hot_identity_small_m(ccq):
    # x = rows of I_K, 16 at a time (the register-decode mma.sync kernel): y[m][n] = w[n][m], so
    # every weight the fused kernel decodes is observed exactly
    n, k = 272, 320
    codes, scales, alpha, beta = synth.w2_format_random(n, k, 1400)
    W = w2_weight(ccq, codes, scales, alpha, beta)
    eye = synth.one_hot_rows(k).cuda()
    ref = oracle.bf16_to_f64(oracle.dequant_w2(codes, scales, alpha, beta)).T
    for j in range(0, k, 16):
        y = ccq.ccq_w2a16_gemm(W, eye[j:j + 16].contiguous()).float().cpu().numpy()
        assert np.array_equal(y, ref[j:j + 16].astype(np.float32)), j


def test_gemm_one_hot_identity_tcgen05(ccq):
    # x = I_K with K >= 33 rows runs the tcgen05 kernel: decoded BF16 weights in shared memory
    n, k = 528, 576
    codes, scales, alpha, beta = synth.w2_format_random(n, k, 1401)
    W = w2_weight(ccq, codes, scales, alpha, beta)
    y = ccq.ccq_w2a16_gemm(W, synth.one_hot_rows(k).cuda()).float().cpu().numpy()
    ref = oracle.bf16_to_f64(oracle.dequant_w2(codes, scales, alpha, beta)).T
    assert np.array_equal(y, ref.astype(np.float32))


def test_gemm_small_linear(ccq):
    w = synth.weights_normal(256, 256, 1001)
    codes, scales, alpha, beta = oracle.encode_w2(w, 64)
    W = w2_weight(ccq, codes, scales, alpha, beta)
    x = synth.activations(4, 256, 1002)
    y = ccq.ccq_w2a16_gemm(W, x.cuda()).float().cpu().numpy()
    ref = oracle.gemm_f64(synth.bf16_bits(x), oracle.dequant_w2(codes, scales, alpha, beta))
    e = rel_err(y, ref)
    assert e <= TOL
    assert e <= 4e-3  # fp32 accumulation + one BF16 output rounding


# m = 32: the largest call on the decode-sized kernel (one 32-token chunk); 33: the smallest on tcgen05
@pytest.mark.parametrize("m,n,k", [(1, 16, 64), (3, 48, 192), (8, 256, 512), (9, 272, 576), (17, 128, 1088),
                                   (32, 256, 1024), (33, 256, 1024), (1, 8192, 8192), (16, 8192, 8192),
                                   (48, 256, 256), (130, 272, 576), (300, 512, 1088), (128, 8192, 8192)])
def test_gemm_shapes(ccq, m, n, k):
    codes, scales, alpha, beta = synth.w2_format_random(n, k, 1500 + m + n + k)
    W = w2_weight(ccq, codes, scales, alpha, beta)
    x = synth.activations(m, k, 1501 + m)
    y = ccq.ccq_w2a16_gemm(W, x.cuda()).float().cpu().numpy()
    ref = oracle.gemm_f64(synth.bf16_bits(x), oracle.dequant_w2(codes, scales, alpha, beta))
    e = rel_err(y, ref)
    assert e <= TOL
    assert e <= 4e-3


def test_gemm_m0_and_determinism(ccq):
    codes, scales, alpha, beta = synth.w2_format_random(256, 1024, 1600)
    W = w2_weight(ccq, codes, scales, alpha, beta)
    x = synth.activations(16, 1024, 1601).cuda()
    y0 = ccq.ccq_w2a16_gemm(W, x[:0])
    assert y0.shape == (0, 256)
    a = bits_of(ccq.ccq_w2a16_gemm(W, x))
    b = bits_of(ccq.ccq_w2a16_gemm(W, x))
    assert np.array_equal(a, b)


# ----------------------------------------------------------------------------------------------
# MoE FFN
# ----------------------------------------------------------------------------------------------
def moe_weights(ccq, E, H, I, seed):
    c13, s13, a13, b13 = synth.w2_format_random(E * 2 * I, H, seed)
    c2, s2, a2, b2 = synth.w2_format_random(E * H, I, seed + 1)
    W13 = ccq.CcqWeight(ccq.CCQ_FMT_W2_CCQ_G64, 2 * I, H, c13, s13, a13, b13, experts=E)
    W2 = ccq.CcqWeight(ccq.CCQ_FMT_W2_CCQ_G64, H, I, c2, s2, a2, b2, experts=E)
    dec13 = oracle.dequant_w2(c13, s13, a13, b13).reshape(E, 2 * I, H)
    dec2 = oracle.dequant_w2(c2, s2, a2, b2).reshape(E, H, I)
    return W13, W2, dec13, dec2


def run_moe(ccq, W13, W2, x, ids, rw):
    ids_t = torch.from_numpy(np.ascontiguousarray(ids, np.int32)).cuda()
    rw_t = torch.from_numpy(np.ascontiguousarray(rw, np.float32)).cuda()
    T, H = x.shape
    ws = ccq.workspace(ccq.ccq_moe_workspace_size(T, ids.shape[1], H, W13.n // 2, W13.experts))
    y = ccq.ccq_moe_w2a16_forward(W13, W2, x.cuda(), ids_t, rw_t, ws=ws)
    st = ccq.ccq_check_device_error(ws)
    return y.float().cpu().numpy(), st


# (104, 8, 2): 26 rows per expert, the decode-sized kernel with experts over one 32-token chunk;
# (112, 8, 2): 28 rows per expert, the smallest MoE layer on the tcgen05 kernel
@pytest.mark.parametrize("T,E,topk", [(5, 8, 2), (40, 4, 1), (24, 16, 4), (104, 8, 2), (112, 8, 2)])
def test_moe_small_full(ccq, T, E, topk):
    H, I = 256, 128
    W13, W2, d13, d2 = moe_weights(ccq, E, H, I, 2000 + T)
    x = synth.activations(T, H, 2002 + T)
    ids, rw = synth.routing_uniform(T, E, topk, 2003 + T)
    y, st = run_moe(ccq, W13, W2, x, ids, rw)
    assert st == ccq.CCQ_OK
    xb = synth.bf16_bits(x)
    ref = oracle.moe_f64(xb, d13, d2, ids, rw, round_h=True)
    ref64 = oracle.moe_f64(xb, d13, d2, ids, rw, round_h=False)
    assert rel_err(y, ref) <= TOL
    assert rel_err(y, ref64) <= TOL


def test_moe_skewed_and_empty_experts(ccq):
    # every token on expert 2 (more tokens than one mma tile), experts 0,1,3..7 empty except one pair
    H, I, E, T = 256, 192, 8, 37
    W13, W2, d13, d2 = moe_weights(ccq, E, H, I, 2100)
    x = synth.activations(T, H, 2101)
    ids = np.full((T, 2), 2, np.int32)
    ids[:, 1] = 5
    rw = np.full((T, 2), 0.5, np.float32)
    y, st = run_moe(ccq, W13, W2, x, ids, rw)
    assert st == ccq.CCQ_OK
    ref = oracle.moe_f64(synth.bf16_bits(x), d13, d2, ids, rw, round_h=True)
    assert rel_err(y, ref) <= TOL


def test_moe_invalid_ids_reported_and_skipped(ccq):
    H, I, E, T = 256, 128, 6, 7
    W13, W2, d13, d2 = moe_weights(ccq, E, H, I, 2200)
    x = synth.activations(T, H, 2201)
    ids, rw = synth.routing_uniform(T, E, 3, 2202)
    ids[1, 0] = E        # out of range
    ids[3, 2] = -1       # out of range
    ids[4, 1] = ids[4, 0]  # repeated within a token
    y, st = run_moe(ccq, W13, W2, x, ids, rw)
    assert st == ccq.CCQ_ERR_DEVICE_CHECK
    keep = ids.copy()
    keep[1, 0] = -1
    keep[3, 2] = -1
    keep[4, 1] = -1
    ref = oracle.moe_f64(synth.bf16_bits(x), d13, d2, keep, rw, round_h=True)
    assert rel_err(y, ref) <= TOL


def test_moe_token_permutation_invariance(ccq):
    H, I, E, T = 256, 128, 8, 16
    W13, W2, _, _ = moe_weights(ccq, E, H, I, 2300)
    x = synth.activations(T, H, 2301)
    ids, rw = synth.routing_uniform(T, E, 2, 2302)
    y, _ = run_moe(ccq, W13, W2, x, ids, rw)
    perm = synth.rng(2303).permutation(T)
    yp, _ = run_moe(ccq, W13, W2, x[perm], ids[perm], rw[perm])
    assert np.array_equal(yp, y[perm])


def test_moe_decode_layer_full_size_sampled(ccq):
    # the decode-sized MoE layer: 32 tokens, hidden 8192, 64 experts of 8192x3584x2 / 3584x8192,
    # top-8 uniform routing with softmax weights; checked on sampled tokens against the oracle
    T, H, I, E, topk = 32, 8192, 3584, 64, 8
    c13, s13, a13, b13 = synth.w2_format_random(E * 2 * I, H, 3000)
    c2, s2, a2, b2 = synth.w2_format_random(E * H, I, 3001)
    W13 = ccq.CcqWeight(ccq.CCQ_FMT_W2_CCQ_G64, 2 * I, H, c13, s13, a13, b13, experts=E)
    W2 = ccq.CcqWeight(ccq.CCQ_FMT_W2_CCQ_G64, H, I, c2, s2, a2, b2, experts=E)
    x = synth.activations(T, H, 3002)
    ids, rw = synth.routing_uniform(T, E, topk, 3003)
    y, st = run_moe(ccq, W13, W2, x, ids, rw)
    assert st == ccq.CCQ_OK
    xb = synth.bf16_bits(x)
    sample = [0, 13, 31]
    ref = np.zeros((len(sample), H))
    for e in sorted({int(ids[t, j]) for t in sample for j in range(topk)}):
        d13 = oracle.dequant_w2(c13[e * 2 * I:(e + 1) * 2 * I], s13[e * 2 * I:(e + 1) * 2 * I],
                                a13[e * 2 * I:(e + 1) * 2 * I], b13[e * 2 * I:(e + 1) * 2 * I])
        d2 = oracle.dequant_w2(c2[e * H:(e + 1) * H], s2[e * H:(e + 1) * H], a2[e * H:(e + 1) * H],
                               b2[e * H:(e + 1) * H])
        for si, t in enumerate(sample):
            for j in range(topk):
                if ids[t, j] == e:
                    ref[si] += float(rw[t, j]) * oracle.expert_ffn_f64(xb[t:t + 1], d13, d2, round_h=True)[0]
    assert rel_err(y[sample], ref) <= TOL


@pytest.mark.parametrize("T,E,topk,H,I,zipf", [(256, 8, 2, 256, 128, False), (512, 16, 4, 1024, 512, True),
                                               (700, 4, 1, 576, 192, False)])
def test_moe_prefill_full(ccq, T, E, topk, H, I, zipf):
    # prefill-sized (>= 28 rows per expert on average): tcgen05 grouped GEMMs
    W13, W2, d13, d2 = moe_weights(ccq, E, H, I, 2400 + T)
    x = synth.activations(T, H, 2401 + T, outlier_frac=0.01)
    ids, rw = (synth.routing_zipf(T, E, topk, 2402 + T) if zipf else synth.routing_uniform(T, E, topk, 2402 + T))
    y, st = run_moe(ccq, W13, W2, x, ids, rw)
    assert st == ccq.CCQ_OK
    xb = synth.bf16_bits(x)
    ref = oracle.moe_f64(xb, d13, d2, ids, rw, round_h=True)
    assert rel_err(y, ref) <= TOL
    assert rel_err(y, oracle.moe_f64(xb, d13, d2, ids, rw, round_h=False)) <= TOL


def test_moe_prefill_layer_full_size_sampled(ccq):
    # the prefill-sized MoE layer: 4096 tokens, hidden 8192, 64 experts, top-8 with Zipf(1.1) expert
    # popularity, activations N(0,1) with 1% of channels x20; checked on sampled tokens
    T, H, I, E, topk = 4096, 8192, 3584, 64, 8
    c13, s13, a13, b13 = synth.w2_format_random(E * 2 * I, H, 3100)
    c2, s2, a2, b2 = synth.w2_format_random(E * H, I, 3101)
    W13 = ccq.CcqWeight(ccq.CCQ_FMT_W2_CCQ_G64, 2 * I, H, c13, s13, a13, b13, experts=E)
    W2 = ccq.CcqWeight(ccq.CCQ_FMT_W2_CCQ_G64, H, I, c2, s2, a2, b2, experts=E)
    x = synth.activations(T, H, 3102, outlier_frac=0.01, outlier_scale=20.0)
    ids, rw = synth.routing_zipf(T, E, topk, 3103, s=1.1)
    y, st = run_moe(ccq, W13, W2, x, ids, rw)
    assert st == ccq.CCQ_OK
    xb = synth.bf16_bits(x)
    sample = [0, 1, 2047, 4095]
    ref = np.zeros((len(sample), H))
    for e in sorted({int(ids[t, j]) for t in sample for j in range(topk)}):
        sl13, sl2 = slice(e * 2 * I, (e + 1) * 2 * I), slice(e * H, (e + 1) * H)
        d13 = oracle.dequant_w2(c13[sl13], s13[sl13], a13[sl13], b13[sl13])
        d2 = oracle.dequant_w2(c2[sl2], s2[sl2], a2[sl2], b2[sl2])
        for si, t in enumerate(sample):
            for j in range(topk):
                if ids[t, j] == e:
                    ref[si] += float(rw[t, j]) * oracle.expert_ffn_f64(xb[t:t + 1], d13, d2, round_h=True)[0]
    assert rel_err(y[sample], ref) <= TOL


# ----------------------------------------------------------------------------------------------
# W4 per-channel (the mixed W4/W2 expert stack: WINT2 page's quantization_config)
# ----------------------------------------------------------------------------------------------
def w4_weight(ccq, codes, scales, experts=1):
    n = codes.shape[0] // experts
    return ccq.CcqWeight(ccq.CCQ_FMT_W4_PER_CHANNEL, n, codes.shape[1] * 2, codes, scales, experts=experts)


def test_gemm_w4_one_hot_identity_both_paths(ccq):
    n, k = 272, 576
    codes, scales = synth.w4_format_random(n, k, 5000)
    W = w4_weight(ccq, codes, scales)
    ref = oracle.bf16_to_f64(oracle.dequant_w4(codes, scales)).T.astype(np.float32)
    eye = synth.one_hot_rows(k).cuda()
    for j in range(0, 64, 16):  # register-decode mma.sync kernel
        y = ccq.ccq_w2a16_gemm(W, eye[j:j + 16].contiguous()).float().cpu().numpy()
        assert np.array_equal(y, ref[j:j + 16]), j
    y = ccq.ccq_w2a16_gemm(W, eye).float().cpu().numpy()  # tcgen05 kernel
    assert np.array_equal(y, ref)


@pytest.mark.parametrize("m,n,k", [(1, 256, 512), (9, 272, 576), (16, 1024, 2048), (33, 256, 1024),
                                   (64, 512, 1024), (300, 272, 576), (1, 8192, 8192)])
def test_gemm_w4_shapes(ccq, m, n, k):
    codes, scales = synth.w4_format_random(n, k, 5100 + m + n)
    W = w4_weight(ccq, codes, scales)
    x = synth.activations(m, k, 5101 + m)
    y = ccq.ccq_w2a16_gemm(W, x.cuda()).float().cpu().numpy()
    ref = oracle.gemm_f64(synth.bf16_bits(x), oracle.dequant_w4(codes, scales))
    e = rel_err(y, ref)
    assert e <= TOL
    assert e <= 4e-3


# formats by name: "ccq" (W2 g64, fp32 scales), "q4" (W2 g64, 4-bit scales), "w4" (per channel),
# "std" (WINT2-Standard); FMT_SEED gives each a number for the seeds
FMT_SEED = {"ccq": 2, "q4": 3, "w4": 4, "std": 5, "w275": 6, "w25": 7}


def moe_weights_fmt(ccq, E, H, I, seed, fmt13, fmt2):
    def make(rows, k, s, fmt):
        if fmt == "q4":  # CCQ W2 with 4-bit group scales
            c, sq, sup, a, b = synth.w2q4_format_random(rows, k, s)
            return q4_weight(ccq, c, sq, sup, a, b, experts=E), oracle.dequant_w2q4(c, sq, sup, a, b)
        if fmt == "w4":
            c, sc = synth.w4_format_random(rows, k, s)
            return (ccq.CcqWeight(ccq.CCQ_FMT_W4_PER_CHANNEL, rows // E, k, c, sc, experts=E),
                    oracle.dequant_w4(c, sc))
        if fmt == "std":
            c, sc = synth.std_format_random(rows, k, s)
            return (ccq.CcqWeight(ccq.CCQ_FMT_W2_STD_G64, rows // E, k, c, sc, experts=E),
                    oracle.dequant_w2std(c, sc))
        if fmt in ("w275", "w25"):
            kind = 1 if fmt == "w275" else 2
            c, sup = synth.emb_format_random(kind, rows, k, s)
            return emb_weight(ccq, kind, c, sup, experts=E), emb_oracle(kind, c, sup)
        assert fmt == "ccq"
        c, sc, a, b = synth.w2_format_random(rows, k, s)
        return (ccq.CcqWeight(ccq.CCQ_FMT_W2_CCQ_G64, rows // E, k, c, sc, a, b, experts=E),
                oracle.dequant_w2(c, sc, a, b))
    W13, d13 = make(E * 2 * I, H, seed, fmt13)
    W2, d2 = make(E * H, I, seed + 1, fmt2)
    return W13, W2, d13.reshape(E, 2 * I, H), d2.reshape(E, H, I)


@pytest.mark.parametrize("fmts", [("w4", "ccq"), ("ccq", "w4"), ("w4", "w4")])
@pytest.mark.parametrize("T", [6, 300])
def test_moe_mixed_formats(ccq, fmts, T):
    E, H, I, topk = 8, 512, 256, 2
    W13, W2, d13, d2 = moe_weights_fmt(ccq, E, H, I, 5200 + T + 10 * FMT_SEED[fmts[0]], *fmts)
    x = synth.activations(T, H, 5201 + T)
    ids, rw = synth.routing_uniform(T, E, topk, 5202 + T)
    y, st = run_moe(ccq, W13, W2, x, ids, rw)
    assert st == ccq.CCQ_OK
    ref = oracle.moe_f64(synth.bf16_bits(x), d13, d2, ids, rw, round_h=True)
    assert rel_err(y, ref) <= TOL


@pytest.mark.parametrize("M", [1, 8, 64, 300])
def test_mixed_stack_layer_by_layer(ccq, M):
    # 8 MoE layers: the first 2 with W4 per-channel experts, the last 6 with CCQ W2 g64 (scaled-down
    # shapes); fresh uniform routing per layer; x_{l+1} = RMSnorm(MoE_l(x_l)) -- random weights grow
    # the activations by 10-1000x per layer, so without the norm a model keeps between layers the
    # stack overflows bf16 by the last layer; every layer checked against the oracle on the GPU's own
    # input to that layer
    E, H, I, topk = 8, 512, 256, 4
    x = synth.activations(M, H, 5300 + M).cuda()
    for layer in range(8):
        fmt = "w4" if layer < 2 else "ccq"
        W13, W2, d13, d2 = moe_weights_fmt(ccq, E, H, I, 5400 + 100 * layer, fmt, fmt)
        ids, rw = synth.routing_uniform(M, E, topk, 5500 + 100 * layer + M)
        ids_t = torch.from_numpy(ids).cuda()
        rw_t = torch.from_numpy(rw).cuda()
        ws = ccq.workspace(ccq.ccq_moe_workspace_size(M, topk, H, I, E))
        y = ccq.ccq_moe_w2a16_forward(W13, W2, x, ids_t, rw_t, ws=ws)
        assert ccq.ccq_check_device_error(ws) == ccq.CCQ_OK
        ref = oracle.moe_f64(bits_of(x), d13, d2, ids, rw, round_h=True)
        assert rel_err(y.float().cpu().numpy(), ref) <= TOL, layer
        yf = y.float()
        x = (yf * torch.rsqrt(yf.pow(2).mean(dim=1, keepdim=True) + 1e-12)).to(torch.bfloat16)


# ----------------------------------------------------------------------------------------------
# CCQ W2 with 4-bit group scales (CCQ §3.4 Scale Compression; 2.06 bpw)
# ----------------------------------------------------------------------------------------------
def q4_weight(ccq, codes, sq, sup, alpha, beta, experts=1):
    n = codes.shape[0] // experts
    return ccq.CcqWeight(ccq.CCQ_FMT_W2_CCQ_G64_Q4SCALE, n, codes.shape[1] * 4, codes, None, alpha, beta,
                         experts=experts, scale_q4=sq, super_scale=sup)


@pytest.mark.parametrize("n,k,E", [(16, 128, 1), (48, 384, 3), (272, 640, 2), (1024, 8192, 1)])
def test_dequant_q4_bitexact(ccq, n, k, E):
    codes, sq, sup, a, b = synth.w2q4_format_random(n * E, k, 6000 + n + k)
    W = q4_weight(ccq, codes, sq, sup, a, b, experts=E)
    got = bits_of(ccq.ccq_dequant_bf16(W)).reshape(n * E, k)
    assert np.array_equal(got, oracle.dequant_w2q4(codes, sq, sup, a, b))


def test_dequant_q4_encoded_bitexact(ccq):
    w = synth.weights_normal(64, 512, 6001)
    codes, sq, sup, a, b, _ = ccq.ccq_encode_host_q4(w, 64)
    got = bits_of(ccq.ccq_dequant_bf16(q4_weight(ccq, codes, sq, sup, a, b)))[0]
    assert np.array_equal(got, oracle.dequant_w2q4(codes, sq, sup, a, b))


def test_gemm_q4_one_hot_identity_both_paths(ccq):
    n, k = 272, 640  # 5 scale bytes per row: odd, and a stage that ends inside the row
    codes, sq, sup, a, b = synth.w2q4_format_random(n, k, 6100)
    W = q4_weight(ccq, codes, sq, sup, a, b)
    ref = oracle.bf16_to_f64(oracle.dequant_w2q4(codes, sq, sup, a, b)).T.astype(np.float32)
    eye = synth.one_hot_rows(k).cuda()
    for j in range(0, k, 16):  # register-decode mma.sync kernel
        y = ccq.ccq_w2a16_gemm(W, eye[j:j + 16].contiguous()).float().cpu().numpy()
        assert np.array_equal(y, ref[j:j + 16]), j
    y = ccq.ccq_w2a16_gemm(W, eye).float().cpu().numpy()  # tcgen05 kernel
    assert np.array_equal(y, ref)


@pytest.mark.parametrize("m,n,k", [(1, 256, 512), (9, 272, 640), (16, 1024, 2048), (64, 512, 1024),
                                   (300, 272, 640), (1, 8192, 8192), (128, 8192, 8192)])
def test_gemm_q4_shapes(ccq, m, n, k):
    codes, sq, sup, a, b = synth.w2q4_format_random(n, k, 6200 + m + n)
    W = q4_weight(ccq, codes, sq, sup, a, b)
    x = synth.activations(m, k, 6201 + m)
    y = ccq.ccq_w2a16_gemm(W, x.cuda()).float().cpu().numpy()
    ref = oracle.gemm_f64(synth.bf16_bits(x), oracle.dequant_w2q4(codes, sq, sup, a, b))
    e = rel_err(y, ref)
    assert e <= TOL
    assert e <= 4e-3


@pytest.mark.parametrize("fmts", [("q4", "q4"), ("q4", "ccq"), ("ccq", "q4"), ("w4", "q4")])
@pytest.mark.parametrize("T", [6, 300])
def test_moe_q4_formats(ccq, fmts, T):
    E, H, I, topk = 8, 512, 256, 2
    W13, W2, d13, d2 = moe_weights_fmt(ccq, E, H, I, 6300 + T + 10 * FMT_SEED[fmts[0]] + FMT_SEED[fmts[1]], *fmts)
    x = synth.activations(T, H, 6301 + T)
    ids, rw = synth.routing_uniform(T, E, topk, 6302 + T)
    y, st = run_moe(ccq, W13, W2, x, ids, rw)
    assert st == ccq.CCQ_OK
    ref = oracle.moe_f64(synth.bf16_bits(x), d13, d2, ids, rw, round_h=True)
    assert rel_err(y, ref) <= TOL


# ----------------------------------------------------------------------------------------------
# device encoder: identical bytes to the host encoder and the oracle's brute-force Algorithm 1
# ----------------------------------------------------------------------------------------------
@pytest.mark.parametrize("n,k", [(6, 128), (33, 576), (64, 1024)])
def test_encode_device_matches_oracle(ccq, n, k):
    w = synth.weights_normal(n, k, 7000 + n + k)
    w[min(2, n - 1), 64:128] = 0.0  # an all-zero group
    wd = torch.from_numpy(w).cuda()
    for flags in (0, ccq.CCQ_ENC_LITERAL_EQ1, ccq.CCQ_ENC_REFIT_SCALE,
                  ccq.CCQ_ENC_LITERAL_EQ1 | ccq.CCQ_ENC_REFIT_SCALE):
        c, s, a, b = (t.cpu().numpy() for t in ccq.ccq_encode_device(wd, 64, flags))
        oc, os_, oa, ob = oracle.encode_w2(w, 64, flags)
        assert np.array_equal(a, oa) and np.array_equal(b, ob), flags
        assert np.array_equal(s, os_), flags
        assert np.array_equal(c, oc), flags


def test_encode_device_matches_host_at_size(ccq):
    # a full-width expert slice (the oracle's brute force is too slow here; the host encoder is
    # itself checked against the oracle): 256 rows of the decode layer's gate/up weight
    w = synth.weights_normal(256, 8192, 7100)
    c, s, a, b = (t.cpu().numpy() for t in ccq.ccq_encode_device(torch.from_numpy(w).cuda(), 64, 0))
    hc, hs, ha, hb, _ = ccq.ccq_encode_host(w, 64, 0)
    assert np.array_equal(a, ha) and np.array_equal(b, hb)
    assert np.array_equal(s, hs)
    assert np.array_equal(c, hc)


# ----------------------------------------------------------------------------------------------
# WINT2-Standard, the plain 2-bit comparison format of CCQ "Inference Performance", Table 4
# ----------------------------------------------------------------------------------------------
def std_weight(ccq, codes, scales, experts=1):
    n = codes.shape[0] // experts
    return ccq.CcqWeight(ccq.CCQ_FMT_W2_STD_G64, n, codes.shape[1] * 4, codes, scales, experts=experts)


@pytest.mark.parametrize("n,k,E", [(16, 64, 1), (48, 192, 3), (1024, 8192, 1)])
def test_dequant_std_bitexact(ccq, n, k, E):
    codes, scales = synth.std_format_random(n * E, k, 8000 + n + k)
    got = bits_of(ccq.ccq_dequant_bf16(std_weight(ccq, codes, scales, experts=E))).reshape(n * E, k)
    assert np.array_equal(got, oracle.dequant_w2std(codes, scales))


def test_quantize_std_device_matches_oracle(ccq):
    w = synth.weights_normal(40, 1088, 8100)
    # group 0 of row 0: amax 0.5, so s = 0.25, and every rounding tie (+-s/2, +-3s/2) and both clips
    w[0, :64] = np.resize(np.array([0.5, -0.5, 0.375, -0.375, 0.125, -0.125, 0.0, 0.25, -0.25, 0.4, -0.4],
                                   np.float32), 64)
    w[1, 64:128] = 0.0                                   # all-zero group: s = 0, levels 0
    w[2, 128:192] = np.float32(2.0 ** -149)              # amax/2 rounds to 0: s = 0
    # subnormal s = 2^-127, quotients k/16: ties at +-1/2 and +-3/2 among them
    w[3, 192:256] = np.float32(2.0 ** -131) * np.arange(-32, 32, dtype=np.float32)
    w[4, 256:320] *= 1e4                                 # large values
    c, sc = (t.cpu().numpy() for t in ccq.ccq_quantize_std_device(torch.from_numpy(w).cuda()))
    oc, osc = oracle.quantize_w2std(w)
    assert np.array_equal(sc, osc)
    assert np.array_equal(c, oc)


def test_gemm_std_one_hot_identity_both_paths(ccq):
    n, k = 272, 576
    codes, scales = synth.std_format_random(n, k, 8200)
    W = std_weight(ccq, codes, scales)
    ref = oracle.bf16_to_f64(oracle.dequant_w2std(codes, scales)).T.astype(np.float32)
    eye = synth.one_hot_rows(k).cuda()
    for j in range(0, k, 16):  # register-decode mma.sync kernel
        y = ccq.ccq_w2a16_gemm(W, eye[j:j + 16].contiguous()).float().cpu().numpy()
        assert np.array_equal(y, ref[j:j + 16]), j
    y = ccq.ccq_w2a16_gemm(W, eye).float().cpu().numpy()  # tcgen05 kernel
    assert np.array_equal(y, ref)


@pytest.mark.parametrize("m,n,k", [(1, 256, 512), (4, 1024, 4096), (9, 272, 576), (33, 256, 1088),
                                   (64, 512, 1024), (300, 272, 576), (1, 8192, 8192), (128, 8192, 8192)])
def test_gemm_std_shapes(ccq, m, n, k):
    codes, scales = synth.std_format_random(n, k, 8300 + m + n)
    W = std_weight(ccq, codes, scales)
    x = synth.activations(m, k, 8301 + m)
    y = ccq.ccq_w2a16_gemm(W, x.cuda()).float().cpu().numpy()
    ref = oracle.gemm_f64(synth.bf16_bits(x), oracle.dequant_w2std(codes, scales))
    e = rel_err(y, ref)
    assert e <= TOL
    assert e <= 4e-3


@pytest.mark.parametrize("fmts", [("std", "std"), ("std", "ccq"), ("ccq", "std"), ("w4", "std")])
@pytest.mark.parametrize("T", [6, 300])
def test_moe_std_formats(ccq, fmts, T):
    E, H, I, topk = 8, 512, 256, 2
    W13, W2, d13, d2 = moe_weights_fmt(ccq, E, H, I, 8400 + T + 10 * FMT_SEED[fmts[0]] + FMT_SEED[fmts[1]], *fmts)
    x = synth.activations(T, H, 8401 + T)
    ids, rw = synth.routing_uniform(T, E, topk, 8402 + T)
    y, st = run_moe(ccq, W13, W2, x, ids, rw)
    assert st == ccq.CCQ_OK
    ref = oracle.moe_f64(synth.bf16_bits(x), d13, d2, ids, rw, round_h=True)
    assert rel_err(y, ref) <= TOL


def test_moe_std_quantized_layer_matches_oracle(ccq):
    # weights through the device quantizer (not random codes), decode-sized fused path
    E, H, I, topk, T = 8, 1024, 512, 2, 16
    def q(rows, k, seed):
        w = synth.weights_normal(rows, k, seed)
        c, sc = (t.cpu().numpy() for t in ccq.ccq_quantize_std_device(torch.from_numpy(w).cuda()))
        return std_weight(ccq, c, sc, experts=E), oracle.dequant_w2std(c, sc)
    W13, d13 = q(E * 2 * I, H, 8500)
    W2, d2 = q(E * H, I, 8501)
    x = synth.activations(T, H, 8502)
    ids, rw = synth.routing_uniform(T, E, topk, 8503)
    y, st = run_moe(ccq, W13, W2, x, ids, rw)
    assert st == ccq.CCQ_OK
    ref = oracle.moe_f64(synth.bf16_bits(x), d13.reshape(E, 2 * I, H), d2.reshape(E, H, I), ids, rw, round_h=True)
    assert rel_err(y, ref) <= TOL


# ----------------------------------------------------------------------------------------------
# formats with the scale in the redundant bits (CCQ §3.5 Algorithm 2): (4,3,2) 2.75 bpw and
# hybrid (3,3,2)+(3,4,2) 2.5 bpw; decode-sized token counts run the register-decode kernel, larger
# ones the tcgen05 kernel
# ----------------------------------------------------------------------------------------------
def emb_weight(ccq, kind, codes, sup, experts=1):
    fmt = ccq.CCQ_FMT_W275_432 if kind == 1 else ccq.CCQ_FMT_W25_HYBRID
    n = codes.shape[0] // experts
    k = codes.shape[1] // (22 if kind == 1 else 20) * 64
    return ccq.CcqWeight(fmt, n, k, codes, None, experts=experts, super_scale=sup)


def emb_oracle(kind, codes, sup):
    codes = np.ascontiguousarray(codes)
    return oracle.dequant_emb(kind, codes if kind == 1 else codes.view(np.uint16), sup)


@pytest.mark.parametrize("kind", [1, 2])
@pytest.mark.parametrize("n,k,E", [(16, 512, 1), (48, 1024, 3), (1024, 8192, 1)])
def test_dequant_emb_bitexact(ccq, kind, n, k, E):
    codes, sup = synth.emb_format_random(kind, n * E, k, 9000 + n + k + kind)
    got = bits_of(ccq.ccq_dequant_bf16(emb_weight(ccq, kind, codes, sup, experts=E))).reshape(n * E, k)
    assert np.array_equal(got, emb_oracle(kind, codes, sup))


@pytest.mark.parametrize("kind", [1, 2])
@pytest.mark.parametrize("n,k", [(6, 512), (33, 1024)])
def test_encode_emb_device_matches_oracle(ccq, kind, n, k):
    w = synth.weights_normal(n, k, 9100 + n + kind)
    w[min(2, n - 1)] = 0.0                       # an all-zero row (super scale 0)
    w[0, 64:128] = 0.0                           # an all-zero group
    fmt = ccq.CCQ_FMT_W275_432 if kind == 1 else ccq.CCQ_FMT_W25_HYBRID
    c, sup = (t.cpu().numpy() for t in ccq.ccq_encode_emb_device(fmt, torch.from_numpy(w).cuda()))
    oc, osup = oracle.encode_emb(kind, w)
    assert np.array_equal(sup, osup)
    assert np.array_equal(c if kind == 1 else c.view(np.uint16), oc)


@pytest.mark.parametrize("kind", [1, 2])
def test_gemm_emb_one_hot_identity(ccq, kind):
    n, k = 272, 1024
    codes, sup = synth.emb_format_random(kind, n, k, 9200 + kind)
    W = emb_weight(ccq, kind, codes, sup)
    ref = oracle.bf16_to_f64(emb_oracle(kind, codes, sup)).T.astype(np.float32)
    eye = synth.one_hot_rows(k).cuda()
    for j in range(0, 64, 16):  # 16 tokens: the register-decode kernel; all k rows: the tcgen05 kernel
        y = ccq.ccq_w2a16_gemm(W, eye[j:j + 16].contiguous()).float().cpu().numpy()
        assert np.array_equal(y, ref[j:j + 16]), j
    y = ccq.ccq_w2a16_gemm(W, eye).float().cpu().numpy()
    assert np.array_equal(y, ref)


@pytest.mark.parametrize("kind", [1, 2])
@pytest.mark.parametrize("m,n,k", [(1, 256, 512), (4, 1024, 4096), (33, 272, 1024), (128, 512, 1536),
                                   (300, 272, 1024), (1, 8192, 8192)])
def test_gemm_emb_shapes(ccq, kind, m, n, k):
    if kind == 1 and k % 512:
        k += 512 - k % 512
    codes, sup = synth.emb_format_random(kind, n, k, 9300 + m + n + kind)
    W = emb_weight(ccq, kind, codes, sup)
    x = synth.activations(m, k, 9301 + m)
    y = ccq.ccq_w2a16_gemm(W, x.cuda()).float().cpu().numpy()
    ref = oracle.gemm_f64(synth.bf16_bits(x), emb_oracle(kind, codes, sup))
    e = rel_err(y, ref)
    assert e <= TOL
    assert e <= 4e-3


@pytest.mark.parametrize("fmts", [("w275", "w275"), ("w25", "w25"), ("ccq", "w275"), ("w25", "ccq")])
@pytest.mark.parametrize("T", [6, 300])
def test_moe_emb_formats(ccq, fmts, T):
    E, H, I, topk = 8, 1024, 512, 2
    W13, W2, d13, d2 = moe_weights_fmt(ccq, E, H, I, 9400 + T + 10 * FMT_SEED[fmts[0]] + FMT_SEED[fmts[1]], *fmts)
    x = synth.activations(T, H, 9401 + T)
    ids, rw = synth.routing_uniform(T, E, topk, 9402 + T)
    y, st = run_moe(ccq, W13, W2, x, ids, rw)
    assert st == ccq.CCQ_OK
    ref = oracle.moe_f64(synth.bf16_bits(x), d13, d2, ids, rw, round_h=True)
    assert rel_err(y, ref) <= TOL


@pytest.mark.parametrize("kind", [1, 2])
def test_moe_emb_encoded_layer_matches_oracle(ccq, kind):
    # weights through the device encoder, decode-sized token count (the register-decode kernel)
    E, H, I, topk, T = 8, 1024, 512, 2, 16
    fmt = ccq.CCQ_FMT_W275_432 if kind == 1 else ccq.CCQ_FMT_W25_HYBRID

    def q(rows, k, seed):
        w = synth.weights_normal(rows, k, seed)
        c, sup = (t.cpu().numpy() for t in ccq.ccq_encode_emb_device(fmt, torch.from_numpy(w).cuda()))
        return emb_weight(ccq, kind, c, sup, experts=E), emb_oracle(kind, c, sup)

    W13, d13 = q(E * 2 * I, H, 9500 + kind)
    W2, d2 = q(E * H, I, 9510 + kind)
    x = synth.activations(T, H, 9502)
    ids, rw = synth.routing_uniform(T, E, topk, 9503)
    y, st = run_moe(ccq, W13, W2, x, ids, rw)
    assert st == ccq.CCQ_OK
    ref = oracle.moe_f64(synth.bf16_bits(x), d13.reshape(E, 2 * I, H), d2.reshape(E, H, I), ids, rw, round_h=True)
    assert rel_err(y, ref) <= TOL


@pytest.mark.parametrize("kind", [1, 2])
@pytest.mark.parametrize("m", [17, 32, 33, 40, 48, 57, 64])
def test_gemm_emb_path_boundary(ccq, kind, m):
    # up to 32 tokens the decode-sized kernel; from 33 one 128-token tile on the tcgen05 kernel
    n, k = 512, 1024
    codes, sup = synth.emb_format_random(kind, n, k, 9600 + m + kind)
    W = emb_weight(ccq, kind, codes, sup)
    x = synth.activations(m, k, 9601 + m)
    y = ccq.ccq_w2a16_gemm(W, x.cuda()).float().cpu().numpy()
    ref = oracle.gemm_f64(synth.bf16_bits(x), emb_oracle(kind, codes, sup))
    assert rel_err(y, ref) <= 4e-3


@pytest.mark.parametrize("fmts", [("w275", "w275"), ("w25", "w25")])
@pytest.mark.parametrize("T,zipf", [(48, False), (104, False), (112, False), (200, False), (240, True)])
def test_moe_emb_path_boundary(ccq, fmts, T, zipf):
    # 12 and 26 rows per expert on average (decode-sized kernel, some experts over one 32-token chunk
    # at 26), 28, 50 and 60 (tcgen05 kernel), with experts that span several chunks (and, under Zipf
    # routing, experts with none)
    E, H, I, topk = 8, 1024, 512, 2
    W13, W2, d13, d2 = moe_weights_fmt(ccq, E, H, I, 9700 + T + FMT_SEED[fmts[0]], *fmts)
    x = synth.activations(T, H, 9701 + T)
    if zipf:
        ids, rw = synth.routing_zipf(T, E, topk, 9702 + T, s=1.1)
    else:
        ids, rw = synth.routing_uniform(T, E, topk, 9702 + T)
    y, st = run_moe(ccq, W13, W2, x, ids, rw)
    assert st == ccq.CCQ_OK
    ref = oracle.moe_f64(synth.bf16_bits(x), d13, d2, ids, rw, round_h=True)
    assert rel_err(y, ref) <= TOL


# ----------------------------------------------------------------------------------------------
# failure detection: bounded waits give up, report, and leave the context usable
# ----------------------------------------------------------------------------------------------
@pytest.mark.parametrize("kind", [0, 1])
def test_bounded_wait_reports_timeout_and_context_survives(ccq, kind):
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    ccq.ccq_selftest_bounded_wait(ws, kind, limit_us=20000)
    assert ccq.ccq_check_device_error(ws) == ccq.CCQ_ERR_TIMEOUT
    assert ccq.ccq_check_device_error(ws) == ccq.CCQ_OK  # the check clears the word
    # the same context still computes exactly
    n, k = 256, 512
    codes, scales, a, b = synth.w2_format_random(n, k, 9900 + kind)
    W = w2_weight(ccq, codes, scales, a, b)
    eye = synth.one_hot_rows(k)[:16].contiguous().cuda()
    y = ccq.ccq_w2a16_gemm(W, eye).float().cpu().numpy()
    ref = oracle.bf16_to_f64(oracle.dequant_w2(codes, scales, a, b)).T.astype(np.float32)[:16]
    assert np.array_equal(y, ref)
