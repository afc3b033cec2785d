/*
 * CPU oracle for the CCQ WINT2 weight-only matmul and the MoE expert FFN built on it.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline
 * leg may load this library.  It shares no code, header, table or constant generator with the
 * CUDA path in extreme_bit_weight_b200/; it is written from the definitions in
 *   [CCQ]  "CCQ: Convolutional Code for Extreme Low-bit Quantization in LLMs" (arXiv 2507.07145)
 *   [WINT2] FastDeploy "WINT2 Quantization" documentation page
 *   [GPTQ] course lesson "GPTQ and AWQ" (E6.4), worked example and Part 2 specification
 * Everything is plain loops; floating point results are fp64 unless the definition fixes a
 * narrower type (the fp32 code-cluster FMA and the BF16 weight rounding).
 *
 * Parity pins for each function are in tests/test_oracle_pins.py.  One function is
 * "parity unpinned": the encode *quality* (MSE of the chosen codes) has no published number;
 * only its optimality (argmin) and round-trip properties are pinned.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <fenv.h>
#include <limits.h>

/* ------------------------------------------------------------------------------------------
 * Convolutional-code codebook, [CCQ] §3.1 "Definition of Convolutional Code Codebook", Fig. 1.
 *
 * A configuration (L, N, S): each state has L bits, a code covers N states, and each step to the
 * next state brings S new ("transition") bits while the state keeps L-S bits of its predecessor.
 * The stored code is the first state's L bits followed by the S transition bits of each later
 * step, so a code has T = L + (N-1)S bits (§3.1, the formula after Fig. 1).  The codebook row with
 * index `code` lists the N states that the code walks through.
 *
 * This builds the table by walking the state graph (state_{i+1} = (state_i << S | b) mod 2^L),
 * not by shifting windows out of the code: the two agree, and tests check that they do against
 * the shift lists printed in [CCQ] Table 1.
 * ------------------------------------------------------------------------------------------ */
int oracle_code_bits(int L, int N, int S) { return L + (N - 1) * S; }

int oracle_codebook(int L, int N, int S, int32_t *out /* [2^T][N] */)
{
    if (L <= 0 || N <= 0 || S <= 0 || S > L) return -1;
    int T = oracle_code_bits(L, N, S);
    if (T > 24) return -1;
    uint32_t ncodes = 1u << T, smask = (1u << L) - 1u, bmask = (1u << S) - 1u;
    for (uint32_t first = 0; first <= smask; ++first) {
        /* enumerate every sequence of N-1 transitions of S bits each */
        uint32_t ntrans = 1u << ((N - 1) * S);
        for (uint32_t tr = 0; tr < ntrans; ++tr) {
            uint32_t code = first;
            uint32_t state = first;
            int32_t states[64];
            states[0] = (int32_t)state;
            for (int i = 1; i < N; ++i) {
                /* transition bits in the order they are stored: earliest step first */
                uint32_t b = (tr >> ((N - 1 - i) * S)) & bmask;
                state = ((state << S) | b) & smask;
                states[i] = (int32_t)state;
                code = (code << S) | b;
            }
            if (code >= ncodes) return -2;
            for (int i = 0; i < N; ++i) out[(size_t)code * N + i] = states[i];
        }
    }
    return 0;
}

/* ------------------------------------------------------------------------------------------
 * BF16 round-to-nearest-even from fp32 (IEEE-754 binary32 -> bfloat16: keep the top 16 bits,
 * rounding the dropped 16 with ties to even; NaN stays NaN).
 * ------------------------------------------------------------------------------------------ */
uint16_t oracle_bf16_bits(float x)
{
    uint32_t u;
    memcpy(&u, &x, 4);
    if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu)) return (uint16_t)((u >> 16) | 0x0040u);
    uint32_t lower = u & 0xFFFFu;
    uint32_t upper = u >> 16;
    if (lower > 0x8000u || (lower == 0x8000u && (upper & 1u))) upper += 1u;
    return (uint16_t)upper;
}

float oracle_bf16_to_float(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* ------------------------------------------------------------------------------------------
 * Code-cluster decode of one stored byte, [CCQ] §3.3 Eq. 1 and §3.5 Algorithm 3
 * ("Dequantization with Code Cluster"): the byte q (read as unsigned, "UINT8" in §3.3) is
 * mapped back to a convolutional code by round(q * s_code + zp_code).  Readings: the product and
 * sum are one fp32 fused multiply-add (fmaf), and round is to nearest with ties to even.
 * ------------------------------------------------------------------------------------------ */
int32_t oracle_cluster_code(uint8_t q, float code_scale, float code_zero)
{
    float t = fmaf((float)q, code_scale, code_zero);
    /* Outside the int32 range (never produced by an encoder) the rounded value saturates to the
     * nearest int32 and NaN gives 0; only the low 15 bits of the code are used afterwards. */
    if (!(t == t)) return 0;
    if (t >= 2147483648.0f) return INT32_MAX;
    if (t < -2147483648.0f) return INT32_MIN;
    int old = fegetround();
    fesetround(FE_TONEAREST);
    float r = nearbyintf(t);
    fesetround(old);
    return (int32_t)r;
}

/* ------------------------------------------------------------------------------------------
 * W2 dequantization, (L,N,S) = (6,4,3) with code cluster, group size g, [CCQ] §3.5 Algorithm 3
 * and Table 1 row (6,4,3).
 *
 * Layout ([WINT2]: four weights per 8-bit storage element; [CCQ] Algorithm 1 reshape to groups
 * of g/N vectors of N): codes[n][k/4], byte j of row n holds weights k = 4j .. 4j+3, one (6,4,3)
 * code of 4 states; scales[n][k/g]; code_scale[n], code_zero[n] per output channel (§3.3
 * clusters the codes channel by channel).
 *
 * Per weight: C = cluster code of the byte; the codebook row of C (reduced mod 2^15, since the
 * state windows only cover the low T bits) gives the 4 states u_0..u_3; the weight is
 * (u_i - zp) * s with zp = 32 (the midpoint of the 6-bit state range: reading of the unnamed
 * zero-point) and s = bf16(scale), and the product is rounded once to BF16 ([WINT2]: weights are
 * decoded to BF16).  (u - 32) * bf16(s) is exact in fp64, so there is exactly one rounding.
 * Output: BF16 bit patterns, [n][k].
 * ------------------------------------------------------------------------------------------ */
static int32_t *g_cb643 = NULL;

static const int32_t *codebook_643(void)
{
    if (!g_cb643) {
        int32_t *cb = (int32_t *)malloc(sizeof(int32_t) * 4 * 32768);
        if (!cb) return NULL;
        if (oracle_codebook(6, 4, 3, cb) != 0) { free(cb); return NULL; }
        g_cb643 = cb;
    }
    return g_cb643;
}

static uint16_t dequant_state(int32_t u, float scale)
{
    double s = (double)oracle_bf16_to_float(oracle_bf16_bits(scale));
    double w = (double)(u - 32) * s; /* exact: 6-bit integer times 8-bit significand */
    return oracle_bf16_bits((float)w);
}

int oracle_dequant_w2(const uint8_t *codes, const float *scales, const float *code_scale,
                      const float *code_zero, int n, int k, int group, uint16_t *out)
{
    const int32_t *cb = codebook_643();
    if (!cb || n < 0 || k < 0 || group <= 0 || k % 4 || k % group) return -1;
    int ng = k / group;
#pragma omp parallel for schedule(static)
    for (int r = 0; r < n; ++r) {
        for (int kk = 0; kk < k; ++kk) {
            uint8_t q = codes[(size_t)r * (k / 4) + kk / 4];
            int32_t C = oracle_cluster_code(q, code_scale[r], code_zero[r]);
            uint32_t idx = ((uint32_t)C) & 0x7FFFu;
            int32_t u = cb[(size_t)idx * 4 + (kk % 4)];
            out[(size_t)r * k + kk] = dequant_state(u, scales[(size_t)r * ng + kk / group]);
        }
    }
    return 0;
}

/* ------------------------------------------------------------------------------------------
 * 4-bit group scales, [CCQ] §3.4 "Scale Compression" and §3.5 Algorithm 3 (first line):
 * s = ((s_q >> s_shift) & s_mask) * s_super, s_mask = 0xF for (6,4,3) (Table 1), one fp32 super
 * scale per output channel.  Storage (the pages fix only the formula; reading): two 4-bit group
 * scales per byte, scale_q4[n][ceil(k/g / 2)], group G in byte G/2, the low nibble holding the even
 * group (s_shift = 4 * (G mod 2)).  The group scale is the fp32 product q4 * s_super; the weight
 * rule is then the one above, w = bf16((u - 32) * bf16(s)).
 * ------------------------------------------------------------------------------------------ */
static float q4_group_scale(const uint8_t *sq_row, float super, int G)
{
    int q = (sq_row[G >> 1] >> (4 * (G & 1))) & 0xF;
    return (float)q * super; /* one fp32 multiply (the file is built without contraction) */
}

int oracle_dequant_w2q4(const uint8_t *codes, const uint8_t *scale_q4, const float *super,
                        const float *code_scale, const float *code_zero, int n, int k, int group,
                        uint16_t *out)
{
    const int32_t *cb = codebook_643();
    if (!cb || n < 0 || k < 0 || group <= 0 || k % 4 || k % group) return -1;
    int ng = k / group, nb = (ng + 1) / 2;
#pragma omp parallel for schedule(static)
    for (int r = 0; r < n; ++r) {
        for (int kk = 0; kk < k; ++kk) {
            uint8_t q = codes[(size_t)r * (k / 4) + kk / 4];
            int32_t C = oracle_cluster_code(q, code_scale[r], code_zero[r]);
            uint32_t idx = ((uint32_t)C) & 0x7FFFu;
            int32_t u = cb[(size_t)idx * 4 + (kk % 4)];
            float s = q4_group_scale(scale_q4 + (size_t)r * nb, super[r], kk / group);
            out[(size_t)r * k + kk] = dequant_state(u, s);
        }
    }
    return 0;
}

/* ------------------------------------------------------------------------------------------
 * "WINT2-Standard": plain 2-bit scalar weights, the comparison format of [CCQ] Table 4 (the pages
 * compare against it but do not define it; reading): codes[n][k/4], field i of byte j (bits 2i,
 * 2i+1) is weight 4j+i, level q - 2 (zero-point 2 = 2^(bits-1), as the CCQ format's 32 = 2^(L-1)),
 * group scales scales[n][k/64] used as bf16: w = bf16((q - 2) * bf16(s)).
 * Quantizer (round to nearest): s = bf16(max|w_g| / 2), q = clip(round_half_even(w / s) + 2, 0, 3)
 * in fp64 (q = 2 when s = 0).
 * ------------------------------------------------------------------------------------------ */
static uint16_t dequant_std_level(int q, float scale)
{
    double s = (double)oracle_bf16_to_float(oracle_bf16_bits(scale));
    return oracle_bf16_bits((float)((double)(q - 2) * s)); /* exact product, one rounding */
}

int oracle_dequant_w2std(const uint8_t *codes, const float *scales, int n, int k, int group, uint16_t *out)
{
    if (n < 0 || k < 0 || group <= 0 || k % 4 || k % group) return -1;
    int ng = k / group;
#pragma omp parallel for schedule(static)
    for (int r = 0; r < n; ++r)
        for (int kk = 0; kk < k; ++kk) {
            int q = (codes[(size_t)r * (k / 4) + kk / 4] >> (2 * (kk % 4))) & 3;
            out[(size_t)r * k + kk] = dequant_std_level(q, scales[(size_t)r * ng + kk / group]);
        }
    return 0;
}

int oracle_quantize_w2std(const float *w, int n, int k, int group, uint8_t *codes, float *scales)
{
    if (n < 0 || k <= 0 || group <= 0 || k % 4 || k % group) return -1;
    int ng = k / group;
#pragma omp parallel for schedule(static)
    for (int r = 0; r < n; ++r) {
        int old = fegetround();
        fesetround(FE_TONEAREST);
        for (int g = 0; g < ng; ++g) {
            double amax = 0.0;
            for (int i = 0; i < group; ++i) {
                double a = fabs((double)w[(size_t)r * k + g * group + i]);
                if (a > amax) amax = a;
            }
            float s = oracle_bf16_to_float(oracle_bf16_bits((float)(amax / 2.0)));
            scales[(size_t)r * ng + g] = s;
            for (int i = 0; i < group; i += 4) {
                uint8_t byte = 0;
                for (int t = 0; t < 4; ++t) {
                    double v = s > 0.0f ? (double)w[(size_t)r * k + g * group + i + t] / (double)s : 0.0;
                    double q = nearbyint(v) + 2.0;
                    if (q < 0.0) q = 0.0;
                    if (q > 3.0) q = 3.0;
                    byte |= (uint8_t)((int)q << (2 * t));
                }
                codes[(size_t)r * (k / 4) + (g * group + i) / 4] = byte;
            }
        }
        fesetround(old);
    }
    return 0;
}

/* ------------------------------------------------------------------------------------------
 * Formats without code cluster whose group scale sits in the group's redundant bits: [CCQ] §3.2
 * "Hybrid Encoding", §3.4 "Scale Compression" (redundant bits; Eq. 5, first case), §3.5
 * Algorithm 2 ("Dequantization without Code Cluster"), Table 1 rows (4,3,2) and (3,3,2)(3,4,2).
 *
 * kind 1, (L,N,S) = (4,3,2), 2.75 bpw.  A group of 64 weights is 22 one-byte codes W_q[0..21].
 *   Code j < 21 covers weights 3j..3j+2 (its 3 states; Table 1 shifts [4,2,0], mask 0xF).  The
 *   last code covers weight 63 with its first state (its top 4 bits); its low 4 bits, redundant
 *   for the weights, hold the group's 4-bit scale (s_mask 0xF).  codes[n][k/64 * 22].
 * kind 2, hybrid (3,3,2)+(3,4,2), 2.5 bpw.  A group is ten 16-bit words W_q[0..9] (uint16,
 *   codes[n][k/64 * 10]).  Word j < 9 covers weights 7j..7j+6: a (3,3,2) code in its top 7 bits
 *   (states at shifts 13, 11, 9) then a (3,4,2) code in its low 9 bits (shifts 6, 4, 2, 0); Table
 *   1 mask 0x7.  The last word covers weight 63 with its top 3 bits and holds a 13-bit scale in
 *   its low 13 bits (s_mask 0x1FFF).
 * Decode (Algorithm 2): s = (last code & s_mask) * s_super[n], one fp32 multiply (reading, as for
 * the code-cluster format's 4-bit scales); w = bf16((u - zp) * bf16(s)) with zp = 2^(L-1), 8 and
 * 4 (reading, as CCQ's 32).  The states come from the codebooks built by walking the state graph.
 * ------------------------------------------------------------------------------------------ */
static int32_t *g_cb432 = NULL, *g_cb332 = NULL, *g_cb342 = NULL;

static int emb_codebooks(void)
{
    if (!g_cb432) {
        int32_t *a = (int32_t *)malloc(sizeof(int32_t) * 256 * 3);
        int32_t *b = (int32_t *)malloc(sizeof(int32_t) * 128 * 3);
        int32_t *c = (int32_t *)malloc(sizeof(int32_t) * 512 * 4);
        if (!a || !b || !c || oracle_codebook(4, 3, 2, a) || oracle_codebook(3, 3, 2, b) ||
            oracle_codebook(3, 4, 2, c)) {
            free(a); free(b); free(c);
            return -1;
        }
        g_cb332 = b;
        g_cb342 = c;
        g_cb432 = a;
    }
    return 0;
}

/* words per group, scale mask, zero-point, raw-scale divisor 2^(L-1) - 1 */
static int emb_words(int kind) { return kind == 1 ? 22 : 10; }
static uint32_t emb_smask(int kind) { return kind == 1 ? 0xFu : 0x1FFFu; }
static int emb_zp(int kind) { return kind == 1 ? 8 : 4; }

/* state of weight i (0..63) of a group whose codes are W[0..words) */
static int32_t emb_state(int kind, const uint32_t *W, int i)
{
    if (kind == 1) return g_cb432[(size_t)W[i / 3] * 3 + i % 3];
    uint32_t word = W[i / 7];
    int t = i % 7;
    return t < 3 ? g_cb332[(size_t)(word >> 9) * 3 + t] : g_cb342[(size_t)(word & 0x1FFu) * 4 + (t - 3)];
}

static double emb_level(int32_t u, int zp, float s_bf16)
{
    return (double)oracle_bf16_to_float(oracle_bf16_bits((float)((double)(u - zp) * (double)s_bf16)));
}

static void emb_load_group(int kind, const void *codes, size_t row, int nwords_row, int g, uint32_t *W)
{
    int nw = emb_words(kind);
    for (int j = 0; j < nw; ++j) {
        size_t at = row * (size_t)nwords_row + (size_t)g * nw + j;
        W[j] = kind == 1 ? ((const uint8_t *)codes)[at] : ((const uint16_t *)codes)[at];
    }
}

int oracle_dequant_emb(int kind, const void *codes, const float *super, int n, int k, uint16_t *out)
{
    if ((kind != 1 && kind != 2) || emb_codebooks() || n < 0 || k < 0 || k % 64) return -1;
    int ng = k / 64, nw = emb_words(kind), zp = emb_zp(kind);
#pragma omp parallel for schedule(static)
    for (int r = 0; r < n; ++r)
        for (int g = 0; g < ng; ++g) {
            uint32_t W[22];
            emb_load_group(kind, codes, (size_t)r, ng * nw, g, W);
            float s = (float)(W[nw - 1] & emb_smask(kind)) * super[r];
            float sb = oracle_bf16_to_float(oracle_bf16_bits(s));
            for (int i = 0; i < 64; ++i)
                out[(size_t)r * k + (size_t)g * 64 + i] =
                    oracle_bf16_bits((float)emb_level(emb_state(kind, W, i), zp, sb));
        }
    return 0;
}

/* Encoder (the pages print none for these formats; plain reading of Algorithm 1 and §3.4):
 * raw group scale r_g = max|w_g| / (2^(L-1) - 1) (fp32: 7 or 3); s_super = max_g r_g / (2^b - 1)
 * (fp32; b = 4 or 13 scale bits); q_g = clip(round-half-even(r_g / s_super), 0, 2^b - 1) in fp64
 * (0 when s_super = 0); the group scale is fl32(q_g * s_super).  Each full code is the one, over all
 * codes of its width, whose decoded weights have the least squared error to the group's weights
 * (ties to the smallest code); the last code's weight state is chosen the same way over its 2^L
 * values, and its low bits are q_g. */
int oracle_encode_emb(int kind, const float *w, int n, int k, void *codes, float *super)
{
    if ((kind != 1 && kind != 2) || emb_codebooks() || n < 0 || k <= 0 || k % 64) return -1;
    int ng = k / 64, nw = emb_words(kind), zp = emb_zp(kind);
    int L = kind == 1 ? 4 : 3;
    double rdiv = kind == 1 ? 7.0 : 3.0, qmax = (double)emb_smask(kind);
#pragma omp parallel for schedule(static)
    for (int r = 0; r < n; ++r) {
        const float *wr = w + (size_t)r * k;
        float *raw = (float *)malloc(sizeof(float) * (size_t)ng);
        if (!raw) continue;
        double smax = 0.0;
        for (int g = 0; g < ng; ++g) {
            double amax = 0.0;
            for (int i = 0; i < 64; ++i) {
                double a = fabs((double)wr[g * 64 + i]);
                if (a > amax) amax = a;
            }
            raw[g] = (float)(amax / rdiv);
            if ((double)raw[g] > smax) smax = (double)raw[g];
        }
        float sup = (float)(smax / qmax);
        super[r] = sup;
        int old = fegetround();
        fesetround(FE_TONEAREST);
        for (int g = 0; g < ng; ++g) {
            double qq = sup > 0.0f ? nearbyint((double)raw[g] / (double)sup) : 0.0;
            if (qq < 0.0) qq = 0.0;
            if (qq > qmax) qq = qmax;
            uint32_t q = (uint32_t)qq;
            float sb = oracle_bf16_to_float(oracle_bf16_bits((float)q * sup));
            const float *v = wr + g * 64;
            uint32_t W[22];
            if (kind == 1) {
                for (int j = 0; j < 21; ++j) {
                    double best = INFINITY;
                    uint32_t bc = 0;
                    for (uint32_t c = 0; c < 256; ++c) {
                        double e = 0.0;
                        for (int t = 0; t < 3; ++t) {
                            double d = (double)v[3 * j + t] - emb_level(g_cb432[c * 3 + t], zp, sb);
                            e += d * d;
                        }
                        if (e < best) { best = e; bc = c; }
                    }
                    W[j] = bc;
                }
            } else {
                for (int j = 0; j < 9; ++j) {
                    double best = INFINITY;
                    uint32_t b7 = 0, b9 = 0;
                    for (uint32_t c = 0; c < 128; ++c) {
                        double e = 0.0;
                        for (int t = 0; t < 3; ++t) {
                            double d = (double)v[7 * j + t] - emb_level(g_cb332[c * 3 + t], zp, sb);
                            e += d * d;
                        }
                        if (e < best) { best = e; b7 = c; }
                    }
                    best = INFINITY;
                    for (uint32_t c = 0; c < 512; ++c) {
                        double e = 0.0;
                        for (int t = 0; t < 4; ++t) {
                            double d = (double)v[7 * j + 3 + t] - emb_level(g_cb342[c * 4 + t], zp, sb);
                            e += d * d;
                        }
                        if (e < best) { best = e; b9 = c; }
                    }
                    W[j] = (b7 << 9) | b9;
                }
            }
            /* the last code: weight 63 in its top L bits, the scale in the rest */
            double best = INFINITY;
            uint32_t bu = 0;
            for (uint32_t u = 0; u < (1u << L); ++u) {
                double d = (double)v[63] - emb_level((int32_t)u, zp, sb);
                if (d * d < best) { best = d * d; bu = u; }
            }
            W[nw - 1] = (bu << (kind == 1 ? 4 : 13)) | q;
            for (int j = 0; j < nw; ++j) {
                size_t at = (size_t)r * ng * nw + (size_t)g * nw + j;
                if (kind == 1) ((uint8_t *)codes)[at] = (uint8_t)W[j];
                else ((uint16_t *)codes)[at] = (uint16_t)W[j];
            }
        }
        fesetround(old);
        free(raw);
    }
    return 0;
}

/* ------------------------------------------------------------------------------------------
 * W4 per-channel dequantization ([WINT2] quantization_config "wint4", "per_channel"; [GPTQ]
 * Part 2 pack_int4/unpack_int4): codes[n][k/2], two signed 4-bit codes per byte, the first code
 * of a pair in the low nibble; the code is sign-extended; w = bf16(q * bf16(scale[n])).
 * ------------------------------------------------------------------------------------------ */
int oracle_dequant_w4(const uint8_t *codes, const float *scales, int n, int k, uint16_t *out)
{
    if (n < 0 || k < 0 || k % 2) return -1;
    for (int r = 0; r < n; ++r) {
        double s = (double)oracle_bf16_to_float(oracle_bf16_bits(scales[r]));
        for (int kk = 0; kk < k; ++kk) {
            uint8_t b = codes[(size_t)r * (k / 2) + kk / 2];
            int nib = (kk % 2 == 0) ? (b & 0xF) : (b >> 4);
            int q = nib >= 8 ? nib - 16 : nib;
            out[(size_t)r * k + kk] = oracle_bf16_bits((float)((double)q * s));
        }
    }
    return 0;
}

/* ------------------------------------------------------------------------------------------
 * Dense product over decoded weights: y[m][n] = sum_k x[m][k] * w[n][k], fp64, plain loops.
 * x and w are BF16 bit patterns ([WINT2]: activations BF16, weights decoded to BF16).
 * ------------------------------------------------------------------------------------------ */
void oracle_gemm_bf16_f64(const uint16_t *x, const uint16_t *w, int m, int n, int k, double *y)
{
#pragma omp parallel for collapse(2) schedule(static)
    for (int i = 0; i < m; ++i)
        for (int j = 0; j < n; ++j) {
            double acc = 0.0;
            for (int kk = 0; kk < k; ++kk)
                acc += (double)oracle_bf16_to_float(x[(size_t)i * k + kk]) *
                       (double)oracle_bf16_to_float(w[(size_t)j * k + kk]);
            y[(size_t)i * n + j] = acc;
        }
}

/* ------------------------------------------------------------------------------------------
 * MoE expert FFN for one token set, fp64.  For token t with experts e_j and routing weights r_j
 * (j < topk): g = x_t W_gate(e)^T, u = x_t W_up(e)^T, h = SiLU(g) * u with SiLU(z) = z/(1+e^-z),
 * y_t = sum_j r_j * (h W_down(e)^T).  The gate/up weights of expert e are rows [0, I) and
 * [I, 2I) of its decoded W13 ([E][2I][H]); W_down is [E][H][I].  Routing weights are used as
 * given.  round_h != 0 rounds h to BF16 before the down projection (the activation the GPU path
 * stores); 0 keeps fp64.
 * Weights come in decoded BF16 bit form (from oracle_dequant_*), so any weight format works.
 * Invalid expert ids (outside [0, E)) contribute nothing to their token.
 * ------------------------------------------------------------------------------------------ */
static void expert_ffn_token(const uint16_t *xt, int H, int I, const uint16_t *wg, const uint16_t *wu,
                             const uint16_t *wd, int round_h, double *h, double *out /* [H] */)
{
    for (int i = 0; i < I; ++i) {
        double g = 0.0, u = 0.0;
        for (int c = 0; c < H; ++c) {
            double xv = (double)oracle_bf16_to_float(xt[c]);
            g += xv * (double)oracle_bf16_to_float(wg[(size_t)i * H + c]);
            u += xv * (double)oracle_bf16_to_float(wu[(size_t)i * H + c]);
        }
        double hv = g / (1.0 + exp(-g)) * u;
        if (round_h) hv = (double)oracle_bf16_to_float(oracle_bf16_bits((float)hv));
        h[i] = hv;
    }
    for (int c = 0; c < H; ++c) {
        double acc = 0.0;
        for (int i = 0; i < I; ++i) acc += h[i] * (double)oracle_bf16_to_float(wd[(size_t)c * I + i]);
        out[c] = acc;
    }
}

/* One expert's FFN (no routing weight) for T tokens: out[t] = SiLU(x_t Wg^T) * (x_t Wu^T) Wd^T. */
int oracle_expert_ffn_f64(const uint16_t *x /* [T][H] */, int T, int H, int I,
                          const uint16_t *w13 /* [2I][H] */, const uint16_t *w2 /* [H][I] */,
                          int round_h, double *out /* [T][H] */)
{
    int fail = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : fail)
    for (int t = 0; t < T; ++t) {
        double *h = (double *)malloc(sizeof(double) * (size_t)I);
        if (!h) { fail = 1; continue; }
        expert_ffn_token(x + (size_t)t * H, H, I, w13, w13 + (size_t)I * H, w2, round_h, h, out + (size_t)t * H);
        free(h);
    }
    return fail ? -1 : 0;
}

int oracle_moe_f64(const uint16_t *x /* [T][H] */, int T, int H, int I, int E,
                   const uint16_t *w13 /* [E][2I][H] */, const uint16_t *w2 /* [E][H][I] */,
                   const int32_t *ids /* [T][topk] */, const float *rw /* [T][topk] */, int topk,
                   int round_h, double *y /* [T][H] */)
{
    int fail = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : fail)
    for (int t = 0; t < T; ++t) {
        double *h = (double *)malloc(sizeof(double) * (size_t)I);
        double *o = (double *)malloc(sizeof(double) * (size_t)H);
        if (!h || !o) { free(h); free(o); fail = 1; continue; }
        for (int c = 0; c < H; ++c) y[(size_t)t * H + c] = 0.0;
        for (int j = 0; j < topk; ++j) {
            int e = ids[(size_t)t * topk + j];
            if (e < 0 || e >= E) continue;
            double r = (double)rw[(size_t)t * topk + j];
            const uint16_t *wg = w13 + (size_t)e * 2 * I * H;
            expert_ffn_token(x + (size_t)t * H, H, I, wg, wg + (size_t)I * H, w2 + (size_t)e * H * I,
                             round_h, h, o);
            for (int c = 0; c < H; ++c) y[(size_t)t * H + c] += r * o[c];
        }
        free(h);
        free(o);
    }
    return fail ? -1 : 0;
}

/* ------------------------------------------------------------------------------------------
 * Encoder, [CCQ] §3.1 Algorithm 1 "Convolutional Code Quantization", then §3.3 code cluster
 * (Eq. 1), then optionally §3.4 scale optimisation (Eq. 2-4).
 *
 * Steps, for the (6,4,3) configuration, group size g (g % 4 == 0), zero-point 32:
 *  1. group scale (Algorithm 1 line "group scale <- W_g", formula not given; reading):
 *     s = bf16(max|w| / 31) over the group, so the largest magnitude lands on level +31.
 *  2. argmin over all 2^15 codebook rows: the code C whose states u_0..u_3 minimise
 *     sum_i (v_i - D(u_i))^2, D(u) = bf16((u-32)*s) the dequantized value (the codebook scaled by
 *     the group scale, Algorithm 1); the sum is fp64 taken in order i = 0..3; ties go to the
 *     smallest C.
 *  3. per output channel: code zero-point beta = min C, code scale alpha = (max C - min C)/255
 *     as an fp32 division (1 when max == min), Eq. 1's asymmetric uniform quantizer of the code.
 *  4. cluster byte (reading of Eq. 1, which maps the searched code to 8 bits): by default the
 *     byte c in 0..255 whose cluster decode gives the smallest error for the vector ("retain only
 *     the frequently used encoding values", §3.3), ties to the smallest c; with flag LITERAL_EQ1,
 *     c = clamp(rint((C - beta)/alpha), 0, 255) computed in fp32.
 *  5. flag REFIT_SCALE: Eq. 4, s <- bf16(sum_i w_i q_i / sum_i q_i^2) over the group with
 *     q_i = u_i - 32 of the chosen bytes (skipped when the sum of squares is 0 or the result is
 *     not positive), then step 4 once more with the new scale.
 * The all-zero group has s = 0; every code then decodes to zero and the tie rule picks C = 0.
 * ------------------------------------------------------------------------------------------ */
#define ORACLE_ENC_LITERAL_EQ1 1u
#define ORACLE_ENC_REFIT_SCALE 2u
/* 4-bit group scales (§3.4 "Scale Compression"; reading of the unstated quantizer): the raw group
 * scales s_g = absmax_g / 31 (fp32) give the channel's super scale s_super = max_g s_g / 15 (fp32)
 * and q4_g = round-half-even(s_g / s_super) in 0..15; the search then uses s_g' = q4_g * s_super.
 * The Eq. 4 refit does not apply (the scale is no longer free). */
#define ORACLE_ENC_Q4_SCALE 4u

static double vec_err(const float *v, const int32_t *st, const double *D)
{
    double e = 0.0;
    for (int i = 0; i < 4; ++i) {
        double d = (double)v[i] - D[st[i]];
        e += d * d;
    }
    return e;
}

static void level_table(float s, double *D)
{
    for (int u = 0; u < 64; ++u) D[u] = (double)oracle_bf16_to_float(dequant_state(u, s));
}

static uint8_t best_byte(const float *v, const double *D, const int32_t *cb, float alpha, float beta)
{
    double best = INFINITY;
    int arg = 0;
    for (int c = 0; c < 256; ++c) {
        int32_t C = oracle_cluster_code((uint8_t)c, alpha, beta);
        const int32_t *st = cb + (size_t)(((uint32_t)C) & 0x7FFFu) * 4;
        double e = vec_err(v, st, D);
        if (e < best) { best = e; arg = c; }
    }
    return (uint8_t)arg;
}

static void encode_row(const float *wr, int k, int group, uint32_t flags, const int32_t *cb,
                       int32_t *C, uint8_t *codes, float *scales, float *alpha, float *beta,
                       uint8_t *q4 /* [ng], Q4 only */, float *super /* Q4 only */)
{
    int ng = k / group, nv = k / 4;
    /* 1 (Q4): raw group scales, the channel's super scale and the 4-bit scale of each group */
    if (flags & ORACLE_ENC_Q4_SCALE) {
        double smax = 0.0;
        for (int g = 0; g < ng; ++g) {
            double amax = 0.0;
            for (int i = 0; i < group; ++i) {
                double a = fabs((double)wr[g * group + i]);
                if (a > amax) amax = a;
            }
            scales[g] = (float)(amax / 31.0);
            if ((double)scales[g] > smax) smax = (double)scales[g];
        }
        float sup = (float)(smax / 15.0);
        *super = sup;
        int old = fegetround();
        fesetround(FE_TONEAREST);
        for (int g = 0; g < ng; ++g) {
            double qq = sup > 0.0f ? nearbyint((double)scales[g] / (double)sup) : 0.0;
            if (qq < 0.0) qq = 0.0;
            if (qq > 15.0) qq = 15.0;
            q4[g] = (uint8_t)qq;
            scales[g] = (float)q4[g] * sup;
        }
        fesetround(old);
    }
    /* 1-2: group scale, then codebook search for every 4-vector */
    for (int g = 0; g < ng; ++g) {
        float s;
        if (flags & ORACLE_ENC_Q4_SCALE) {
            s = scales[g];
        } else {
            double amax = 0.0;
            for (int i = 0; i < group; ++i) {
                double a = fabs((double)wr[g * group + i]);
                if (a > amax) amax = a;
            }
            s = oracle_bf16_to_float(oracle_bf16_bits((float)(amax / 31.0)));
        }
        scales[g] = s;
        double D[64];
        level_table(s, D);
        for (int vq = 0; vq < group / 4; ++vq) {
            const float *v = wr + g * group + vq * 4;
            double best = INFINITY;
            int32_t arg = 0;
            for (int32_t code = 0; code < 32768; ++code) {
                double e = vec_err(v, cb + (size_t)code * 4, D);
                if (e < best) { best = e; arg = code; }
            }
            C[g * (group / 4) + vq] = arg;
        }
    }
    /* 3: per-channel code scale / zero-point */
    int32_t cmin = C[0], cmax = C[0];
    for (int j = 1; j < nv; ++j) {
        if (C[j] < cmin) cmin = C[j];
        if (C[j] > cmax) cmax = C[j];
    }
    float b = (float)cmin;
    float a = (cmax == cmin) ? 1.0f : (float)(cmax - cmin) / 255.0f;
    *alpha = a;
    *beta = b;
    /* 4: cluster byte per vector */
    for (int g = 0; g < ng; ++g) {
        double D[64];
        level_table(scales[g], D);
        for (int vq = 0; vq < group / 4; ++vq) {
            int j = g * (group / 4) + vq;
            const float *v = wr + (size_t)j * 4;
            uint8_t c;
            if (flags & ORACLE_ENC_LITERAL_EQ1) {
                float q = ((float)C[j] - b) / a;
                int old = fegetround();
                fesetround(FE_TONEAREST);
                float qr = nearbyintf(q);
                fesetround(old);
                if (qr < 0.0f) qr = 0.0f;
                if (qr > 255.0f) qr = 255.0f;
                c = (uint8_t)qr;
            } else {
                c = best_byte(v, D, cb, a, b);
            }
            codes[j] = c;
        }
        /* 5: Eq. 4 refit of this group's scale, then one more byte choice */
        if ((flags & ORACLE_ENC_REFIT_SCALE) && !(flags & ORACLE_ENC_Q4_SCALE)) {
            double num = 0.0, den = 0.0;
            for (int vq = 0; vq < group / 4; ++vq) {
                int j = g * (group / 4) + vq;
                int32_t Cq = oracle_cluster_code(codes[j], a, b);
                const int32_t *st = cb + (size_t)(((uint32_t)Cq) & 0x7FFFu) * 4;
                for (int i = 0; i < 4; ++i) {
                    double q = (double)(st[i] - 32);
                    num += (double)wr[(size_t)j * 4 + i] * q;
                    den += q * q;
                }
            }
            if (den > 0.0 && num / den > 0.0) {
                float s2 = oracle_bf16_to_float(oracle_bf16_bits((float)(num / den)));
                if (s2 > 0.0f) {
                    scales[g] = s2;
                    double D2[64];
                    level_table(s2, D2);
                    if (!(flags & ORACLE_ENC_LITERAL_EQ1))
                        for (int vq = 0; vq < group / 4; ++vq) {
                            int j = g * (group / 4) + vq;
                            codes[j] = best_byte(wr + (size_t)j * 4, D2, cb, a, b);
                        }
                }
            }
        }
    }
}

int oracle_encode_w2(const float *w, int n, int k, int group, uint32_t flags, uint8_t *codes,
                     float *scales, float *alpha, float *beta)
{
    const int32_t *cb = codebook_643();
    if (!cb || n < 0 || k <= 0 || group <= 0 || group % 4 || k % group) return -1;
    int ng = k / group, nv = k / 4;
    int fail = 0;
    /* rows are independent; the loop runs them on all host threads */
#pragma omp parallel for schedule(dynamic, 1) reduction(| : fail)
    for (int r = 0; r < n; ++r) {
        int32_t *C = (int32_t *)malloc(sizeof(int32_t) * (size_t)nv);
        if (!C) { fail = 1; continue; }
        encode_row(w + (size_t)r * k, k, group, flags & ~ORACLE_ENC_Q4_SCALE, cb, C, codes + (size_t)r * nv,
                   scales + (size_t)r * ng, alpha + r, beta + r, NULL, NULL);
        free(C);
    }
    return fail ? -1 : 0;
}

/* Encoder for the 4-bit scale format: codes, packed scale_q4[n][ceil(ng/2)] (even group in the
 * low nibble), super[n], alpha[n], beta[n].  flags: ORACLE_ENC_LITERAL_EQ1 only. */
int oracle_encode_w2q4(const float *w, int n, int k, int group, uint32_t flags, uint8_t *codes,
                       uint8_t *scale_q4, float *super, float *alpha, float *beta)
{
    const int32_t *cb = codebook_643();
    if (!cb || n < 0 || k <= 0 || group <= 0 || group % 4 || k % group) return -1;
    if (flags & ORACLE_ENC_REFIT_SCALE) return -1;
    int ng = k / group, nv = k / 4, nb = (ng + 1) / 2;
    int fail = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : fail)
    for (int r = 0; r < n; ++r) {
        int32_t *C = (int32_t *)malloc(sizeof(int32_t) * (size_t)nv);
        float *sc = (float *)malloc(sizeof(float) * (size_t)ng);
        uint8_t *q4 = (uint8_t *)malloc((size_t)ng);
        if (!C || !sc || !q4) { fail = 1; free(C); free(sc); free(q4); continue; }
        encode_row(w + (size_t)r * k, k, group, flags | ORACLE_ENC_Q4_SCALE, cb, C, codes + (size_t)r * nv, sc,
                   alpha + r, beta + r, q4, super + r);
        uint8_t *dst = scale_q4 + (size_t)r * nb;
        for (int b = 0; b < nb; ++b) dst[b] = 0;
        for (int g = 0; g < ng; ++g) dst[g >> 1] |= (uint8_t)(q4[g] << (4 * (g & 1)));
        free(C);
        free(sc);
        free(q4);
    }
    return fail ? -1 : 0;
}

/* Error of the encoded weights: sum over all weights of (w - decoded)^2, fp64. */
double oracle_w2_sq_error(const float *w, const uint8_t *codes, const float *scales, const float *alpha,
                          const float *beta, int n, int k, int group)
{
    uint16_t *d = (uint16_t *)malloc(sizeof(uint16_t) * (size_t)n * k);
    if (!d) return -1.0;
    if (oracle_dequant_w2(codes, scales, alpha, beta, n, k, group, d) != 0) { free(d); return -1.0; }
    double e = 0.0;
    for (size_t i = 0; i < (size_t)n * k; ++i) {
        double dd = (double)w[i] - (double)oracle_bf16_to_float(d[i]);
        e += dd * dd;
    }
    free(d);
    return e;
}

/* ------------------------------------------------------------------------------------------
 * W4 per-channel round-to-nearest ([GPTQ] Part 2 "rtn": clip(round(w/scale), -8, 7), np.round
 * ties to even; pack_int4 layout, first code in the low nibble).  Reading for the per-channel
 * scale (not printed anywhere): s = bf16(max|w_row| / 7).  w/s is taken in fp64.
 * ------------------------------------------------------------------------------------------ */
int oracle_quantize_w4(const float *w, int n, int k, uint8_t *codes, float *scales)
{
    if (n < 0 || k <= 0 || k % 2) return -1;
    for (int r = 0; r < n; ++r) {
        double amax = 0.0;
        for (int i = 0; i < k; ++i) {
            double a = fabs((double)w[(size_t)r * k + i]);
            if (a > amax) amax = a;
        }
        float s = oracle_bf16_to_float(oracle_bf16_bits((float)(amax / 7.0)));
        scales[r] = s;
        for (int i = 0; i < k; i += 2) {
            int q[2];
            for (int h = 0; h < 2; ++h) {
                double v = (s > 0.0f) ? (double)w[(size_t)r * k + i + h] / (double)s : 0.0;
                int old = fegetround();
                fesetround(FE_TONEAREST);
                double qr = nearbyint(v);
                fesetround(old);
                if (qr < -8.0) qr = -8.0;
                if (qr > 7.0) qr = 7.0;
                q[h] = (int)qr;
            }
            codes[(size_t)r * (k / 2) + i / 2] = (uint8_t)((q[0] & 0xF) | ((q[1] & 0xF) << 4));
        }
    }
    return 0;
}
