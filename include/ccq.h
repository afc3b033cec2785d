/*
 * ccq.h - C ABI of libccq.so: CCQ WINT2 (W2A16) weight-only matmul and MoE expert FFN on NVIDIA
 * B200 (sm_100a).
 *
 * The method is "CCQ: Convolutional Code for Extreme Low-bit Quantization in LLMs"
 * (arXiv 2507.07145), in the deployed form that FastDeploy's "WINT2 Quantization" page describes:
 * weights are stored offline as INT8 bytes holding four 2-bit-equivalent weights each, decoded to
 * BF16 in real time and multiplied against BF16 activations; activations are not quantized.
 *
 * Conventions for every entry point:
 *  - Pointers marked (device) are CUDA device pointers; (host) are ordinary host memory.  The
 *    caller owns every buffer.  The library keeps no state between calls and never allocates
 *    device memory; scratch space is the caller's workspace `ws` of `ws_bytes` bytes
 *    (size it with the matching *_workspace_size call; 256-byte alignment).
 *  - Device calls are asynchronous on `stream` (0 = legacy default stream).  Argument errors that
 *    the host can see (null pointers, shapes, alignment, workspace too small, unsupported format)
 *    are returned synchronously before anything is launched.  Errors only the device can see (an
 *    expert id outside [0, E), a repeated expert id within one token) set an error word in the
 *    workspace; the offending (token, slot) pair is skipped; ccq_check_device_error() reports it.
 *    No entry point traps, asserts, exits or throws.
 *  - BF16 tensors are raw 16-bit bfloat16 bit patterns, row-major.
 *  - Calls on different streams are independent when each has its own workspace.
 */
#ifndef CCQ_H
#define CCQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *ccq_stream_t; /* same object as cudaStream_t */

typedef enum {
    CCQ_OK = 0,
    CCQ_ERR_INVALID_ARG = 1,  /* bad pointer, shape, alignment or workspace size */
    CCQ_ERR_UNSUPPORTED = 2,  /* format or shape this build does not implement */
    CCQ_ERR_CUDA = 3,         /* a CUDA runtime call failed (launch, copy, attribute) */
    CCQ_ERR_DEVICE_CHECK = 4, /* the device recorded an invalid routing entry (see above) */
    CCQ_ERR_TIMEOUT = 5       /* a bounded device-side wait gave up */
} ccq_status;

/* Weight formats.
 * CCQ_FMT_W2_CCQ_G64: CCQ configuration (L,N,S) = (6,4,3) with code cluster, group size 64
 *   (CCQ §3.3 "Code Cluster"; §3.5 Table 1 row (6,4,3); Algorithm 3).  Per output row n:
 *     codes[n][k/4]  uint8, byte j holds weights k = 4j..4j+3 of row n;
 *     scales[n][k/64] fp32 group scales (used as bf16_rn(scale));
 *     alpha[n], beta[n] fp32 code scale / code zero-point of the channel.
 *   Decode of weight k of row n (byte q = codes[n][k/4], i = k mod 4, g = k/64):
 *     C = round_half_even(fmaf(q, alpha[n], beta[n]))         (Eq. 1 inverted, Algorithm 3)
 *     u = ((uint32)C >> (9 - 3i)) & 0x3F                      (Table 1 shifts [9,6,3,0], mask 0x3F)
 *     w = bf16_rn((u - 32) * bf16_rn(scales[n][g]))           (weight zero-point 32)
 *   The fast matmul kernels need every code in [0, 2^16): alpha >= 0, beta >= 0 and
 *   beta + 255*alpha < 65535 (the host encoder's output always has 0 <= C < 2^15).  Outside that
 *   domain their results are unspecified; ccq_dequant_bf16 is exact for any alpha/beta.
 * CCQ_FMT_W4_PER_CHANNEL: signed 4-bit codes -8..7, two per byte, first code of a pair in the low
 *   nibble ("GPTQ and AWQ" lesson, pack_int4 layout); one scale per output row
 *   (WINT2 page, quantization_config "wint4" / "per_channel"):
 *     codes[n][k/2] uint8, scales[n] fp32; w = bf16_rn(sext4(nibble) * bf16_rn(scales[n])).
 * CCQ_FMT_W2_CCQ_G64_Q4SCALE: the CCQ paper's 2.06-bpw form of CCQ_FMT_W2_CCQ_G64 (§3.4 "Scale
 *   Compression", Eq. 5, Algorithm 3 first line: s = ((s_q >> s_shift) & 0xF) * s_super).  The
 *   codes, alpha and beta are as for CCQ_FMT_W2_CCQ_G64; the group scales are 4-bit:
 *     scale_q4[n][k/128] uint8, group g in byte g/2, the low nibble holding the even group;
 *     super_scale[n] fp32;
 *     group scale s = fl32(q4 * super_scale[n]) (one fp32 multiply), then the same weight rule
 *     w = bf16_rn((u - 32) * bf16_rn(s)).  `scales` is unused (NULL).  k must be a multiple of 128.
 * CCQ_FMT_W2_STD_G64: "WINT2-Standard", the plain 2-bit scalar format the CCQ paper measures
 *   against (Inference Performance, Table 4; the paper does not define it, this is the plain
 *   reading).  Same storage as CCQ_FMT_W2_CCQ_G64 without alpha/beta (NULL):
 *     codes[n][k/4] uint8, bits 2i..2i+1 of byte j hold the level q of weight k = 4j + i;
 *     scales[n][k/64] fp32 group scales (used as bf16_rn(scale));
 *     w = bf16_rn((q - 2) * bf16_rn(scales[n][k/64]))          (levels -2, -1, 0, 1).
 * CCQ_FMT_W275_432 and CCQ_FMT_W25_HYBRID: the CCQ formats without code cluster whose group scale
 *   sits in the group's redundant bits (§3.2 "Hybrid Encoding", §3.4 "Scale Compression", §3.5
 *   Algorithm 2, Table 1 rows (4,3,2) and (3,3,2)(3,4,2)).  Per row: `codes` is the row's groups of
 *   64 weights back to back, and super_scale[n] is fp32; scales, alpha, beta, scale_q4 are unused.
 *   CCQ_FMT_W275_432, (L,N,S) = (4,3,2), 2.75 bpw: a group is 22 one-byte codes; code j < 21
 *     holds weights 3j..3j+2 as states (c >> 4) & 15, (c >> 2) & 15, c & 15; code 21 holds weight
 *     63 in its top nibble and the group's 4-bit scale q in its low nibble.  Zero-point 8.
 *     k must be a multiple of 512 (row pitch a multiple of 16 bytes).
 *   CCQ_FMT_W25_HYBRID, (3,3,2)+(3,4,2), 2.5 bpw: a group is ten little-endian 16-bit words; word
 *     j < 9 holds weights 7j..7j+6 as states (x >> 13, 11, 9, 6, 4, 2, 0) & 7; word 9 holds weight
 *     63 in its top 3 bits and the 13-bit scale q in its low 13 bits.  Zero-point 4.  k must be a
 *     multiple of 256.
 *   Weight: w = bf16_rn((u - zp) * bf16_rn(fl32(q * super_scale[n]))).
 *   They run on both matmul kernels, chosen by token count as for the other formats.
 */
enum {
    CCQ_FMT_W2_CCQ_G64 = 1,
    CCQ_FMT_W4_PER_CHANNEL = 2,
    CCQ_FMT_W2_CCQ_G64_Q4SCALE = 3,
    CCQ_FMT_W2_STD_G64 = 4,
    CCQ_FMT_W275_432 = 5,
    CCQ_FMT_W25_HYBRID = 6
};

/* One linear layer, or `num_experts` layers of the same shape stacked back to back: expert e's
 * arrays start at codes + e*n*(k/4) (W2) or e*n*(k/2) (W4), scales + e*n*(k/64) (W2) or e*n (W4),
 * alpha/beta/super_scale + e*n, scale_q4 + e*n*(k/128); for CCQ_FMT_W275_432 / CCQ_FMT_W25_HYBRID
 * codes + e*n*(k/64)*22 / 20.  All device pointers, 16-byte aligned.
 * y = x W^T: W is [n][k]. */
typedef struct {
    int32_t fmt;          /* CCQ_FMT_* */
    int32_t n;            /* output features (rows of W), multiple of 16 */
    int32_t k;            /* input features, multiple of 64 */
    int32_t group;        /* 64 for the W2 formats; ignored for W4 */
    const uint8_t *codes; /* (device) packed code stream */
    const float *scales;  /* (device) group scales (W2) or channel scales (W4) */
    const float *alpha;   /* (device) CCQ code scale per row; NULL for W4 and STD */
    const float *beta;    /* (device) CCQ code zero-point per row; NULL for W4 and STD */
    const uint8_t *scale_q4;   /* (device) Q4SCALE: packed 4-bit group scales; NULL otherwise */
    const float *super_scale;  /* (device) Q4SCALE: super scale per row; NULL otherwise */
} ccq_weight;

/* Encoder flags for ccq_encode_host. */
enum {
    CCQ_ENC_LITERAL_EQ1 = 1u,  /* cluster byte = clamp(rint((C - beta)/alpha), 0, 255) (Eq. 1 as printed) */
    CCQ_ENC_REFIT_SCALE = 2u   /* one Eq. 4 scale refit per group, then re-choose the bytes */
};

/* ccq_encode_host - offline CCQ (6,4,3) code-cluster quantization of one weight matrix on host
 * threads (CCQ §3.1 Algorithm 1, §3.3 Eq. 1, §3.4 Eq. 2-4).
 *   w       (host) fp32 [n][k], row-major; k % group == 0, group % 4 == 0
 *   group   group size (64 for the WINT2 format)
 *   flags   CCQ_ENC_* bits
 *   threads host threads to use (<= 0: all hardware threads)
 *   codes   (host) out uint8 [n][k/4];  scales (host) out fp32 [n][k/group] (BF16-representable)
 *   alpha, beta (host) out fp32 [n]
 *   sq_err  (host, may be NULL) out: sum of squared errors of the decoded weights
 * Per group: scale s = bf16(max|w|/31); each 4-vector takes the (6,4,3) code minimising the
 * squared error of its decoded values (trellis search, ties to the smallest code); per row
 * beta = min code, alpha = (max code - min code)/255 (1 if equal); each vector then takes the byte
 * 0..255 whose decoded values are closest (ties to the smallest byte), or the literal Eq. 1 byte.
 * Returns CCQ_ERR_INVALID_ARG on null pointers or bad shapes. */
ccq_status ccq_encode_host(const float *w, int32_t n, int32_t k, int32_t group, uint32_t flags,
                           int32_t threads, uint8_t *codes, float *scales, float *alpha, float *beta,
                           double *sq_err);

/* ccq_encode_device - ccq_encode_host on the GPU: the same algorithm (CCQ §3.1 Algorithm 1, §3.3
 * Eq. 1, §3.4 Eq. 4), the same fp64 arithmetic in the same order and the same tie rules, so the
 * outputs are identical to ccq_encode_host's for the same input and flags.
 *   w       (device) fp32 [n][k]; group must be 64 (CCQ_ERR_UNSUPPORTED otherwise), k % 64 == 0
 *   flags   CCQ_ENC_LITERAL_EQ1 and/or CCQ_ENC_REFIT_SCALE
 *   codes (device) out [n][k/4]; scales (device) out [n][k/64]; alpha, beta (device) out [n]
 *   ws      (device) scratch of ccq_encode_device_workspace_size(n, k) bytes
 * Asynchronous on `stream`; argument errors return before any launch.  No paper counterpart as an
 * interface: the paper encodes offline and does not say where. */
size_t ccq_encode_device_workspace_size(int32_t n, int32_t k);
ccq_status ccq_encode_device(const float *w, int32_t n, int32_t k, int32_t group, uint32_t flags,
                             uint8_t *codes, float *scales, float *alpha, float *beta, void *ws,
                             size_t ws_bytes, ccq_stream_t stream);

/* ccq_encode_host_q4 - ccq_encode_host for CCQ_FMT_W2_CCQ_G64_Q4SCALE (CCQ §3.4 "Scale
 * Compression"; the pages give no quantizer for the 4-bit scales, this is the plain reading):
 *   raw group scale r_g = max|w_g|/31 (fp32); super_scale[n] = max_g r_g / 15 (fp32);
 *   q4_g = clip(round_half_even(r_g / super), 0, 15) (in fp64); the codes are then searched and
 *   clustered exactly as by ccq_encode_host at the group scales fl32(q4_g * super).
 *   w (host) fp32 [n][k], k % 128 == 0 (group 64); flags: CCQ_ENC_LITERAL_EQ1 only (the Eq. 4
 *   refit does not apply to a quantized scale); codes (host) out [n][k/4]; scale_q4 (host) out
 *   [n][k/128]; super_scale, alpha, beta (host) out fp32 [n]; sq_err as for ccq_encode_host.
 * Returns CCQ_ERR_INVALID_ARG on null pointers, bad shapes or flags. */
ccq_status ccq_encode_host_q4(const float *w, int32_t n, int32_t k, int32_t group, uint32_t flags,
                              int32_t threads, uint8_t *codes, uint8_t *scale_q4, float *super_scale,
                              float *alpha, float *beta, double *sq_err);

/* ccq_quantize_std_device - round-to-nearest quantization to CCQ_FMT_W2_STD_G64 on the GPU (the
 * pages print no quantizer for WINT2-Standard; this is the plain one):
 *   per group of 64: s = bf16_rn(max|w| / 2); level q - 2 = clip(round_half_even(w / s), -2, 1),
 *   q = 2 where s == 0.  Decided by exact fp32 comparisons with s/2 and 3s/2 (both exact for a
 *   BF16 s), identical to the rounding of the exact quotient.
 *   w (device) fp32 [n][k], k % 64 == 0; codes (device) out [n][k/4]; scales (device) out
 *   [n][k/64] (BF16-representable).  Asynchronous on `stream`; argument errors (null pointers,
 *   bad shapes, misaligned pointers: all three 16-byte aligned) return before any launch. */
ccq_status ccq_quantize_std_device(const float *w, int32_t n, int32_t k, uint8_t *codes, float *scales,
                                   ccq_stream_t stream);

/* ccq_encode_emb_device - encoder for CCQ_FMT_W275_432 / CCQ_FMT_W25_HYBRID on the GPU (the pages
 * print no encoder for these formats; plain reading of Algorithm 1 and §3.4):
 *   raw group scale r_g = max|w_g| / (2^(L-1) - 1) (fp32; 7 or 3); super_scale[n] = max_g r_g /
 *   (2^b - 1) (fp32; b = 4 or 13 scale bits); q_g = clip(round_half_even(r_g / super), 0, 2^b - 1)
 *   in fp64 (0 when super is 0); group scale bf16(fl32(q_g * super)).  Every full code is the one,
 *   over all codes of its width, whose decoded weights have the least squared error (fp64, ties to
 *   the smallest code); the last code's state is the nearest level for weight 63.
 *   fmt    CCQ_FMT_W275_432 or CCQ_FMT_W25_HYBRID (else CCQ_ERR_UNSUPPORTED)
 *   w      (device) fp32 [n][k], k % 64 == 0;  codes (device) out [n][k/64 * (22 or 20) bytes];
 *   super_scale (device) out fp32 [n].  Asynchronous on `stream`; argument errors (null or
 *   misaligned pointers, bad shapes) return before any launch. */
ccq_status ccq_encode_emb_device(int32_t fmt, const float *w, int32_t n, int32_t k, uint8_t *codes,
                                 float *super_scale, ccq_stream_t stream);

/* ccq_quantize_w4_host - W4 per-channel round-to-nearest ("GPTQ and AWQ" Part 2 rtn/pack_int4):
 * s = bf16(max|w_row|/7), q = clip(round_half_even(w/s), -8, 7) (w/s in fp64), two codes per byte,
 * first in the low nibble.  w (host) fp32 [n][k], k even; codes (host) out [n][k/2]; scales (host)
 * out [n]. */
ccq_status ccq_quantize_w4_host(const float *w, int32_t n, int32_t k, int32_t threads, uint8_t *codes,
                                float *scales);

/* ccq_dequant_bf16 - decode `num_experts` stacked weights to BF16 [E][n][k] in device memory.
 * Test and inspection only: the GEMM entry points never write decoded weights to memory.
 * Exact for every input (no fast-path domain limit). */
ccq_status ccq_dequant_bf16(const ccq_weight *w, int32_t num_experts, void *out_bf16,
                            ccq_stream_t stream);

/* ccq_gemm_workspace_size - bytes of workspace ccq_w2a16_gemm needs for this weight and m. */
size_t ccq_gemm_workspace_size(const ccq_weight *w, int32_t m);

/* ccq_w2a16_gemm - y[m][n] = x[m][k] * W^T with W decoded on the fly (never stored), fp32
 * accumulation, BF16 output.  The GEMV / small-M shapes of CCQ's "Inference Performance"
 * section (Table 4) and the dense prefill shape.
 *   w      single layer (num_experts = 1), any CCQ_FMT_* format
 *   x_bf16 (device) BF16 [m][k], 16-byte aligned;  m >= 0 (m == 0 is a no-op)
 *   y_bf16 (device) BF16 [m][n], 16-byte aligned
 *   ws     (device) workspace of ccq_gemm_workspace_size(w, m) bytes (may be NULL if that is 0)
 * Dispatch: m <= 32 runs the register-decode tensor-core kernel (decoded weights go straight into
 * mma operands in registers); m >= 33 runs the tcgen05/TMEM kernel (decoded weights go to shared
 * memory tiles that the tensor core reads). */
ccq_status ccq_w2a16_gemm(const ccq_weight *w, const void *x_bf16, int32_t m, void *y_bf16, void *ws,
                          size_t ws_bytes, ccq_stream_t stream);

/* ccq_w2a16_gemm_noalloc - ccq_w2a16_gemm for callers that cannot allocate device memory.
 * No counterpart in the paper: it exists for host code that is handed only input and output
 * pointers (e.g. a plugin whose host framework owns and pre-plans all device memory) or that must
 * not call cudaMalloc/cudaFree (which can synchronize the device) on its critical path.  It
 * computes the same result as ccq_w2a16_gemm with the same arguments, but takes its scratch from
 * a fixed array inside the library (ccq_w2a16_gemm_noalloc_max_scratch() bytes per device, held
 * by every GPU that loads the library until the process exits) and calls no allocator.
 *   - Shapes whose workspace (ccq_gemm_workspace_size) exceeds that size return
 *     CCQ_ERR_UNSUPPORTED before anything is launched.
 *   - The first call on each device looks up the array's device address (with that device
 *     current) and caches it; make that first call before any stream capture.
 *   - All calls share the one array and it keeps the last call's contents (every byte a call
 *     reads it writes first).  Calls that may overlap on the GPU (different streams, or several
 *     threads) race on it: serialize them. */
ccq_status ccq_w2a16_gemm_noalloc(const ccq_weight *w, const void *x_bf16, int32_t m, void *y_bf16,
                                  ccq_stream_t stream);
/* ccq_w2a16_gemm_noalloc_max_scratch - bytes of the fixed scratch array (per device). */
size_t ccq_w2a16_gemm_noalloc_max_scratch(void);

/* ccq_moe_workspace_size - workspace bytes of ccq_moe_w2a16_forward for these sizes. */
size_t ccq_moe_workspace_size(int32_t T, int32_t topk, int32_t H, int32_t I, int32_t num_experts);

/* ccq_moe_w2a16_forward - one MoE FFN layer whose expert weights are CCQ-quantized (the grouped
 * GEMM use of CCQ's "Inference Performance" section, Table 5; MoE-only scope per the WINT2 page):
 *   y[t] = sum_j routing_w[t][j] * ( SiLU(x_t Wg_e^T) * (x_t Wu_e^T) ) Wd_e^T,  e = expert_ids[t][j]
 * with SiLU(z) = z / (1 + exp(-z)).  The activation h = SiLU(.)*(.) is rounded to BF16 before the
 * down projection; the top-k sum runs in fp32 in fixed j order and is rounded to BF16 once.
 *   w13        E stacked gate/up weights: n = 2I (rows [0,I) gate, [I,2I) up), k = H
 *   w2         E stacked down weights: n = H, k = I
 *   x_bf16     (device) BF16 [T][H];   y_bf16 (device) BF16 [T][H] (may not alias x)
 *   expert_ids (device) int32 [T][topk], each in [0, E) and distinct within a token
 *   routing_w  (device) fp32 [T][topk], used as given (no renormalisation)
 *   ws         (device) workspace of ccq_moe_workspace_size(...) bytes
 * The formats may be mixed (w13 and w2 need not share a format).  Dispatch by the mean rows per
 * expert, T * topk / E: below 28 the register-decode kernel, from 28 the tcgen05 kernel. */
ccq_status ccq_moe_w2a16_forward(const ccq_weight *w13, const ccq_weight *w2, int32_t num_experts,
                                 const void *x_bf16, int32_t T, const int32_t *expert_ids,
                                 const float *routing_w, int32_t topk, void *y_bf16, void *ws,
                                 size_t ws_bytes, ccq_stream_t stream);

/* ccq_moe_w2a16_forward_traced - ccq_moe_w2a16_forward that also records CUDA events on `stream`
 * between its steps, for per-kernel timing: events[0] before routing, [1] after routing,
 * [2] after activation packing, [3] after the gate/up kernel, [4] after the group-sum kernel,
 * [5] after the down kernel, [6] after the combine.  When the decode-sized path runs both
 * projections as one fused launch (the same 2-bit format on both: CCQ or STD with fp32 group-scale
 * rows a multiple of 16 bytes, CCQ with 4-bit scales, or the same (4,3,2) / hybrid format),
 * [3], [4] and [5] are all recorded after that launch.  `events` (host) holds
 * CCQ_MOE_TRACE_POINTS cudaEvent_t handles created by the caller (NULL: no events).  No paper
 * counterpart: a measurement hook. */
enum { CCQ_MOE_TRACE_POINTS = 7 };
ccq_status ccq_moe_w2a16_forward_traced(const ccq_weight *w13, const ccq_weight *w2, int32_t num_experts,
                                        const void *x_bf16, int32_t T, const int32_t *expert_ids,
                                        const float *routing_w, int32_t topk, void *y_bf16, void *ws,
                                        size_t ws_bytes, ccq_stream_t stream, void *const *events);

/* ccq_check_device_error - wait for `stream`, read and clear the error word at the start of a
 * workspace used by ccq_moe_w2a16_forward.  CCQ_OK, or CCQ_ERR_DEVICE_CHECK / CCQ_ERR_TIMEOUT. */
ccq_status ccq_check_device_error(void *ws, ccq_stream_t stream);

/* ccq_selftest_bounded_wait - failure-detection self-test (no paper counterpart).  Launches one
 * CTA whose bounded wait can never be satisfied, with the same wait primitive the matmul kernels
 * use: kind 0 waits on an mbarrier phase that nothing completes, kind 1 on a global counter that
 * nothing increments.  The wait gives up after limit_us microseconds (1 .. 2 000 000), records
 * CCQ_ERR_TIMEOUT in the error word at the start of `ws`, and the kernel returns; the context stays
 * usable.  ws (device): at least 16 bytes, 16-byte aligned (a MoE workspace will do; bytes 8..11
 * are overwritten).  Read the result with ccq_check_device_error. */
ccq_status ccq_selftest_bounded_wait(void *ws, int32_t kind, int32_t limit_us, ccq_stream_t stream);

/* ccq_status_string - static description of a status code. */
const char *ccq_status_string(ccq_status s);

/* ccq_build_info - static string naming the target architecture and build options. */
const char *ccq_build_info(void);

#ifdef __cplusplus
}
#endif

#endif /* CCQ_H */
