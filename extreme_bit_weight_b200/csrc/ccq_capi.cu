// C ABI of libccq: argument validation, workspace layout, TMA descriptor encoding and dispatch.
// Declarations and the contract of every entry point are in include/ccq.h.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include <algorithm>
#include <mutex>
#include <type_traits>

#include "../../include/ccq.h"
#include "ccq_device.cuh"
#include "ccq_kernels.cuh"

using namespace ccq;

namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

bool make_map(CUtensorMap *m, CUtensorMapDataType dt, int rank, const void *base, const cuuint64_t *dims,
              const cuuint64_t *strides, const cuuint32_t *box, CUtensorMapSwizzle swz) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint32_t es[3] = {1, 1, 1};
    CUresult r = fn(m, dt, (cuuint32_t)rank, const_cast<void *>(base), dims, strides, box, es,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline size_t up256(size_t x) { return (x + 255) & ~size_t(255); }
inline int ceil_div(int a, int b) { return (a + b - 1) / b; }

ccq_status check_weight(const ccq_weight *w, int experts) {
    if (!w || experts <= 0) return CCQ_ERR_INVALID_ARG;
    if (w->fmt != CCQ_FMT_W2_CCQ_G64 && w->fmt != CCQ_FMT_W4_PER_CHANNEL && w->fmt != CCQ_FMT_W2_CCQ_G64_Q4SCALE &&
        w->fmt != CCQ_FMT_W2_STD_G64 && w->fmt != CCQ_FMT_W275_432 && w->fmt != CCQ_FMT_W25_HYBRID)
        return CCQ_ERR_UNSUPPORTED;
    if (w->n <= 0 || w->k <= 0 || w->n % 16 || w->k % 64) return CCQ_ERR_INVALID_ARG;
    if (!w->codes || !aligned16(w->codes)) return CCQ_ERR_INVALID_ARG;
    if (w->fmt == CCQ_FMT_W275_432 || w->fmt == CCQ_FMT_W25_HYBRID) {
        if (w->group != 64) return CCQ_ERR_UNSUPPORTED;
        // the code rows' pitch must be a multiple of 16 bytes (TMA)
        if (w->k % (w->fmt == CCQ_FMT_W275_432 ? 512 : 256)) return CCQ_ERR_INVALID_ARG;
        if (!w->super_scale || !aligned16(w->super_scale)) return CCQ_ERR_INVALID_ARG;
        if ((size_t)experts * w->n > (size_t)INT32_MAX) return CCQ_ERR_INVALID_ARG;
        return CCQ_OK;
    }
    if (w->fmt == CCQ_FMT_W2_CCQ_G64_Q4SCALE) {
        if (w->group != 64) return CCQ_ERR_UNSUPPORTED;
        if (w->k % 128 || !w->scale_q4 || !w->super_scale || !w->alpha || !w->beta) return CCQ_ERR_INVALID_ARG;
        if (!aligned16(w->scale_q4) || !aligned16(w->super_scale) || !aligned16(w->alpha) || !aligned16(w->beta))
            return CCQ_ERR_INVALID_ARG;
    } else {
        if (!w->scales || !aligned16(w->scales)) return CCQ_ERR_INVALID_ARG;
    }
    if (w->fmt == CCQ_FMT_W2_CCQ_G64) {
        if (w->group != 64) return CCQ_ERR_UNSUPPORTED;
        if (!w->alpha || !w->beta) return CCQ_ERR_INVALID_ARG;
    }
    if (w->fmt == CCQ_FMT_W2_STD_G64 && w->group != 64) return CCQ_ERR_UNSUPPORTED;
    if ((size_t)experts * w->n > (size_t)INT32_MAX) return CCQ_ERR_INVALID_ARG;
    return CCQ_OK;
}

// Formats with the scale in the redundant bits: 1 = (4,3,2), 2 = hybrid, 0 otherwise.
inline int emb_kind(const ccq_weight *w) {
    return w->fmt == CCQ_FMT_W275_432 ? 1 : w->fmt == CCQ_FMT_W25_HYBRID ? 2 : 0;
}

// The weight-format fields of a kernel parameter block.
template <class Params>
void set_format(Params &p, const ccq_weight *w) {
    p.emb = emb_kind(w);
    p.scales = w->scales;
    p.alpha = w->alpha;
    p.beta = w->beta;
    p.w4 = w->fmt == CCQ_FMT_W4_PER_CHANNEL;
    p.q4 = w->fmt == CCQ_FMT_W2_CCQ_G64_Q4SCALE;
    p.std2 = w->fmt == CCQ_FMT_W2_STD_G64;
    p.scale_q4 = w->scale_q4;
    p.super_scale = w->super_scale;
}

// Level offset of the decoders' BF16 values for this format (the gsq table's L).
float level_of(const ccq_weight *w) {
    return gsq_level(w->fmt == CCQ_FMT_W4_PER_CHANNEL, w->fmt == CCQ_FMT_W2_STD_G64);
}

// --- decode-sized path ----------------------------------------------------------------------
int pick_nt(double rows_per_expert, int fmt = CCQ_FMT_W2_CCQ_G64) {
    if (rows_per_expert <= 8.0) return 1;
    // W4 code tiles are twice as wide; the embedded-scale decodes hold more registers per group
    if (rows_per_expert <= 16.0 || fmt == CCQ_FMT_W4_PER_CHANNEL || fmt == CCQ_FMT_W275_432 ||
        fmt == CCQ_FMT_W25_HYBRID)
        return 2;
    return 4;
}

struct DecodeMaps {
    CUtensorMap codes, xa, gs, sc;
    bool tma_scales;
};

bool decode_maps(DecodeMaps &m, const ccq_weight *w, int experts, const uint16_t *xa, const float *gs, int P,
                 int nt) {
    const int K = w->k;
    const bool w4 = w->fmt == CCQ_FMT_W4_PER_CHANNEL;
    const int emb = emb_kind(w);
    const cuuint64_t rows = (cuuint64_t)experts * w->n;
    const cuuint32_t emb_row = emb == 1 ? 176u : 160u;  // 8 groups of 22 / 20 bytes
    const cuuint64_t row_bytes = (cuuint64_t)(w4 ? K / 2 : emb ? K / 64 * (emb == 1 ? 22 : 20) : K / 4);
    {
        // embedded-scale formats: one unswizzled box of a stage's 8 groups per row
        cuuint64_t dims[2] = {row_bytes, rows};
        cuuint64_t str[1] = {row_bytes};
        cuuint32_t box[2] = {emb ? emb_row : 128u, 128};
        if (!make_map(&m.codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, w->codes, dims, str, box,
                      emb ? CU_TENSOR_MAP_SWIZZLE_NONE : CU_TENSOR_MAP_SWIZZLE_128B))
            return false;
    }
    {
        cuuint64_t dims[3] = {16, (cuuint64_t)P, (cuuint64_t)(K / 16)};
        cuuint64_t str[2] = {32, (cuuint64_t)P * 32};
        cuuint32_t box[3] = {16, (cuuint32_t)(8 * nt), 32};
        if (!make_map(&m.xa, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, xa, dims, str, box, CU_TENSOR_MAP_SWIZZLE_NONE))
            return false;
    }
    {
        // gsq table: [P][gsum_ld(K)] float4 entries; the map stops at K/64 groups so that a stage
        // running past the last group reads zeros
        const int ld = gsum_ld(K);
        cuuint64_t dims[2] = {(cuuint64_t)(4 * (K / 64)), (cuuint64_t)P};
        cuuint64_t str[1] = {(cuuint64_t)ld * 16};
        cuuint32_t box[2] = {32, (cuuint32_t)(8 * nt)};
        if (!make_map(&m.gs, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, gs, dims, str, box, CU_TENSOR_MAP_SWIZZLE_NONE))
            return false;
    }
    // group scales [rows][K/64] fp32: staged by TMA when the row pitch is a multiple of 16 bytes
    m.tma_scales = !w4 && !emb && w->fmt != CCQ_FMT_W2_CCQ_G64_Q4SCALE && (K / 64) % 4 == 0;
    if (m.tma_scales) {
        cuuint64_t dims[2] = {(cuuint64_t)(K / 64), rows};
        cuuint64_t str[1] = {(cuuint64_t)(K / 64) * 4};
        cuuint32_t box[2] = {8, 128};
        if (!make_map(&m.sc, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, w->scales, dims, str, box, CU_TENSOR_MAP_SWIZZLE_NONE))
            return false;
    } else {
        m.sc = m.gs;  // unused
    }
    return true;
}

// Token counts from which the tcgen05 kernel runs (dense GEMM: m; MoE: mean rows per expert).  The
// decode-sized kernel takes at most 32 tokens of an expert per pass over its weight, and it is
// bound by the decode, so a second 32-token chunk costs a second full decode: a dense call of 33
// to 47 tokens took 60 us against 39 us on the tcgen05 kernel (8192 x 8192), and a MoE layer with
// 32 / 40 tokens per expert 2.27 / 2.83 ms against 1.84 / 1.86 ms.  With 24 tokens per expert
// (few experts over 32) the decode-sized kernel still wins, 1.64 against about 1.83 ms.
constexpr int kTcMinM = 33;
constexpr double kTcMinRowsPerExpert = 28.0;
// 128-token sub-tiles per tcgen05 tile: 1 while experts average at most 96 rows (a half-empty
// 256-token tile would double the MMA time, which bounds the kernel there, and few experts spill
// into a second 128-token tile), else 2 (a second tile would decode the weights again)
int tc_mt(double rows_per_expert) { return rows_per_expert > 96.0 ? 2 : 1; }

struct GemmWs {
    size_t xa, gs, partial, xt, work, total;
    int P, ksplit, spp, row_blocks, nt;
    bool tc;
};

int sm_count() {
    static int n = 0;
    if (n == 0) {
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            n = 148;
    }
    return n;
}

GemmWs gemm_layout(const ccq_weight *w, int m) {
    GemmWs L{};
    if (m >= kTcMinM) {
        L.tc = true;
        L.P = m;
        L.xt = 0;
        size_t off = up256((size_t)m * w->k * 2);
        // split-K when the (token tile, row tile) items cannot fill the SMs: ranges of kg groups
        // (a multiple of 4, one code stage), as many ranges as keep every item on its own SM
        const int nk = w->k / 64;
        const int items = ceil_div(m, 128 * tc_mt((double)m)) * ceil_div(w->n, 256);
        const int sms = sm_count();
        L.ksplit = 1;
        L.spp = nk;
        if (2 * items <= sms && nk >= 8) {
            const int want = std::max(1, std::min(sms / items, nk / 4));
            L.spp = ((ceil_div(nk, want) + 3) / 4) * 4;  // groups per split
            L.ksplit = ceil_div(nk, L.spp);
        }
        L.partial = off;
        if (L.ksplit > 1) off = up256(off + (size_t)L.ksplit * m * w->n * 4);
        L.total = off;
        return L;
    }
    L.P = (m + 3) & ~3;
    L.nt = pick_nt((double)m, w->fmt);
    const int K = w->k, N = w->n;
    const int nst = ceil_div(K, 512);
    L.row_blocks = ceil_div(N, 256);
    int want = std::max(1, ceil_div(2 * 148, L.row_blocks));
    want = std::min(want, nst);
    L.spp = ceil_div(nst, want);
    L.ksplit = ceil_div(nst, L.spp);
    size_t off = 0;
    L.work = off;  // the decode kernel's work counter, zeroed by the activation packing
    off = up256(off + 16);
    L.xa = off;
    off = up256(off + (size_t)L.P * K * 2);
    L.gs = off;
    off = up256(off + (size_t)L.P * gsum_ld(K) * 16);
    L.partial = off;
    if (L.ksplit > 1) off = up256(off + (size_t)L.ksplit * m * N * 4);
    L.total = off;
    return L;
}

struct MoeWs {
    size_t err, seg, cursor, dep, tok, rwp, inv, xa_x, gs_x, xa_h, gs_h, tiles, tcount, slot, total;
    int P, max_tiles;
    bool tc;
};

MoeWs moe_layout(int T, int topk, int H, int I, int E) {
    MoeWs L{};
    const int pairs = T * topk;
    L.P = (pairs + 3) & ~3;
    L.tc = (double)pairs / E >= kTcMinRowsPerExpert;
    L.max_tiles = L.P / 128 + E + 1;  // (expert, 128-token tile) entries: at most one partial tile per expert
    size_t off = 0;
    L.err = off; off = up256(off + 16);
    L.seg = off; off = up256(off + sizeof(int) * (size_t)(E + 1));
    L.cursor = off; off = up256(off + sizeof(int) * (size_t)E);
    // per-expert counters of the fused launch, then the work counters of the fused launch and of
    // the two separate launches
    L.dep = off; off = up256(off + sizeof(int) * (size_t)(E + 3));
    L.tok = off; off = up256(off + sizeof(int) * (size_t)L.P);
    L.rwp = off; off = up256(off + sizeof(float) * (size_t)L.P);
    L.inv = off; off = up256(off + sizeof(int) * (size_t)pairs);
    // activation operand of the first projection and of the second (XA + group sums for the
    // decode-sized kernel, the plain permuted-column layout for the tcgen05 kernel)
    L.xa_x = off; off = up256(off + (size_t)L.P * H * 2);
    L.gs_x = off; if (!L.tc) off = up256(off + (size_t)L.P * gsum_ld(H) * 16);
    L.xa_h = off; off = up256(off + (size_t)L.P * I * 2);
    L.gs_h = off; if (!L.tc) off = up256(off + (size_t)L.P * gsum_ld(I) * 16);
    L.tiles = off; off = up256(off + sizeof(int2) * (size_t)L.max_tiles);
    L.tcount = off; off = up256(off + 16);
    L.slot = off; off = up256(off + (size_t)L.P * H * 4);
    L.total = off;
    return L;
}

bool tc_maps(CUtensorMap &ta, CUtensorMap &tcodes, const ccq_weight *w, int experts, const uint16_t *a, int P) {
    const int K = w->k;
    {
        cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)P};
        cuuint64_t str[1] = {(cuuint64_t)K * 2};
        cuuint32_t box[2] = {64, 128};
        if (!make_map(&ta, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B))
            return false;
    }
    if (const int emb = emb_kind(w)) {
        // rows of K/64 groups of 22 or 20 bytes; a code stage (4 groups) is one 112- or 80-byte box
        const cuuint64_t row_bytes = (cuuint64_t)(K / 64) * (emb == 1 ? 22 : 20);
        cuuint64_t dims[2] = {row_bytes, (cuuint64_t)experts * w->n};
        cuuint64_t str[1] = {row_bytes};
        cuuint32_t box[2] = {emb == 1 ? 112u : 80u, 128};
        if (!make_map(&tcodes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, w->codes, dims, str, box, CU_TENSOR_MAP_SWIZZLE_NONE))
            return false;
    } else {
        const cuuint64_t row_bytes = (cuuint64_t)(w->fmt == CCQ_FMT_W4_PER_CHANNEL ? K / 2 : K / 4);
        cuuint64_t dims[2] = {row_bytes, (cuuint64_t)experts * w->n};
        cuuint64_t str[1] = {row_bytes};
        cuuint32_t box[2] = {64, 128};
        if (!make_map(&tcodes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, w->codes, dims, str, box, CU_TENSOR_MAP_SWIZZLE_64B))
            return false;
    }
    return true;
}

inline ccq_status cuda_status(cudaError_t e) { return e == cudaSuccess ? CCQ_OK : CCQ_ERR_CUDA; }

inline cudaError_t trace(void *const *events, int i, cudaStream_t s) {
    if (!events || !events[i]) return cudaSuccess;
    return cudaEventRecord(static_cast<cudaEvent_t>(events[i]), s);
}

}  // namespace

extern "C" {

const char *ccq_status_string(ccq_status s) {
    switch (s) {
        case CCQ_OK: return "ok";
        case CCQ_ERR_INVALID_ARG: return "invalid argument";
        case CCQ_ERR_UNSUPPORTED: return "unsupported format or shape";
        case CCQ_ERR_CUDA: return "CUDA runtime error";
        case CCQ_ERR_DEVICE_CHECK: return "device-side check failed (invalid routing entry)";
        case CCQ_ERR_TIMEOUT: return "bounded device wait timed out";
    }
    return "unknown status";
}

const char *ccq_build_info(void) {
    return "libccq: sm_100a; decode-sized path: register decode -> mma.sync m16n8k16 bf16 (TMA-staged); "
           "prefill path: decode -> swizzled smem -> tcgen05.mma kind::f16, TMEM fp32 accumulators";
}

ccq_status ccq_dequant_bf16(const ccq_weight *w, int32_t num_experts, void *out_bf16, ccq_stream_t stream) {
    ccq_status st = check_weight(w, num_experts);
    if (st != CCQ_OK) return st;
    if (!out_bf16 || !aligned16(out_bf16)) return CCQ_ERR_INVALID_ARG;
    return cuda_status(launch_dequant(w->fmt, w->codes, w->scales, w->alpha, w->beta, num_experts * w->n, w->k,
                                      static_cast<uint16_t *>(out_bf16), (cudaStream_t)stream, w->scale_q4,
                                      w->super_scale));
}

size_t ccq_gemm_workspace_size(const ccq_weight *w, int32_t m) {
    if (!w || m <= 0 || w->n <= 0 || w->k <= 0) return 0;
    return gemm_layout(w, m).total;
}

ccq_status ccq_w2a16_gemm(const ccq_weight *w, const void *x_bf16, int32_t m, void *y_bf16, void *ws,
                          size_t ws_bytes, ccq_stream_t stream) {
    ccq_status st = check_weight(w, 1);
    if (st != CCQ_OK) return st;
    if (m < 0) return CCQ_ERR_INVALID_ARG;
    if (m == 0) return CCQ_OK;
    if (!x_bf16 || !y_bf16 || !aligned16(x_bf16) || !aligned16(y_bf16)) return CCQ_ERR_INVALID_ARG;
    const GemmWs L = gemm_layout(w, m);
    if (!ws || ws_bytes < L.total || (reinterpret_cast<uintptr_t>(ws) & 255u)) return CCQ_ERR_INVALID_ARG;
    cudaStream_t s = (cudaStream_t)stream;
    uint8_t *base = static_cast<uint8_t *>(ws);
    if (L.tc) {
        uint16_t *xt = reinterpret_cast<uint16_t *>(base + L.xt);
        cudaError_t e = launch_pack_xt(static_cast<const uint16_t *>(x_bf16), nullptr, m, w->k, xt, s);
        if (e != cudaSuccess) return CCQ_ERR_CUDA;
        CUtensorMap ta, tcodes;
        if (!tc_maps(ta, tcodes, w, 1, xt, m)) return CCQ_ERR_CUDA;
        TcGemmParams p{};
        p.N = w->n;
        p.K = w->k;
        p.row_block_stride = 256;
        p.half_stride = 128;
        p.n_tiles = ceil_div(w->n, 256);
        const int mt = tc_mt((double)m);
        p.m_tile = 128 * mt;
        p.static_tiles = ceil_div(m, p.m_tile);
        p.M = m;
        p.out_ld = w->n;
        set_format(p, w);
        p.ksplit = L.ksplit;
        p.kg = L.spp;
        if (L.ksplit > 1) {
            p.mode = EPI_PARTIAL_F32;
            p.out = base + L.partial;
            p.out_split_stride = (size_t)m * w->n;
        } else {
            p.mode = EPI_BF16;
            p.out = y_bf16;
        }
        const int grid = std::min(sm_count(), p.static_tiles * p.n_tiles * L.ksplit);
        e = launch_tc_gemm_w2(p, ta, tcodes, mt, grid, s);
        if (e == cudaSuccess && L.ksplit > 1)
            e = launch_splitk_reduce(reinterpret_cast<const float *>(base + L.partial), L.ksplit, (size_t)m * w->n, m,
                                     w->n, static_cast<uint16_t *>(y_bf16), s);
        return cuda_status(e);
    }
    uint16_t *xa = reinterpret_cast<uint16_t *>(base + L.xa);
    float *gs = reinterpret_cast<float *>(base + L.gs);
    int *work = reinterpret_cast<int *>(base + L.work);
    cudaError_t e = launch_pack_xa(static_cast<const uint16_t *>(x_bf16), nullptr, m, L.P, w->k,
                                   level_of(w), xa, gs, s, work, emb_kind(w));
    if (e != cudaSuccess) return CCQ_ERR_CUDA;
    DecodeMaps maps;
    if (!decode_maps(maps, w, 1, xa, gs, L.P, L.nt)) return CCQ_ERR_CUDA;
    DecodeGemmParams p{};
    p.N = w->n;
    p.K = w->k;
    p.row_block_stride = 256;
    p.half_stride = 128;
    p.num_stages = ceil_div(w->k, 512);
    p.stages_per_split = L.spp;
    p.seg_off = nullptr;
    p.M = m;
    p.P = L.P;
    p.out_ld = w->n;
    p.err = nullptr;
    if (L.ksplit > 1) {
        p.mode = EPI_PARTIAL_F32;
        p.out = base + L.partial;
        p.out_split_stride = (size_t)m * w->n;
    } else {
        p.mode = EPI_BF16;
        p.out = y_bf16;
    }
    p.tma_scales = maps.tma_scales;
    set_format(p, w);
    p.work = work;
    e = launch_decode_gemm_w2(p, maps.codes, maps.xa, maps.gs, maps.sc, L.row_blocks, L.ksplit, 1, L.nt, s);
    if (e != cudaSuccess) return CCQ_ERR_CUDA;
    if (L.ksplit > 1) {
        e = launch_splitk_reduce(reinterpret_cast<const float *>(base + L.partial), L.ksplit, (size_t)m * w->n, m,
                                 w->n, static_cast<uint16_t *>(y_bf16), s);
        if (e != cudaSuccess) return CCQ_ERR_CUDA;
    }
    return CCQ_OK;
}

size_t ccq_moe_workspace_size(int32_t T, int32_t topk, int32_t H, int32_t I, int32_t num_experts) {
    if (T <= 0 || topk <= 0 || H <= 0 || I <= 0 || num_experts <= 0) return 0;
    return moe_layout(T, topk, H, I, num_experts).total;
}

ccq_status ccq_moe_w2a16_forward(const ccq_weight *w13, const ccq_weight *w2, int32_t num_experts,
                                 const void *x_bf16, int32_t T, const int32_t *expert_ids,
                                 const float *routing_w, int32_t topk, void *y_bf16, void *ws, size_t ws_bytes,
                                 ccq_stream_t stream) {
    return ccq_moe_w2a16_forward_traced(w13, w2, num_experts, x_bf16, T, expert_ids, routing_w, topk, y_bf16, ws,
                                        ws_bytes, stream, nullptr);
}

ccq_status ccq_moe_w2a16_forward_traced(const ccq_weight *w13, const ccq_weight *w2, int32_t num_experts,
                                        const void *x_bf16, int32_t T, const int32_t *expert_ids,
                                        const float *routing_w, int32_t topk, void *y_bf16, void *ws,
                                        size_t ws_bytes, ccq_stream_t stream, void *const *events) {
    ccq_status st = check_weight(w13, num_experts);
    if (st != CCQ_OK) return st;
    st = check_weight(w2, num_experts);
    if (st != CCQ_OK) return st;
    if (T < 0 || topk <= 0 || topk > 64) return CCQ_ERR_INVALID_ARG;
    const int H = w13->k, I = w13->n / 2;
    if (w13->n % 2 || w2->n != H || w2->k != I || I % 64) return CCQ_ERR_INVALID_ARG;
    if (T == 0) return CCQ_OK;
    if (!x_bf16 || !y_bf16 || !expert_ids || !routing_w || !aligned16(x_bf16) || !aligned16(y_bf16))
        return CCQ_ERR_INVALID_ARG;
    if (x_bf16 == y_bf16) return CCQ_ERR_INVALID_ARG;
    const MoeWs L = moe_layout(T, topk, H, I, num_experts);
    if (!ws || ws_bytes < L.total || (reinterpret_cast<uintptr_t>(ws) & 255u)) return CCQ_ERR_INVALID_ARG;
    cudaStream_t s = (cudaStream_t)stream;
    uint8_t *base = static_cast<uint8_t *>(ws);
    uint32_t *err = reinterpret_cast<uint32_t *>(base + L.err);
    int *seg = reinterpret_cast<int *>(base + L.seg);
    int *cursor = reinterpret_cast<int *>(base + L.cursor);
    int *dep = reinterpret_cast<int *>(base + L.dep);
    int *tok = reinterpret_cast<int *>(base + L.tok);
    float *rwp = reinterpret_cast<float *>(base + L.rwp);
    int *inv = reinterpret_cast<int *>(base + L.inv);
    uint16_t *xa_x = reinterpret_cast<uint16_t *>(base + L.xa_x);
    float *gs_x = reinterpret_cast<float *>(base + L.gs_x);
    uint16_t *xa_h = reinterpret_cast<uint16_t *>(base + L.xa_h);
    float *gs_h = reinterpret_cast<float *>(base + L.gs_h);
    float *slot = reinterpret_cast<float *>(base + L.slot);
    const int pairs = T * topk;

    cudaError_t e = trace(events, 0, s);
    if (e == cudaSuccess) e = cudaMemsetAsync(base + L.err, 0, 16, s);
    if (e == cudaSuccess) e = cudaMemsetAsync(base + L.tok, 0, sizeof(int) * (size_t)L.P, s);
    if (e == cudaSuccess) e = cudaMemsetAsync(base + L.rwp, 0, sizeof(float) * (size_t)L.P, s);
    if (e == cudaSuccess)
        e = launch_moe_route(expert_ids, routing_w, T, topk, num_experts, seg, cursor, tok, rwp, inv, dep, err, s);
    if (e == cudaSuccess) e = trace(events, 1, s);
    if (e != cudaSuccess) return CCQ_ERR_CUDA;
    if (L.tc) {
        // prefill-sized: tcgen05 grouped GEMMs over (expert, 256-token tile) entries
        int2 *tiles = reinterpret_cast<int2 *>(base + L.tiles);
        int *tcount = reinterpret_cast<int *>(base + L.tcount);
        const int mt = tc_mt((double)pairs / num_experts);
        const int m_tile = 128 * mt;
        e = launch_pack_xt(static_cast<const uint16_t *>(x_bf16), tok, pairs, H, xa_x, s);
        if (e == cudaSuccess) e = launch_build_tiles(seg, num_experts, m_tile, tiles, tcount, s);
        if (e == cudaSuccess) e = trace(events, 2, s);
        if (e != cudaSuccess) return CCQ_ERR_CUDA;
        CUtensorMap ta1, tc1, ta2, tc2;
        if (!tc_maps(ta1, tc1, w13, num_experts, xa_x, L.P) || !tc_maps(ta2, tc2, w2, num_experts, xa_h, L.P))
            return CCQ_ERR_CUDA;
        TcGemmParams q1{};
        q1.N = w13->n;
        q1.K = H;
        q1.row_block_stride = 128;
        q1.half_stride = I;
        q1.n_tiles = ceil_div(I, 128);
        q1.tile_list = tiles;
        q1.tile_count = tcount;
        q1.m_tile = m_tile;
        q1.seg_off = seg;
        q1.mode = EPI_GATEUP;
        q1.out = xa_h;
        q1.out_ld = I;
        q1.I = I;
        q1.err = err;
        set_format(q1, w13);
        e = launch_tc_gemm_w2(q1, ta1, tc1, mt, std::min(sm_count(), L.max_tiles * q1.n_tiles), s);
        if (e == cudaSuccess) e = trace(events, 3, s);
        if (e == cudaSuccess) e = trace(events, 4, s);
        TcGemmParams q2 = q1;
        q2.N = H;
        q2.K = I;
        q2.row_block_stride = 256;
        q2.half_stride = 128;
        q2.n_tiles = ceil_div(H, 256);
        q2.mode = EPI_DOWN;
        q2.out = slot;
        q2.out_ld = H;
        q2.rw = rwp;
        q2.I = 0;
        set_format(q2, w2);
        if (e == cudaSuccess) e = launch_tc_gemm_w2(q2, ta2, tc2, mt, std::min(sm_count(), L.max_tiles * q2.n_tiles), s);
        if (e == cudaSuccess) e = trace(events, 5, s);
        if (e == cudaSuccess) e = launch_moe_combine(slot, inv, T, topk, H, static_cast<uint16_t *>(y_bf16), s);
        if (e == cudaSuccess) e = trace(events, 6, s);
        return cuda_status(e);
    }
    e = launch_pack_xa(static_cast<const uint16_t *>(x_bf16), tok, pairs, L.P, H, level_of(w13), xa_x, gs_x, s,
                       nullptr, emb_kind(w13));
    if (e == cudaSuccess) e = trace(events, 2, s);
    if (e != cudaSuccess) return CCQ_ERR_CUDA;
    const int nt1 = pick_nt((double)pairs / num_experts, w13->fmt);
    const int nt2 = pick_nt((double)pairs / num_experts, w2->fmt);

    // gate/up projection with the SiLU gate fused in its epilogue -> h (activation operand layout)
    DecodeMaps m1;
    if (!decode_maps(m1, w13, num_experts, xa_x, gs_x, L.P, nt1)) return CCQ_ERR_CUDA;
    DecodeGemmParams p1{};
    p1.N = w13->n;
    p1.K = H;
    p1.row_block_stride = 128;
    p1.half_stride = I;
    p1.num_stages = ceil_div(H, 512);
    p1.stages_per_split = p1.num_stages;
    p1.seg_off = seg;
    p1.P = L.P;
    p1.mode = EPI_GATEUP;
    p1.out = xa_h;
    p1.h_P = L.P;
    p1.I = I;
    p1.err = err;
    p1.tma_scales = m1.tma_scales;
    set_format(p1, w13);

    // down projection, scaled by each pair's routing weight -> fp32 slots
    DecodeMaps m2;
    if (!decode_maps(m2, w2, num_experts, xa_h, gs_h, L.P, nt2)) return CCQ_ERR_CUDA;
    DecodeGemmParams p2{};
    p2.N = H;
    p2.K = I;
    p2.row_block_stride = 256;
    p2.half_stride = 128;
    p2.num_stages = ceil_div(I, 512);
    p2.stages_per_split = p2.num_stages;
    p2.seg_off = seg;
    p2.P = L.P;
    p2.mode = EPI_DOWN;
    p2.out = slot;
    p2.out_ld = H;
    p2.rw = rwp;
    p2.err = err;
    p2.tma_scales = m2.tma_scales;
    set_format(p2, w2);

    // Both projections in the same 2-bit format (CCQ or STD with TMA-staged fp32 scales, or CCQ
    // with 4-bit scales) and the same token tiling: one fused launch, in which the gate/up
    // epilogue also writes h's group-sum table and each down unit starts once its expert's
    // gate/up units are done.  Otherwise (or if the device refuses the cooperative launch) two
    // launches with the group sums computed in between.
    p1.h_perm = emb_kind(w2);  // h in the down projection's operand order
    bool fused = !p1.w4 && !p2.w4 && nt1 == nt2 && p1.std2 == p2.std2 && p1.emb == p2.emb &&
                 ((p1.tma_scales && p2.tma_scales && !p1.q4 && !p2.q4) || (p1.q4 && p2.q4) || p1.emb != 0);
    if (fused) {
        p1.dep = dep;
        p1.fuse_gsq = gs_h;
        p1.fuse_gsq_ld = gsum_ld(I);
        p1.fuse_level = level_of(w2);
        p1.work = dep + num_experts;
        p2.dep = dep;
        e = launch_decode_moe_fused(p1, m1.codes, m1.xa, m1.gs, m1.sc, ceil_div(I, 128), p2, m2.codes, m2.xa, m2.gs,
                                    m2.sc, ceil_div(H, 256), num_experts, nt1, s);
        if (e == cudaErrorCooperativeLaunchTooLarge || e == cudaErrorNotSupported) {
            (void)cudaGetLastError();  // not launched: take the two-launch path
            fused = false;
        } else {
            if (e == cudaSuccess) e = trace(events, 3, s);
            if (e == cudaSuccess) e = trace(events, 4, s);
            if (e == cudaSuccess) e = trace(events, 5, s);
        }
    }
    if (!fused) {
        p1.dep = p2.dep = nullptr;
        p1.fuse_gsq = nullptr;
        p1.work = dep + num_experts + 1;
        p2.work = dep + num_experts + 2;
        e = launch_decode_gemm_w2(p1, m1.codes, m1.xa, m1.gs, m1.sc, ceil_div(I, 128), 1, num_experts, nt1, s);
        if (e == cudaSuccess) e = trace(events, 3, s);
        if (e == cudaSuccess)
            e = launch_gsum_from_xa(xa_h, pairs, L.P, I, level_of(w2), gs_h, s, emb_kind(w2));
        if (e == cudaSuccess) e = trace(events, 4, s);
        if (e == cudaSuccess)
            e = launch_decode_gemm_w2(p2, m2.codes, m2.xa, m2.gs, m2.sc, ceil_div(H, 256), 1, num_experts, nt2, s);
        if (e == cudaSuccess) e = trace(events, 5, s);
    }
    if (e == cudaSuccess) e = launch_moe_combine(slot, inv, T, topk, H, static_cast<uint16_t *>(y_bf16), s);
    if (e == cudaSuccess) e = trace(events, 6, s);
    return cuda_status(e);
}

ccq_status ccq_encode_emb_device(int32_t fmt, const float *w, int32_t n, int32_t k, uint8_t *codes,
                                 float *super_scale, ccq_stream_t stream) {
    if (fmt != CCQ_FMT_W275_432 && fmt != CCQ_FMT_W25_HYBRID) return CCQ_ERR_UNSUPPORTED;
    if (!w || !codes || !super_scale || n < 0 || k <= 0 || k % 64) return CCQ_ERR_INVALID_ARG;
    if (!aligned16(w) || !aligned16(codes) || !aligned16(super_scale)) return CCQ_ERR_INVALID_ARG;
    if ((long long)n * (k / 64) > 0x3FFFFFFFll) return CCQ_ERR_INVALID_ARG;
    return cuda_status(launch_encode_emb(fmt == CCQ_FMT_W275_432 ? 1 : 2, w, n, k, codes, super_scale,
                                         (cudaStream_t)stream));
}

ccq_status ccq_quantize_std_device(const float *w, int32_t n, int32_t k, uint8_t *codes, float *scales,
                                   ccq_stream_t stream) {
    if (!w || !codes || !scales || n < 0 || k <= 0 || k % 64) return CCQ_ERR_INVALID_ARG;
    if (!aligned16(w) || !aligned16(codes) || !aligned16(scales)) return CCQ_ERR_INVALID_ARG;
    if ((size_t)n * (k / 64) > (size_t)INT32_MAX * 64) return CCQ_ERR_INVALID_ARG;
    return cuda_status(launch_quantize_std(w, n, k, codes, scales, (cudaStream_t)stream));
}

ccq_status ccq_selftest_bounded_wait(void *ws, int32_t kind, int32_t limit_us, ccq_stream_t stream) {
    if (!ws || (reinterpret_cast<uintptr_t>(ws) & 15u) || (kind != 0 && kind != 1)) return CCQ_ERR_INVALID_ARG;
    if (limit_us < 1 || limit_us > 2000000) return CCQ_ERR_INVALID_ARG;
    uint32_t *err = static_cast<uint32_t *>(ws);
    int *never = reinterpret_cast<int *>(static_cast<uint8_t *>(ws) + 8);
    return cuda_status(launch_bounded_wait_probe(err, never, kind, (uint64_t)limit_us * 1000u, (cudaStream_t)stream));
}

ccq_status ccq_check_device_error(void *ws, ccq_stream_t stream) {
    if (!ws) return CCQ_ERR_INVALID_ARG;
    uint32_t h[2] = {0, 0};
    cudaStream_t s = (cudaStream_t)stream;
    if (cudaMemcpyAsync(h, ws, sizeof(h), cudaMemcpyDeviceToHost, s) != cudaSuccess) return CCQ_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return CCQ_ERR_CUDA;
    if (h[0] == 0) return CCQ_OK;
    if (cudaMemsetAsync(ws, 0, sizeof(h), s) != cudaSuccess) return CCQ_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return CCQ_ERR_CUDA;
    return (h[0] & DEV_ERR_TIMEOUT) ? CCQ_ERR_TIMEOUT : CCQ_ERR_DEVICE_CHECK;
}

}  // extern "C"
