// Device-side CCQ (6,4,3) code-cluster encoder: the same algorithm, arithmetic and tie rules as the
// host encoder (ccq_encode_host), so the two produce identical bytes.
//
// "CCQ: Convolutional Code for Extreme Low-bit Quantization in LLMs": §3.1 Algorithm 1 (group
// scale, codebook scaled by it, argmin over the codebook), §3.3 Eq. 1 (the channel's code
// cluster), §3.4 Eq. 2-4 (closed-form scale refit).  Three launches:
//   1. per 64-weight group: scale s = bf16(max|w|/31); per 4-vector the (6,4,3) code minimising
//      ((e0 + e1) + e2) + e3, e_i = (w_i - level_i)^2 in fp64, ties to the smallest code, found by
//      the 64-state trellis (consecutive states share 3 bits) -- one thread per vector;
//   2. per row: beta = min code, alpha = (max - min)/255 (1 if equal);
//   3. per row and 16 groups: the byte 0..255 whose decoded values are closest (ties to the
//      smallest byte), or the literal Eq. 1 byte; optionally one Eq. 4 refit per group.
// All fp64 sums and products are written as explicitly rounded operations (no contraction into
// fused multiply-adds), in the host encoder's order.
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/ccq.h"
#include "ccq_device.cuh"
#include "ccq_kernels.cuh"

namespace ccq {
namespace {

constexpr int kGroup = 64;
constexpr int kVecPerGroup = kGroup / 4;

__device__ __forceinline__ float to_bf16(float x) { return bf16_bits_to_float(float_to_bf16_bits(x)); }

// decoded level of state u at group scale s: bf16((u - 32) * bf16(s)), as a double
__device__ __forceinline__ double level(int u, float s) {
    const float sb = to_bf16(s);
    return (double)to_bf16((float)__dmul_rn((double)(u - 32), (double)sb));
}

// code of byte c under (alpha, beta): round half to even of one fp32 FMA (saturating, NaN -> 0)
__device__ __forceinline__ int32_t cluster_code(int c, float alpha, float beta) {
    const float t = __fmaf_rn((float)c, alpha, beta);
    if (!(t == t)) return 0;
    if (t >= 2147483648.0f) return INT32_MAX;
    if (t < -2147483648.0f) return INT32_MIN;
    return __float2int_rn(t);
}

// ---- 1: group scales and searched codes ---------------------------------------------------------
// block = 16 groups x 16 vectors (256 threads); one group's 16 threads are 16 consecutive lanes
__global__ void __launch_bounds__(256) enc_codes_kernel(const float *__restrict__ w, int n, int k,
                                                        float *__restrict__ scales, int32_t *__restrict__ C) {
    __shared__ double D[16][64];
    const int ng = k / kGroup;
    const int gl = threadIdx.x >> 4, vq = threadIdx.x & 15;  // group within the block, vector within the group
    const long long gidx = (long long)blockIdx.x * 16 + gl;   // global group index (row-major over n x ng)
    const bool live = gidx < (long long)n * ng;
    const long long gsafe = live ? gidx : 0;
    const int r = (int)(gsafe / ng), g = (int)(gsafe % ng);
    const float *v = w + (size_t)r * k + (size_t)g * kGroup + 4 * vq;
    float x[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) x[i] = v[i];
    // max |w| over the group (exact in any order)
    double amax = 0.0;
#pragma unroll
    for (int i = 0; i < 4; ++i) amax = fmax(amax, fabs((double)x[i]));
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) amax = fmax(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o, 16));
    const float s = to_bf16((float)__ddiv_rn(amax, 31.0));
#pragma unroll
    for (int j = 0; j < 4; ++j) D[gl][vq * 4 + j] = level(vq * 4 + j, s);
    __syncthreads();
    if (!live) return;
    if (vq == 0) scales[(size_t)r * ng + g] = s;
    const double *Dg = D[gl];
    // trellis: cost of the best walk ending in each state, and its code prefix
    double cost[64];
    int32_t pre[64];
#pragma unroll 8
    for (int u = 0; u < 64; ++u) {
        const double d = __dsub_rn((double)x[0], Dg[u]);
        cost[u] = __dmul_rn(d, d);
        pre[u] = u;
    }
#pragma unroll 1
    for (int i = 1; i < 4; ++i) {
        double nc[64];
        int32_t np[64];
#pragma unroll 1
        for (int u = 0; u < 64; ++u) {
            const double d = __dsub_rn((double)x[i], Dg[u]);
            const double e = __dmul_rn(d, d);
            const int lo = u >> 3;  // the 3 bits this state shares with its predecessor
            double best = __longlong_as_double(0x7FF0000000000000ll);  // +inf
            int32_t bp = 0;
#pragma unroll
            for (int h = 0; h < 8; ++h) {
                const int p = (h << 3) | lo;
                const double c = __dadd_rn(cost[p], e);
                const int32_t code = (pre[p] << 3) | (u & 7);
                if (c < best || (c == best && code < bp)) {
                    best = c;
                    bp = code;
                }
            }
            nc[u] = best;
            np[u] = bp;
        }
#pragma unroll 8
        for (int u = 0; u < 64; ++u) {
            cost[u] = nc[u];
            pre[u] = np[u];
        }
    }
    double best = __longlong_as_double(0x7FF0000000000000ll);
    int32_t arg = 0;
#pragma unroll 1
    for (int u = 0; u < 64; ++u)
        if (cost[u] < best || (cost[u] == best && pre[u] < arg)) {
            best = cost[u];
            arg = pre[u];
        }
    C[(size_t)r * (k / 4) + (size_t)g * kVecPerGroup + vq] = arg;
}

// ---- 2: the channel's code scale and zero-point -------------------------------------------------
__global__ void __launch_bounds__(256) enc_alpha_kernel(const int32_t *__restrict__ C, int n, int k,
                                                        float *__restrict__ alpha, float *__restrict__ beta) {
    const int r = blockIdx.x;
    const int nv = k / 4;
    int32_t lo = INT32_MAX, hi = INT32_MIN;
    for (int j = threadIdx.x; j < nv; j += blockDim.x) {
        const int32_t c = C[(size_t)r * nv + j];
        lo = min(lo, c);
        hi = max(hi, c);
    }
    __shared__ int32_t slo[8], shi[8];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        lo = min(lo, __shfl_xor_sync(0xFFFFFFFFu, lo, o));
        hi = max(hi, __shfl_xor_sync(0xFFFFFFFFu, hi, o));
    }
    if ((threadIdx.x & 31) == 0) {
        slo[threadIdx.x >> 5] = lo;
        shi[threadIdx.x >> 5] = hi;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int i = 1; i < (int)(blockDim.x >> 5); ++i) {
            lo = min(lo, slo[i]);
            hi = max(hi, shi[i]);
        }
        lo = min(lo, slo[0]);
        hi = max(hi, shi[0]);
        beta[r] = (float)lo;
        alpha[r] = hi == lo ? 1.0f : __fdiv_rn((float)(hi - lo), 255.0f);
    }
}

// ---- 3: cluster bytes (and the optional refit) --------------------------------------------------
// block = (row, 16 groups): 16 vectors per group, one thread each; the row's byte -> states table
// and the groups' level tables in shared memory
__device__ __forceinline__ uint8_t best_byte(const float *x, const double *Dg, const uint8_t (*st)[4]) {
    double best = __longlong_as_double(0x7FF0000000000000ll);
    int arg = 0;
#pragma unroll 1
    for (int c = 0; c < 256; ++c) {
        double err = 0.0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const double d = __dsub_rn((double)x[i], Dg[st[c][i]]);
            err = __dadd_rn(err, __dmul_rn(d, d));
        }
        if (err < best) {
            best = err;
            arg = c;
        }
    }
    return (uint8_t)arg;
}

__global__ void __launch_bounds__(256) enc_bytes_kernel(const float *__restrict__ w, const int32_t *__restrict__ C,
                                                        int n, int k, uint32_t flags, float *__restrict__ scales,
                                                        const float *__restrict__ alpha,
                                                        const float *__restrict__ beta, uint8_t *__restrict__ codes) {
    __shared__ uint8_t st[256][4];
    __shared__ double D[16][64];
    __shared__ float s2sh[16];
    const int ng = k / kGroup;
    const int chunks = (ng + 15) / 16;
    const int r = blockIdx.x / chunks, g0 = (blockIdx.x % chunks) * 16;
    const float a = alpha[r], b = beta[r];
    {
        const uint32_t Cc = (uint32_t)cluster_code(threadIdx.x, a, b);
#pragma unroll
        for (int i = 0; i < 4; ++i) st[threadIdx.x][i] = (uint8_t)((Cc >> (9 - 3 * i)) & 0x3Fu);
    }
    const int gl = threadIdx.x >> 4, vq = threadIdx.x & 15, g = g0 + gl;
    const bool live = g < ng;
    const float s = live ? scales[(size_t)r * ng + g] : 0.0f;
#pragma unroll
    for (int j = 0; j < 4; ++j) D[gl][vq * 4 + j] = level(vq * 4 + j, s);
    __syncthreads();
    const int j = g * kVecPerGroup + vq;  // vector index within the row
    float x[4] = {0.f, 0.f, 0.f, 0.f};
    if (live)
#pragma unroll
        for (int i = 0; i < 4; ++i) x[i] = w[(size_t)r * k + (size_t)j * 4 + i];
    uint8_t byte = 0;
    if (live) {
        if (flags & CCQ_ENC_LITERAL_EQ1) {
            float qq = rintf(__fdiv_rn(__fsub_rn((float)C[(size_t)r * (k / 4) + j], b), a));
            qq = fminf(255.0f, fmaxf(0.0f, qq));
            byte = (uint8_t)qq;
        } else {
            byte = best_byte(x, D[gl], st);
        }
    }
    if (flags & CCQ_ENC_REFIT_SCALE) {
        // Eq. 4 for the group, summed in the host encoder's order (vector by vector, i = 0..3)
        __shared__ uint8_t bsh[16][16];
        bsh[gl][vq] = byte;
        __syncthreads();
        if (live && vq == 0) {
            double num = 0.0, den = 0.0;
            for (int q = 0; q < kVecPerGroup; ++q) {
                const int jj = g * kVecPerGroup + q;
                for (int i = 0; i < 4; ++i) {
                    const double lev = (double)st[bsh[gl][q]][i] - 32.0;
                    num = __dadd_rn(num, __dmul_rn((double)w[(size_t)r * k + (size_t)jj * 4 + i], lev));
                    den = __dadd_rn(den, __dmul_rn(lev, lev));
                }
            }
            float s2 = 0.0f;
            if (den > 0.0 && __ddiv_rn(num, den) > 0.0) s2 = to_bf16((float)__ddiv_rn(num, den));
            s2sh[gl] = s2;
        }
        __syncthreads();
        const float s2 = live ? s2sh[gl] : 0.0f;
        if (s2 > 0.0f) {
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) D[gl][vq * 4 + jj] = level(vq * 4 + jj, s2);
        }
        __syncthreads();
        if (live && s2 > 0.0f) {
            if (vq == 0) scales[(size_t)r * ng + g] = s2;
            if (!(flags & CCQ_ENC_LITERAL_EQ1)) byte = best_byte(x, D[gl], st);
        }
    }
    if (live) codes[(size_t)r * (k / 4) + j] = byte;
}

// ---- formats with the scale in the redundant bits (§3.2, §3.4, Algorithm 2) -----------------------
// kind 1, (4,3,2): 22 one-byte codes per 64 weights, states at shifts 4, 2, 0 (mask 0xF), zero-point
//   8, 4-bit scale in code 21's low nibble.
// kind 2, hybrid (3,3,2)+(3,4,2): 10 little-endian 16-bit words per 64 weights; word j < 9 = a 7-bit
//   (3,3,2) code (states at 4, 2, 0 of it) above a 9-bit (3,4,2) code (states at 6, 4, 2, 0), mask
//   0x7, zero-point 4; 13-bit scale in word 9's low 13 bits.
// Scale: raw r_g = max|w_g| / (7 or 3) (fp32), super = max_g r_g / (15 or 8191) (fp32), q_g =
// clip(round-half-even(r_g / super), 0, 15 or 8191) (0 when super = 0), s = bf16(fl32(q_g * super)).
// Each full code is the argmin of its decoded weights' squared error over every code of its width
// (ties to the smallest); the last code's state is the nearest level for weight 63.

__device__ __forceinline__ double emb_raw(const float *g, int kind) {
    double amax = 0.0;
    for (int i = 0; i < 64; ++i) amax = fmax(amax, fabs((double)g[i]));
    return (double)__double2float_rn(__ddiv_rn(amax, kind == 1 ? 7.0 : 3.0));
}

// 1: one block per row: its super scale
__global__ void __launch_bounds__(128) enc_emb_super_kernel(int kind, const float *__restrict__ w, int n, int k,
                                                            float *__restrict__ super) {
    __shared__ double red[128];
    const int r = blockIdx.x, ng = k / 64;
    double m = 0.0;
    for (int g = threadIdx.x; g < ng; g += blockDim.x) m = fmax(m, emb_raw(w + (size_t)r * k + (size_t)g * 64, kind));
    red[threadIdx.x] = m;
    __syncthreads();
    for (int h = 64; h > 0; h >>= 1) {
        if (threadIdx.x < h) red[threadIdx.x] = fmax(red[threadIdx.x], red[threadIdx.x + h]);
        __syncthreads();
    }
    if (threadIdx.x == 0) super[r] = __double2float_rn(__ddiv_rn(red[0], kind == 1 ? 15.0 : 8191.0));
}

// squared error of n consecutive weights v[0..n) against states taken from code c at the given shifts
template <int N>
__device__ __forceinline__ double emb_err(const double *v, uint32_t c, const int (&sh)[N], uint32_t mask,
                                          const double *lev) {
    double e = 0.0;
#pragma unroll
    for (int t = 0; t < N; ++t) {
        const double d = __dsub_rn(v[t], lev[(c >> sh[t]) & mask]);
        e = __dadd_rn(e, __dmul_rn(d, d));
    }
    return e;
}

// 2: one warp per (row, group); lane j searches code j
__global__ void __launch_bounds__(256) enc_emb_codes_kernel(int kind, const float *__restrict__ w, int n, int k,
                                                            const float *__restrict__ super,
                                                            uint8_t *__restrict__ codes) {
    __shared__ double sv[8][64];
    __shared__ double slev[8][16];
    const int wv = threadIdx.x >> 5, lane = threadIdx.x & 31, ng = k / 64;
    const long long unit = (long long)blockIdx.x * 8 + wv;
    if (unit >= (long long)n * ng) return;  // whole warps only: no barrier below
    const int r = (int)(unit / ng), g = (int)(unit % ng);
    const float *gw = w + (size_t)r * k + (size_t)g * 64;
    sv[wv][lane] = (double)gw[lane];
    sv[wv][lane + 32] = (double)gw[lane + 32];
    __syncwarp();
    const float sup = super[r];
    const double raw = emb_raw(gw, kind);
    const double qmax = kind == 1 ? 15.0 : 8191.0;
    double qq = sup > 0.0f ? rint(__ddiv_rn(raw, (double)sup)) : 0.0;
    qq = fmin(fmax(qq, 0.0), qmax);
    const uint32_t q = (uint32_t)qq;
    const float sb = to_bf16(__fmul_rn((float)q, sup));
    const int zp = kind == 1 ? 8 : 4, L = kind == 1 ? 4 : 3;
    if (lane < (1 << L)) slev[wv][lane] = (double)to_bf16(__fmul_rn((float)(lane - zp), sb));
    __syncwarp();
    const double *v = sv[wv], *lev = slev[wv];
    const int nw = kind == 1 ? 22 : 10;
    uint8_t *dst = codes + ((size_t)r * ng + g) * (size_t)(kind == 1 ? 22 : 20);
    if (lane < nw - 1) {
        if (kind == 1) {
            const int sh[3] = {4, 2, 0};
            double best = INFINITY;
            uint32_t bc = 0;
            for (uint32_t c = 0; c < 256; ++c) {
                const double e = emb_err<3>(v + 3 * lane, c, sh, 0xFu, lev);
                if (e < best) { best = e; bc = c; }
            }
            dst[lane] = (uint8_t)bc;
        } else {
            const int sh7[3] = {4, 2, 0}, sh9[4] = {6, 4, 2, 0};
            double best = INFINITY;
            uint32_t b7 = 0, b9 = 0;
            for (uint32_t c = 0; c < 128; ++c) {
                const double e = emb_err<3>(v + 7 * lane, c, sh7, 0x7u, lev);
                if (e < best) { best = e; b7 = c; }
            }
            best = INFINITY;
            for (uint32_t c = 0; c < 512; ++c) {
                const double e = emb_err<4>(v + 7 * lane + 3, c, sh9, 0x7u, lev);
                if (e < best) { best = e; b9 = c; }
            }
            reinterpret_cast<uint16_t *>(dst)[lane] = (uint16_t)((b7 << 9) | b9);
        }
    } else if (lane == nw - 1) {
        double best = INFINITY;
        uint32_t bu = 0;
        for (uint32_t u = 0; u < (1u << L); ++u) {
            const double d = __dsub_rn(v[63], lev[u]);
            const double e = __dmul_rn(d, d);
            if (e < best) { best = e; bu = u; }
        }
        if (kind == 1) dst[21] = (uint8_t)((bu << 4) | q);
        else reinterpret_cast<uint16_t *>(dst)[9] = (uint16_t)((bu << 13) | q);
    }
}

}  // namespace

cudaError_t launch_encode_emb(int kind, const float *w, int rows, int K, void *codes, float *super, cudaStream_t s) {
    if (rows <= 0) return cudaSuccess;
    enc_emb_super_kernel<<<rows, 128, 0, s>>>(kind, w, rows, K, super);
    const long long units = (long long)rows * (K / 64);
    enc_emb_codes_kernel<<<(unsigned)((units + 7) / 8), 256, 0, s>>>(kind, w, rows, K, super,
                                                                     static_cast<uint8_t *>(codes));
    return cudaGetLastError();
}

}  // namespace ccq

using namespace ccq;

extern "C" size_t ccq_encode_device_workspace_size(int32_t n, int32_t k) {
    if (n <= 0 || k <= 0) return 0;
    return ((size_t)n * (size_t)(k / 4) * sizeof(int32_t) + 255) & ~size_t(255);
}

extern "C" ccq_status ccq_encode_device(const float *w, int32_t n, int32_t k, int32_t group, uint32_t flags,
                                        uint8_t *codes, float *scales, float *alpha, float *beta, void *ws,
                                        size_t ws_bytes, ccq_stream_t stream) {
    if (!w || !codes || !scales || !alpha || !beta) return CCQ_ERR_INVALID_ARG;
    if (n < 0 || k <= 0 || group != kGroup || k % kGroup) return group != kGroup ? CCQ_ERR_UNSUPPORTED
                                                                                   : CCQ_ERR_INVALID_ARG;
    if (flags & ~uint32_t(CCQ_ENC_LITERAL_EQ1 | CCQ_ENC_REFIT_SCALE)) return CCQ_ERR_INVALID_ARG;
    if (n == 0) return CCQ_OK;
    if (!ws || ws_bytes < ccq_encode_device_workspace_size(n, k)) return CCQ_ERR_INVALID_ARG;
    cudaStream_t s = (cudaStream_t)stream;
    int32_t *C = static_cast<int32_t *>(ws);
    const long long groups = (long long)n * (k / kGroup);
    const long long blocks1 = (groups + 15) / 16;
    if (blocks1 > 0x7FFFFFFFll) return CCQ_ERR_INVALID_ARG;
    enc_codes_kernel<<<(unsigned)blocks1, 256, 0, s>>>(w, n, k, scales, C);
    enc_alpha_kernel<<<n, 256, 0, s>>>(C, n, k, alpha, beta);
    const int chunks = (k / kGroup + 15) / 16;
    if ((long long)n * chunks > 0x7FFFFFFFll) return CCQ_ERR_INVALID_ARG;
    enc_bytes_kernel<<<n * chunks, 256, 0, s>>>(w, C, n, k, flags, scales, alpha, beta, codes);
    return cudaGetLastError() == cudaSuccess ? CCQ_OK : CCQ_ERR_CUDA;
}
