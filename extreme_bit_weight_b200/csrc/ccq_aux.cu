// Auxiliary kernels of libccq (sm_100a): exact BF16 dequantization (inspection / tests),
// activation packing into the decode-sized kernel's operand layout, split-K reduction, and the
// MoE routing / combine steps around the expert matmuls.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>
#include <vector>

#include "../../include/ccq.h"
#include "ccq_device.cuh"
#include "ccq_kernels.cuh"

namespace ccq {

cudaError_t kernel_setup(const void *kern, int smem, int threads, int want_regs, int *per_sm) {
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    struct Entry {
        const void *kern;
        int dev, smem, threads, per_sm;
    };
    static std::mutex mu;
    static std::vector<Entry> done;
    {
        std::lock_guard<std::mutex> g(mu);
        for (const Entry &e : done)
            if (e.kern == kern && e.dev == dev && e.smem == smem && e.threads == threads) {
                if (per_sm) *per_sm = e.per_sm;
                return cudaSuccess;
            }
    }
    cudaFuncAttributes fa{};
    err = cudaFuncGetAttributes(&fa, kern);
    if (err != cudaSuccess) return err;
    if (want_regs && fa.numRegs != want_regs) return cudaErrorInvalidConfiguration;
    err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (err != cudaSuccess) return err;
    int n = 0;
    err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, threads, smem);
    if (err != cudaSuccess) return err;
    std::lock_guard<std::mutex> g(mu);
    done.push_back({kern, dev, smem, threads, n});
    if (per_sm) *per_sm = n;
    return cudaSuccess;
}

namespace {

// ------------------------------------------------------------------------------------------------
// Exact dequantization (CCQ §3.5 Algorithm 3 for W2; signed nibbles for W4).  One thread per
// stored byte.  The code is rounded with cvt.rni (round to nearest even, saturating at the int32
// range, NaN -> 0), so this kernel is exact for any alpha/beta, unlike the fast path.
// ------------------------------------------------------------------------------------------------
// scales == NULL: 4-bit group scales, s = fl32(q4 * super[r]) (CCQ §3.4 "Scale Compression"),
// two per byte of scale_q4[r][K/128], the even group in the low nibble.
__global__ void dequant_w2_kernel(const uint8_t *__restrict__ codes, const float *__restrict__ scales,
                                  const float *__restrict__ alpha, const float *__restrict__ beta, int rows,
                                  int K, uint16_t *__restrict__ out, const uint8_t *__restrict__ scale_q4,
                                  const float *__restrict__ super) {
    const size_t nbytes = (size_t)rows * (K / 4);
    const int kb = K / 4, ng = K / 64;
    for (size_t idx = blockIdx.x * (size_t)blockDim.x + threadIdx.x; idx < nbytes;
         idx += (size_t)gridDim.x * blockDim.x) {
        const int r = (int)(idx / kb), j = (int)(idx % kb);
        const float t = __fmaf_rn((float)codes[idx], __ldg(alpha + r), __ldg(beta + r));
        const uint32_t C = (uint32_t)__float2int_rn(t);
        const int G = (4 * j) / 64;
        float sraw;
        if (scales) {
            sraw = __ldg(scales + (size_t)r * ng + G);
        } else {
            const uint32_t q = (__ldg(scale_q4 + (size_t)r * (K / 128) + G / 2) >> (4 * (G & 1))) & 0xFu;
            sraw = __fmul_rn((float)q, __ldg(super + r));
        }
        const float s = bf16_bits_to_float(float_to_bf16_bits(sraw));
        uint16_t o[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int u = (int)((C >> (9 - 3 * i)) & 0x3Fu);
            o[i] = float_to_bf16_bits(__fmul_rn((float)(u - 32), s));
        }
        uint2 v;
        v.x = (uint32_t)o[0] | ((uint32_t)o[1] << 16);
        v.y = (uint32_t)o[2] | ((uint32_t)o[3] << 16);
        *reinterpret_cast<uint2 *>(out + (size_t)r * K + 4 * j) = v;
    }
}

__global__ void dequant_w4_kernel(const uint8_t *__restrict__ codes, const float *__restrict__ scales, int rows,
                                  int K, uint16_t *__restrict__ out) {
    const size_t nbytes = (size_t)rows * (K / 2);
    const int kb = K / 2;
    for (size_t idx = blockIdx.x * (size_t)blockDim.x + threadIdx.x; idx < nbytes;
         idx += (size_t)gridDim.x * blockDim.x) {
        const int r = (int)(idx / kb), j = (int)(idx % kb);
        const uint32_t b = codes[idx];
        const float s = bf16_bits_to_float(float_to_bf16_bits(__ldg(scales + r)));
        const int q0 = (int)((b & 0xFu) ^ 8u) - 8, q1 = (int)((b >> 4) ^ 8u) - 8;
        const uint32_t v = (uint32_t)float_to_bf16_bits(__fmul_rn((float)q0, s)) |
                           ((uint32_t)float_to_bf16_bits(__fmul_rn((float)q1, s)) << 16);
        *reinterpret_cast<uint32_t *>(out + (size_t)r * K + 2 * j) = v;
    }
}

// WINT2-Standard (CCQ "Inference Performance", Table 4's comparison format): field i of byte j is the
// level q of weight 4j+i, w = bf16((q - 2) * bf16(s)) (an exact product).  One thread per byte.
__global__ void dequant_std_kernel(const uint8_t *__restrict__ codes, const float *__restrict__ scales, int rows,
                                   int K, uint16_t *__restrict__ out) {
    const size_t nbytes = (size_t)rows * (K / 4);
    const int kb = K / 4, ng = K / 64;
    for (size_t idx = blockIdx.x * (size_t)blockDim.x + threadIdx.x; idx < nbytes;
         idx += (size_t)gridDim.x * blockDim.x) {
        const int r = (int)(idx / kb), j = (int)(idx % kb);
        const uint32_t b = codes[idx];
        const float s = bf16_bits_to_float(float_to_bf16_bits(__ldg(scales + (size_t)r * ng + (4 * j) / 64)));
        uint16_t o[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) o[i] = float_to_bf16_bits(__fmul_rn((float)((int)((b >> (2 * i)) & 3u) - 2), s));
        uint2 v;
        v.x = (uint32_t)o[0] | ((uint32_t)o[1] << 16);
        v.y = (uint32_t)o[2] | ((uint32_t)o[3] << 16);
        *reinterpret_cast<uint2 *>(out + (size_t)r * K + 4 * j) = v;
    }
}

// Formats with the group scale in the redundant bits (CCQ §3.5 Algorithm 2; Table 1 rows (4,3,2) and
// (3,3,2)(3,4,2)), one thread per (row, group).  kind 1: 22 one-byte codes per group, states at
// shifts 4, 2, 0 (mask 0xF, zero-point 8), code 21 = weight 63's state (top nibble) and the 4-bit
// scale (low nibble).  kind 2: ten little-endian 16-bit words, states at shifts 13, 11, 9, 6, 4, 2,
// 0 (mask 0x7, zero-point 4), word 9 = weight 63's state (top 3 bits) and the 13-bit scale.
// s = bf16(fl32(q * super[row])); w = bf16((u - zp) * s), an exact product rounded once.
__global__ void dequant_emb_kernel(int kind, const uint8_t *__restrict__ codes, const float *__restrict__ super,
                                   int rows, int K, uint16_t *__restrict__ out) {
    const int ng = K / 64, gb = kind == 1 ? 22 : 20;
    const int kShift[7] = {13, 11, 9, 6, 4, 2, 0};
    for (size_t idx = blockIdx.x * (size_t)blockDim.x + threadIdx.x; idx < (size_t)rows * ng;
         idx += (size_t)gridDim.x * blockDim.x) {
        const int r = (int)(idx / ng), g = (int)(idx % ng);
        const uint8_t *c = codes + idx * gb;
        const uint32_t q = kind == 1 ? (c[21] & 0xFu) : (((uint32_t)c[18] | ((uint32_t)c[19] << 8)) & 0x1FFFu);
        const float s = bf16_bits_to_float(float_to_bf16_bits(__fmul_rn((float)q, __ldg(super + r))));
        uint16_t *o = out + (size_t)r * K + (size_t)g * 64;
        for (int i = 0; i < 64; ++i) {
            int u;
            if (kind == 1) {
                const int j = i < 63 ? i / 3 : 21, sh = i < 63 ? 4 - 2 * (i % 3) : 4;
                u = (c[j] >> sh) & 0xF;
                u -= 8;
            } else {
                const int j = i < 63 ? i / 7 : 9, sh = i < 63 ? kShift[i % 7] : 13;
                const uint32_t word = (uint32_t)c[2 * j] | ((uint32_t)c[2 * j + 1] << 8);
                u = (int)((word >> sh) & 0x7u) - 4;
            }
            o[i] = float_to_bf16_bits(__fmul_rn((float)u, s));
        }
    }
}

// Failure-detection self-test: one CTA whose bounded waits can never be satisfied -- kind 0 an
// mbarrier phase that nothing completes, kind 1 a global counter that nothing increments (it is
// zeroed first).  Each wait gives up after limit_ns and records DEV_ERR_TIMEOUT in the error word,
// as the matmul kernels' waits do; the kernel then returns normally.
__global__ void bounded_wait_probe_kernel(uint32_t *err, int *never, int kind, uint64_t limit_ns) {
    __shared__ uint64_t bar;
    if (threadIdx.x != 0) return;
    if (kind == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
        (void)mbar_wait(&bar, 0, err, limit_ns);  // nobody arrives
    } else {
        *never = 0;
        __threadfence();
        (void)wait_counter(never, 1, err, limit_ns);  // nobody adds
    }
}

// WINT2-Standard round-to-nearest, one warp per (row, 64-column group); lane l holds columns 2l,
// 2l+1.  s = bf16(max|w| / 2); the level round_half_even(w / s) clipped to [-2, 1] is decided by
// comparing w with s/2 and 3s/2, which are exact in fp32 for a BF16 s, so the decision equals the
// rounding of the exact quotient (ties: -3s/2 -> -2, +-s/2 -> 0, 3s/2 -> 2 clipped to 1).
__device__ __forceinline__ uint32_t std_field(float w, float s) {
    if (!(s > 0.0f)) return 2u;
    const float h = 0.5f * s, t = 1.5f * s;
    return w <= -t ? 0u : w < -h ? 1u : w <= h ? 2u : 3u;
}

__global__ void quantize_std_kernel(const float *__restrict__ w, int rows, int K, uint8_t *__restrict__ codes,
                                    float *__restrict__ scales) {
    const int ng = K / 64, lane = threadIdx.x & 31;
    const size_t units = (size_t)rows * ng;
    const size_t warps = (size_t)gridDim.x * (blockDim.x >> 5);
    for (size_t u = blockIdx.x * (size_t)(blockDim.x >> 5) + (threadIdx.x >> 5); u < units; u += warps) {
        const size_t r = u / ng, g = u % ng;
        const float2 v = __ldg(reinterpret_cast<const float2 *>(w + r * K + g * 64) + lane);
        float a = fmaxf(fabsf(v.x), fabsf(v.y));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xFFFFFFFFu, a, o));
        const float s = bf16_bits_to_float(float_to_bf16_bits(a * 0.5f));
        const uint32_t nib = std_field(v.x, s) | (std_field(v.y, s) << 2);
        const uint32_t hi = __shfl_down_sync(0xFFFFFFFFu, nib, 1);
        if ((lane & 1) == 0) codes[r * (K / 4) + g * 16 + lane / 2] = (uint8_t)(nib | (hi << 4));
        if (lane == 0) scales[r * ng + g] = s;
    }
}

// ------------------------------------------------------------------------------------------------
// Activation operand packing.  One thread per (operand row p, 64-column group G): reads the
// group's 64 BF16 values of source row tok_of[p] (or p), writes them in the XA order and the
// group sum S(p, G) (fp32, summed in column order) into the gsq table.
//
// gsq[p][G] = {L*S(p,G), L*S(p+1,G), L*S(p,G), L*S(p+1,G)} (float4, row pitch gsum_ld(K) groups,
// S = 0 past row P_valid - 1): L is the weight format's level offset, and the float4 is exactly the
// accumulator start of one mma C fragment (tokens p, p+1 for both of its rows), so the matmul
// kernel fills it with one 16-byte shared-memory read.  Padding groups [K/64, gsum_ld) are never
// read (the tensor map stops at K/64).
// ------------------------------------------------------------------------------------------------
__device__ __forceinline__ void store_gsq(float *gsq, int pr, int G, int ld, int P_valid, float v) {
    float *mine = gsq + ((size_t)pr * ld + G) * 4;
    mine[0] = v;
    mine[2] = v;
    if (pr + 1 == P_valid) {  // no next row: its half of this entry reads zero
        mine[1] = 0.0f;
        mine[3] = 0.0f;
    }
    if (pr > 0) {  // the previous row's entry holds this row as its second token
        float *prev = gsq + ((size_t)(pr - 1) * ld + G) * 4;
        prev[1] = v;
        prev[3] = v;
    }
}

// Four threads per (operand row p, group G): thread tig handles columns 16*tig .. 16*tig+15 of the
// group (one 16-column block of the XA order) and the four lanes sum the group in a fixed order.
__global__ void pack_xa_kernel(const uint16_t *__restrict__ x, const int *__restrict__ tok_of, int P_valid,
                               int P, int K, float level, uint16_t *__restrict__ xa, float *__restrict__ gsq,
                               int *zero_ctr) {
    pdl_wait();     // x, tok_of: written by earlier work
    pdl_trigger();  // the matmul may load its prologue meanwhile; it waits for this grid's results
    if (zero_ctr && blockIdx.x == 0 && threadIdx.x == 0) *zero_ctr = 0;
    const int ng = K / 64, ld = gsum_ld(K);
    const size_t total = (size_t)P_valid * ng * 4;  // a multiple of 4: the lanes of one group stay together
    for (size_t idx = blockIdx.x * (size_t)blockDim.x + threadIdx.x; idx < ((total + 31) & ~size_t(31));
         idx += (size_t)gridDim.x * blockDim.x) {
        const bool live = idx < total;
        const size_t q = live ? idx : 0;
        const int tig = (int)(q & 3);
        const int pr = (int)((q >> 2) / ng), G = (int)((q >> 2) % ng);
        const int src = tok_of ? __ldg(tok_of + pr) : pr;
        const uint4 *blk = reinterpret_cast<const uint4 *>(x + (size_t)src * K + (size_t)G * 64 + 16 * tig);
        const uint4 w0 = __ldg(blk), w1 = __ldg(blk + 1);
        const uint32_t ws[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
        uint16_t v[16];
#pragma unroll
        for (int h = 0; h < 8; ++h) {
            v[2 * h] = (uint16_t)(ws[h] & 0xFFFFu);
            v[2 * h + 1] = (uint16_t)(ws[h] >> 16);
        }
        float sum = 0.0f;
#pragma unroll
        for (int k = 0; k < 16; ++k) sum += bf16_bits_to_float(v[k]);
        // group sum over the four 16-column blocks, in block order
        const float s1 = __shfl_down_sync(0xFFFFFFFFu, sum, 1, 4);
        const float s2 = __shfl_down_sync(0xFFFFFFFFu, sum, 2, 4);
        const float s3 = __shfl_down_sync(0xFFFFFFFFu, sum, 3, 4);
        if (!live) continue;
        if (tig == 0) store_gsq(gsq, pr, G, ld, P_valid, level * (((sum + s1) + s2) + s3));
        // this block's 4 runs of 4 values: (i) -> j = 0..3 contiguous
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            uint2 o;
            o.x = (uint32_t)v[0 + i] | ((uint32_t)v[4 + i] << 16);
            o.y = (uint32_t)v[8 + i] | ((uint32_t)v[12 + i] << 16);
            *reinterpret_cast<uint2 *>(xa + xa_index((size_t)pr, (size_t)G * 64 + 16 * tig + i, (size_t)P)) = o;
        }
    }
}

// The (4,3,2) and hybrid operand orders (perm 1, 2; xa_index_perm): one warp per (operand row, group);
// lane l takes columns 2l, 2l+1, writes them to their positions and the warp sums L(k) x_k (every
// product is exact: an 8-bit level times a BF16 value) in a fixed shuffle order.
__global__ void pack_xa_perm_kernel(const uint16_t *__restrict__ x, const int *__restrict__ tok_of, int P_valid,
                                    int P, int K, uint16_t *__restrict__ xa, float *__restrict__ gsq, int *zero_ctr,
                                    int perm) {
    pdl_wait();
    pdl_trigger();
    if (zero_ctr && blockIdx.x == 0 && threadIdx.x == 0) *zero_ctr = 0;
    const int ng = K / 64, ld = gsum_ld(K), lane = threadIdx.x & 31;
    const size_t warps = (size_t)gridDim.x * (blockDim.x >> 5);
    for (size_t u = blockIdx.x * (size_t)(blockDim.x >> 5) + (threadIdx.x >> 5); u < (size_t)P_valid * ng;
         u += warps) {
        const int pr = (int)(u / ng), G = (int)(u % ng);
        const int src = tok_of ? __ldg(tok_of + pr) : pr;
        const uint32_t w2 = __ldg(reinterpret_cast<const uint32_t *>(x + (size_t)src * K + (size_t)G * 64) + lane);
        const uint16_t v0 = (uint16_t)(w2 & 0xFFFFu), v1 = (uint16_t)(w2 >> 16);
        const int k0 = 2 * lane;
        float sum = perm_level(perm, k0) * bf16_bits_to_float(v0) + perm_level(perm, k0 + 1) * bf16_bits_to_float(v1);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xFFFFFFFFu, sum, o);
        xa[xa_index_perm((size_t)pr, (size_t)G * 64 + k0, (size_t)P, perm)] = v0;
        xa[xa_index_perm((size_t)pr, (size_t)G * 64 + k0 + 1, (size_t)P, perm)] = v1;
        if (lane == 0) store_gsq(gsq, pr, G, ld, P_valid, sum);
    }
}

__global__ void gsum_from_xa_perm_kernel(const uint16_t *__restrict__ xa, int P_valid, int P, int K,
                                         float *__restrict__ gsq, int perm) {
    const int ng = K / 64, ld = gsum_ld(K);
    for (size_t idx = blockIdx.x * (size_t)blockDim.x + threadIdx.x; idx < (size_t)P_valid * ng;
         idx += (size_t)gridDim.x * blockDim.x) {
        const int pr = (int)(idx / ng), G = (int)(idx % ng);
        float sum = 0.0f;
        for (int k = 0; k < 64; ++k)
            sum += perm_level(perm, k) *
                   bf16_bits_to_float(xa[xa_index_perm((size_t)pr, (size_t)G * 64 + k, (size_t)P, perm)]);
        store_gsq(gsq, pr, G, ld, P_valid, sum);
    }
}

__global__ void gsum_from_xa_kernel(const uint16_t *__restrict__ xa, int P_valid, int P, int K, float level,
                                    float *__restrict__ gsq) {
    const int ng = K / 64, ld = gsum_ld(K);
    const size_t total = (size_t)P_valid * ng;
    for (size_t idx = blockIdx.x * (size_t)blockDim.x + threadIdx.x; idx < total;
         idx += (size_t)gridDim.x * blockDim.x) {
        const int pr = (int)(idx / ng), G = (int)(idx % ng);
        float sum = 0.0f;
        for (int k = 0; k < 64; ++k)
            sum += bf16_bits_to_float(xa[xa_index((size_t)pr, (size_t)G * 64 + k, (size_t)P)]);
        store_gsq(gsq, pr, G, ld, P_valid, level * sum);
    }
}

__global__ void splitk_reduce_kernel(const float *__restrict__ partial, int ksplit, size_t split_stride, int M,
                                     int N, uint16_t *__restrict__ y) {
    pdl_wait();  // the partial sums of the matmul before
    pdl_trigger();
    const size_t total = (size_t)M * N;
    for (size_t idx = blockIdx.x * (size_t)blockDim.x + threadIdx.x; idx < total;
         idx += (size_t)gridDim.x * blockDim.x) {
        float s = 0.0f;
        for (int k = 0; k < ksplit; ++k) s += partial[(size_t)k * split_stride + idx];
        y[idx] = float_to_bf16_bits(s);
    }
}

// ------------------------------------------------------------------------------------------------
// MoE routing.  One CTA.  Pass 1 validates each (token, slot) pair (expert id in [0,E) and not a
// repeat within its token) and counts pairs per expert; a scan gives each expert's contiguous
// segment of operand rows; pass 2 places each valid pair in its expert's segment.  The order
// inside a segment does not affect any result (every operand row is computed independently).
// Invalid pairs get inv = -1 and are reported in the error word.
// ------------------------------------------------------------------------------------------------
__global__ void moe_route_kernel(const int *__restrict__ ids, const float *__restrict__ rw, int T, int topk,
                                 int E, int *__restrict__ seg_off, int *__restrict__ cursor,
                                 int *__restrict__ tok_of, float *__restrict__ rw_perm, int *__restrict__ inv,
                                 int *__restrict__ dep, uint32_t *err) {
    extern __shared__ int sh[];
    int *cnt = sh;          // [E]
    int *off = sh + E;      // [E+1]
    for (int i = threadIdx.x; i < E; i += blockDim.x) cnt[i] = 0;
    // per-expert completion counters of the fused matmul launch, then the matmuls' work counters
    for (int i = threadIdx.x; dep && i < E + 3; i += blockDim.x) dep[i] = 0;
    __syncthreads();
    const int npairs = T * topk;
    for (int q = threadIdx.x; q < npairs; q += blockDim.x) {
        const int t = q / topk, j = q % topk;
        const int e = ids[q];
        bool ok = (e >= 0 && e < E);
        if (!ok) record_error(err, DEV_ERR_BAD_EXPERT, (uint32_t)q);
        if (ok)
            for (int jj = 0; jj < j; ++jj)
                if (ids[t * topk + jj] == e) {
                    ok = false;
                    record_error(err, DEV_ERR_DUP_EXPERT, (uint32_t)q);
                    break;
                }
        inv[q] = ok ? -2 : -1;  // -2: valid, not yet placed
        if (ok) atomicAdd(&cnt[e], 1);
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        int s = 0;
        for (int i = 0; i < E; ++i) {
            off[i] = s;
            s += cnt[i];
        }
        off[E] = s;
    }
    __syncthreads();
    for (int i = threadIdx.x; i <= E; i += blockDim.x) seg_off[i] = off[i];
    for (int i = threadIdx.x; i < E; i += blockDim.x) cnt[i] = 0;
    __syncthreads();
    for (int q = threadIdx.x; q < npairs; q += blockDim.x) {
        if (inv[q] != -2) continue;
        const int e = ids[q];
        const int pos = off[e] + atomicAdd(&cnt[e], 1);
        tok_of[pos] = q / topk;
        rw_perm[pos] = rw[q];
        inv[q] = pos;
    }
    __syncthreads();
    for (int i = threadIdx.x; i < E; i += blockDim.x) cursor[i] = cnt[i];
}

// y[t] = bf16( sum_j slot[inv[t][j]] ), fixed j order, fp32; invalid pairs skipped.
__global__ void moe_combine_kernel(const float *__restrict__ slot, const int *__restrict__ inv, int T, int topk,
                                   int H, uint16_t *__restrict__ y) {
    const int H4 = H / 4;
    const size_t total = (size_t)T * H4;
    for (size_t idx = blockIdx.x * (size_t)blockDim.x + threadIdx.x; idx < total;
         idx += (size_t)gridDim.x * blockDim.x) {
        const int t = (int)(idx / H4), c4 = (int)(idx % H4);
        float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int j = 0; j < topk; ++j) {
            const int pr = __ldg(inv + t * topk + j);
            if (pr < 0) continue;
            const float4 v = __ldg(reinterpret_cast<const float4 *>(slot + (size_t)pr * H) + c4);
            s.x += v.x;
            s.y += v.y;
            s.z += v.z;
            s.w += v.w;
        }
        uint2 o;
        o.x = pack_bf16x2(s.x, s.y);
        o.y = pack_bf16x2(s.z, s.w);
        *reinterpret_cast<uint2 *>(y + (size_t)t * H + 4 * c4) = o;
    }
}

inline int grid_for(size_t work, int threads) {
    size_t b = (work + threads - 1) / threads;
    if (b > 148 * 16) b = 148 * 16;
    return b < 1 ? 1 : (int)b;
}

}  // namespace

cudaError_t launch_dequant(int fmt, const uint8_t *codes, const float *scales, const float *alpha,
                           const float *beta, int rows, int K, uint16_t *out, cudaStream_t s,
                           const uint8_t *scale_q4, const float *super) {
    if (rows == 0) return cudaSuccess;
    if (fmt == CCQ_FMT_W2_CCQ_G64 || fmt == CCQ_FMT_W2_CCQ_G64_Q4SCALE) {
        const bool q4 = fmt == CCQ_FMT_W2_CCQ_G64_Q4SCALE;
        dequant_w2_kernel<<<grid_for((size_t)rows * K / 4, 256), 256, 0, s>>>(
            codes, q4 ? nullptr : scales, alpha, beta, rows, K, out, scale_q4, super);
    } else if (fmt == CCQ_FMT_W2_STD_G64) {
        dequant_std_kernel<<<grid_for((size_t)rows * K / 4, 256), 256, 0, s>>>(codes, scales, rows, K, out);
    } else if (fmt == CCQ_FMT_W275_432 || fmt == CCQ_FMT_W25_HYBRID) {
        dequant_emb_kernel<<<grid_for((size_t)rows * (K / 64), 128), 128, 0, s>>>(fmt == CCQ_FMT_W275_432 ? 1 : 2, codes,
                                                                                   super, rows, K, out);
    } else {
        dequant_w4_kernel<<<grid_for((size_t)rows * K / 2, 256), 256, 0, s>>>(codes, scales, rows, K, out);
    }
    return cudaGetLastError();
}

cudaError_t launch_bounded_wait_probe(uint32_t *err, int *never, int kind, uint64_t limit_ns, cudaStream_t s) {
    bounded_wait_probe_kernel<<<1, 32, 0, s>>>(err, never, kind, limit_ns);
    return cudaGetLastError();
}

cudaError_t launch_quantize_std(const float *w, int rows, int K, uint8_t *codes, float *scales, cudaStream_t s) {
    if (rows <= 0) return cudaSuccess;
    quantize_std_kernel<<<grid_for((size_t)rows * (K / 64) * 32, 256), 256, 0, s>>>(w, rows, K, codes, scales);
    return cudaGetLastError();
}

cudaError_t launch_pack_xa(const uint16_t *x, const int *tok_of, int P_valid, int P, int K, float level,
                           uint16_t *xa, float *gsq, cudaStream_t s, int *zero_ctr, int perm) {
    if (P_valid <= 0) return cudaSuccess;
    if (perm != 0)
        return launch_pdl(pack_xa_perm_kernel, dim3(grid_for((size_t)P_valid * (K / 64) * 32, 256)), dim3(256), 0, s,
                          x, tok_of, P_valid, P, K, xa, gsq, zero_ctr, perm);
    return launch_pdl(pack_xa_kernel, dim3(grid_for((size_t)P_valid * (K / 64) * 4, 128)), dim3(128), 0, s, x, tok_of,
                      P_valid, P, K, level, xa, gsq, zero_ctr);
}

cudaError_t launch_gsum_from_xa(const uint16_t *xa, int P_valid, int P, int K, float level, float *gsq,
                                cudaStream_t s, int perm) {
    if (P_valid <= 0) return cudaSuccess;
    if (perm != 0) {
        gsum_from_xa_perm_kernel<<<grid_for((size_t)P_valid * (K / 64), 128), 128, 0, s>>>(xa, P_valid, P, K, gsq,
                                                                                           perm);
        return cudaGetLastError();
    }
    gsum_from_xa_kernel<<<grid_for((size_t)P_valid * (K / 64), 128), 128, 0, s>>>(xa, P_valid, P, K, level, gsq);
    return cudaGetLastError();
}

cudaError_t launch_splitk_reduce(const float *partial, int ksplit, size_t split_stride, int M, int N,
                                 uint16_t *y, cudaStream_t s) {
    if ((size_t)M * N == 0) return cudaSuccess;
    return launch_pdl(splitk_reduce_kernel, dim3(grid_for((size_t)M * N, 256)), dim3(256), 0, s, partial, ksplit,
                      split_stride, M, N, y);
}

cudaError_t launch_moe_route(const int *ids, const float *rw, int T, int topk, int E, int *seg_off, int *cursor,
                             int *tok_of, float *rw_perm, int *inv, int *dep, uint32_t *err, cudaStream_t s) {
    const size_t sh = sizeof(int) * (2 * (size_t)E + 1);
    if (sh > 48 * 1024) {
        cudaError_t e = kernel_setup(reinterpret_cast<const void *>(moe_route_kernel), (int)sh, 1024, 0, nullptr);
        if (e != cudaSuccess) return e;
    }
    moe_route_kernel<<<1, 1024, sh, s>>>(ids, rw, T, topk, E, seg_off, cursor, tok_of, rw_perm, inv, dep, err);
    return cudaGetLastError();
}

cudaError_t launch_moe_combine(const float *slot, const int *inv, int T, int topk, int H, uint16_t *y,
                               cudaStream_t s) {
    if (T == 0) return cudaSuccess;
    moe_combine_kernel<<<grid_for((size_t)T * (H / 4), 256), 256, 0, s>>>(slot, inv, T, topk, H, y);
    return cudaGetLastError();
}

}  // namespace ccq
