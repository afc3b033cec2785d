// Decode-sized CCQ W2A16 grouped matmul (the GEMV / small-M shapes of the CCQ paper's Table 4 and
// the small-M grouped GEMM of Table 5), sm_100a.
//
// One CTA = one expert x two 128-row halves of its weight x one k range (split-K) x all of the
// expert's tokens (in chunks of 8*NT).  A producer warp streams, per 512-column stage:
//   * the two halves' code bytes, [128 rows][128 B] each, by TMA with the 128-byte swizzle;
//   * the activation operand slice in the XA layout (see ccq_kernels.cuh) and its group sums.
// Eight consumer warps decode the bytes in registers and feed them straight into
// mma.sync.m16n8k16 (BF16 in, fp32 accumulate) as the A operand -- weights on the M side, tokens
// on the N side -- so no decoded weight is ever written to memory.
//
// Decode (CCQ §3.3 Eq. 1 inverted and §3.5 Algorithm 3, Table 1 row (6,4,3)):
//   code  C = round_half_even(fma(q, alpha, beta))   fp32 FMA; the rounding is an add of
//         1.5*2^23 (exact for codes in [0, 2^16): one fp32 add rounds to the nearest integer);
//   state u_i = (C >> (9 - 3i)) & 63;
//   the tensor core receives the BF16 value 128 + u_i (exact), and each 64-column group (one
//   scale) is accumulated on its own: the accumulator starts at -160 * sum_k x_k, so after the
//   group it holds sum_k x_k (u_k - 32) exactly up to fp32 rounding; it is then scaled by
//   bf16(scale) and added to the running fp32 sum.  This equals the BF16 weight definition
//   w = bf16((u - 32) * bf16(scale)) up to the final rounding of each weight (it skips that
//   per-weight rounding and keeps the exact product); with a one-hot activation the result is
//   exactly the decoded weight.
// Two bytes of the same row are paired into one 32-bit register with one integer multiply-add
// (the second byte's rounding constant is offset so that the float exponent bits cancel), then
// each state window is one shift and one mask-and-or.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "ccq_device.cuh"
#include "ccq_kernels.cuh"

namespace ccq {
namespace {

constexpr int kConsumerWarps = 8;
constexpr int kThreads = (kConsumerWarps + 1) * 32;
constexpr int kCodeTileBytes = 128 * 128;  // [128 rows][128 B] = 8 groups of 16 bytes

template <int NT>
struct Smem {
    static constexpr int MP = 8 * NT;
    static constexpr int kStages = NT >= 4 ? 3 : 4;  // ring depth within the 227 KB per CTA
    static constexpr int kXaBytes = 32 * MP * 16 * 2;  // [G*4+i = 32][MP][16] bf16
    static constexpr int kGsBytes = MP * 8 * 4;        // [MP][8] fp32
    static constexpr int kStageBytes = ((2 * kCodeTileBytes + kXaBytes + kGsBytes) + 1023) & ~1023;
    static constexpr int kTotal = kStages * kStageBytes + 1024;  // + alignment slack
    static_assert(kTotal + 64 <= 227 * 1024, "shared memory per CTA");
    static constexpr uint32_t kTxBytes = 2 * kCodeTileBytes + kXaBytes + kGsBytes;
};

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}

__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ uint64_t u2_pack(uint32_t lo, uint32_t hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "r"(lo), "r"(hi));
    return r;
}
__device__ __forceinline__ void u2_unpack(uint64_t v, uint32_t &lo, uint32_t &hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=r"(lo), "=r"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}

struct RowDecode {
    uint64_t ab;    // {alpha, alpha}
    uint64_t bb;    // {beta, beta}
};

// The constants of the decode, held in registers so the compiler keeps the integer multiply.
struct DecodeConsts {
    uint64_t neg_magic;  // {-2^23, -2^23}: byte value from its 0x4B0000bb bit pattern
    uint64_t round_mag;  // {1.5*2^23, 1.5*2^23 - 0x4B40}
    uint32_t mul16;      // 65536
};

// Decode one 32-bit word (4 consecutive bytes of one row) into the eight BF16x2 registers
//   R[2i]   = (128 + u_i(byte0), 128 + u_i(byte1)),  R[2i+1] = (.. byte2, .. byte3)
__device__ __forceinline__ void decode_word(uint32_t w, const RowDecode &rd, const DecodeConsts &k,
                                            uint32_t R[8]) {
    const uint32_t magic = 0x4B000000u;
    uint64_t c01 = u2_pack(prmt(w, magic, 0x7650u), prmt(w, magic, 0x7651u));
    uint64_t c23 = u2_pack(prmt(w, magic, 0x7652u), prmt(w, magic, 0x7653u));
    c01 = f2_add(c01, k.neg_magic);
    c23 = f2_add(c23, k.neg_magic);
    uint64_t t01 = f2_fma(c01, rd.ab, rd.bb);
    uint64_t t23 = f2_fma(c23, rd.ab, rd.bb);
    t01 = f2_add(t01, k.round_mag);
    t23 = f2_add(t23, k.round_mag);
    uint32_t r0, r1, r2, r3;
    u2_unpack(t01, r0, r1);
    u2_unpack(t23, r2, r3);
    uint32_t X01, X23;
    asm("mad.lo.u32 %0, %1, %2, %3;" : "=r"(X01) : "r"(r1), "r"(k.mul16), "r"(r0));
    asm("mad.lo.u32 %0, %1, %2, %3;" : "=r"(X23) : "r"(r3), "r"(k.mul16), "r"(r2));
    const uint32_t M = 0x003F003Fu, E = 0x43004300u;
    R[0] = ((X01 >> 9) & M) | E;
    R[1] = ((X23 >> 9) & M) | E;
    R[2] = ((X01 >> 6) & M) | E;
    R[3] = ((X23 >> 6) & M) | E;
    R[4] = ((X01 >> 3) & M) | E;
    R[5] = ((X23 >> 3) & M) | E;
    R[6] = (X01 & M) | E;
    R[7] = (X23 & M) | E;
}

__device__ __forceinline__ void mma_bf16(float *c, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ float silu(float z) { return z / (1.0f + __expf(-z)); }

template <int NT>
__global__ void __launch_bounds__(kThreads, 1)
decode_gemm_w2_kernel(const __grid_constant__ CUtensorMap tm_codes, const __grid_constant__ CUtensorMap tm_xa,
                      const __grid_constant__ CUtensorMap tm_gs, const DecodeGemmParams p) {
    using S = Smem<NT>;
    constexpr int MP = S::MP;
    constexpr int kStages = S::kStages;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ uint64_t full_bar[kStages], empty_bar[kStages];

    const int e = blockIdx.z;
    const int rb = blockIdx.x;
    const int ks = blockIdx.y;
    const int seg0 = p.seg_off ? __ldg(p.seg_off + e) : 0;
    const int Me = p.seg_off ? __ldg(p.seg_off + e + 1) - seg0 : p.M;
    const int s_begin = ks * p.stages_per_split;
    const int s_end = min(p.num_stages, s_begin + p.stages_per_split);
    if (Me <= 0 || s_begin >= s_end) return;
    const int nchunks = (Me + MP - 1) / MP;
    const int nst = s_end - s_begin;
    const int total_iters = nchunks * nst;
    const int localA = rb * p.row_block_stride;       // first local row of half A
    const int localB = localA + p.half_stride;        // first local row of half B
    const int rowA = e * p.N + localA, rowB = e * p.N + localB;
    const int ngroups = p.K / 64;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&full_bar[i], 1);
            mbar_init(&empty_bar[i], kConsumerWarps);
        }
        fence_mbar_init();
    }
    __syncthreads();

    if (warp == kConsumerWarps) {
        // ---------------- producer ----------------
        if (lane == 0) {
            prefetch_tensormap(&tm_codes);
            prefetch_tensormap(&tm_xa);
            prefetch_tensormap(&tm_gs);
            bool ok = true;
            for (int it = 0; it < total_iters && ok; ++it) {
                const int slot = it % kStages;
                if (it >= kStages) ok = mbar_wait(&empty_bar[slot], ((it / kStages) - 1) & 1, p.err);
                if (!ok) break;
                const int c = it / nst, st = s_begin + it % nst;
                uint8_t *base = smem + slot * S::kStageBytes;
                mbar_arrive_expect_tx(&full_bar[slot], S::kTxBytes);
                tma_load_2d(base, &tm_codes, &full_bar[slot], st * 128, rowA);
                tma_load_2d(base + kCodeTileBytes, &tm_codes, &full_bar[slot], st * 128, rowB);
                tma_load_3d(base + 2 * kCodeTileBytes, &tm_xa, &full_bar[slot], 0, seg0 + c * MP, st * 32);
                tma_load_2d(base + 2 * kCodeTileBytes + S::kXaBytes, &tm_gs, &full_bar[slot], st * 8,
                            seg0 + c * MP);
            }
            // every issued copy must land before the CTA may exit
            const int issued = ok ? total_iters : 0;
            for (int it = max(0, issued - kStages); it < issued && ok; ++it)
                ok = mbar_wait(&full_bar[it % kStages], (it / kStages) & 1, p.err);
        }
        return;
    }

    // ---------------- consumers ----------------
    const int g = lane >> 2, tig = lane & 3;
    const int wrow = warp * 16;  // this warp's 16 rows inside each 128-row half
    // local rows (within the expert) of the four rows this thread decodes
    int lrow[4] = {localA + wrow + g, localA + wrow + g + 8, localB + wrow + g, localB + wrow + g + 8};
    RowDecode rd[4];
    bool rvalid[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        rvalid[r] = lrow[r] < p.N;
        const int grow = e * p.N + (rvalid[r] ? lrow[r] : 0);
        const float a = __ldg(p.alpha + grow), b = __ldg(p.beta + grow);
        rd[r].ab = f2_pack(a, a);
        rd[r].bb = f2_pack(b, b);
    }
    DecodeConsts kc;
    kc.neg_magic = f2_pack(-8388608.0f, -8388608.0f);
    kc.round_mag = f2_pack(12582912.0f, 12582912.0f - 19264.0f);
    kc.mul16 = 65536u + (uint32_t)(p.K >> 30);  // == 65536; kept opaque so it stays a multiply

    float acc[2][NT][4];
#pragma unroll
    for (int t = 0; t < 2; ++t)
#pragma unroll
        for (int n = 0; n < NT; ++n)
#pragma unroll
            for (int q = 0; q < 4; ++q) acc[t][n][q] = 0.0f;

    const uint32_t swz = (uint32_t)g;  // row & 7 for rows wrow+g and wrow+g+8

    for (int it = 0; it < total_iters; ++it) {
        const int slot = it % kStages;
        const int c = it / nst, st = s_begin + it % nst;
        if (!mbar_wait(&full_bar[slot], (it / kStages) & 1, p.err)) break;
        const uint8_t *base = smem + slot * S::kStageBytes;
        const uint8_t *codesA = base, *codesB = base + kCodeTileBytes;
        const uint8_t *xa = base + 2 * kCodeTileBytes;
        const float *gs = reinterpret_cast<const float *>(base + 2 * kCodeTileBytes + S::kXaBytes);
        const int g_lim = min(8, ngroups - st * 8);
#pragma unroll 1
        for (int G = 0; G < g_lim; ++G) {
            const int gg = st * 8 + G;
            float sc[4];
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                const int grow = e * p.N + (rvalid[r] ? lrow[r] : 0);
                sc[r] = bf16_bits_to_float(float_to_bf16_bits(__ldg(p.scales + (size_t)grow * ngroups + gg)));
            }
            const uint32_t off0 = (uint32_t)(wrow + g) * 128u + ((((uint32_t)G) ^ swz) << 4) + 4u * tig;
            const uint32_t off1 = off0 + 8u * 128u;
            const uint32_t w0 = *reinterpret_cast<const uint32_t *>(codesA + off0);
            const uint32_t w1 = *reinterpret_cast<const uint32_t *>(codesA + off1);
            const uint32_t w2 = *reinterpret_cast<const uint32_t *>(codesB + off0);
            const uint32_t w3 = *reinterpret_cast<const uint32_t *>(codesB + off1);
            uint32_t RA0[8], RA1[8], RB0[8], RB1[8];
            decode_word(w0, rd[0], kc, RA0);
            decode_word(w1, rd[1], kc, RA1);
            decode_word(w2, rd[2], kc, RB0);
            decode_word(w3, rd[3], kc, RB1);
            float cg[2][NT][4];
#pragma unroll
            for (int n = 0; n < NT; ++n) {
                const float gs0 = gs[(n * 8 + 2 * tig) * 8 + G];
                const float gs1 = gs[(n * 8 + 2 * tig + 1) * 8 + G];
#pragma unroll
                for (int t = 0; t < 2; ++t) {
                    cg[t][n][0] = gs0;
                    cg[t][n][1] = gs1;
                    cg[t][n][2] = gs0;
                    cg[t][n][3] = gs1;
                }
            }
#pragma unroll
            for (int i = 0; i < 4; ++i) {
#pragma unroll
                for (int n = 0; n < NT; ++n) {
                    const uint2 b = *reinterpret_cast<const uint2 *>(
                        xa + ((size_t)((G * 4 + i) * MP + n * 8 + g) * 16 + tig * 4) * 2);
                    mma_bf16(cg[0][n], RA0[2 * i], RA1[2 * i], RA0[2 * i + 1], RA1[2 * i + 1], b.x, b.y);
                    mma_bf16(cg[1][n], RB0[2 * i], RB1[2 * i], RB0[2 * i + 1], RB1[2 * i + 1], b.x, b.y);
                }
            }
#pragma unroll
            for (int n = 0; n < NT; ++n) {
                acc[0][n][0] = fmaf(sc[0], cg[0][n][0], acc[0][n][0]);
                acc[0][n][1] = fmaf(sc[0], cg[0][n][1], acc[0][n][1]);
                acc[0][n][2] = fmaf(sc[1], cg[0][n][2], acc[0][n][2]);
                acc[0][n][3] = fmaf(sc[1], cg[0][n][3], acc[0][n][3]);
                acc[1][n][0] = fmaf(sc[2], cg[1][n][0], acc[1][n][0]);
                acc[1][n][1] = fmaf(sc[2], cg[1][n][1], acc[1][n][1]);
                acc[1][n][2] = fmaf(sc[3], cg[1][n][2], acc[1][n][2]);
                acc[1][n][3] = fmaf(sc[3], cg[1][n][3], acc[1][n][3]);
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty_bar[slot]);

        if (st == s_end - 1) {
            // ---------------- epilogue for token chunk c ----------------
#pragma unroll
            for (int n = 0; n < NT; ++n) {
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int tok = c * MP + n * 8 + 2 * tig + (q & 1);
                    if (tok >= Me) continue;
                    const int hr = q >> 1;  // 0: row g, 1: row g+8
                    if (p.mode == EPI_GATEUP) {
                        const int r = lrow[hr];  // gate row; its up row is r + half_stride
                        if (r >= p.I) continue;
                        const float h = silu(acc[0][n][q]) * acc[1][n][q];
                        const size_t pr = (size_t)(seg0 + tok);
                        reinterpret_cast<uint16_t *>(p.out)[xa_index(pr, (size_t)r, (size_t)p.h_P)] =
                            float_to_bf16_bits(h);
                        continue;
                    }
#pragma unroll
                    for (int t = 0; t < 2; ++t) {
                        const int r = lrow[2 * t + hr];
                        if (!rvalid[2 * t + hr]) continue;
                        const float v = acc[t][n][q];
                        const size_t m = (size_t)(seg0 + tok);
                        if (p.mode == EPI_PARTIAL_F32) {
                            reinterpret_cast<float *>(p.out)[(size_t)ks * p.out_split_stride + m * p.out_ld + r] = v;
                        } else if (p.mode == EPI_BF16) {
                            reinterpret_cast<uint16_t *>(p.out)[m * p.out_ld + r] = float_to_bf16_bits(v);
                        } else {  // EPI_DOWN
                            reinterpret_cast<float *>(p.out)[m * p.out_ld + r] = __ldg(p.rw + m) * v;
                        }
                    }
                }
            }
#pragma unroll
            for (int t = 0; t < 2; ++t)
#pragma unroll
                for (int n = 0; n < NT; ++n)
#pragma unroll
                    for (int q = 0; q < 4; ++q) acc[t][n][q] = 0.0f;
        }
    }
}

template <int NT>
cudaError_t launch_nt(const DecodeGemmParams &p, const CUtensorMap &a, const CUtensorMap &b,
                      const CUtensorMap &c, int row_blocks, int ksplit, int experts, cudaStream_t s) {
    auto kern = decode_gemm_w2_kernel<NT>;
    const int smem = Smem<NT>::kTotal;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (err != cudaSuccess) return err;
    dim3 grid(row_blocks, ksplit, experts);
    kern<<<grid, kThreads, smem, s>>>(a, b, c, p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode_gemm_w2(const DecodeGemmParams &p, const CUtensorMap &tm_codes,
                                  const CUtensorMap &tm_xa, const CUtensorMap &tm_gs, int row_blocks,
                                  int ksplit, int experts, int nt, cudaStream_t s) {
    switch (nt) {
        case 1: return launch_nt<1>(p, tm_codes, tm_xa, tm_gs, row_blocks, ksplit, experts, s);
        case 2: return launch_nt<2>(p, tm_codes, tm_xa, tm_gs, row_blocks, ksplit, experts, s);
        case 4: return launch_nt<4>(p, tm_codes, tm_xa, tm_gs, row_blocks, ksplit, experts, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace ccq
