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

constexpr int kRowWarps = 8;                       // warps per 16-row slot set (256 rows per CTA)
constexpr int kConsumerWarps = 2 * kRowWarps;       // two warps per row slot: groups 0-3 / 4-7 of a stage
constexpr int kThreads = kConsumerWarps * 32;       // lane 0 of warp 0 also issues the TMA loads
constexpr int kCodeTileBytes = 128 * 128;  // [128 rows][128 B] = 8 groups of 16 bytes

template <int NT, bool W4 = false>
struct Smem {
    static constexpr int MP = 8 * NT;
    static constexpr int kCodeBytes = (W4 ? 2 : 1) * 2 * kCodeTileBytes;  // both halves, one stage
    static constexpr int kXaBytes = 32 * MP * 16 * 2;  // [G*4+i = 32][MP][16] bf16
    static constexpr int kGsBytes = MP * 8 * 4;        // [MP][8] fp32
    static constexpr int kScBytes = W4 ? 0 : 2 * 128 * 8 * 4;  // [2 halves][128 rows][8 groups] fp32 scales
    static constexpr int kStageBytes = ((kCodeBytes + kXaBytes + kGsBytes + kScBytes) + 1023) & ~1023;
    static constexpr int kRedBytes = kRowWarps * 32 * 2 * NT * 4 * 4;  // partial sums of the second warp half
    static constexpr int kStages = ((227 * 1024 - 2048 - kRedBytes) / kStageBytes) < 4
                                       ? ((227 * 1024 - 2048 - kRedBytes) / kStageBytes) : 4;  // ring depth
    static constexpr int kTotal = kStages * kStageBytes + kRedBytes + 1024;  // + alignment slack
    static_assert(kTotal + 64 <= 227 * 1024, "shared memory per CTA");
    static constexpr uint32_t kTxBytes = kCodeBytes + kXaBytes + kGsBytes;  // + kScBytes with TMA scales
    static_assert(kStages >= 2, "ring depth");
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
// (a & m) | e in one three-input logic op
__device__ __forceinline__ uint32_t and_or(uint32_t a, uint32_t m, uint32_t e) {
    uint32_t d;
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(a), "r"(m), "r"(e));
    return d;
}

struct RowDecode {
    uint64_t ab;    // {alpha, alpha}: code scale of the row
    uint64_t bb;    // {beta, beta}: code zero-point of the row
};

// The constants of the decode, held in registers: the integer multiply stays a multiply and the
// window mask/exponent pair feeds one three-input logic op.
struct DecodeConsts {
    uint64_t neg_magic;  // {-2^23, -2^23}: byte value from its 0x4B0000bb bit pattern
    uint64_t round_mag;  // {1.5*2^23, 1.5*2^23 - 0x4B40}: round to integer; second byte pre-cancels
    uint32_t mul16;      // 65536
    uint32_t wmask;      // 0x003F003F: one 6-bit state window per 16-bit half
    uint32_t wexp;       // 0x43004300: BF16 exponent of 128 in both halves
};

// Decode one 32-bit word (4 consecutive bytes of one row) into the eight BF16x2 registers
//   R[2i]   = (128 + u_i(byte0), 128 + u_i(byte1)),  R[2i+1] = (.. byte2, .. byte3)
__device__ __forceinline__ void decode_word(uint32_t w, const RowDecode &rd, const DecodeConsts &k,
                                            uint32_t R[8]) {
    const uint32_t magic = 0x4B000000u;
    uint64_t c01 = u2_pack(prmt(w, magic, 0x7650u), prmt(w, magic, 0x7651u));
    uint64_t c23 = u2_pack(prmt(w, magic, 0x7652u), prmt(w, magic, 0x7653u));
    c01 = f2_add(c01, k.neg_magic);                       // the bytes, exact
    c23 = f2_add(c23, k.neg_magic);
    uint64_t t01 = f2_fma(c01, rd.ab, rd.bb);             // q*alpha + beta, one fp32 rounding
    uint64_t t23 = f2_fma(c23, rd.ab, rd.bb);
    t01 = f2_add(t01, k.round_mag);                       // round half to even to an integer
    t23 = f2_add(t23, k.round_mag);
    uint32_t r0, r1, r2, r3;
    u2_unpack(t01, r0, r1);
    u2_unpack(t23, r2, r3);
    uint32_t X01, X23;
    asm("mad.lo.u32 %0, %1, %2, %3;" : "=r"(X01) : "r"(r1), "r"(k.mul16), "r"(r0));
    asm("mad.lo.u32 %0, %1, %2, %3;" : "=r"(X23) : "r"(r3), "r"(k.mul16), "r"(r2));
    R[0] = and_or(X01 >> 9, k.wmask, k.wexp);
    R[1] = and_or(X23 >> 9, k.wmask, k.wexp);
    R[2] = and_or(X01 >> 6, k.wmask, k.wexp);
    R[3] = and_or(X23 >> 6, k.wmask, k.wexp);
    R[4] = and_or(X01 >> 3, k.wmask, k.wexp);
    R[5] = and_or(X23 >> 3, k.wmask, k.wexp);
    R[6] = and_or(X01, k.wmask, k.wexp);
    R[7] = and_or(X23, k.wmask, k.wexp);
}

// W4: one 32-bit word = 8 signed 4-bit codes (first of a pair in the low nibble).  Register i holds
// codes i and i+4 as BF16 (128 + (q + 8)) -- the sign bit of each nibble flipped, OR-ed into the
// exponent pattern of 128 -- so one shift and one three-input logic op per register.
__device__ __forceinline__ void decode_word_w4(uint32_t w, uint32_t m4, uint32_t x4, uint32_t R[4]) {
    asm("lop3.b32 %0, %1, %2, %3, 0x6A;" : "=r"(R[0]) : "r"(w), "r"(m4), "r"(x4));
    asm("lop3.b32 %0, %1, %2, %3, 0x6A;" : "=r"(R[1]) : "r"(w >> 4), "r"(m4), "r"(x4));
    asm("lop3.b32 %0, %1, %2, %3, 0x6A;" : "=r"(R[2]) : "r"(w >> 8), "r"(m4), "r"(x4));
    asm("lop3.b32 %0, %1, %2, %3, 0x6A;" : "=r"(R[3]) : "r"(w >> 12), "r"(m4), "r"(x4));
}

__device__ __forceinline__ void mma_bf16(float *c, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// d = a*b + c with c given separately (the group's starting value)
__device__ __forceinline__ void mma_bf16_c(float *d, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                           uint32_t b1, float c0, float c1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%10,%11,%10,%11};"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(c0), "f"(c1));
}

// fp32 value of bf16_rn(x): one conversion, the BF16 bits land in the high half
__device__ __forceinline__ float round_bf16(float x) { return __uint_as_float(pack_bf16x2(0.0f, x)); }

__device__ __forceinline__ float silu(float z) { return z / (1.0f + __expf(-z)); }

// One 64-column group of one stage for this thread: 4 code words (rows g, g+8 of both halves),
// decode, 4 x NT x 2 mma, per-group rescale.  All shared-memory offsets are compile-time
// constants once G is unrolled.
template <int NT, bool W4>
__device__ __forceinline__ void group_step(const int G, const uint8_t *codes, uint32_t cbase, uint32_t cswz,
                                           const uint8_t *xa, const uint8_t *gsb, const float sc[4],
                                           const RowDecode rd[4], const DecodeConsts &kc, float (&acc)[2][NT][4]) {
    constexpr int MP = 8 * NT;
    // A fragments per state window i: RA0/RA1 = rows g / g+8 of half A, RB0/RB1 of half B;
    // [2i] and [2i+1] are the k-pairs (j=0,1) and (j=2,3) of the window
    uint32_t RA0[8], RA1[8], RB0[8], RB1[8];
    if constexpr (!W4) {
        const uint32_t coff = cbase + (((uint32_t)G << 4) ^ cswz);
        const uint32_t w0 = *reinterpret_cast<const uint32_t *>(codes + coff);
        const uint32_t w1 = *reinterpret_cast<const uint32_t *>(codes + coff + 1024);
        const uint32_t w2 = *reinterpret_cast<const uint32_t *>(codes + kCodeTileBytes + coff);
        const uint32_t w3 = *reinterpret_cast<const uint32_t *>(codes + kCodeTileBytes + coff + 1024);
        decode_word(w0, rd[0], kc, RA0);
        decode_word(w1, rd[1], kc, RA1);
        decode_word(w2, rd[2], kc, RB0);
        decode_word(w3, rd[3], kc, RB1);
    } else {
        // 32 bytes per row and group: this thread's 8 bytes sit in 16-byte chunk 2(G%4) + tig/2 of
        // the 128-byte line (box G/4); cbase holds 8*(tig&1) and the row offset, cswz the row swizzle
        const int box = (G >> 2) * (2 * kCodeTileBytes);
        const uint32_t coff = cbase + ((((uint32_t)(2 * (G & 3))) << 4) ^ cswz);
        const uint2 q0 = *reinterpret_cast<const uint2 *>(codes + box + coff);
        const uint2 q1 = *reinterpret_cast<const uint2 *>(codes + box + coff + 1024);
        const uint2 q2 = *reinterpret_cast<const uint2 *>(codes + box + kCodeTileBytes + coff);
        const uint2 q3 = *reinterpret_cast<const uint2 *>(codes + box + kCodeTileBytes + coff + 1024);
        uint32_t t[4];
        decode_word_w4(q0.x, kc.wmask, kc.wexp, t);
        RA0[0] = t[0]; RA0[2] = t[1]; RA0[4] = t[2]; RA0[6] = t[3];
        decode_word_w4(q0.y, kc.wmask, kc.wexp, t);
        RA0[1] = t[0]; RA0[3] = t[1]; RA0[5] = t[2]; RA0[7] = t[3];
        decode_word_w4(q1.x, kc.wmask, kc.wexp, t);
        RA1[0] = t[0]; RA1[2] = t[1]; RA1[4] = t[2]; RA1[6] = t[3];
        decode_word_w4(q1.y, kc.wmask, kc.wexp, t);
        RA1[1] = t[0]; RA1[3] = t[1]; RA1[5] = t[2]; RA1[7] = t[3];
        decode_word_w4(q2.x, kc.wmask, kc.wexp, t);
        RB0[0] = t[0]; RB0[2] = t[1]; RB0[4] = t[2]; RB0[6] = t[3];
        decode_word_w4(q2.y, kc.wmask, kc.wexp, t);
        RB0[1] = t[0]; RB0[3] = t[1]; RB0[5] = t[2]; RB0[7] = t[3];
        decode_word_w4(q3.x, kc.wmask, kc.wexp, t);
        RB1[0] = t[0]; RB1[2] = t[1]; RB1[4] = t[2]; RB1[6] = t[3];
        decode_word_w4(q3.y, kc.wmask, kc.wexp, t);
        RB1[1] = t[0]; RB1[3] = t[1]; RB1[5] = t[2]; RB1[7] = t[3];
    }
    // group sums of the activations times the format's level offset (160 for W2, 136 for W4)
    const float off = W4 ? -136.0f : -160.0f;
#pragma unroll
    for (int n = 0; n < NT; ++n) {
        // the group's starting value: the activation sum times the level offset
        const float gs0 = off * *reinterpret_cast<const float *>(gsb + n * 256 + G * 4);
        const float gs1 = off * *reinterpret_cast<const float *>(gsb + n * 256 + 32 + G * 4);
        float cA[4], cB[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint2 b = *reinterpret_cast<const uint2 *>(xa + ((G * 4 + i) * MP + n * 8) * 32);
            if (i == 0) {
                mma_bf16_c(cA, RA0[0], RA1[0], RA0[1], RA1[1], b.x, b.y, gs0, gs1);
                mma_bf16_c(cB, RB0[0], RB1[0], RB0[1], RB1[1], b.x, b.y, gs0, gs1);
            } else {
                mma_bf16(cA, RA0[2 * i], RA1[2 * i], RA0[2 * i + 1], RA1[2 * i + 1], b.x, b.y);
                mma_bf16(cB, RB0[2 * i], RB1[2 * i], RB0[2 * i + 1], RB1[2 * i + 1], b.x, b.y);
            }
        }
        acc[0][n][0] = fmaf(sc[0], cA[0], acc[0][n][0]);
        acc[0][n][1] = fmaf(sc[0], cA[1], acc[0][n][1]);
        acc[0][n][2] = fmaf(sc[1], cA[2], acc[0][n][2]);
        acc[0][n][3] = fmaf(sc[1], cA[3], acc[0][n][3]);
        acc[1][n][0] = fmaf(sc[2], cB[0], acc[1][n][0]);
        acc[1][n][1] = fmaf(sc[2], cB[1], acc[1][n][1]);
        acc[1][n][2] = fmaf(sc[3], cB[2], acc[1][n][2]);
        acc[1][n][3] = fmaf(sc[3], cB[3], acc[1][n][3]);
    }
}

template <int NT, bool TMA_SC, bool W4>
__global__ void __launch_bounds__(kThreads, 1)
decode_gemm_w2_kernel(const __grid_constant__ CUtensorMap tm_codes, const __grid_constant__ CUtensorMap tm_xa,
                      const __grid_constant__ CUtensorMap tm_gs, const __grid_constant__ CUtensorMap tm_sc,
                      const DecodeGemmParams p) {
    using S = Smem<NT, W4>;
    constexpr int MP = S::MP;
    constexpr int kStages = S::kStages;
    constexpr int kCodeOff = 0;                       // code tiles of the stage
    constexpr int kXaOff = S::kCodeBytes;             // activation operand slice
    constexpr int kGsOff = S::kCodeBytes + S::kXaBytes;
    constexpr int kScOff = kGsOff + S::kGsBytes;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ uint64_t full_bar[kStages], empty_bar[kStages], red_full, red_empty;

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
    const bool producer = threadIdx.x == 0;
    if (producer) {
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&full_bar[i], 1);
            mbar_init(&empty_bar[i], kConsumerWarps);
        }
        mbar_init(&red_full, kRowWarps);
        mbar_init(&red_empty, kRowWarps);
        fence_mbar_init();
        prefetch_tensormap(&tm_codes);
        prefetch_tensormap(&tm_xa);
        prefetch_tensormap(&tm_gs);
        if (TMA_SC) prefetch_tensormap(&tm_sc);
    }
    __syncthreads();

    // TMA loads of iteration `it` (token chunk, 512-column stage) into its ring slot
    auto issue = [&](int it) {
        const int slot = it % kStages;
        const int c = it / nst, st = s_begin + it % nst;
        uint8_t *base = smem + slot * S::kStageBytes;
        mbar_arrive_expect_tx(&full_bar[slot], S::kTxBytes + ((TMA_SC && !W4) ? S::kScBytes : 0));
        if (TMA_SC && !W4) {
            uint8_t *sc = base + kScOff;
            tma_load_2d(sc, &tm_sc, &full_bar[slot], st * 8, rowA);
            tma_load_2d(sc + S::kScBytes / 2, &tm_sc, &full_bar[slot], st * 8, rowB);
        }
        // W2: 128 code bytes per row per stage; W4: 256, as two 128-byte boxes
#pragma unroll
        for (int bx = 0; bx < (W4 ? 2 : 1); ++bx) {
            const int x = st * (W4 ? 256 : 128) + bx * 128;
            tma_load_2d(base + kCodeOff + bx * 2 * kCodeTileBytes, &tm_codes, &full_bar[slot], x, rowA);
            tma_load_2d(base + kCodeOff + bx * 2 * kCodeTileBytes + kCodeTileBytes, &tm_codes, &full_bar[slot], x, rowB);
        }
        tma_load_3d(base + kXaOff, &tm_xa, &full_bar[slot], 0, seg0 + c * MP, st * 32);
        tma_load_2d(base + kGsOff, &tm_gs, &full_bar[slot], st * 8, seg0 + c * MP);
    };
    if (producer)
        for (int it = 0; it < min(kStages - 1, total_iters); ++it) issue(it);

    // ---------------- consumers ----------------
    const int g = lane >> 2, tig = lane & 3;
    const int wslot = warp & (kRowWarps - 1);  // row slot: 16 rows inside each 128-row half
    const int khalf = warp / kRowWarps;        // 0: groups 0-3 of every stage, 1: groups 4-7
    const int wrow = wslot * 16;
    // local rows (within the expert) of the four rows this thread decodes
    int lrow[4] = {localA + wrow + g, localA + wrow + g + 8, localB + wrow + g, localB + wrow + g + 8};
    RowDecode rd[4];
    bool rvalid[4];
    float sc_row[4];  // W4: per-channel scales, bf16-rounded
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        rvalid[r] = lrow[r] < p.N;
        const int grow = e * p.N + (rvalid[r] ? lrow[r] : 0);
        if constexpr (!W4) {
            const float a = __ldg(p.alpha + grow), b = __ldg(p.beta + grow);
            rd[r].ab = f2_pack(a, a);
            rd[r].bb = f2_pack(b, b);
            sc_row[r] = 0.0f;
        } else {
            rd[r].ab = rd[r].bb = 0;
            sc_row[r] = round_bf16(__ldg(p.scales + grow));
        }
    }
    DecodeConsts kc;
    const uint32_t opaque = (uint32_t)(p.K >> 30);  // == 0; keeps the constants in registers
    kc.neg_magic = f2_pack(-8388608.0f, -8388608.0f);
    kc.round_mag = f2_pack(12582912.0f, 12582912.0f - 19264.0f);
    kc.mul16 = 65536u + opaque;
    kc.wmask = (W4 ? 0x000F000Fu : 0x003F003Fu) ^ opaque;  // one state window / one nibble per half
    kc.wexp = (W4 ? 0x43084308u : 0x43004300u) ^ opaque;   // BF16 128 (W4: and the nibble sign flip)

    float acc[2][NT][4];
#pragma unroll
    for (int t = 0; t < 2; ++t)
#pragma unroll
        for (int n = 0; n < NT; ++n)
#pragma unroll
            for (int q = 0; q < 4; ++q) acc[t][n][q] = 0.0f;

    // per-thread shared-memory offsets inside a stage
    const uint32_t cbase = (uint32_t)(wrow + g) * 128u +
                           (W4 ? 8u * ((uint32_t)tig & 1u) : 4u * (uint32_t)tig);  // code word of row wrow+g
    const uint32_t cswz = ((uint32_t)g << 4) ^ (W4 ? (((uint32_t)tig >> 1) << 4) : 0u);  // 128B swizzle (+ W4 chunk)
    const uint32_t xa_thr = (uint32_t)g * 32u + (uint32_t)tig * 8u;  // B fragment of token g, lane tig
    const uint32_t gs_thr = (uint32_t)(2 * tig) * 32u;               // group sums of token 2*tig
    const uint32_t sc_thr = (uint32_t)(wrow + g) * 32u;              // scales of row wrow+g

    bool ok = true;
    int consumed = 0;  // iterations whose loads this thread has seen land
    for (int it = 0; it < total_iters; ++it) {
        const int slot = it % kStages;
        const int c = it / nst, st = s_begin + it % nst;
        if (producer && it + kStages - 1 < total_iters) {
            // refill the slot every warp released at iteration it-1 (kStages-1 stages of lookahead)
            const int nx = it + kStages - 1;
            if (nx >= kStages) ok = mbar_wait(&empty_bar[nx % kStages], ((nx / kStages) - 1) & 1, p.err);
            if (ok) issue(nx);
        }
        if (!ok || !mbar_wait(&full_bar[slot], (it / kStages) & 1, p.err)) {
            ok = false;
            break;
        }
        consumed = it + 1;
        const uint8_t *base = smem + slot * S::kStageBytes;
        const uint8_t *xa = base + kXaOff + xa_thr;
        const uint8_t *gsb = base + kGsOff + gs_thr;
        if (W4) {
            // per-channel scales; groups beyond K read TMA zero fill (activations 0) and add nothing
            const int Gh = 4 * khalf;
#pragma unroll
            for (int G = 0; G < 4; ++G)
                group_step<NT, W4>(Gh + G, base, cbase, cswz, xa, gsb, sc_row, rd, kc, acc);
        } else if (TMA_SC) {
            // full stage: groups beyond K read TMA zero fill (scale 0, activations 0) and add nothing
            const uint8_t *scb = base + kScOff + sc_thr;
            {
                // this warp's four groups of the stage: offsets are immediates
                const int Gh = 4 * khalf;
                const uint8_t *xah = xa + Gh * 4 * MP * 32;
                const uint8_t *gsh = gsb + Gh * 4;
                const uint8_t *sch = scb + Gh * 4;
                const uint32_t cswz_h = cswz ^ ((uint32_t)Gh << 4);
#pragma unroll
                for (int G = 0; G < 4; ++G) {
                    float sc[4];
                    sc[0] = round_bf16(*reinterpret_cast<const float *>(sch + G * 4));
                    sc[1] = round_bf16(*reinterpret_cast<const float *>(sch + 256 + G * 4));
                    sc[2] = round_bf16(*reinterpret_cast<const float *>(sch + 4096 + G * 4));
                    sc[3] = round_bf16(*reinterpret_cast<const float *>(sch + 4096 + 256 + G * 4));
                    group_step<NT, W4>(G, base, cbase, cswz_h, xah, gsh, sc, rd, kc, acc);
                }
            }
        } else {
            const int g_lim = min(8, ngroups - st * 8);
#pragma unroll 1
            for (int G = 4 * khalf; G < min(g_lim, 4 * khalf + 4); ++G) {
                const int gg = st * 8 + G;
                float sc[4];
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    const int grow = e * p.N + (rvalid[r] ? lrow[r] : 0);
                    sc[r] = round_bf16(__ldg(p.scales + (size_t)grow * ngroups + gg));
                }
                group_step<NT, W4>(G, base, cbase, cswz, xa, gsb, sc, rd, kc, acc);
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty_bar[slot]);

        if (st == s_end - 1) {
            // ---------------- epilogue for token chunk c ----------------
            // the second warp of each row slot hands its partial sums to the first (bounded waits)
            float *red = reinterpret_cast<float *>(smem + kStages * S::kStageBytes) + (wslot * 32 + lane) * (2 * NT * 4);
            if (khalf == 1) {
                if (c > 0 && !mbar_wait(&red_empty, (c - 1) & 1, p.err)) break;
#pragma unroll
                for (int t = 0; t < 2; ++t)
#pragma unroll
                    for (int n = 0; n < NT; ++n)
#pragma unroll
                        for (int q = 0; q < 4; ++q) red[(t * NT + n) * 4 + q] = acc[t][n][q];
                __syncwarp();
                if (lane == 0) mbar_arrive(&red_full);
            } else {
                if (!mbar_wait(&red_full, c & 1, p.err)) break;
#pragma unroll
                for (int t = 0; t < 2; ++t)
#pragma unroll
                    for (int n = 0; n < NT; ++n)
#pragma unroll
                        for (int q = 0; q < 4; ++q) acc[t][n][q] += red[(t * NT + n) * 4 + q];
                __syncwarp();
                if (lane == 0) mbar_arrive(&red_empty);
            }
#pragma unroll
            for (int n = 0; n < NT && khalf == 0; ++n) {
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
    if (producer && !ok) {
        // after a failed wait: let the copies already issued land before the CTA exits (bounded)
        const int issued = min(total_iters, consumed + kStages - 1);
        for (int it = consumed; it < issued; ++it)
            if (!mbar_wait(&full_bar[it % kStages], (it / kStages) & 1, p.err)) break;
    }
}

template <int NT>
cudaError_t launch_nt(const DecodeGemmParams &p, const CUtensorMap &a, const CUtensorMap &b,
                      const CUtensorMap &c, const CUtensorMap &d, int row_blocks, int ksplit, int experts,
                      cudaStream_t s) {
    void (*kern)(CUtensorMap, CUtensorMap, CUtensorMap, CUtensorMap, DecodeGemmParams) = nullptr;
    int smem = 0;
    if constexpr (NT <= 2) {  // W4 keeps at most 16 tokens per chunk (its code tiles are twice as wide)
        if (p.w4) {
            kern = decode_gemm_w2_kernel<NT, false, true>;
            smem = Smem<NT, true>::kTotal;
        }
    }
    if (!p.w4) {
        kern = p.tma_scales ? decode_gemm_w2_kernel<NT, true, false> : decode_gemm_w2_kernel<NT, false, false>;
        smem = Smem<NT, false>::kTotal;
    }
    if (!kern) return cudaErrorInvalidValue;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (err != cudaSuccess) return err;
    dim3 grid(row_blocks, ksplit, experts);
    kern<<<grid, kThreads, smem, s>>>(a, b, c, d, p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode_gemm_w2(const DecodeGemmParams &p, const CUtensorMap &tm_codes,
                                  const CUtensorMap &tm_xa, const CUtensorMap &tm_gs, const CUtensorMap &tm_sc,
                                  int row_blocks, int ksplit, int experts, int nt, cudaStream_t s) {
    if (p.w4 && nt > 2) return cudaErrorInvalidValue;  // W4 tiles hold at most 16 tokens per chunk
    switch (nt) {
        case 1: return launch_nt<1>(p, tm_codes, tm_xa, tm_gs, tm_sc, row_blocks, ksplit, experts, s);
        case 2: return launch_nt<2>(p, tm_codes, tm_xa, tm_gs, tm_sc, row_blocks, ksplit, experts, s);
        case 4: return launch_nt<4>(p, tm_codes, tm_xa, tm_gs, tm_sc, row_blocks, ksplit, experts, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace ccq
