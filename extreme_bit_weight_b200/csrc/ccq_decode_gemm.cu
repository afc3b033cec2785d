// Decode-sized CCQ W2A16 grouped matmul (the GEMV / small-M shapes of the CCQ paper's Table 4 and
// the small-M grouped GEMM of Table 5), sm_100a.
//
// Work unit = one expert x two 128-row halves of its weight x one k range (split-K) x all of the
// expert's tokens (in chunks of 8*NT).  The kernel is persistent: each CTA takes its next unit from
// the launch's work counter (without one: units b, b + gridDim.x, ...), and one producer thread
// streams every 512-column stage of all of them through one shared-memory ring (so the next unit's
// first stages load while the current unit finishes):
//   * the two halves' code bytes, [128 rows][128 B] each, by TMA with the 128-byte swizzle;
//   * their group scales, the activation operand slice in the XA layout (see ccq_kernels.cuh)
//     and its gsq group-sum table;
//   * with a unit's first stage, the unit's per-row alpha/beta (or W4 channel scales).
// Eight consumer warps, one per 16-row slot of both halves (sixteen, two per slot splitting a stage's
// groups, when the scale rows cannot be staged by TMA), decode the bytes in registers and feed them
// straight into mma.sync.m16n8k16 (BF16 in, fp32 accumulate) as the A operand -- weights on the M
// side, tokens on the N side -- so no decoded weight is ever written to memory.  The producer warpgroup gives
// its registers to the consumer warpgroups (setmaxnreg), so the issue work never slows a consumer.
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

#include <algorithm>
#include <utility>

#include "ccq_device.cuh"
#include "ccq_kernels.cuh"

namespace ccq {
namespace {

constexpr int kRowWarps = 8;                       // warps per 16-row slot set (256 rows per CTA)
constexpr int kProducerWarps = 4;                   // one warpgroup; lane 0 of its first warp issues the loads
// Consumer layout.  KH = 2: two warps per row slot, groups 0-3 / 4-7 of a stage, whose sums meet at
// the end of a chunk (640 threads).  KH = 1: one warp per row slot takes all 8 groups (384 threads,
// each consumer with twice the registers).
// Register split: the CTA launches with kLaunchRegs per thread (the most its threads can have), the
// producer warpgroup hands registers back and the consumer warpgroups take them.  The split must
// fit in the launch allocation, or the consumers' increase would wait for registers forever; the
// launcher also checks that the compiled kernel really launches with kLaunchRegs.
template <int KH>
struct Cfg {
    static constexpr int kConsumerWarps = kRowWarps * KH;
    static constexpr int kThreads = (kConsumerWarps + kProducerWarps) * 32;
    static constexpr int kLaunchRegs = KH == 2 ? 96 : 168;
    // the producer warpgroup keeps what the consumers leave: its issue loop (and, KH 1, the scale
    // expanders holding three rows' loads in flight) then runs without spills
    static constexpr int kProducerRegs = KH == 2 ? 32 : 40;
    static constexpr int kConsumerRegs = KH == 2 ? 112 : 232;
    static constexpr int kGroups = 8 / KH;  // groups of a stage per consumer warp
    static_assert(kProducerWarps * 32 * kProducerRegs + kConsumerWarps * 32 * kConsumerRegs <= kThreads * kLaunchRegs,
                  "register split exceeds the launch allocation");
    static_assert(kProducerRegs % 8 == 0 && kConsumerRegs % 8 == 0 && kConsumerRegs <= 256, "setmaxnreg counts");
    static_assert(65536 / kThreads >= kLaunchRegs, "launch registers");
};
constexpr int kCodeTileBytes = 128 * 128;  // [128 rows][128 B] = 8 groups of 16 bytes

// The code rows of the formats with the scale in the codes (EMBK 1: (4,3,2), 8 groups x 22 bytes per
// stage and row; 2: hybrid, 8 x 20), as unswizzled TMA boxes
template <int EMBK>
constexpr int kEmbRow = EMBK == 1 ? 176 : 160;

template <int NT, bool W4 = false, bool Q4 = false, int EMBK = 0>
struct Smem {
    static constexpr int MP = 8 * NT;
    static constexpr int kCodeBytes = EMBK ? 2 * 128 * kEmbRow<EMBK> : (W4 ? 2 : 1) * 2 * kCodeTileBytes;  // both halves
    static constexpr int kXaBytes = 32 * MP * 16 * 2;  // [G*4+i = 32][MP][16] bf16
    static constexpr int kGsBytes = MP * 8 * 16;       // [MP][8] gsq float4 entries
    // [2 halves][128 rows][8 groups] fp32 scales (none for W4; 4-bit scales are expanded into it by
    // the producer warpgroup)
    static constexpr int kScBytes = (W4 || EMBK) ? 0 : 2 * 128 * 8 * 4;
    // [4][128] fp32: alpha A, alpha B, beta A, beta B (W4: scales A, B)
    static constexpr int kRowsBytes = 2048;
    static constexpr int kStageBytes = ((kCodeBytes + kXaBytes + kGsBytes + kScBytes + kRowsBytes) + 1023) & ~1023;
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
// (a & m) | E, E an immediate: the logic op reads two registers
template <uint32_t E>
__device__ __forceinline__ uint32_t and_or_e(uint32_t a, uint32_t m) {
    uint32_t d;
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(a), "r"(m), "n"(E));
    return d;
}

struct RowDecode {
    uint64_t ab;    // {alpha, alpha}: code scale of the row
    uint64_t bb;    // {beta, beta}: code zero-point of the row
};

// The constants of the decode, held in registers: the integer multiply stays a multiply, and the
// window mask is the logic op's register operand while the BF16 exponent pattern is its immediate
// (a logic op that reads three registers, mask and exponent both in registers, was 2-3% slower).
struct DecodeConsts {
    uint64_t neg_magic;  // {-2^23, -2^23}: byte value from its 0x4B0000bb bit pattern
    uint64_t round_mag;  // {1.5*2^23, 1.5*2^23 - 0x4B40}: round to integer; second byte pre-cancels
    uint32_t mul16;      // 65536
    uint32_t wmask;      // 0x003F003F: one 6-bit state window per 16-bit half
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
    R[0] = and_or_e<0x43004300u>(X01 >> 9, k.wmask);
    R[1] = and_or_e<0x43004300u>(X23 >> 9, k.wmask);
    R[2] = and_or_e<0x43004300u>(X01 >> 6, k.wmask);
    R[3] = and_or_e<0x43004300u>(X23 >> 6, k.wmask);
    R[4] = and_or_e<0x43004300u>(X01 >> 3, k.wmask);
    R[5] = and_or_e<0x43004300u>(X23 >> 3, k.wmask);
    R[6] = and_or_e<0x43004300u>(X01, k.wmask);
    R[7] = and_or_e<0x43004300u>(X23, k.wmask);
}

// W4: one 32-bit word = 8 signed 4-bit codes (first of a pair in the low nibble).  Register i holds
// codes i and i+4 as BF16 (128 + (q + 8)) -- the sign bit of each nibble flipped, OR-ed into the
// exponent pattern of 128 -- so one shift and one three-input logic op per register.
__device__ __forceinline__ void decode_word_w4(uint32_t w, uint32_t m4, uint32_t R[4]) {
    constexpr uint32_t x4 = 0x43084308u;  // BF16 128 in both halves, and the nibble sign flip
    asm("lop3.b32 %0, %1, %2, %3, 0x6A;" : "=r"(R[0]) : "r"(w), "r"(m4), "n"(x4));
    asm("lop3.b32 %0, %1, %2, %3, 0x6A;" : "=r"(R[1]) : "r"(w >> 4), "r"(m4), "n"(x4));
    asm("lop3.b32 %0, %1, %2, %3, 0x6A;" : "=r"(R[2]) : "r"(w >> 8), "r"(m4), "n"(x4));
    asm("lop3.b32 %0, %1, %2, %3, 0x6A;" : "=r"(R[3]) : "r"(w >> 12), "r"(m4), "n"(x4));
}

// WINT2-Standard: one 32-bit word = 16 plain 2-bit fields (field i of byte j at bits 2i of the byte),
// laid out like a CCQ word: R[2i] = (128 + f_i(byte0), 128 + f_i(byte1)), R[2i+1] = (.. byte2, ..
// byte3).  Bytes 0,1 and 2,3 are first spread into the two 16-bit halves of one register each.
__device__ __forceinline__ void decode_word_std(uint32_t w, const DecodeConsts &k, uint32_t R[8]) {
    const uint32_t X01 = prmt(w, 0u, 0x4140u), X23 = prmt(w, 0u, 0x4342u);
    R[0] = and_or_e<0x43004300u>(X01, k.wmask);
    R[1] = and_or_e<0x43004300u>(X23, k.wmask);
    R[2] = and_or_e<0x43004300u>(X01 >> 2, k.wmask);
    R[3] = and_or_e<0x43004300u>(X23 >> 2, k.wmask);
    R[4] = and_or_e<0x43004300u>(X01 >> 4, k.wmask);
    R[5] = and_or_e<0x43004300u>(X23 >> 4, k.wmask);
    R[6] = and_or_e<0x43004300u>(X01 >> 6, k.wmask);
    R[7] = and_or_e<0x43004300u>(X23 >> 6, k.wmask);
}

__device__ __forceinline__ void mma_bf16(float *c, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// d = a*b + q: q is the group's starting value, read as one float4 from the gsq table
__device__ __forceinline__ void mma_bf16_q(float *d, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                           uint32_t b1, const float4 &q) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%10,%11,%12,%13};"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(q.x), "f"(q.y), "f"(q.z), "f"(q.w));
}

// fp32 value of bf16_rn(x): one conversion, the BF16 bits land in the high half
__device__ __forceinline__ float round_bf16(float x) { return __uint_as_float(pack_bf16x2(0.0f, x)); }

__device__ __forceinline__ float silu(float z) { return z / (1.0f + __expf(-z)); }

// Shared-memory reads at a base address plus a compile-time offset, written as one instruction
// with an immediate offset (no address arithmetic per read).
template <int OFF>
__device__ __forceinline__ uint32_t lds32_at(uint32_t a) {
    uint32_t v;
    asm volatile("ld.shared.b32 %0, [%1+%2];" : "=r"(v) : "r"(a), "n"(OFF));
    return v;
}
template <int OFF>
__device__ __forceinline__ uint2 lds64_at(uint32_t a) {
    uint2 v;
    asm volatile("ld.shared.v2.b32 {%0, %1}, [%2+%3];" : "=r"(v.x), "=r"(v.y) : "r"(a), "n"(OFF));
    return v;
}
template <int OFF>
__device__ __forceinline__ float4 lds128f_at(uint32_t a) {
    float4 v;
    asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4+%5];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "r"(a), "n"(OFF));
    return v;
}

// f(std::integral_constant<int, 0>{}), ..., f(std::integral_constant<int, N-1>{})
template <class F, int... Is>
__device__ __forceinline__ void static_for_impl(F &&f, std::integer_sequence<int, Is...>) {
    (f(std::integral_constant<int, Is>{}), ...);
}
template <int N, class F>
__device__ __forceinline__ void static_for(F &&f) {
    static_for_impl(f, std::make_integer_sequence<int, N>{});
}

// The mma part of one 64-column group G: 4 state windows x NT token tiles x 2 halves, each token
// tile's accumulators starting from its gsq entry, then the per-group rescale into acc.
//   xs: shared address of this thread's B fragments in the stage (group 0, window 0, tile 0)
//   gs: shared address of this thread's gsq entries in the stage (group 0, tile 0)
template <int NT, int G>
__device__ __forceinline__ void group_mma(const uint32_t (&RA0)[8], const uint32_t (&RA1)[8], const uint32_t (&RB0)[8],
                                          const uint32_t (&RB1)[8], uint32_t xs, uint32_t gs, const float sc[4],
                                          float (&acc)[2][NT][4]) {
    constexpr int MP = 8 * NT;
    static_for<NT>([&](auto nc) {
        constexpr int n = decltype(nc)::value;
        const float4 q = lds128f_at<G * 16 + n * 8 * 128>(gs);
        float cA[4], cB[4];
        static_for<4>([&](auto ic) {
            constexpr int i = decltype(ic)::value;
            const uint2 b = lds64_at<((G * 4 + i) * MP + n * 8) * 32>(xs);
            if constexpr (i == 0) {
                mma_bf16_q(cA, RA0[0], RA1[0], RA0[1], RA1[1], b.x, b.y, q);
                mma_bf16_q(cB, RB0[0], RB1[0], RB0[1], RB1[1], b.x, b.y, q);
            } else {
                mma_bf16(cA, RA0[2 * i], RA1[2 * i], RA0[2 * i + 1], RA1[2 * i + 1], b.x, b.y);
                mma_bf16(cB, RB0[2 * i], RB1[2 * i], RB0[2 * i + 1], RB1[2 * i + 1], b.x, b.y);
            }
        });
        acc[0][n][0] = fmaf(sc[0], cA[0], acc[0][n][0]);
        acc[0][n][1] = fmaf(sc[0], cA[1], acc[0][n][1]);
        acc[0][n][2] = fmaf(sc[1], cA[2], acc[0][n][2]);
        acc[0][n][3] = fmaf(sc[1], cA[3], acc[0][n][3]);
        acc[1][n][0] = fmaf(sc[2], cB[0], acc[1][n][0]);
        acc[1][n][1] = fmaf(sc[2], cB[1], acc[1][n][1]);
        acc[1][n][2] = fmaf(sc[3], cB[2], acc[1][n][2]);
        acc[1][n][3] = fmaf(sc[3], cB[3], acc[1][n][3]);
    });
}

// One 2-bit group (CCQ, or STD plain fields): the four code words of this thread (rows g, g+8 of
// both halves) at ca, ca+1024, and one code tile further.
template <int NT, int G, bool STD = false>
__device__ __forceinline__ void group_w2(uint32_t ca, uint32_t xs, uint32_t gs, const float sc[4],
                                         const RowDecode rd[4], const DecodeConsts &kc, float (&acc)[2][NT][4]) {
    uint32_t RA0[8], RA1[8], RB0[8], RB1[8];
    if constexpr (STD) {
        decode_word_std(lds32_at<0>(ca), kc, RA0);
        decode_word_std(lds32_at<1024>(ca), kc, RA1);
        decode_word_std(lds32_at<kCodeTileBytes>(ca), kc, RB0);
        decode_word_std(lds32_at<kCodeTileBytes + 1024>(ca), kc, RB1);
    } else {
        decode_word(lds32_at<0>(ca), rd[0], kc, RA0);
        decode_word(lds32_at<1024>(ca), rd[1], kc, RA1);
        decode_word(lds32_at<kCodeTileBytes>(ca), rd[2], kc, RB0);
        decode_word(lds32_at<kCodeTileBytes + 1024>(ca), rd[3], kc, RB1);
    }
    group_mma<NT, G>(RA0, RA1, RB0, RB1, xs, gs, sc, acc);
}

// One W4 group: 8 bytes per row (16 nibbles), same row arrangement as W2.
template <int NT, int G>
__device__ __forceinline__ void group_w4(uint32_t ca, uint32_t xs, uint32_t gs, const float sc[4],
                                         const DecodeConsts &kc, float (&acc)[2][NT][4]) {
    uint32_t R[4][8];
    const uint2 q[4] = {lds64_at<0>(ca), lds64_at<1024>(ca), lds64_at<kCodeTileBytes>(ca),
                        lds64_at<kCodeTileBytes + 1024>(ca)};
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        uint32_t t[4];
        decode_word_w4(q[r].x, kc.wmask, t);
        R[r][0] = t[0]; R[r][2] = t[1]; R[r][4] = t[2]; R[r][6] = t[3];
        decode_word_w4(q[r].y, kc.wmask, t);
        R[r][1] = t[0]; R[r][3] = t[1]; R[r][5] = t[2]; R[r][7] = t[3];
    }
    group_mma<NT, G>(R[0], R[1], R[2], R[3], xs, gs, sc, acc);
}

template <int OFF>
__device__ __forceinline__ uint32_t lds16_at(uint32_t a) {
    uint16_t v;
    asm volatile("ld.shared.u16 %0, [%1+%2];" : "=h"(v) : "r"(a), "n"(OFF));
    return v;
}
template <int OFF>
__device__ __forceinline__ uint32_t lds8_at(uint32_t a) {
    uint16_t v;
    asm volatile("ld.shared.u8 %0, [%1+%2];" : "=h"(v) : "r"(a), "n"(OFF));
    return v;
}

// (4,3,2) format: one row's part of group G for this thread (operand order w275_pos): the word of
// codes 4tig..4tig+3, code 16+tig and the extra code's byte, decoded into the eight A-fragment
// registers as BF16 2^(7-T) + u (T = 0, 2, 3: shift-0 states as they are, shift-2 states two bits
// up, shift-4 states moved down by one), and the group's scale bf16(fl32(q * super)), q the low
// nibble of code 21.  rb: the row's code line; o_w = 4 tig, o_b = 16 + tig, o_e = 20 + (tig == 3),
// sh_e: the extra state's shift (4 - 2 tig, or 4 for tig 3).
template <int G>
__device__ __forceinline__ void decode_w275_row(uint32_t rb, uint32_t o_w, uint32_t o_b, uint32_t o_e, uint32_t sh_e,
                                                float sup, uint32_t (&R)[8], float &s) {
    uint32_t W;
    if constexpr ((G & 1) == 0) {
        W = lds32_at<22 * G>(rb + o_w);  // group start 22 G: 4-byte aligned for even G
    } else {
        W = lds16_at<22 * G>(rb + o_w) | (lds16_at<22 * G + 2>(rb + o_w) << 16);
    }
    const uint32_t b16 = lds8_at<22 * G>(rb + o_b);
    const uint32_t ex = lds8_at<22 * G>(rb + o_e);
    const uint32_t q = lds8_at<22 * G + 21>(rb) & 0xFu;
    const uint32_t W8 = W >> 8, W1 = W >> 1, W9 = W >> 9;
    R[0] = and_or(W, 0x000F000Fu, 0x43004300u);   // shift-0 states of bytes 0, 2: 128 + u
    R[1] = and_or(W8, 0x000F000Fu, 0x43004300u);  // bytes 1, 3
    R[2] = and_or(W, 0x003C003Cu, 0x42004200u);   // shift-2 states: 32 + u
    R[3] = and_or(W8, 0x003C003Cu, 0x42004200u);
    R[4] = and_or(W1, 0x00780078u, 0x41804180u);  // shift-4 states, one bit down: 16 + u
    R[5] = and_or(W9, 0x00780078u, 0x41804180u);
    R[6] = and_or(b16 * 0x10001u, 0x003C000Fu, 0x42004300u);  // code 16+tig: shift 0 | shift 2
    R[7] = and_or(((ex >> sh_e) << 16) + (b16 >> 1), 0x000F0078u, 0x43004180u);  // its shift 4 | the extra
    s = round_bf16(__fmul_rn(__uint_as_float(0x4B000000u | q) - 8388608.0f, sup));
}

// Hybrid format: one row's part of group G for this thread (operand order hyb_pos): words 2tig and
// 2tig+1 (one 32-bit load), each state pair of the two words in one register as BF16 2^(7-T) + u (T 4
// for states 0-4 moved down to bit 4, 2 for state 5, 0 for state 6), the extra pair (word 8's states
// at shifts sha and shb, or word 8's state 6 and word 9's first state) at T = 0, and the group's scale
// bf16(fl32(q * super)), q the low 13 bits of word 9.  rb: the row's code line; o_w = 4 tig.
template <int G>
__device__ __forceinline__ void decode_hyb_row(uint32_t rb, uint32_t o_w, uint32_t sha, uint32_t shb, float sup,
                                               uint32_t (&R)[8], float &s) {
    const uint32_t W = lds32_at<20 * G>(rb + o_w);  // group start 20 G: 4-byte aligned
    const uint32_t W89 = lds32_at<20 * G + 16>(rb);  // words 8, 9
    const uint32_t q = (W89 >> 16) & 0x1FFFu;
    R[0] = and_or(W >> 9, 0x00700070u, 0x41004100u);  // state 0 (shift 13): 8 + u
    R[1] = and_or(W >> 7, 0x00700070u, 0x41004100u);  // state 1 (shift 11)
    R[2] = and_or(W >> 5, 0x00700070u, 0x41004100u);  // state 2 (shift 9)
    R[3] = and_or(W >> 2, 0x00700070u, 0x41004100u);  // state 3 (shift 6)
    R[4] = and_or(W, 0x00700070u, 0x41004100u);       // state 4 (shift 4)
    R[5] = and_or(W, 0x001C001Cu, 0x42004200u);       // state 5 (shift 2): 32 + u
    R[6] = and_or(W, 0x00070007u, 0x43004300u);       // state 6 (shift 0): 128 + u
    R[7] = and_or(((W89 >> shb) << 16) | ((W89 >> sha) & 0x7u), 0x00070007u, 0x43004300u);
    s = round_bf16(__fmul_rn(__uint_as_float(0x4B000000u | q) - 8388608.0f, sup));
}

// One work unit of the persistent kernel: expert e, 256-row block rb (two 128-row halves), k split ks.
// A unit walks its stages starting at s_begin + rot (wrapping): units that run at the same time
// then read different 128-byte column slabs of their rows, which spreads the loads over the DRAM
// channels instead of having every CTA hit the same address interleave.
struct Unit {
    int e, ks, seg0, Me, s_begin, s_end, nchunks, localA, localB, nA, nB, rot;
    int phase;  // fused launch: 0 gate/up, 1 down (always 0 otherwise)
};

// The four tensor maps of one matmul: codes, activation operand, gsq table, group scales.
struct MapSet {
    CUtensorMap codes, xa, gs, sc;
};

// Fills U for unit u; false when the unit has no work (an expert without tokens).
template <int MP>
__device__ __forceinline__ bool load_unit(const DecodeGemmParams &p, int u, Unit &U) {
    const int rb = u % p.row_blocks, t = u / p.row_blocks;
    U.ks = t % p.ksplit;
    U.e = t / p.ksplit;
    U.seg0 = p.seg_off ? __ldg(p.seg_off + U.e) : 0;
    U.Me = p.seg_off ? __ldg(p.seg_off + U.e + 1) - U.seg0 : p.M;
    U.s_begin = U.ks * p.stages_per_split;
    U.s_end = min(p.num_stages, U.s_begin + p.stages_per_split);
    if (U.Me <= 0 || U.s_begin >= U.s_end) return false;
    U.nchunks = (U.Me + MP - 1) / MP;
    U.localA = rb * p.row_block_stride;
    U.localB = U.localA + p.half_stride;
    U.nA = max(0, min(128, p.N - U.localA));
    U.nB = max(0, min(128, p.N - U.localB));
    U.rot = u % (U.s_end - U.s_begin);
    U.phase = 0;
    return true;
}

// Unit u of the whole launch: fused launches number the gate/up units first, then the down units.
template <int MP, bool FUSED>
__device__ __forceinline__ bool load_unit_any(const DecodeGemmParams &p, const DecodeGemmParams &p2, int u, Unit &U) {
    if (!FUSED || u < p.units) return load_unit<MP>(p, u, U);
    const bool ok = load_unit<MP>(p2, u - p.units, U);
    U.phase = 1;
    return ok;
}

__device__ __forceinline__ void red_release_gpu_add(int *ptr, int v) {
    asm volatile("red.release.gpu.global.add.s32 [%0], %1;" ::"l"(ptr), "r"(v) : "memory");
}
__device__ __forceinline__ void fence_proxy_async_global() {
    asm volatile("fence.proxy.async.global;" ::: "memory");
}

// 1D bulk copy global -> shared completing on an mbarrier (16-byte aligned, size a multiple of 16)
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_u32(dst)),
                 "l"(src), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ float lds_f32(uint32_t a) {
    float v;
    asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(a));
    return v;
}

// Persistent: each CTA takes units from the work counter (or walks units b, b + gridDim.x, ...); its
// producer streams every stage of every unit through one ring, so the next unit's first stages load
// while this unit finishes.
// FUSED: the launch holds the MoE gate/up units (p, m1) followed by the down units (p2, m2).
// STD: WINT2-Standard plain 2-bit fields (no per-row constants).  KH: consumer layout (Cfg; KH = 2
// only for fp32 scales that TMA does not stage).  EMBK: 1 / 2 = the (4,3,2) / hybrid formats.
template <int NT, bool TMA_SC, bool W4, bool FUSED, bool Q4 = false, bool STD = false, int KH = 2,
          int EMBK = 0>
__global__ void __launch_bounds__(Cfg<KH>::kThreads, 1)
decode_gemm_w2_kernel(const __grid_constant__ MapSet m1, const __grid_constant__ MapSet m2,
                      const __grid_constant__ DecodeGemmParams p, const __grid_constant__ DecodeGemmParams p2) {
    static_assert(KH == 2 || W4 || TMA_SC || Q4 || EMBK, "one warp per row slot needs staged scales");
    static_assert(!Q4 || (KH == 1 && !TMA_SC), "4-bit scales: expanded by the producer warpgroup");
    static_assert(!EMBK || (KH == 1 && !TMA_SC && !W4 && !Q4 && !STD), "embedded scales come with the codes");
    using S = Smem<NT, W4, Q4, EMBK>;
    constexpr bool W275 = EMBK != 0;  // (formats with the scale in the codes: super scale per row, no scale region)
    constexpr int kERow = EMBK ? kEmbRow<EMBK> : 0;
    constexpr int kCodeHalf = EMBK ? 128 * kERow : kCodeTileBytes;  // second half's code tile
    using C = Cfg<KH>;
    constexpr int MP = S::MP;
    constexpr int kStages = S::kStages;
    constexpr int kCodeOff = 0;                       // code tiles of the stage
    constexpr int kXaOff = S::kCodeBytes;             // activation operand slice
    constexpr int kGsOff = S::kCodeBytes + S::kXaBytes;
    constexpr int kScOff = kGsOff + S::kGsBytes;
    constexpr int kRowsOff = kScOff + S::kScBytes;    // per-row constants of the unit (its first stage)
    extern __shared__ uint8_t smem_raw[];
    // 1024-byte aligned start (the 128-byte swizzle repeats every 1024 bytes)
    uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    __shared__ uint64_t full_bar[kStages], empty_bar[kStages], red_full, red_empty;
    __shared__ float epi_gs[FUSED ? kRowWarps : 1][FUSED ? MP : 1];  // fused gate/up epilogue sums
    __shared__ uint64_t epi_bar[2];  // fused gate/up epilogue: the 8 first-half warps meet twice per chunk
    // Q4: the stage each ring slot holds, published by the producer for the scale expanders (warps
    // 1-3 of the producer warpgroup), which complete the slot's full barrier once they have written
    // its fp32 scales
    struct StageDesc {
        int rowA, rowB, nA, nB, st, phase;  // phase < 0: the end marker
    };
    __shared__ StageDesc sdesc[Q4 ? kStages : 1];
    __shared__ uint64_t desc_bar[Q4 ? kStages : 1];
    constexpr int kExpanderWarps = 3;

    const int units = p.units + (FUSED ? p2.units : 0);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    pdl_trigger();  // a dependent grid cannot fit beside this one; it is scheduled as CTAs retire
    if (threadIdx.x == 0) {
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&full_bar[i], Q4 ? 1 + kExpanderWarps : 1);
            if (Q4) mbar_init(&desc_bar[i], 1);
            mbar_init(&empty_bar[i], C::kConsumerWarps);
        }
        mbar_init(&red_full, kRowWarps);
        mbar_init(&red_empty, kRowWarps);
        mbar_init(&epi_bar[0], kRowWarps);
        mbar_init(&epi_bar[1], kRowWarps);
        fence_mbar_init();
        prefetch_tensormap(&m1.codes);
        prefetch_tensormap(&m1.xa);
        prefetch_tensormap(&m1.gs);
        if (TMA_SC) prefetch_tensormap(&m1.sc);
        if (FUSED) {
            prefetch_tensormap(&m2.codes);
            prefetch_tensormap(&m2.xa);
            prefetch_tensormap(&m2.gs);
            prefetch_tensormap(&m2.sc);
        }
    }
    __syncthreads();

    // ---------------- producer (lane 0 of the first producer warp) ----------------
    // Its state lives in shared memory (only thread 0 touches it), so that the consumers' register
    // budget does not pay for it.  pi = next iteration to load (over all of this CTA's units); it
    // goes to ring slot `slot` in ring round `round` and covers token chunk c, 512-column stage st
    // of unit U.
    struct Producer {
        Unit U;
        int u, pi, slot, round, c, i, st;  // i: position of stage st within the chunk's walk
        bool done;
    };
    __shared__ Producer P_;
    Producer &P = P_;
    // Unit descriptors, by unit ordinal modulo kUnitRing, written by the producer before the unit's
    // first load and read by the consumers after that load lands.  The producer runs at most
    // kStages iterations (so at most kStages units) ahead of the slowest consumer, whose unit --
    // epilogue included -- therefore keeps its entry.  After the last unit the producer posts an
    // end marker (e < 0) through one more ring slot that carries no data.
    constexpr int kUnitRing = kStages + 2;
    __shared__ Unit udesc[kUnitRing];
    __shared__ int p_ord;  // producer: ordinal of unit P.U
    // The next unit index.  With a work counter a CTA takes the next unit when it is ready for one,
    // so units of unequal cost (16-stage gate/up against 7-stage down units, experts with two
    // token chunks, experts without tokens) even out across CTAs; the counter hands out every
    // gate/up unit before any down unit, and gate/up units wait on nothing, so the down units'
    // waits always end.  Without one, CTA b takes units b, b + gridDim.x, ...
    auto p_next = [&]() -> int {
        if (p.work) return atomicAdd(p.work, 1);
        const int u = P.u;
        P.u += gridDim.x;
        return u;
    };
    auto p_seek = [&]() {  // the next unit with work
        Unit U;
        int u = p_next();
        while (u < units && !load_unit_any<MP, FUSED>(p, p2, u, U)) u = p_next();
        P.U = U;
        P.done = u >= units;
        if (!P.done) udesc[p_ord++ % kUnitRing] = U;
        P.c = 0;
        P.i = 0;
        P.st = P.done ? 0 : U.s_begin + U.rot;
    };
    auto issue_next = [&]() {
        const Unit U = P.U;
        const int slot = P.slot, c = P.c, i = P.i, st = P.st;
        const DecodeGemmParams &q = (FUSED && U.phase) ? p2 : p;
        const MapSet &m = (FUSED && U.phase) ? m2 : m1;
        uint8_t *base = smem + slot * S::kStageBytes;
        uint64_t *bar = &full_bar[slot];
        const int rowA = U.e * q.N + U.localA, rowB = U.e * q.N + U.localB;
        const bool first = c == 0 && i == 0;
        if (FUSED && U.phase == 1 && first) {
            // the down unit reads h and its gsq table: every gate/up unit of the expert must be done
            if (!wait_counter(q.dep + U.e, q.dep_need, q.err)) {
                P.done = true;  // consumers time out on this stage and stop
                return;
            }
            fence_proxy_async_global();  // the generic-proxy writes of h are visible to TMA from here
        }
        if constexpr (Q4) {
            // the stage this slot will hold, for the scale expanders (the slot is free: the empty
            // barrier was passed before this call)
            sdesc[slot] = StageDesc{rowA, rowB, U.nA, U.nB, st, U.phase};
            mbar_arrive(&desc_bar[slot]);
        }
        const uint32_t row_bytes = (first && !STD) ? (uint32_t)(U.nA + U.nB) * 4u * ((W4 || W275) ? 1u : 2u) : 0u;
        mbar_arrive_expect_tx(bar, S::kTxBytes + ((TMA_SC && !W4) ? S::kScBytes : 0) + row_bytes);
        if (first && !STD) {
            // the unit's per-row constants: alpha, beta (W2), the channel scales (W4) or the super
            // scales ((4,3,2)) of both halves
            const float *ra = W4 ? q.scales : W275 ? q.super_scale : q.alpha;
            if (U.nA) bulk_g2s(base + kRowsOff, ra + rowA, U.nA * 4u, bar);
            if (U.nB) bulk_g2s(base + kRowsOff + 512, ra + rowB, U.nB * 4u, bar);
            if (!W4 && !W275) {
                if (U.nA) bulk_g2s(base + kRowsOff + 1024, q.beta + rowA, U.nA * 4u, bar);
                if (U.nB) bulk_g2s(base + kRowsOff + 1536, q.beta + rowB, U.nB * 4u, bar);
            }
        }
        if (TMA_SC && !W4) {
            uint8_t *sc = base + kScOff;
            tma_load_2d(sc, &m.sc, bar, st * 8, rowA);
            tma_load_2d(sc + S::kScBytes / 2, &m.sc, bar, st * 8, rowB);
        }
        // W2: 128 code bytes per row per stage; W4: 256, as two 128-byte boxes; (4,3,2): one 176-byte box
#pragma unroll
        for (int bx = 0; bx < (W4 ? 2 : 1); ++bx) {
            const int x = W275 ? st * kERow : st * (W4 ? 256 : 128) + bx * 128;
            tma_load_2d(base + kCodeOff + bx * 2 * kCodeTileBytes, &m.codes, bar, x, rowA);
            tma_load_2d(base + kCodeOff + bx * 2 * kCodeTileBytes + kCodeHalf, &m.codes, bar, x, rowB);
        }
        tma_load_3d(base + kXaOff, &m.xa, bar, 0, U.seg0 + c * MP, st * 32);
        tma_load_2d(base + kGsOff, &m.gs, bar, st * 32, U.seg0 + c * MP);
        ++P.pi;
        if (slot + 1 == kStages) {
            P.slot = 0;
            ++P.round;
        } else {
            P.slot = slot + 1;
        }
        if (i + 1 == U.s_end - U.s_begin) {
            P.i = 0;
            P.st = U.s_begin + U.rot;
            if (c + 1 == U.nchunks) {
                p_seek();
            } else {
                P.c = c + 1;
            }
        } else {
            P.i = i + 1;
            P.st = st + 1 == U.s_end ? U.s_begin : st + 1;
        }
    };
    if (warp >= C::kConsumerWarps) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(C::kProducerRegs));
        if (warp == C::kConsumerWarps && lane == 0) {
            // the work counter, the activation operand and its gsq table come from the kernel before
            // (with programmatic launch this grid may start while it still runs); everything the
            // consumers and expanders do follows this thread's loads
            pdl_wait();
            P.u = blockIdx.x;
            P.pi = P.slot = P.round = 0;
            p_ord = 0;
            p_seek();
            bool pok = true;
            while (!P.done) {
                // a slot is free once every consumer warp released its last use (ring round - 1)
                if (P.pi >= kStages && !mbar_wait(&empty_bar[P.slot], (P.round & 1) ^ 1, p.err)) {
                    pok = false;
                    break;
                }
                issue_next();
            }
            if (pok && !(P.pi >= kStages && !mbar_wait(&empty_bar[P.slot], (P.round & 1) ^ 1, p.err))) {
                // end marker: a ring slot without loads whose descriptor stops the consumers (and
                // the scale expanders, which then complete the slot's barrier too)
                Unit end{};
                end.e = -1;
                udesc[p_ord++ % kUnitRing] = end;
                if constexpr (Q4) {
                    sdesc[P.slot] = StageDesc{0, 0, 0, 0, 0, -1};
                    mbar_arrive(&desc_bar[P.slot]);
                }
                mbar_arrive(&full_bar[P.slot]);
            } else {
                pok = false;
            }
            if (!pok) {
                // consumers stopped releasing: let the copies in flight land before exiting (bounded)
                for (int j = max(0, P.pi - kStages); j < P.pi; ++j)
                    if (!mbar_wait(&full_bar[j % kStages], (j / kStages) & 1, p.err)) break;
            }
        } else if (Q4 && warp > C::kConsumerWarps) {
            // scale expanders: for each slot in ring order, the 4-bit scales of the stage's rows ->
            // bf16(fl32(q4 * super[row])) as fp32 in the [half][row][8 groups] layout the consumers
            // read (rounded here once per scale, so the consumers use them as they are)
            const int et = (warp - C::kConsumerWarps - 1) * 32 + lane;  // 0..95
            for (int j = 0;; ++j) {
                const int slot = j % kStages;
                if (!mbar_wait(&desc_bar[slot], (j / kStages) & 1, p.err)) break;
                const StageDesc d = sdesc[slot];
                if (d.phase >= 0) {
                    const DecodeGemmParams &q = (FUSED && d.phase) ? p2 : p;
                    const int qpr = q.K / 128;  // scale bytes per row
                    float *sc = reinterpret_cast<float *>(smem + slot * S::kStageBytes + kScOff);
                    // rows et, et + 96, et + 192 (< 256): every load issued before any is used
                    constexpr int kR = (256 + 32 * kExpanderWarps - 1) / (32 * kExpanderWarps);
                    float sup[kR];
                    uint32_t bytes[kR][4];
#pragma unroll
                    for (int k = 0; k < kR; ++k) {
                        const int idx = et + 32 * kExpanderWarps * k;
                        const int half = idx >> 7, r = idx & 127;
                        const bool live = idx < 256 && r < (half ? d.nB : d.nA);
                        const int row = (half ? d.rowB : d.rowA) + r;
                        sup[k] = live ? __ldg(q.super_scale + row) : 0.0f;
                        const uint8_t *src = q.scale_q4 + (size_t)(live ? row : 0) * qpr;
#pragma unroll
                        for (int b = 0; b < 4; ++b) {
                            const int at = 4 * d.st + b;  // groups 8 st + 2b, 8 st + 2b + 1
                            bytes[k][b] = (live && at < qpr) ? (uint32_t)__ldg(src + at) : 0u;
                        }
                    }
#pragma unroll
                    for (int k = 0; k < kR; ++k) {
                        const int idx = et + 32 * kExpanderWarps * k;
                        if (idx >= 256) break;
                        float v[8];
#pragma unroll
                        for (int b = 0; b < 4; ++b) {
                            v[2 * b] = round_bf16(__fmul_rn((float)(bytes[k][b] & 0xFu), sup[k]));
                            v[2 * b + 1] = round_bf16(__fmul_rn((float)(bytes[k][b] >> 4), sup[k]));
                        }
                        float4 *dst = reinterpret_cast<float4 *>(sc + idx * 8);  // [half][row][8]
                        dst[0] = make_float4(v[0], v[1], v[2], v[3]);
                        dst[1] = make_float4(v[4], v[5], v[6], v[7]);
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&full_bar[slot]);
                if (d.phase < 0) break;
            }
        }
        return;
    }
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(C::kConsumerRegs));

    // ---------------- consumers ----------------
    const int g = lane >> 2, tig = lane & 3;
    const int wslot = warp & (kRowWarps - 1);  // row slot: 16 rows inside each 128-row half
    const int khalf = KH == 2 ? warp / kRowWarps : 0;  // KH 2: 0 = groups 0-3 of every stage, 1 = 4-7
    const int Gh = 4 * khalf;
    const int wrow = wslot * 16;

    DecodeConsts kc;
    const uint32_t opaque = (uint32_t)(p.K >> 30);  // == 0; keeps the constants in registers
    kc.neg_magic = f2_pack(-8388608.0f, -8388608.0f);
    kc.round_mag = f2_pack(12582912.0f, 12582912.0f - 19264.0f);
    kc.mul16 = 65536u + opaque;
    // one state window / one nibble / one 2-bit field per half
    kc.wmask = (W4 ? 0x000F000Fu : STD ? 0x00030003u : 0x003F003Fu) ^ opaque;

    // per-thread shared-memory offsets inside a stage, for this warp's groups Gh..Gh+kGroups-1
    constexpr int kG = C::kGroups;
    uint32_t coff[kG];
#pragma unroll
    for (int G = 0; G < kG; ++G) {
        if constexpr (!W4) {
            // word tig of row wrow+g in 16-byte chunk (Gh+G) ^ g (128-byte swizzle)
            coff[G] = kCodeOff + (uint32_t)(wrow + g) * 128u + 4u * (uint32_t)tig + ((uint32_t)((Gh + G) ^ g) << 4);
        } else {
            // 32 bytes per row and group: this thread's 8 bytes sit in chunk (2G' + tig/2) ^ g of the
            // 128-byte line of box khalf (KH 2; G' = G) or of box G/4 (KH 1; G' = G mod 4)
            const int box = KH == 2 ? khalf : G >> 2, Gb = G & 3;
            coff[G] = kCodeOff + (uint32_t)box * (2u * kCodeTileBytes) + (uint32_t)(wrow + g) * 128u +
                      8u * ((uint32_t)tig & 1u) + ((uint32_t)((2 * Gb + (tig >> 1)) ^ g) << 4);
        }
    }
    const uint32_t xa_thr = kXaOff + (uint32_t)(Gh * 4 * MP * 32) + (uint32_t)g * 32u + (uint32_t)tig * 8u;
    const uint32_t gs_thr = kGsOff + (uint32_t)(2 * tig) * 128u + (uint32_t)Gh * 16u;  // token pair 2tig, 2tig+1
    const uint32_t sc_thr = kScOff + (uint32_t)(wrow + g) * 32u + (uint32_t)Gh * 4u;   // row wrow+g, groups Gh..
    const uint32_t rows_thr = kRowsOff + (uint32_t)(wrow + g) * 4u;                     // row wrow+g of half A
    const uint32_t sbase = smem_u32(smem);
    // (4,3,2): this thread's four code lines (rows g, g+8 of both halves) and byte offsets
    uint32_t w_row[4] = {0, 0, 0, 0};
#pragma unroll
    for (int r = 0; r < 4; ++r)
        w_row[r] = kCodeOff + (uint32_t)(r >> 1) * (uint32_t)kCodeHalf + (uint32_t)(wrow + g + 8 * (r & 1)) * kERow;
    const uint32_t w_ow = 4u * (uint32_t)tig, w_ob = 16u + (uint32_t)tig, w_oe = 20u + (tig == 3 ? 1u : 0u);
    const uint32_t w_she = tig < 3 ? 4u - 2u * (uint32_t)tig : 4u;
    // hybrid: the extra pair's shifts in words 8-9 (word 8's states 2tig, 2tig+1; tig 3: its state 6 and
    // word 9's state 0, at bit 16 + 13)
    const uint32_t h_sha = tig == 0 ? 13u : tig == 1 ? 9u : tig == 2 ? 4u : 0u;
    const uint32_t h_shb = tig == 0 ? 11u : tig == 1 ? 6u : tig == 2 ? 2u : 29u;

    bool ok = true;
    int it = 0, slot = 0, round = 0, cc = 0;  // iteration (over all units), ring slot and round, chunk count
    int ec = 0;                               // fused gate/up chunks done (epilogue meeting parity)
    RowDecode rd[4];
    float sc_row[4];  // W4: per-channel scales, bf16-rounded
    float acc[2][NT][4];
#pragma unroll
    for (int t = 0; t < 2; ++t)
#pragma unroll
        for (int n = 0; n < NT; ++n)
#pragma unroll
            for (int q = 0; q < 4; ++q) acc[t][n][q] = 0.0f;
    // walk: unit ordinal cu, token chunk c, position i of stage st in the chunk's rotated walk
    int cu = 0, c = 0, i = 0, st = 0;
    for (;;) {
        if (!ok || !mbar_wait(&full_bar[slot], round & 1, p.err)) {
            ok = false;
            break;
        }
        const Unit &U = udesc[cu % kUnitRing];  // written before this unit's first load was issued
        if (U.e < 0) break;                     // the producer's end marker
        const DecodeGemmParams &pq = (FUSED && U.phase) ? p2 : p;
        const bool first = c == 0 && i == 0;
        if (first) st = U.s_begin + U.rot;
        const uint32_t sb = sbase + (uint32_t)(slot * S::kStageBytes);
        if (first && !STD) {
            // this unit's per-row constants arrived with its first stage
            const uint32_t ra = sb + rows_thr;
            const float r0 = lds_f32(ra), r1 = lds_f32(ra + 32), r2 = lds_f32(ra + 512), r3 = lds_f32(ra + 544);
            if constexpr (W275) {
                sc_row[0] = r0; sc_row[1] = r1; sc_row[2] = r2; sc_row[3] = r3;  // super scales
            } else if constexpr (!W4) {
                const float b0 = lds_f32(ra + 1024), b1 = lds_f32(ra + 1056), b2 = lds_f32(ra + 1536),
                            b3 = lds_f32(ra + 1568);
                rd[0].ab = f2_pack(r0, r0); rd[0].bb = f2_pack(b0, b0);
                rd[1].ab = f2_pack(r1, r1); rd[1].bb = f2_pack(b1, b1);
                rd[2].ab = f2_pack(r2, r2); rd[2].bb = f2_pack(b2, b2);
                rd[3].ab = f2_pack(r3, r3); rd[3].bb = f2_pack(b3, b3);
            } else {
                sc_row[0] = round_bf16(r0); sc_row[1] = round_bf16(r1);
                sc_row[2] = round_bf16(r2); sc_row[3] = round_bf16(r3);
            }
        }
        if (W4) {
            // per-channel scales; groups beyond K read TMA zero fill (activations 0) and add nothing
            const uint32_t xs = sb + xa_thr, gs = sb + gs_thr;
            static_for<kG>([&](auto Gc) {
                constexpr int G = decltype(Gc)::value;
                group_w4<NT, G>(sb + coff[G], xs, gs, sc_row, kc, acc);
            });
        } else if (W275) {
            // (4,3,2) / hybrid: all 8 groups of the stage; each group's scale comes with its codes.  Groups
            // beyond K read zero codes (scale 0) and zero activations and add nothing.
            const uint32_t xs = sb + xa_thr, gs = sb + gs_thr;
            static_for<8>([&](auto Gc) {
                constexpr int G = decltype(Gc)::value;
                uint32_t RA0[8], RA1[8], RB0[8], RB1[8];
                float sc[4];
                if constexpr (EMBK == 1) {
                    decode_w275_row<G>(sb + w_row[0], w_ow, w_ob, w_oe, w_she, sc_row[0], RA0, sc[0]);
                    decode_w275_row<G>(sb + w_row[1], w_ow, w_ob, w_oe, w_she, sc_row[1], RA1, sc[1]);
                    decode_w275_row<G>(sb + w_row[2], w_ow, w_ob, w_oe, w_she, sc_row[2], RB0, sc[2]);
                    decode_w275_row<G>(sb + w_row[3], w_ow, w_ob, w_oe, w_she, sc_row[3], RB1, sc[3]);
                } else {
                    decode_hyb_row<G>(sb + w_row[0], w_ow, h_sha, h_shb, sc_row[0], RA0, sc[0]);
                    decode_hyb_row<G>(sb + w_row[1], w_ow, h_sha, h_shb, sc_row[1], RA1, sc[1]);
                    decode_hyb_row<G>(sb + w_row[2], w_ow, h_sha, h_shb, sc_row[2], RB0, sc[2]);
                    decode_hyb_row<G>(sb + w_row[3], w_ow, h_sha, h_shb, sc_row[3], RB1, sc[3]);
                }
                group_mma<NT, G>(RA0, RA1, RB0, RB1, xs, gs, sc, acc);
            });
        } else if (TMA_SC || Q4) {
            // full stage (scales staged by TMA, or expanded from 4 bits by the producer warpgroup):
            // groups beyond K read zero scales and activations and add nothing
            // this warp's groups, four at a time: groups 4Q..4Q+3 sit 16Q bytes further in the scale
            // rows, 16 MP 32 Q bytes further in the XA slice, 64Q in the gsq entries, and in the
            // 128-byte-swizzled chunk (G ^ g) ^ 4Q, i.e. with code address bit 6 flipped
            auto quad = [&](int Q) {
                const uint32_t sa = sb + sc_thr + 16u * (uint32_t)Q;
                const uint32_t xs = sb + xa_thr + (uint32_t)(Q * 16 * MP * 32), gs = sb + gs_thr + 64u * (uint32_t)Q;
                const uint32_t cflip = (uint32_t)Q << 6;
                const float4 s0 = lds128f_at<0>(sa);
                const float4 s1 = lds128f_at<256>(sa);
                const float4 s2 = lds128f_at<4096>(sa);
                const float4 s3 = lds128f_at<4096 + 256>(sa);
                const float v0[4] = {s0.x, s0.y, s0.z, s0.w}, v1[4] = {s1.x, s1.y, s1.z, s1.w};
                const float v2[4] = {s2.x, s2.y, s2.z, s2.w}, v3[4] = {s3.x, s3.y, s3.z, s3.w};
                static_for<4>([&](auto Gc) {
                    constexpr int G = decltype(Gc)::value;
                    // (4-bit scales arrive rounded by the expanders)
                    const float sc[4] = {Q4 ? v0[G] : round_bf16(v0[G]), Q4 ? v1[G] : round_bf16(v1[G]),
                                         Q4 ? v2[G] : round_bf16(v2[G]), Q4 ? v3[G] : round_bf16(v3[G])};
                    group_w2<NT, G, STD>(sb + (coff[G] ^ cflip), xs, gs, sc, rd, kc, acc);
                });
            };
            if constexpr (NT >= 4) {
                // (4 token tiles: one quad's code at a time keeps the accumulators in registers)
#pragma unroll 1
                for (int Q = 0; Q < kG / 4; ++Q) quad(Q);
            } else {
                static_for<kG / 4>([&](auto Qc) { quad(decltype(Qc)::value); });
            }
        } else {
            const int ngroups = pq.K / 64;
            const int g_lim = min(kG, ngroups - st * 8 - Gh);
#pragma unroll 1
            for (int G = 0; G < g_lim; ++G) {
                const int gg = st * 8 + Gh + G;
                float sc[4];
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    // local row of row r (g, g+8 of half A, then of half B); rows past N read row 0
                    const int lr = (r < 2 ? U.localA : U.localB) + wrow + g + 8 * (r & 1);
                    const int grow = U.e * pq.N + (lr < pq.N ? lr : 0);
                    sc[r] = round_bf16(__ldg(pq.scales + (size_t)grow * ngroups + gg));
                }
                const uint32_t ca = kCodeOff + (uint32_t)(wrow + g) * 128u + 4u * (uint32_t)tig +
                                    ((uint32_t)((Gh + G) ^ g) << 4);
                group_w2<NT, 0, STD>(sb + ca, sb + xa_thr + G * 4 * MP * 32, sb + gs_thr + G * 16, sc, rd, kc,
                                     acc);
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty_bar[slot]);
        if (++slot == kStages) { slot = 0; ++round; }
        ++it;
        st = st + 1 == U.s_end ? U.s_begin : st + 1;
        if (++i < U.s_end - U.s_begin) continue;
        i = 0;

        // ---------------- epilogue for token chunk c ----------------
        // KH 2: the second warp of each row slot hands its partial sums to the first (bounded waits)
        float *red = reinterpret_cast<float *>(smem + kStages * S::kStageBytes) + (wslot * 32 + lane) * (2 * NT * 4);
        if (KH == 1) {
            // one warp per row slot: its sums are complete
        } else if (khalf == 1) {
            if (cc > 0 && !mbar_wait(&red_empty, (cc - 1) & 1, p.err)) {
                ok = false;
                break;
            }
#pragma unroll
            for (int t = 0; t < 2; ++t)
#pragma unroll
                for (int n = 0; n < NT; ++n)
#pragma unroll
                    for (int q = 0; q < 4; ++q) red[(t * NT + n) * 4 + q] = acc[t][n][q];
            __syncwarp();
            if (lane == 0) mbar_arrive(&red_full);
        } else {
            if (!mbar_wait(&red_full, cc & 1, p.err)) {
                ok = false;
                break;
            }
#pragma unroll
            for (int t = 0; t < 2; ++t)
#pragma unroll
                for (int n = 0; n < NT; ++n)
#pragma unroll
                    for (int q = 0; q < 4; ++q) acc[t][n][q] += red[(t * NT + n) * 4 + q];
            __syncwarp();
            if (lane == 0) mbar_arrive(&red_empty);
        }
        ++cc;
        // local rows (within the expert) of the four rows this thread decoded
        const int lrow[4] = {U.localA + wrow + g, U.localA + wrow + g + 8, U.localB + wrow + g,
                             U.localB + wrow + g + 8};
        const bool rvalid[4] = {wrow + g < U.nA, wrow + g + 8 < U.nA, wrow + g < U.nB, wrow + g + 8 < U.nB};
        float hsum[NT][2];  // fused gate/up: sums of the stored BF16 h over this thread's two rows
#pragma unroll
        for (int n = 0; n < NT; ++n) hsum[n][0] = hsum[n][1] = 0.0f;
#pragma unroll
        for (int n = 0; n < NT && khalf == 0; ++n) {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int tok = c * MP + n * 8 + 2 * tig + (q & 1);
                if (tok >= U.Me) continue;
                const int hr = q >> 1;  // 0: row g, 1: row g+8
                if (pq.mode == EPI_GATEUP) {
                    const int r = lrow[hr];  // gate row; its up row is r + half_stride
                    if (r >= pq.I) continue;
                    const float h = silu(acc[0][n][q]) * acc[1][n][q];
                    const size_t pr = (size_t)(U.seg0 + tok);
                    const uint16_t hb = float_to_bf16_bits(h);
                    reinterpret_cast<uint16_t *>(pq.out)[xa_index_perm(pr, (size_t)r, (size_t)pq.h_P, pq.h_perm)] = hb;
                    if constexpr (FUSED) {
                        // (4,3,2) or hybrid down weight: each column carries its own level offset
                        const float lw = pq.h_perm ? perm_level(pq.h_perm, r & 63) : 1.0f;
                        hsum[n][q & 1] += lw * bf16_bits_to_float(hb);
                    }
                    continue;
                }
#pragma unroll
                for (int t = 0; t < 2; ++t) {
                    const int r = lrow[2 * t + hr];
                    if (!rvalid[2 * t + hr]) continue;
                    const float v = acc[t][n][q];
                    const size_t m = (size_t)(U.seg0 + tok);
                    if (pq.mode == EPI_PARTIAL_F32) {
                        reinterpret_cast<float *>(pq.out)[(size_t)U.ks * pq.out_split_stride + m * pq.out_ld + r] = v;
                    } else if (pq.mode == EPI_BF16) {
                        reinterpret_cast<uint16_t *>(pq.out)[m * pq.out_ld + r] = float_to_bf16_bits(v);
                    } else {  // EPI_DOWN
                        reinterpret_cast<float *>(pq.out)[m * pq.out_ld + r] = __ldg(pq.rw + m) * v;
                    }
                }
            }
        }
        if constexpr (FUSED) {
            if (U.phase == 0 && khalf == 0) {
                // The down operand's gsq table for this chunk's tokens over the unit's two 64-column
                // groups of h (row slots 0-3 and 4-7): per warp, sum the 16 rows over g in a fixed
                // shuffle order; then the four row slots of a group, in slot order.
#pragma unroll
                for (int n = 0; n < NT; ++n)
#pragma unroll
                    for (int j = 0; j < 2; ++j) {
                        float v = hsum[n][j];
                        v += __shfl_xor_sync(0xFFFFFFFFu, v, 4);
                        v += __shfl_xor_sync(0xFFFFFFFFu, v, 8);
                        v += __shfl_xor_sync(0xFFFFFFFFu, v, 16);
                        if (g == 0) epi_gs[wslot][n * 8 + 2 * tig + j] = v;
                    }
                // bounded meeting points (a plain barrier could wait forever for a warp that left
                // after a timed-out wait)
                __syncwarp();
                if (lane == 0) mbar_arrive(&epi_bar[0]);
                if (!mbar_wait(&epi_bar[0], ec & 1, p.err)) {
                    ok = false;
                    break;
                }
                if ((wslot & 3) == 0 && lane < MP / 2) {
                    const int t0 = c * MP + 2 * lane;  // token pair (t0, t0 + 1) of the expert
                    if (t0 < U.Me) {
                        float s0 = 0.0f, s1 = 0.0f;
#pragma unroll
                        for (int w = 0; w < 4; ++w) {
                            s0 += epi_gs[wslot + w][2 * lane];
                            s1 += epi_gs[wslot + w][2 * lane + 1];
                        }
                        if (t0 + 1 >= U.Me) s1 = 0.0f;
                        const int G = U.localA / 64 + (wslot >> 2);
                        const float L = pq.h_perm ? 1.0f : pq.fuse_level;  // (perm 1: levels applied per column)
                        reinterpret_cast<float4 *>(pq.fuse_gsq)[(size_t)(U.seg0 + t0) * pq.fuse_gsq_ld + G] =
                            make_float4(L * s0, L * s1, L * s0, L * s1);
                    }
                }
                // epi_gs reusable, and every store of the chunk issued before the publication below
                __syncwarp();
                if (lane == 0) mbar_arrive(&epi_bar[1]);
                if (!mbar_wait(&epi_bar[1], ec & 1, p.err)) {
                    ok = false;
                    break;
                }
                ++ec;
                if (c + 1 == U.nchunks && warp == 0 && lane == 0) {
                    // publish the finished unit: its h and gsq writes, ordered by the barrier above
                    __threadfence();
                    fence_proxy_async_global();
                    red_release_gpu_add(pq.dep + U.e, 1);
                }
            }
        }
#pragma unroll
        for (int t = 0; t < 2; ++t)
#pragma unroll
            for (int n = 0; n < NT; ++n)
#pragma unroll
                for (int q = 0; q < 4; ++q) acc[t][n][q] = 0.0f;
        if (++c == U.nchunks) {
            c = 0;
            ++cu;
        }
    }
}

using DecodeKernel = void (*)(MapSet, MapSet, DecodeGemmParams, DecodeGemmParams);

// Checks the kernel's launch register count (the register split assumes kLaunchRegs), sets its
// dynamic shared memory and returns the CTAs that fit per SM (once per kernel and device).
template <int KH>
cudaError_t prepare_kernel(DecodeKernel kern, int smem, int *per_sm = nullptr) {
    return kernel_setup(reinterpret_cast<const void *>(kern), smem, Cfg<KH>::kThreads, Cfg<KH>::kLaunchRegs, per_sm);
}

// Consumer layout for the fp32-scale 2-bit kernels (CCQ and STD); 4-bit scales, the embedded-scale
// formats and W4 always take KH = 1; unstaged fp32 scales (rows whose scale pitch is not a multiple of
// 16 bytes) KH = 2.
constexpr int kFastKH = 1;

int device_sms(cudaError_t &err) {
    int dev = 0, sms = 0;
    err = cudaGetDevice(&dev);
    if (err == cudaSuccess) err = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    return sms;
}

template <int NT>
cudaError_t launch_nt(const DecodeGemmParams &p, const CUtensorMap &a, const CUtensorMap &b,
                      const CUtensorMap &c, const CUtensorMap &d, int row_blocks, int ksplit, int experts,
                      cudaStream_t s) {
    DecodeKernel kern = nullptr;
    int smem = 0, kh = 2;
    if constexpr (NT <= 2) {  // W4 keeps at most 16 tokens per chunk (its code tiles are twice as wide)
        if (p.w4) {
            kern = decode_gemm_w2_kernel<NT, false, true, false, false, false, 1>;
            kh = 1;
            smem = Smem<NT, true>::kTotal;
        }
    }
    if (p.emb == 1 || p.emb == 2) {
        kern = p.emb == 1 ? decode_gemm_w2_kernel<NT, false, false, false, false, false, 1, 1>
                          : decode_gemm_w2_kernel<NT, false, false, false, false, false, 1, 2>;
        kh = 1;
        smem = p.emb == 1 ? Smem<NT, false, false, 1>::kTotal : Smem<NT, false, false, 2>::kTotal;
    } else if (!p.w4 && p.std2) {
        kern = p.tma_scales ? decode_gemm_w2_kernel<NT, true, false, false, false, true, kFastKH>
                            : decode_gemm_w2_kernel<NT, false, false, false, false, true>;
        kh = p.tma_scales ? kFastKH : 2;
        smem = Smem<NT, false>::kTotal;
    } else if (!p.w4 && p.q4) {
        kern = decode_gemm_w2_kernel<NT, false, false, false, true, false, 1>;
        kh = 1;
        smem = Smem<NT, false, true>::kTotal;
    } else if (!p.w4) {
        kern = p.tma_scales ? decode_gemm_w2_kernel<NT, true, false, false, false, false, kFastKH>
                            : decode_gemm_w2_kernel<NT, false, false, false>;
        kh = p.tma_scales ? kFastKH : 2;
        smem = Smem<NT, false>::kTotal;
    }
    if (!kern) return cudaErrorInvalidValue;
    cudaError_t err = kh == 1 ? prepare_kernel<1>(kern, smem) : prepare_kernel<2>(kern, smem);
    if (err != cudaSuccess) return err;
    const int threads = kh == 1 ? Cfg<1>::kThreads : Cfg<2>::kThreads;
    DecodeGemmParams q = p;
    q.row_blocks = row_blocks;
    q.ksplit = ksplit;
    q.units = row_blocks * ksplit * experts;
    if (q.units <= 0) return cudaSuccess;
    const int sms = device_sms(err);
    if (err != cudaSuccess) return err;
    MapSet m{a, b, c, d};
    return launch_pdl(kern, dim3(std::min(q.units, sms)), dim3(threads), (size_t)smem, s, m, m, q, q);
}

template <int NT>
cudaError_t launch_fused_nt(const DecodeGemmParams &p1, const MapSet &m1, int row_blocks1, const DecodeGemmParams &p2,
                            const MapSet &m2, int row_blocks2, int experts, cudaStream_t s) {
    // fp32 group scales staged by TMA, or 4-bit scales read by the consumers (both projections alike)
    DecodeKernel kern = p1.emb == 1 ? decode_gemm_w2_kernel<NT, false, false, true, false, false, 1, 1>
                        : p1.emb == 2 ? decode_gemm_w2_kernel<NT, false, false, true, false, false, 1, 2>
                        : p1.q4     ? decode_gemm_w2_kernel<NT, false, false, true, true, false, 1>
                        : p1.std2   ? decode_gemm_w2_kernel<NT, true, false, true, false, true, kFastKH>
                                    : decode_gemm_w2_kernel<NT, true, false, true, false, false, kFastKH>;
    const int kh = (p1.q4 || p1.emb) ? 1 : kFastKH;
    const int smem = p1.emb == 1 ? Smem<NT, false, false, 1>::kTotal
                     : p1.emb == 2 ? Smem<NT, false, false, 2>::kTotal
                     : p1.q4     ? Smem<NT, false, true>::kTotal
                                 : Smem<NT, false>::kTotal;
    int per_sm = 0;
    cudaError_t err = kh == 1 ? prepare_kernel<1>(kern, smem, &per_sm) : prepare_kernel<2>(kern, smem, &per_sm);
    if (err != cudaSuccess) return err;
    const int threads = kh == 1 ? Cfg<1>::kThreads : Cfg<2>::kThreads;
    DecodeGemmParams q1 = p1, q2 = p2;
    q1.row_blocks = row_blocks1;
    q1.ksplit = 1;
    q1.units = row_blocks1 * experts;
    q2.row_blocks = row_blocks2;
    q2.ksplit = 1;
    q2.units = row_blocks2 * experts;
    q2.dep_need = row_blocks1;
    if (q1.units + q2.units <= 0) return cudaSuccess;
    // down units wait for other CTAs' gate/up units: every CTA must be resident at once, which a
    // cooperative launch guarantees (or refuses)
    if (per_sm < 1) return cudaErrorCooperativeLaunchTooLarge;
    const int sms = device_sms(err);
    if (err != cudaSuccess) return err;
    const int grid = std::min(q1.units + q2.units, sms * per_sm);
    MapSet a = m1, b = m2;
    void *args[] = {&a, &b, &q1, &q2};
    err = cudaLaunchCooperativeKernel(reinterpret_cast<const void *>(kern), dim3(grid), dim3(threads), args, smem, s);
    if (err != cudaSuccess) return err;
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

cudaError_t launch_decode_moe_fused(const DecodeGemmParams &p1, const CUtensorMap &a1, const CUtensorMap &b1,
                                    const CUtensorMap &c1, const CUtensorMap &d1, int row_blocks1,
                                    const DecodeGemmParams &p2, const CUtensorMap &a2, const CUtensorMap &b2,
                                    const CUtensorMap &c2, const CUtensorMap &d2, int row_blocks2, int experts,
                                    int nt, cudaStream_t s) {
    const bool fp32_sc = !p1.q4 && !p2.q4 && p1.tma_scales && p2.tma_scales, q4_sc = p1.q4 && p2.q4;
    const bool emb_both = p1.emb != 0 && p1.emb == p2.emb;
    if (p1.w4 || p2.w4 || !(fp32_sc || q4_sc || emb_both) || p1.std2 != p2.std2 || p1.emb != p2.emb ||
        (q4_sc && p1.std2) || p1.mode != EPI_GATEUP || p2.mode != EPI_DOWN ||
        !p1.dep || !p2.dep || !p1.fuse_gsq)
        return cudaErrorInvalidValue;
    const MapSet m1{a1, b1, c1, d1}, m2{a2, b2, c2, d2};
    switch (nt) {
        case 1: return launch_fused_nt<1>(p1, m1, row_blocks1, p2, m2, row_blocks2, experts, s);
        case 2: return launch_fused_nt<2>(p1, m1, row_blocks1, p2, m2, row_blocks2, experts, s);
        case 4: return launch_fused_nt<4>(p1, m1, row_blocks1, p2, m2, row_blocks2, experts, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace ccq
