// Prefill-sized CCQ W2A16 grouped matmul on the 5th-generation tensor cores (tcgen05 + TMEM),
// sm_100a.  The grouped GEMM of the CCQ paper's Table 5 at prefill batch sizes, and the dense
// large-M shape.
//
// Tile: 128*MT tokens x 256 weight rows (two 128-row halves of the weight) x K in steps of one
// 64-column group.  Persistent CTAs walk a device-built list of (expert, token-tile) entries
// crossed with the weight's row tiles.  Warp roles:
//   warp 0      TMA producer: activation tiles ([128 tok][64] BF16, 128B swizzle) and code tiles
//               ([128 rows][64 B], 64B swizzle, 4 groups per load)
//   warp 1      TMEM allocation and the single MMA-issuing thread (tcgen05.mma kind::f16,
//               M=128, N=256, K=16, fp32 accumulators in TMEM)
//   warps 2-17  decoders: two threads per weight row of the tile; each decodes its half of the
//               row's code bytes of the group (CCQ §3.3 Eq. 1 inverted / §3.5 Algorithm 3: fp32
//               FMA, ties-to-even rounding, Table 1 shifts) to BF16 w = bf16((u - 32) * bf16(scale))
//               and stores them as the MMA B operand in the canonical K-major 128B-swizzled
//               shared-memory layout
//   warps 18-21 epilogue: tcgen05.ld of the accumulators; SiLU(gate)*up, routing-weight scaling or
//               BF16 conversion; stores to global memory
// Column order: within every 16-column block the decoders emit the 16 weights of one 4-byte word
// window-major (position 4i + j holds state window i of byte j, i.e. column 4j + i), so the
// activation operand is stored with the same permutation (see pack_xt).  Every column is then
// multiplied by its own weight; only the order of the k sum inside a block differs.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "ccq_device.cuh"
#include "ccq_kernels.cuh"

namespace ccq {
namespace {

constexpr int kDecWarps = 16;  // two threads per weight row of the 256-row tile
constexpr int kEpiWarps = 4;
constexpr int kTcThreads = (2 + kDecWarps + kEpiWarps) * 32;  // 704
// Ring depths.  Activation stages: 4 with 128-token tiles, 3 with 256-token tiles (2 for the
// embedded-scale formats, whose code ring is wider), so that enough activation loads are in flight
// to cover their latency.  Decoded-weight stages: 4 / 3 (3 with 128-token tiles of the
// embedded-scale formats), so that the decoders can run ahead of the MMA.
template <int MT, int EMB>
constexpr int kSAof = MT == 1 ? 4 : (EMB ? 2 : 3);
template <int MT, int EMB>
constexpr int kSBof = MT == 1 ? (EMB ? 3 : 4) : 3;
constexpr int kSC = 2;   // code stages (4 groups each)
constexpr int kATile = 128 * 64 * 2;   // 16 KB per 128-token sub-tile
constexpr int kBTile = 256 * 64 * 2;   // 32 KB
// Code bytes per row in one code stage (4 groups; W4: 2): 64 for CCQ, W4 and STD.  The formats with
// the scale in the redundant bits (EMB) have 22 (kind 1) or 20 (kind 2) bytes per group: a kind-1
// stage's 88 bytes start at an 8-byte boundary every other stage, and TMA boxes start at 16-byte
// boundaries, so its box is 112 bytes wide, starting at the 16-byte boundary at or below.
template <int EMB>
constexpr int kCRowOf = EMB == 1 ? 112 : EMB == 2 ? 80 : 64;
template <int EMB>
constexpr int kCTileOf = 2 * 128 * kCRowOf<EMB>;  // two 128-row halves

template <int MT, int EMB = 0>
struct TcSmem {
    static constexpr int kA = kSAof<MT, EMB> * MT * kATile;
    static constexpr int kB = kSBof<MT, EMB> * kBTile;
    static constexpr int kC = kSC * kCTileOf<EMB>;
    static constexpr int kTotal = kA + kB + kC + 1024;
    static_assert(kTotal + 512 <= 227 * 1024, "shared memory per CTA");
};

__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t saddr) {
    uint64_t d = (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)1 << 16;             // leading byte offset (unused for swizzled K-major)
    d |= (uint64_t)(1024 >> 4) << 32;   // stride byte offset: one 8-row x 128 B swizzle atom
    d |= (uint64_t)1 << 46;             // descriptor version for sm_100
    d |= (uint64_t)2 << 61;             // 128-byte swizzle
    return d;
}

// kind::f16 instruction descriptor: fp32 accumulate, BF16 A and B, both K-major, M=128, N=256.
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | ((256u >> 3) << 17) | ((128u >> 4) << 24);

__device__ __forceinline__ void mma_bf16_ss(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a), "l"(b), "r"(kIdesc), "r"(accumulate));
}

__device__ __forceinline__ void mma_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t *r) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t *r) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}
__device__ __forceinline__ uint32_t bsub2(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}
__device__ __forceinline__ uint32_t bmul2(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

__device__ __forceinline__ uint64_t pk2(uint32_t lo, uint32_t hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "r"(lo), "r"(hi));
    return r;
}
__device__ __forceinline__ void upk2(uint64_t v, uint32_t &lo, uint32_t &hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=r"(lo), "=r"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t fadd2(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t ffma2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ uint64_t fpk2(float lo, float hi) { return pk2(__float_as_uint(lo), __float_as_uint(hi)); }

// Per-row and per-thread constants of the W2 decode, held in registers.
struct RowCodeParams {
    uint64_t ab, bb;         // {alpha, alpha}, {beta, beta}
    uint64_t neg, rnd;       // {-2^23, -2^23}; {1.5*2^23, 1.5*2^23 - 0x4B40} (second byte pre-cancels)
    uint32_t mask;           // the state-window mask in a register (0x003F003F; STD: 0x00030003)
};

// (a & m) | E in one logic op: the mask m in a register, the exponent pattern E its immediate
template <uint32_t E>
__device__ __forceinline__ uint32_t and_or_e(uint32_t a, uint32_t m) {
    uint32_t d;
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(a), "r"(m), "n"(E));
    return d;
}

// One 4-byte word of a row -> 16 BF16 weights (u - 32) * s in window-major order, as 8 registers:
// out[2i], out[2i+1] = window i of bytes (0,1) and (2,3).  Byte value, q*alpha + beta (one fp32
// rounding) and the half-to-even rounding to an integer run two bytes per f32x2 instruction.
__device__ __forceinline__ void decode_word_bf16(uint32_t w, const RowCodeParams &rp, uint32_t s2, uint32_t out[8]) {
    const uint32_t magic = 0x4B000000u;
    uint64_t c01 = pk2(prmt(w, magic, 0x7650u), prmt(w, magic, 0x7651u));
    uint64_t c23 = pk2(prmt(w, magic, 0x7652u), prmt(w, magic, 0x7653u));
    c01 = fadd2(c01, rp.neg);
    c23 = fadd2(c23, rp.neg);
    c01 = fadd2(ffma2(c01, rp.ab, rp.bb), rp.rnd);
    c23 = fadd2(ffma2(c23, rp.ab, rp.bb), rp.rnd);
    uint32_t r0, r1, r2, r3;
    upk2(c01, r0, r1);
    upk2(c23, r2, r3);
    const uint32_t X01 = r1 * 65536u + r0;
    const uint32_t X23 = r3 * 65536u + r2;
    const uint32_t M = rp.mask, Z = 0x43204320u;  // Z = bf16x2(160, 160)
    constexpr uint32_t E = 0x43004300u;
    out[0] = bmul2(bsub2(and_or_e<E>(X01 >> 9, M), Z), s2);
    out[1] = bmul2(bsub2(and_or_e<E>(X23 >> 9, M), Z), s2);
    out[2] = bmul2(bsub2(and_or_e<E>(X01 >> 6, M), Z), s2);
    out[3] = bmul2(bsub2(and_or_e<E>(X23 >> 6, M), Z), s2);
    out[4] = bmul2(bsub2(and_or_e<E>(X01 >> 3, M), Z), s2);
    out[5] = bmul2(bsub2(and_or_e<E>(X23 >> 3, M), Z), s2);
    out[6] = bmul2(bsub2(and_or_e<E>(X01, M), Z), s2);
    out[7] = bmul2(bsub2(and_or_e<E>(X23, M), Z), s2);
}

// W4: one word = 8 signed 4-bit codes (low nibble first).  out[i] = BF16 (q_i * s, q_{i+4} * s):
// nibble i and i+4 land in the two halves as 128 + (q + 8), minus 136 exactly, times s once.
__device__ __forceinline__ void decode_word_w4_bf16(uint32_t w, uint32_t s2, uint32_t out[4]) {
    const uint32_t M4 = 0x000F000Fu, X4 = 0x43084308u, Z = 0x43084308u;  // Z = bf16x2(136, 136)
    uint32_t r;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        asm("lop3.b32 %0, %1, %2, %3, 0x6A;" : "=r"(r) : "r"(w >> (4 * i)), "r"(M4), "r"(X4));
        out[i] = bmul2(bsub2(r, Z), s2);
    }
}

// WINT2-Standard: one word = 16 plain 2-bit fields, in the same window-major order as a CCQ word:
// out[2i], out[2i+1] = field i of bytes (0,1) and (2,3), each 128 + q minus 130 exactly, times s.
__device__ __forceinline__ void decode_word_std_bf16(uint32_t w, uint32_t M, uint32_t s2, uint32_t out[8]) {
    const uint32_t X01 = prmt(w, 0u, 0x4140u), X23 = prmt(w, 0u, 0x4342u);
    const uint32_t Z = 0x43024302u;  // Z = bf16x2(130, 130)
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        out[2 * i] = bmul2(bsub2(and_or_e<0x43004300u>(X01 >> (2 * i), M), Z), s2);
        out[2 * i + 1] = bmul2(bsub2(and_or_e<0x43004300u>(X23 >> (2 * i), M), Z), s2);
    }
}

__device__ __forceinline__ float silu(float z) { return z / (1.0f + __expf(-z)); }

// position p of a 16-column block holds column 4*(p%4) + p/4 (and the map is its own inverse)
__host__ __device__ constexpr int perm16(int p) { return ((p & 3) << 2) | (p >> 2); }

// Algorithm 2 formats: the 32 states u[0..31] of this thread's half of a group (natural column
// order) -> the two 16-column blocks of BF16 (u - zp) * s in position order.  Each register pairs
// two states as BF16 (128 + u), subtracts 128 + zp exactly and multiplies by s once.
template <int ZP>
__device__ __forceinline__ void emb_pack(const uint32_t (&u)[32], uint32_t s2, uint32_t (&o)[2][8]) {
    constexpr uint32_t Z = (uint32_t)(0x4300 + ZP) * 0x10001u;  // bf16x2(128 + zp)
#pragma unroll
    for (int b = 0; b < 2; ++b)
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            const uint32_t v = u[16 * b + perm16(2 * q)] | (u[16 * b + perm16(2 * q + 1)] << 16) | 0x43004300u;
            o[b][q] = bmul2(bsub2(v, Z), s2);
        }
}

// kind 1, (4,3,2): code j < 21 holds weights 3j..3j+2 at shifts 4, 2, 0 (mask 0xF); code 21 holds
// weight 63 in its top nibble.  c[] holds codes 10*PT .. 10*PT+11 of the group, one per entry.
template <int PT>
__device__ __forceinline__ void emb1_states(const uint32_t (&c)[12], uint32_t (&u)[32]) {
#pragma unroll
    for (int m = 0; m < 32; ++m) {
        const int wi = 32 * PT + m;
        const int j = wi < 63 ? wi / 3 : 21;
        const int sh = wi < 63 ? 4 - 2 * (wi % 3) : 4;
        u[m] = (c[j - 10 * PT] >> sh) & 0xFu;
    }
}

// kind 2, hybrid: word j < 9 holds weights 7j..7j+6 at shifts 13, 11, 9 (its (3,3,2) code) and 6,
// 4, 2, 0 (its (3,4,2) code), mask 0x7; word 9 holds weight 63 in its top 3 bits.  w[] holds the
// group's ten words two per entry in w[0..4] (word 2i in the low half of w[i]).
template <int PT>
__device__ __forceinline__ void emb2_states(const uint32_t (&w)[12], uint32_t (&u)[32]) {
    constexpr int kShift[7] = {13, 11, 9, 6, 4, 2, 0};
#pragma unroll
    for (int m = 0; m < 32; ++m) {
        const int wi = 32 * PT + m;
        const int j = wi < 63 ? wi / 7 : 9;
        const int sh = wi < 63 ? kShift[wi % 7] : 13;
        u[m] = (w[j >> 1] >> (16 * (j & 1) + sh)) & 0x7u;
    }
}

// Position in a ring of N shared-memory stages: slot and the parity of the current round (no
// division by N in the loops).
template <int N>
struct Ring {
    int slot = 0;
    uint32_t phase = 0;
    __device__ __forceinline__ void advance() {
        if (++slot == N) {
            slot = 0;
            phase ^= 1u;
        }
    }
};

struct TileInfo {
    int e, m0, seg0, Me, nt;
    int ks, g0, g1;  // k split and its 64-column groups [g0, g1)
};

// work item w = ((token tile * n_tiles + row tile) * ksplit + k split)
__device__ __forceinline__ bool tile_of(const TcGemmParams &p, int w, TileInfo &t) {
    const int ksn = p.ksplit > 1 ? p.ksplit : 1;
    const int nk = p.K / 64;
    t.ks = w % ksn;
    w /= ksn;
    t.g0 = ksn > 1 ? t.ks * p.kg : 0;
    t.g1 = ksn > 1 ? min(nk, t.g0 + p.kg) : nk;
    const int li = w / p.n_tiles;
    t.nt = w - li * p.n_tiles;
    const int2 ent = p.tile_list ? p.tile_list[li] : make_int2(0, li);
    t.e = ent.x;
    t.seg0 = p.seg_off ? p.seg_off[t.e] : 0;
    t.Me = p.seg_off ? p.seg_off[t.e + 1] - t.seg0 : p.M;
    t.m0 = ent.y * p.m_tile;
    return true;
}

// STD: WINT2-Standard plain 2-bit fields (no per-row constants)
// EMB: 1 = (4,3,2), 2 = hybrid (3,3,2)+(3,4,2), the formats with the scale in the redundant bits.
template <int MT, bool W4, bool Q4 = false, bool STD = false, int EMB = 0>
__global__ void __launch_bounds__(kTcThreads, 1)
tc_gemm_w2_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_codes,
                  const TcGemmParams p) {
    using S = TcSmem<MT, EMB>;
    constexpr int kCRow = kCRowOf<EMB>;
    constexpr int kCTile = kCTileOf<EMB>;
    constexpr int kSA = kSAof<MT, EMB>;
    constexpr int kSB = kSBof<MT, EMB>;
    extern __shared__ uint8_t smem_raw[];
    // 1024-byte aligned start, kept as an offset from the shared array so that loads and stores
    // through it stay shared-memory instructions
    uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t *sA = smem;
    uint8_t *sB = smem + S::kA;
    uint8_t *sC = smem + S::kA + S::kB;
    __shared__ uint64_t a_full[kSA], a_empty[kSA], b_full[kSB], b_empty[kSB], c_full[kSC], c_empty[kSC];
    __shared__ uint64_t acc_full, acc_empty;
    __shared__ uint32_t tmem_base_slot;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int total_work = (p.tile_count ? *p.tile_count : p.static_tiles) * p.n_tiles * (p.ksplit > 1 ? p.ksplit : 1);
    const int nk = p.K / 64;
    // one code stage holds 64 bytes of every row: 4 groups of W2 codes or 2 groups of W4 codes
    constexpr int kKsPerCode = W4 ? 2 : 4;

    if (threadIdx.x == 0) {
        for (int i = 0; i < kSA; ++i) { mbar_init(&a_full[i], 1); mbar_init(&a_empty[i], 1); }
        for (int i = 0; i < kSB; ++i) { mbar_init(&b_full[i], kDecWarps); mbar_init(&b_empty[i], 1); }
        for (int i = 0; i < kSC; ++i) { mbar_init(&c_full[i], 1); mbar_init(&c_empty[i], kDecWarps); }
        mbar_init(&acc_full, 1);
        mbar_init(&acc_empty, kEpiWarps);
        fence_mbar_init();
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&tmem_base_slot)),
                     "r"(MT * 256));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base_slot;

    if (warp == 0) {
        // ------------------------------ TMA producer ------------------------------
        if (lane == 0) {
            prefetch_tensormap(&tm_a);
            prefetch_tensormap(&tm_codes);
            uint32_t ai = 0, ci = 0;
            Ring<kSA> ra;
            Ring<kSC> rc;
            bool ok = true;
            for (int w = blockIdx.x; w < total_work && ok; w += gridDim.x) {
                TileInfo t;
                tile_of(p, w, t);
                const int localA = t.nt * p.row_block_stride;
                const int rowA = t.e * p.N + localA, rowB = rowA + p.half_stride;
                for (int ks = t.g0; ks < t.g1 && ok; ++ks) {
                    if (ks % kKsPerCode == 0) {
                        const int s = rc.slot;
                        if (ci >= kSC) ok = mbar_wait(&c_empty[s], rc.phase ^ 1u, p.err);
                        if (!ok) break;
                        mbar_arrive_expect_tx(&c_full[s], kCTile);
                        // the stage's first code byte, rounded down to a 16-byte boundary (EMB 1)
                        const int cs_no = ks / kKsPerCode;
                        const int x = EMB == 1 ? (88 * cs_no) & ~15 : EMB == 2 ? 80 * cs_no : 64 * cs_no;
                        tma_load_2d(sC + s * kCTile, &tm_codes, &c_full[s], x, rowA);
                        tma_load_2d(sC + s * kCTile + kCTile / 2, &tm_codes, &c_full[s], x, rowB);
                        ++ci;
                        rc.advance();
                    }
                    const int s = ra.slot;
                    if (ai >= kSA) ok = mbar_wait(&a_empty[s], ra.phase ^ 1u, p.err);
                    if (!ok) break;
                    mbar_arrive_expect_tx(&a_full[s], MT * kATile);
#pragma unroll
                    for (int j = 0; j < MT; ++j)
                        tma_load_2d(sA + (s * MT + j) * kATile, &tm_a, &a_full[s], ks * 64, t.seg0 + t.m0 + j * 128);
                    ++ai;
                    ra.advance();
                }
            }
            // drain: the last copies must land before exit
            for (uint32_t i = (ai > kSA ? ai - kSA : 0); i < ai && ok; ++i)
                ok = mbar_wait(&a_full[i % kSA], (i / kSA) & 1, p.err);
            for (uint32_t i = (ci > kSC ? ci - kSC : 0); i < ci && ok; ++i)
                ok = mbar_wait(&c_full[i % kSC], (i / kSC) & 1, p.err);
        }
    } else if (warp == 1) {
        // ------------------------------ MMA issuer ------------------------------
        if (lane == 0) {
            uint32_t ti = 0;
            Ring<kSA> ra;
            Ring<kSB> rb;
            bool ok = true;
            for (int w = blockIdx.x; w < total_work && ok; w += gridDim.x, ++ti) {
                TileInfo t;
                tile_of(p, w, t);
                if (ti > 0) ok = mbar_wait(&acc_empty, (ti - 1) & 1, p.err);
                if (!ok) break;
                tc_fence_after();
                for (int ks = t.g0; ks < t.g1 && ok; ++ks) {
                    const int sa = ra.slot, sb = rb.slot;
                    ok = mbar_wait(&a_full[sa], ra.phase, p.err) && mbar_wait(&b_full[sb], rb.phase, p.err);
                    if (!ok) break;
                    tc_fence_after();
#pragma unroll
                    for (int j = 0; j < MT; ++j) {
                        const uint32_t abase = smem_u32(sA + (sa * MT + j) * kATile);
                        const uint32_t bbase = smem_u32(sB + sb * kBTile);
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            mma_bf16_ss(tmem + j * 256, smem_desc_sw128(abase + kk * 32),
                                        smem_desc_sw128(bbase + kk * 32), (ks > t.g0 || kk > 0) ? 1u : 0u);
                    }
                    mma_commit(&a_empty[sa]);
                    mma_commit(&b_empty[sb]);
                    ra.advance();
                    rb.advance();
                }
                if (ok) mma_commit(&acc_full);
            }
            // the last MMAs must be complete before TMEM is freed
            if (ok && ti > 0) ok = mbar_wait(&acc_full, (ti - 1) & 1, p.err);
            (void)ok;
        }
    } else if (warp < 2 + kDecWarps) {
        // ------------------------------ decoders ------------------------------
        // two threads per weight row: thread part pt decodes words 2pt, 2pt+1 (W2: bytes 8pt..8pt+7 of
        // the row's 16 bytes of the group; W4: the second 16-byte chunk of the row's 32 bytes)
        // (EMB: each warp decodes one half of 32 rows' groups, so its code path is warp-uniform)
        const int d = threadIdx.x - 64;
        const int r = EMB ? ((d >> 6) << 5) + (d & 31) : d >> 1;  // weight row within the tile, 0..255
        const int pt = EMB ? (d >> 5) & 1 : d & 1;                 // part
        const int half = r >> 7, rr = r & 127;
        uint32_t bi = 0;
        Ring<kSB> rb;
        Ring<kSC> rc;
        bool ok = true;
        RowCodeParams rp;
        rp.neg = fpk2(-8388608.0f, -8388608.0f);
        rp.rnd = fpk2(12582912.0f, 12582912.0f - 19264.0f);
        // (an opaque zero keeps the mask in a register, so the logic op's immediate is the exponent)
        rp.mask = (STD ? 0x00030003u : 0x003F003Fu) ^ (uint32_t)(p.K >> 30);
        for (int w = blockIdx.x; w < total_work && ok; w += gridDim.x) {
            TileInfo t;
            tile_of(p, w, t);
            const int local = t.nt * p.row_block_stride + half * p.half_stride + rr;
            const bool valid = local < p.N;
            const size_t grow = (size_t)t.e * p.N + (valid ? local : 0);
            const float alpha = (W4 || STD || EMB) ? 0.0f : __ldg(p.alpha + grow);
            const float beta = (W4 || STD || EMB) ? 0.0f : __ldg(p.beta + grow);
            rp.ab = fpk2(alpha, alpha);
            rp.bb = fpk2(beta, beta);
            const float *srow = EMB ? nullptr : p.scales + grow * (W4 ? 1 : nk);
            const float sc_row = W4 ? bf16_bits_to_float(float_to_bf16_bits(__ldg(srow))) : 0.0f;
            // W2 group scales, four groups (one code stage) at a time and one stage ahead, so the
            // global read is off the decode's critical path
            const float sup_row = (Q4 || EMB) ? __ldg(p.super_scale + grow) : 0.0f;
            auto load_sc4 = [&](int g0) -> float4 {
                if (W4 || EMB || g0 >= nk) return make_float4(0.f, 0.f, 0.f, 0.f);
                if (Q4) {
                    // 4-bit group scales: groups g0..g0+3 in two bytes (even group in the low nibble)
                    const int qpr = p.K / 128;
                    const uint8_t *qrow = p.scale_q4 + grow * (size_t)qpr;
                    const uint32_t b0 = g0 / 2 < qpr ? __ldg(qrow + g0 / 2) : 0u;
                    const uint32_t b1 = g0 / 2 + 1 < qpr ? __ldg(qrow + g0 / 2 + 1) : 0u;
                    return make_float4(__fmul_rn((float)(b0 & 0xFu), sup_row), __fmul_rn((float)(b0 >> 4), sup_row),
                                       __fmul_rn((float)(b1 & 0xFu), sup_row), __fmul_rn((float)(b1 >> 4), sup_row));
                }
                if ((nk & 3) == 0) return __ldg(reinterpret_cast<const float4 *>(srow + g0));
                return make_float4(__ldg(srow + g0), g0 + 1 < nk ? __ldg(srow + g0 + 1) : 0.f,
                                   g0 + 2 < nk ? __ldg(srow + g0 + 2) : 0.f, g0 + 3 < nk ? __ldg(srow + g0 + 3) : 0.f);
            };
            float4 sc_cur = make_float4(0.f, 0.f, 0.f, 0.f), sc_next = load_sc4(t.g0);
            for (int ks = t.g0; ks < t.g1 && ok; ++ks) {
                if (!W4 && !EMB && (ks & 3) == 0) {
                    sc_cur = sc_next;
                    sc_next = load_sc4(ks + 4);
                }
                const int cs = rc.slot;
                if (ks % kKsPerCode == 0) {
                    ok = mbar_wait(&c_full[cs], rc.phase, p.err);
                    if (!ok) break;
                }
                // this thread's code bytes of group ks (64-byte rows, 64B swizzle; EMB: unswizzled
                // rows of kCRow bytes)
                const uint8_t *crow = sC + cs * kCTile + half * (kCTile / 2) + rr * kCRow;
                const uint32_t swz = ((uint32_t)rr >> 1) & 3u;
                uint2 q2w = make_uint2(0, 0);
                uint4 q4w = make_uint4(0, 0, 0, 0);
                uint32_t ec[12];  // EMB 1: codes 10pt .. 10pt+11 of the group, one per entry; EMB 2:
                                  // the ten words, two per entry, in ec[0..4]
                uint32_t eq = 0;  // EMB: the group's quantized scale
                if constexpr (EMB == 1) {
                    // the group's first code sits (88 * stage) mod 16 + 22 * (ks mod 4) bytes into the
                    // row's line: an even offset, so 16-bit loads are aligned
                    const uint8_t *gb = crow + ((88 * (ks >> 2)) & 15) + 22 * (ks & 3);
                    const uint16_t *g16 = reinterpret_cast<const uint16_t *>(gb + 10 * pt);
#pragma unroll
                    for (int i = 0; i < 6; ++i) {
                        const uint32_t h = g16[i];
                        ec[2 * i] = h & 0xFFu;
                        ec[2 * i + 1] = h >> 8;
                    }
                    // the scale: the low nibble of code 21 (the high byte of the 16-bit word at 20)
                    eq = ((uint32_t)*reinterpret_cast<const uint16_t *>(gb + 20) >> 8) & 0xFu;
                } else if constexpr (EMB == 2) {
                    const uint32_t *g32 = reinterpret_cast<const uint32_t *>(crow + 20 * (ks & 3));
#pragma unroll
                    for (int i = 0; i < 5; ++i) ec[i] = g32[i];
                    eq = (ec[4] >> 16) & 0x1FFFu;
                } else if (!W4) {
                    q2w = *reinterpret_cast<const uint2 *>(crow + ((((uint32_t)(ks & 3)) ^ swz) << 4) + 8 * pt);
                } else {
                    const uint32_t c0 = 2u * (uint32_t)(ks & 1) + (uint32_t)pt;
                    q4w = *reinterpret_cast<const uint4 *>(crow + ((c0 ^ swz) << 4));
                }
                if (ks % kKsPerCode == kKsPerCode - 1 || ks == t.g1 - 1) {
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&c_empty[cs]);
                    rc.advance();
                }
                uint32_t o[2][8];
                if constexpr (EMB != 0) {
                    const float sc = bf16_bits_to_float(float_to_bf16_bits(__fmul_rn((float)eq, sup_row)));
                    const uint32_t s2 = pack_bf16x2(sc, sc);
                    uint32_t u[32];
                    if constexpr (EMB == 1) {
                        if (pt == 0) emb1_states<0>(ec, u);
                        else emb1_states<1>(ec, u);
                        emb_pack<8>(u, s2, o);
                    } else {
                        if (pt == 0) emb2_states<0>(ec, u);
                        else emb2_states<1>(ec, u);
                        emb_pack<4>(u, s2, o);
                    }
                } else if (!W4) {
                    const int gi = ks & 3;
                    const float sraw = gi == 0 ? sc_cur.x : gi == 1 ? sc_cur.y : gi == 2 ? sc_cur.z : sc_cur.w;
                    const float sc = bf16_bits_to_float(float_to_bf16_bits(sraw));
                    const uint32_t s2 = pack_bf16x2(sc, sc);
                    if constexpr (STD) {
                        decode_word_std_bf16(q2w.x, rp.mask, s2, o[0]);
                        decode_word_std_bf16(q2w.y, rp.mask, s2, o[1]);
                    } else {
                        decode_word_bf16(q2w.x, rp, s2, o[0]);
                        decode_word_bf16(q2w.y, rp, s2, o[1]);
                    }
                } else {
                    // block b of 16 columns = words 2b, 2b+1; emit the same window-major order as W2:
                    // positions (4i, 4i+1) <- codes (i, i+4) of word 2b, (4i+2, 4i+3) <- of word 2b+1
                    const uint32_t s2 = pack_bf16x2(sc_row, sc_row);
                    const uint32_t wds[4] = {q4w.x, q4w.y, q4w.z, q4w.w};
#pragma unroll
                    for (int b = 0; b < 2; ++b) {
                        uint32_t r0[4], r1[4];
                        decode_word_w4_bf16(wds[2 * b], s2, r0);
                        decode_word_w4_bf16(wds[2 * b + 1], s2, r1);
                        o[b][0] = r0[0]; o[b][1] = r1[0]; o[b][2] = r0[1]; o[b][3] = r1[1];
                        o[b][4] = r0[2]; o[b][5] = r1[2]; o[b][6] = r0[3]; o[b][7] = r1[3];
                    }
                }
                const int sb = rb.slot;
                if (bi >= kSB) ok = mbar_wait(&b_empty[sb], rb.phase ^ 1u, p.err);
                if (!ok) break;
                uint8_t *brow = sB + sb * kBTile + r * 128;
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    const int wd = 2 * pt + j;  // 16-column block of the group
                    const uint32_t c0 = (uint32_t)(2 * wd) ^ ((uint32_t)r & 7u);
                    const uint32_t c1 = (uint32_t)(2 * wd + 1) ^ ((uint32_t)r & 7u);
                    *reinterpret_cast<uint4 *>(brow + (c0 << 4)) = make_uint4(o[j][0], o[j][1], o[j][2], o[j][3]);
                    *reinterpret_cast<uint4 *>(brow + (c1 << 4)) = make_uint4(o[j][4], o[j][5], o[j][6], o[j][7]);
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&b_full[sb]);
                ++bi;
                rb.advance();
            }
        }
    } else {
        // ------------------------------ epilogue ------------------------------
        const int q = warp & 3;        // TMEM lane quarter this warp may access
        const int m = q * 32 + lane;   // accumulator row = token within the 128-token sub-tile
        uint32_t ti = 0;
        bool ok = true;
        for (int w = blockIdx.x; w < total_work && ok; w += gridDim.x, ++ti) {
            TileInfo t;
            tile_of(p, w, t);
            ok = mbar_wait(&acc_full, ti & 1, p.err);
            if (!ok) break;
            tc_fence_after();
            const int localA = t.nt * p.row_block_stride;
#pragma unroll 1
            for (int j = 0; j < MT; ++j) {
                const int tok = t.m0 + j * 128 + m;
                const bool live = tok < t.Me;
                const size_t prow = (size_t)(t.seg0 + tok);
                const uint32_t tbase = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(j * 256);
                if (p.mode == EPI_GATEUP) {
#pragma unroll 1
                    for (int c = 0; c < 128; c += 16) {  // one 16-column block at a time
                        uint32_t g[16], u[16];
                        tmem_ld16(tbase + c, g);
                        tmem_ld16(tbase + 128 + c, u);
                        tmem_ld_wait();
                        if (!live || localA + c >= p.I) continue;
                        uint32_t h[8];
#pragma unroll
                        for (int pp = 0; pp < 16; pp += 2) {
                            const int c0 = perm16(pp), c1 = perm16(pp + 1);
                            const float h0 = silu(__uint_as_float(g[c0])) * __uint_as_float(u[c0]);
                            const float h1 = silu(__uint_as_float(g[c1])) * __uint_as_float(u[c1]);
                            h[pp / 2] = pack_bf16x2(h0, h1);
                        }
                        uint4 *dst = reinterpret_cast<uint4 *>(static_cast<uint16_t *>(p.out) + prow * p.out_ld + localA + c);
                        dst[0] = make_uint4(h[0], h[1], h[2], h[3]);
                        dst[1] = make_uint4(h[4], h[5], h[6], h[7]);
                    }
                } else {
                    const float rwv = (p.mode == EPI_DOWN && live) ? __ldg(p.rw + prow) : 1.0f;
                    // fp32 outputs: routing-weighted slots, or this k split's partial sums
                    const bool f32 = p.mode == EPI_DOWN || p.mode == EPI_PARTIAL_F32;
                    float *fout = static_cast<float *>(p.out) +
                                  (p.mode == EPI_PARTIAL_F32 ? (size_t)t.ks * p.out_split_stride : 0);
#pragma unroll 1
                    for (int c = 0; c < 256; c += 32) {
                        uint32_t v[32];
                        tmem_ld32(tbase + c, v);
                        tmem_ld_wait();
                        const int lr = localA + (c >= 128 ? p.half_stride - 128 : 0) + c;  // local row of column c
                        if (!live || lr >= p.N) continue;
                        if (f32 && lr + 32 > p.N) {  // partial chunk of rows
                            float *dst = fout + prow * p.out_ld + lr;
#pragma unroll
                            for (int z = 0; z < 32; ++z)
                                if (lr + z < p.N) dst[z] = rwv * __uint_as_float(v[z]);
                        } else if (f32) {
                            float4 *dst = reinterpret_cast<float4 *>(fout + prow * p.out_ld + lr);
#pragma unroll
                            for (int z = 0; z < 8; ++z)
                                dst[z] = make_float4(rwv * __uint_as_float(v[4 * z]), rwv * __uint_as_float(v[4 * z + 1]),
                                                     rwv * __uint_as_float(v[4 * z + 2]), rwv * __uint_as_float(v[4 * z + 3]));
                        } else if (lr + 32 <= p.N) {
                            uint4 *dst = reinterpret_cast<uint4 *>(static_cast<uint16_t *>(p.out) + prow * p.out_ld + lr);
#pragma unroll
                            for (int z = 0; z < 4; ++z)
                                dst[z] = make_uint4(pack_bf16x2(__uint_as_float(v[8 * z]), __uint_as_float(v[8 * z + 1])),
                                                    pack_bf16x2(__uint_as_float(v[8 * z + 2]), __uint_as_float(v[8 * z + 3])),
                                                    pack_bf16x2(__uint_as_float(v[8 * z + 4]), __uint_as_float(v[8 * z + 5])),
                                                    pack_bf16x2(__uint_as_float(v[8 * z + 6]), __uint_as_float(v[8 * z + 7])));
                        } else {  // last, partial chunk of rows (N is a multiple of 16, not of 32)
                            uint16_t *dst = static_cast<uint16_t *>(p.out) + prow * p.out_ld + lr;
#pragma unroll
                            for (int z = 0; z < 32; ++z)
                                if (lr + z < p.N) dst[z] = float_to_bf16_bits(__uint_as_float(v[z]));
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(MT * 256));
    }
}

// Tile list: one entry (expert, token tile) per 128*MT tokens of each expert's segment.
__global__ void build_tiles_kernel(const int *__restrict__ seg_off, int E, int m_tile, int2 *__restrict__ list,
                                   int *__restrict__ count) {
    if (threadIdx.x != 0 || blockIdx.x != 0) return;
    int n = 0;
    for (int e = 0; e < E; ++e) {
        const int Me = seg_off[e + 1] - seg_off[e];
        for (int m = 0; m * m_tile < Me; ++m) list[n++] = make_int2(e, m);
    }
    *count = n;
}

// Prefill activation operand: rows gathered by tok_of (or identity), each 16-column block stored in
// the decoders' window-major order (position p <- column perm16(p)).
__global__ void pack_xt_kernel(const uint16_t *__restrict__ x, const int *__restrict__ tok_of, int P_valid, int K,
                               uint16_t *__restrict__ xt) {
    const int nb = K / 16;
    const size_t total = (size_t)P_valid * nb;
    for (size_t idx = blockIdx.x * (size_t)blockDim.x + threadIdx.x; idx < total;
         idx += (size_t)gridDim.x * blockDim.x) {
        const int pr = (int)(idx / nb), b = (int)(idx % nb);
        const int src = tok_of ? __ldg(tok_of + pr) : pr;
        const uint4 *s = reinterpret_cast<const uint4 *>(x + (size_t)src * K + (size_t)b * 16);
        const uint4 v0 = __ldg(s), v1 = __ldg(s + 1);
        const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
        uint16_t in[16], o[16];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            in[2 * i] = (uint16_t)(w[i] & 0xFFFFu);
            in[2 * i + 1] = (uint16_t)(w[i] >> 16);
        }
#pragma unroll
        for (int pp = 0; pp < 16; ++pp) o[pp] = in[perm16(pp)];
        uint4 *d = reinterpret_cast<uint4 *>(xt + (size_t)pr * K + (size_t)b * 16);
        d[0] = make_uint4((uint32_t)o[0] | ((uint32_t)o[1] << 16), (uint32_t)o[2] | ((uint32_t)o[3] << 16),
                          (uint32_t)o[4] | ((uint32_t)o[5] << 16), (uint32_t)o[6] | ((uint32_t)o[7] << 16));
        d[1] = make_uint4((uint32_t)o[8] | ((uint32_t)o[9] << 16), (uint32_t)o[10] | ((uint32_t)o[11] << 16),
                          (uint32_t)o[12] | ((uint32_t)o[13] << 16), (uint32_t)o[14] | ((uint32_t)o[15] << 16));
    }
}

template <int MT>
cudaError_t launch_tc_mt(const TcGemmParams &p, const CUtensorMap &ta, const CUtensorMap &tc, int grid, cudaStream_t s) {
    auto kern = p.emb == 1 ? tc_gemm_w2_kernel<MT, false, false, false, 1>
                : p.emb == 2 ? tc_gemm_w2_kernel<MT, false, false, false, 2>
                : p.w4       ? tc_gemm_w2_kernel<MT, true>
                : p.q4       ? tc_gemm_w2_kernel<MT, false, true>
                : p.std2     ? tc_gemm_w2_kernel<MT, false, false, true>
                             : tc_gemm_w2_kernel<MT, false>;
    const int smem = p.emb == 1 ? TcSmem<MT, 1>::kTotal : p.emb == 2 ? TcSmem<MT, 2>::kTotal : TcSmem<MT>::kTotal;
    cudaError_t err = kernel_setup(reinterpret_cast<const void *>(kern), smem, kTcThreads, 0, nullptr);
    if (err != cudaSuccess) return err;
    kern<<<grid, kTcThreads, smem, s>>>(ta, tc, p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_tc_gemm_w2(const TcGemmParams &p, const CUtensorMap &tm_a, const CUtensorMap &tm_codes, int mt,
                              int grid, cudaStream_t s) {
    if (mt == 1) return launch_tc_mt<1>(p, tm_a, tm_codes, grid, s);
    if (mt == 2) return launch_tc_mt<2>(p, tm_a, tm_codes, grid, s);
    return cudaErrorInvalidValue;
}

cudaError_t launch_build_tiles(const int *seg_off, int E, int m_tile, int2 *list, int *count, cudaStream_t s) {
    build_tiles_kernel<<<1, 32, 0, s>>>(seg_off, E, m_tile, list, count);
    return cudaGetLastError();
}

cudaError_t launch_pack_xt(const uint16_t *x, const int *tok_of, int P_valid, int K, uint16_t *xt, cudaStream_t s) {
    if (P_valid <= 0) return cudaSuccess;
    size_t work = (size_t)P_valid * (K / 16);
    size_t b = (work + 255) / 256;
    if (b > 148 * 32) b = 148 * 32;
    pack_xt_kernel<<<(int)b, 256, 0, s>>>(x, tok_of, P_valid, K, xt);
    return cudaGetLastError();
}

}  // namespace ccq
