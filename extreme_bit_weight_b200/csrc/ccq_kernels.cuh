// Kernel parameter blocks and launchers shared between the CUDA translation units of libccq.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace ccq {

// Once per (kernel, device, dynamic shared memory size): checks the kernel's launch register count
// (when want_regs != 0), sets its dynamic shared memory limit and computes how many CTAs of
// `threads` threads fit on one SM.  Later calls return the cached result without touching the
// runtime, so a small call's host cost is its launches.  per_sm may be NULL.
cudaError_t kernel_setup(const void *kern, int smem, int threads, int want_regs, int *per_sm);

// Launch `kern` with programmatic stream serialization: the grid may be scheduled while the previous
// kernel in the stream finishes; the kernel itself waits (pdl_wait) before touching that kernel's
// results.  Used for the dense matmul's chain (packing, decode kernel, split-K reduce).
template <class... Params, class... Args>
cudaError_t launch_pdl(void (*kern)(Params...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, args...);
}

// Epilogue modes of the decode-sized grouped kernel.
enum EpiMode : int {
    EPI_PARTIAL_F32 = 0,  // out_f32[ks][m][n] = partial sum over this CTA's k range
    EPI_BF16 = 1,         // out_bf16[m][n] = bf16(acc)
    EPI_GATEUP = 2,       // h = bf16(SiLU(acc_gate) * acc_up) written in the activation-operand layout
    EPI_DOWN = 3          // slot_f32[p][n] = routing_w[p] * acc
};

// Activation-operand ("XA") layout used by the decode-sized kernel.  For an operand of P rows and
// K columns (K % 64 == 0), element (p, k) with G = k/64, r = k%64, tig = r/16, j = (r/4)%4, i = r%4
// sits at  ((((G*4 + i)*P + p)*4 + tig)*4 + j).  Rows of one 16-column block are thus grouped by
// the state window i they meet in the decoded weights, which makes every mma B fragment one
// contiguous, bank-conflict-free 8-byte shared-memory read.  Alongside it the group-sum table
// gsq[p][G] (float4, row pitch gsum_ld(K) entries) holds {L*S(p,G), L*S(p+1,G), L*S(p,G),
// L*S(p+1,G)}: S(p,G) = sum of x[p][k] over group G (fp32, column order; 0 past the last valid row)
// and L the weight format's level offset (gsq_level).
__host__ __device__ inline size_t xa_index(size_t p, size_t k, size_t P) {
    size_t G = k >> 6, r = k & 63, tig = r >> 4, j = (r >> 2) & 3, i = r & 3;
    return ((((G * 4 + i) * P + p) * 4 + tig) * 4 + j);
}
__host__ __device__ inline int gsum_ld(int K) { return ((K / 64) + 3) & ~3; }

// Operand order of the (4,3,2) format (CCQ_FMT_W275_432) in the decode-sized kernel.  Thread tig
// of a fragment quad decodes, per row and 64-column group, the states of codes 4tig..4tig+3 (one
// 32-bit word), of code 16+tig, and one more state (code 20's state tig, or code 21's first state for
// tig 3); a code j < 21 holds weights 3j (its first state, shift 4), 3j+1 (shift 2), 3j+2 (shift 0).
// Its registers, as (slice i, element b) of the mma A fragment:
//   i = 0: the shift-0 states of codes 4tig, 4tig+2, 4tig+1, 4tig+3 (b = 0..3);
//   i = 1: the same codes' shift-2 states;  i = 2: their shift-4 states;
//   i = 3: code 16+tig's shift-0, shift-2 and shift-4 states, then the extra state.
// Each state reaches the tensor core as the BF16 value 2^(7-T) + u with T its bit position in the
// register half (0, 2 or 3), so the group's accumulator starts at sum_k L(k) x_k with
// L = -(2^(7-T) + 8) per position (-136, -40, -24).  w275_pos maps a group column w (0..63) to
// (i, tig, b); w275_level gives L for (i, b).
__host__ __device__ inline void w275_pos(int w, int &i, int &tig, int &b) {
    if (w >= 60) {  // the extra states: weights 60..62 (code 20) and 63 (code 21)
        i = 3;
        tig = w - 60;
        b = 3;
        return;
    }
    const int c = w / 3, x = w % 3;  // code, state index (0: shift 4, 1: shift 2, 2: shift 0)
    if (c >= 16) {
        i = 3;
        tig = c - 16;
        b = 2 - x;  // shift 0, 2, 4 -> b 0, 1, 2
        return;
    }
    tig = c >> 2;
    i = 2 - x;                        // shift 0 -> slice 0, shift 2 -> 1, shift 4 -> 2
    const int cb = c & 3;             // byte of the thread's word
    b = (cb & 1) ? 2 + (cb >> 1) : cb >> 1;  // bytes 0, 2 -> b 0, 1; bytes 1, 3 -> b 2, 3
}
__host__ __device__ inline float w275_level(int i, int b) {
    const int slot = i < 3 ? i : (b < 3 ? b : 0);  // 0: T = 0, 1: T = 2, 2: T = 3
    return slot == 0 ? -136.0f : slot == 1 ? -40.0f : -24.0f;
}
// Operand order of the hybrid (3,3,2)+(3,4,2) format (CCQ_FMT_W25_HYBRID).  A group is ten 16-bit
// words; word j < 9 holds weights 7j + s for its states s = 0..6 (shifts 13, 11, 9, 6, 4, 2, 0).
// Thread tig decodes words 2tig (low half of one 32-bit load) and 2tig+1 (high half): register
// k = 0..6 pairs the two words' state k, as (slice k/2, elements 2 (k mod 2), +1); register 7 holds
// two more states: word 8's states 2tig, 2tig+1 (tig < 3), or word 8's state 6 and word 9's (weight
// 63) for tig 3.  States reach the tensor core as 2^(7-T) + u (T = 4 for states 0-4, 2 for state 5,
// 0 for state 6 and the extra pair), so L = -(2^(7-T) + 4) = -12, -36, -132.
__host__ __device__ inline void hyb_pos(int w, int &i, int &tig, int &b) {
    if (w >= 56) {
        i = 3;
        tig = (w - 56) >> 1;
        b = 2 + (w & 1);
        return;
    }
    const int j = w / 7, st = w % 7;
    tig = j >> 1;
    i = st >> 1;
    b = (st & 1) * 2 + (j & 1);
}
__host__ __device__ inline float hyb_level(int i, int b) {
    const int k = 2 * i + (b >> 1);  // register index
    return k <= 4 ? -12.0f : k == 5 ? -36.0f : -132.0f;
}
// Position (slice, thread, element) and level offset of group column w under operand order perm
// (1: (4,3,2), 2: hybrid).
__host__ __device__ inline void perm_pos(int perm, int w, int &i, int &tig, int &b) {
    if (perm == 1) w275_pos(w, i, tig, b);
    else hyb_pos(w, i, tig, b);
}
__host__ __device__ inline float perm_level(int perm, int w) {
    int i, tig, b;
    perm_pos(perm, w, i, tig, b);
    return perm == 1 ? w275_level(i, b) : hyb_level(i, b);
}
// The decode-sized operand position of element (p, k): perm 0 = the CCQ / STD / W4 order (xa_index),
// 1 = the (4,3,2) order, 2 = the hybrid order.
__host__ __device__ inline size_t xa_index_perm(size_t p, size_t k, size_t P, int perm) {
    if (perm == 0) return xa_index(p, k, P);
    int i, tig, b;
    perm_pos(perm, (int)(k & 63), i, tig, b);
    return (((((k >> 6) * 4 + (size_t)i) * P + p) * 4 + (size_t)tig) * 4 + (size_t)b);
}
// The decoders hand the tensor core BF16 (128 + u) for CCQ state u (weight level u - 32),
// (128 + q + 8) for W4 nibble q and (128 + q) for a STD 2-bit field q (level q - 2): the per-group
// accumulator starts at L * S with L = -160 / -136 / -130.
__host__ __device__ inline float gsq_level(bool w4, bool std2 = false) {
    return w4 ? -136.0f : std2 ? -130.0f : -160.0f;
}

struct DecodeGemmParams {
    const float *scales;  // [rows_total][K/64]
    const float *alpha;   // [rows_total]
    const float *beta;    // [rows_total]
    int N;                // rows per expert
    int K;                // columns
    int row_block_stride; // rows between consecutive row blocks
    int half_stride;      // row offset of the CTA's second 128-row half
    int stages_per_split; // 512-column stages per k split
    int num_stages;       // ceil(K/512)
    // tokens
    const int *seg_off;   // [E+1] row offsets into the activation operand; NULL: one segment [0, M)
    int M;
    int P;                // rows of the activation operand
    // epilogue
    int mode;
    void *out;
    int out_ld;           // leading dimension of out (elements)
    size_t out_split_stride; // EPI_PARTIAL_F32: elements between k splits
    const float *rw;      // EPI_DOWN: routing weight per operand row
    int h_P;              // EPI_GATEUP: rows of the H operand (== P)
    int I;                // EPI_GATEUP: gate rows per expert
    int tma_scales;       // 1: scales staged by TMA with the codes (row pitch a multiple of 16 B)
    int w4;               // 1: W4 per-channel codes (two per byte), scales[row]
    // 1: 4-bit group scales s = fl32(q4 * super[row]) (two per byte, even group in the low nibble)
    int q4;
    const uint8_t *scale_q4;   // [rows_total][K/128]
    const float *super_scale;  // [rows_total]
    int std2;                  // 1: WINT2-Standard plain 2-bit fields (no alpha/beta)
    int emb;                   // 1 / 2: the (4,3,2) / hybrid format (codes with the scale inside; super_scale per row)
    int h_perm;                // EPI_GATEUP: operand order of h for the down projection (xa_index_perm)
    uint32_t *err;
    // work units (set by the launcher): unit u = (expert, k split, row block), row block fastest
    int row_blocks, ksplit, units;
    // zeroed counter from which CTAs take their next unit (NULL: CTA b takes b, b + grid, ...);
    // a fused launch uses the gate/up block's
    int *work;
    // fused MoE launch (gate/up and down in one kernel): the gate/up epilogue also writes the down
    // operand's gsq table and counts finished units per expert in dep[]; a down unit of expert e
    // loads only after dep[e] reaches dep_need
    int *dep;
    float *fuse_gsq;     // gate/up: gsq table of h (row pitch fuse_gsq_ld entries)
    int fuse_gsq_ld;
    float fuse_level;    // level offset of the down weight's format
    int dep_need;        // down: gate/up units per expert
};

// Fused MoE decode: gate/up (p1, maps a1..d1) then down (p2, maps a2..d2) in one cooperative
// persistent launch.  Both must be the same 2-bit format (CCQ or STD with TMA-staged fp32 scales,
// or CCQ with 4-bit scales) with the same token tile count nt.
cudaError_t launch_decode_moe_fused(const DecodeGemmParams &p1, const CUtensorMap &a1, const CUtensorMap &b1,
                                    const CUtensorMap &c1, const CUtensorMap &d1, int row_blocks1,
                                    const DecodeGemmParams &p2, const CUtensorMap &a2, const CUtensorMap &b2,
                                    const CUtensorMap &c2, const CUtensorMap &d2, int row_blocks2, int experts,
                                    int nt, cudaStream_t s);

cudaError_t launch_decode_gemm_w2(const DecodeGemmParams &p, const CUtensorMap &tm_codes,
                                  const CUtensorMap &tm_xa, const CUtensorMap &tm_gs, const CUtensorMap &tm_sc,
                                  int row_blocks, int ksplit, int experts, int nt, cudaStream_t s);

// Prefill-sized tcgen05 kernel.
struct TcGemmParams {
    const float *scales;   // [rows_total][K/64]
    const float *alpha;    // [rows_total]
    const float *beta;     // [rows_total]
    int N;                 // rows per expert
    int K;
    int row_block_stride;  // local row of row tile nt = nt * row_block_stride
    int half_stride;       // second 128-row half of a tile starts half_stride rows later
    int n_tiles;           // row tiles per expert
    const int2 *tile_list; // (expert, token tile) entries; NULL: (0, i) for i < static_tiles
    const int *tile_count; // device count of tile_list entries; NULL: static_tiles
    int static_tiles;
    int m_tile;            // tokens per token tile (128 * MT)
    const int *seg_off;    // [E+1] operand row segments; NULL: one segment of M rows
    int M;
    int mode;              // EPI_GATEUP, EPI_DOWN or EPI_BF16
    void *out;
    int out_ld;
    const float *rw;       // EPI_DOWN: routing weight per operand row
    int I;                 // EPI_GATEUP: gate rows per expert
    int w4;                // 1: W4 per-channel codes (two per byte), scales[row]
    int q4;                // 1: 4-bit group scales (see DecodeGemmParams)
    const uint8_t *scale_q4;
    const float *super_scale;
    int std2;              // 1: WINT2-Standard plain 2-bit fields (no alpha/beta)
    // 1 / 2: the (4,3,2) / hybrid format with the group scale in the redundant bits (codes and
    // super_scale only)
    int emb;
    uint32_t *err;
    // split-K (dense matmul with few tiles): ksplit > 1 splits the 64-column groups into ranges of
    // kg groups (a multiple of 4); each range writes EPI_PARTIAL_F32 sums at out + ks*out_split_stride
    int ksplit, kg;
    size_t out_split_stride;
};

cudaError_t launch_tc_gemm_w2(const TcGemmParams &p, const CUtensorMap &tm_a, const CUtensorMap &tm_codes, int mt,
                              int grid, cudaStream_t s);
cudaError_t launch_build_tiles(const int *seg_off, int E, int m_tile, int2 *list, int *count, cudaStream_t s);
// rows gathered by tok_of (or identity), each 16-column block in the decoders' window-major order
cudaError_t launch_pack_xt(const uint16_t *x, const int *tok_of, int P_valid, int K, uint16_t *xt, cudaStream_t s);

cudaError_t launch_dequant(int fmt, const uint8_t *codes, const float *scales, const float *alpha,
                           const float *beta, int rows, int K, uint16_t *out, cudaStream_t s,
                           const uint8_t *scale_q4 = nullptr, const float *super = nullptr);

// Encoder for the formats with the scale in the redundant bits (kind 1 / 2): w fp32 [rows][K] ->
// codes [rows][K/64 * (22 or 20) bytes] and super [rows].
cudaError_t launch_encode_emb(int kind, const float *w, int rows, int K, void *codes, float *super, cudaStream_t s);

// Failure-detection self-test (see ccq_selftest_bounded_wait in ccq.h).
cudaError_t launch_bounded_wait_probe(uint32_t *err, int *never, int kind, uint64_t limit_ns, cudaStream_t s);

// WINT2-Standard round-to-nearest: w fp32 [rows][K] -> codes [rows][K/4], scales [rows][K/64]
cudaError_t launch_quantize_std(const float *w, int rows, int K, uint8_t *codes, float *scales, cudaStream_t s);

// x (BF16 [rows][K], row r taken from x[tok_of ? tok_of[p] : p]) -> XA operand + group sums.
// zero_ctr (may be NULL): an int the kernel sets to 0 (the following matmul's work counter).
// perm: operand order (xa_index_perm); perms 1 and 2 sum L(k) x_k per group and ignore `level`.
cudaError_t launch_pack_xa(const uint16_t *x, const int *tok_of, int P_valid, int P, int K, float level,
                           uint16_t *xa, float *gsq, cudaStream_t s, int *zero_ctr = nullptr, int perm = 0);
// group-sum table of an operand already in XA layout (rows [0, P_valid))
cudaError_t launch_gsum_from_xa(const uint16_t *xa, int P_valid, int P, int K, float level, float *gsq,
                                cudaStream_t s, int perm = 0);

cudaError_t launch_splitk_reduce(const float *partial, int ksplit, size_t split_stride, int M, int N,
                                 uint16_t *y, cudaStream_t s);

// MoE routing: counts, offsets, placement, inverse map; validates ids; zeroes dep[0, E + 3) (if
// given): the fused launch's per-expert counters and three work counters.
cudaError_t launch_moe_route(const int *ids, const float *rw, int T, int topk, int E, int *seg_off,
                             int *cursor, int *tok_of, float *rw_perm, int *inv, int *dep, uint32_t *err,
                             cudaStream_t s);
cudaError_t launch_moe_combine(const float *slot, const int *inv, int T, int topk, int H, uint16_t *y,
                               cudaStream_t s);

}  // namespace ccq
