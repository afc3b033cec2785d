// Host-side offline encoders of libccq: CCQ (6,4,3) code cluster and W4 per-channel RTN.
//
// CCQ: "CCQ: Convolutional Code for Extreme Low-bit Quantization in LLMs", §3.1 Algorithm 1
// (group scale, codebook scaled by it, argmin over the codebook), §3.3 Eq. 1 (code cluster of the
// channel's codes into a byte), §3.4 Eq. 2-4 (closed-form scale refit).  The argmin over the
// 2^15 codes of the (6,4,3) configuration is found with a 64-state trellis search: consecutive
// states of a code share L-S = 3 bits, so the best code ending in each state can be carried from
// one state to the next (Viterbi), instead of enumerating the codebook.
// W4: "GPTQ and AWQ" lesson, Part 2 (rtn with ties to even, pack_int4 nibble order).
//
// Rows are independent; they are spread over std::thread workers.
#include <algorithm>
#include <atomic>
#include <cfenv>
#include <cmath>
#include <cstdint>
#include <climits>
#include <cstring>
#include <thread>
#include <vector>

#include "../../include/ccq.h"

namespace {

inline uint16_t bf16_rne(float x) {
    uint32_t u;
    std::memcpy(&u, &x, 4);
    if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x7FFFFFu)) return uint16_t((u >> 16) | 0x40u);
    uint32_t rounding = 0x7FFFu + ((u >> 16) & 1u);
    return uint16_t((u + rounding) >> 16);
}
inline float bf16_val(uint16_t b) {
    uint32_t u = uint32_t(b) << 16;
    float f;
    std::memcpy(&f, &u, 4);
    return f;
}
inline float to_bf16(float x) { return bf16_val(bf16_rne(x)); }

// The code of a byte under a channel's (alpha, beta): round-half-even of one fp32 FMA.
inline int32_t cluster_code(int c, float alpha, float beta) {
    float t = std::fmaf(float(c), alpha, beta);
    if (!(t == t)) return 0;
    if (t >= 2147483648.0f) return INT32_MAX;
    if (t < -2147483648.0f) return INT32_MIN;
    return int32_t(std::nearbyintf(t));  // current rounding mode: to nearest even (set by caller)
}

// Decoded level of 6-bit state u at group scale s: bf16((u - 32) * bf16(s)), as a double.
inline void levels(float s, double *D) {
    float sb = to_bf16(s);
    for (int u = 0; u < 64; ++u) D[u] = double(to_bf16(float(double(u - 32) * double(sb))));
}

// Best (6,4,3) code for one 4-vector: minimum of ((e0 + e1) + e2) + e3 over all state walks,
// ties to the smallest code.  The running sum at each state is compared after adding the next
// term, exactly as the full sums would be, and the code prefix breaks ties.
inline int32_t trellis_best(const float *v, const double *D) {
    double e[4][64];
    for (int i = 0; i < 4; ++i)
        for (int u = 0; u < 64; ++u) {
            double d = double(v[i]) - D[u];
            e[i][u] = d * d;
        }
    double cost[64];
    int32_t pre[64];
    for (int u = 0; u < 64; ++u) { cost[u] = e[0][u]; pre[u] = u; }
    for (int i = 1; i < 4; ++i) {
        double nc[64];
        int32_t np[64];
        for (int u = 0; u < 64; ++u) {
            int lo = u >> 3;  // the 3 bits this state shares with its predecessor
            double best = INFINITY;
            int32_t bp = 0;
            for (int h = 0; h < 8; ++h) {
                int p = (h << 3) | lo;
                double c = cost[p] + e[i][u];
                int32_t code = (pre[p] << 3) | (u & 7);
                if (c < best || (c == best && code < bp)) { best = c; bp = code; }
            }
            nc[u] = best;
            np[u] = bp;
        }
        std::memcpy(cost, nc, sizeof(cost));
        std::memcpy(pre, np, sizeof(pre));
    }
    double best = INFINITY;
    int32_t arg = 0;
    for (int u = 0; u < 64; ++u)
        if (cost[u] < best || (cost[u] == best && pre[u] < arg)) { best = cost[u]; arg = pre[u]; }
    return arg;
}

struct ByteTable {
    // states of each byte's code for one channel: st[c][i]
    uint8_t st[256][4];
    void build(float alpha, float beta) {
        for (int c = 0; c < 256; ++c) {
            uint32_t C = uint32_t(cluster_code(c, alpha, beta));
            for (int i = 0; i < 4; ++i) st[c][i] = uint8_t((C >> (9 - 3 * i)) & 0x3Fu);
        }
    }
};

inline uint8_t best_byte(const float *v, const double *D, const ByteTable &bt) {
    double best = INFINITY;
    int arg = 0;
    for (int c = 0; c < 256; ++c) {
        double err = 0.0;
        for (int i = 0; i < 4; ++i) {
            double d = double(v[i]) - D[bt.st[c][i]];
            err += d * d;
        }
        if (err < best) { best = err; arg = c; }
    }
    return uint8_t(arg);
}

// q4 != nullptr: 4-bit group scales (CCQ §3.4 "Scale Compression"): q4[g] and *super_out are
// outputs and scales[] holds the group scales fl32(q4 * super) the search uses.
void encode_row(const float *wr, int k, int group, uint32_t flags, uint8_t *codes, float *scales,
                float *alpha_out, float *beta_out, double *err_out, uint8_t *q4 = nullptr,
                float *super_out = nullptr) {
    const int ng = k / group, nv = k / 4, vpg = group / 4;
    std::vector<int32_t> C(nv);
    std::vector<double> Dall(size_t(ng) * 64);
    if (q4) {
        double smax = 0.0;
        for (int g = 0; g < ng; ++g) {
            double amax = 0.0;
            for (int i = 0; i < group; ++i) amax = std::max(amax, std::fabs(double(wr[g * group + i])));
            scales[g] = float(amax / 31.0);
            smax = std::max(smax, double(scales[g]));
        }
        const float sup = float(smax / 15.0);
        *super_out = sup;
        for (int g = 0; g < ng; ++g) {
            double qq = sup > 0.0f ? std::nearbyint(double(scales[g]) / double(sup)) : 0.0;
            q4[g] = uint8_t(std::min(15.0, std::max(0.0, qq)));
            scales[g] = float(q4[g]) * sup;
        }
    }
    for (int g = 0; g < ng; ++g) {
        float s;
        if (q4) {
            s = scales[g];
        } else {
            double amax = 0.0;
            for (int i = 0; i < group; ++i) amax = std::max(amax, std::fabs(double(wr[g * group + i])));
            s = to_bf16(float(amax / 31.0));
        }
        scales[g] = s;
        double *D = &Dall[size_t(g) * 64];
        levels(s, D);
        for (int q = 0; q < vpg; ++q) C[g * vpg + q] = trellis_best(wr + g * group + q * 4, D);
    }
    int32_t cmin = *std::min_element(C.begin(), C.end());
    int32_t cmax = *std::max_element(C.begin(), C.end());
    float b = float(cmin);
    float a = (cmax == cmin) ? 1.0f : float(cmax - cmin) / 255.0f;
    *alpha_out = a;
    *beta_out = b;
    ByteTable bt;
    bt.build(a, b);
    for (int g = 0; g < ng; ++g) {
        const double *D = &Dall[size_t(g) * 64];
        for (int q = 0; q < vpg; ++q) {
            int j = g * vpg + q;
            if (flags & CCQ_ENC_LITERAL_EQ1) {
                float qq = std::nearbyintf((float(C[j]) - b) / a);
                qq = std::min(255.0f, std::max(0.0f, qq));
                codes[j] = uint8_t(qq);
            } else {
                codes[j] = best_byte(wr + size_t(j) * 4, D, bt);
            }
        }
        if ((flags & CCQ_ENC_REFIT_SCALE) && !q4) {
            double num = 0.0, den = 0.0;
            for (int q = 0; q < vpg; ++q) {
                int j = g * vpg + q;
                for (int i = 0; i < 4; ++i) {
                    double lev = double(bt.st[codes[j]][i]) - 32.0;
                    num += double(wr[size_t(j) * 4 + i]) * lev;
                    den += lev * lev;
                }
            }
            if (den > 0.0 && num / den > 0.0) {
                float s2 = to_bf16(float(num / den));
                if (s2 > 0.0f) {
                    scales[g] = s2;
                    double D2[64];
                    levels(s2, D2);
                    if (!(flags & CCQ_ENC_LITERAL_EQ1))
                        for (int q = 0; q < vpg; ++q) {
                            int j = g * vpg + q;
                            codes[j] = best_byte(wr + size_t(j) * 4, D2, bt);
                        }
                }
            }
        }
    }
    if (err_out) {
        double e = 0.0;
        for (int g = 0; g < ng; ++g) {
            double D[64];
            levels(scales[g], D);
            for (int q = 0; q < vpg; ++q) {
                int j = g * vpg + q;
                for (int i = 0; i < 4; ++i) {
                    double d = double(wr[size_t(j) * 4 + i]) - D[bt.st[codes[j]][i]];
                    e += d * d;
                }
            }
        }
        *err_out = e;
    }
}

template <typename F>
void parallel_rows(int n, int threads, F &&fn) {
    int hw = int(std::thread::hardware_concurrency());
    int nt = threads > 0 ? threads : std::max(1, hw);
    nt = std::max(1, std::min(nt, n));
    std::atomic<int> next{0};
    auto worker = [&]() {
        std::fesetround(FE_TONEAREST);
        for (;;) {
            int r = next.fetch_add(1);
            if (r >= n) break;
            fn(r);
        }
    };
    if (nt == 1) { worker(); return; }
    std::vector<std::thread> pool;
    pool.reserve(nt);
    for (int t = 0; t < nt; ++t) pool.emplace_back(worker);
    for (auto &th : pool) th.join();
}

}  // namespace

extern "C" ccq_status ccq_encode_host(const float *w, int32_t n, int32_t k, int32_t group, uint32_t flags,
                                      int32_t threads, uint8_t *codes, float *scales, float *alpha,
                                      float *beta, double *sq_err) {
    if (!w || !codes || !scales || !alpha || !beta) return CCQ_ERR_INVALID_ARG;
    if (n < 0 || k <= 0 || group <= 0 || group % 4 || k % group) return CCQ_ERR_INVALID_ARG;
    if (flags & ~uint32_t(CCQ_ENC_LITERAL_EQ1 | CCQ_ENC_REFIT_SCALE)) return CCQ_ERR_INVALID_ARG;
    if (n == 0) { if (sq_err) *sq_err = 0.0; return CCQ_OK; }
    std::vector<double> errs(sq_err ? size_t(n) : 0);
    const int ng = k / group;
    parallel_rows(n, threads, [&](int r) {
        encode_row(w + size_t(r) * k, k, group, flags, codes + size_t(r) * (k / 4), scales + size_t(r) * ng,
                   alpha + r, beta + r, sq_err ? &errs[r] : nullptr);
    });
    if (sq_err) {
        double e = 0.0;
        for (double v : errs) e += v;
        *sq_err = e;
    }
    return CCQ_OK;
}

extern "C" ccq_status ccq_encode_host_q4(const float *w, int32_t n, int32_t k, int32_t group, uint32_t flags,
                                         int32_t threads, uint8_t *codes, uint8_t *scale_q4, float *super_scale,
                                         float *alpha, float *beta, double *sq_err) {
    if (!w || !codes || !scale_q4 || !super_scale || !alpha || !beta) return CCQ_ERR_INVALID_ARG;
    if (n < 0 || k <= 0 || group <= 0 || group % 4 || k % (2 * group)) return CCQ_ERR_INVALID_ARG;
    if (flags & ~uint32_t(CCQ_ENC_LITERAL_EQ1)) return CCQ_ERR_INVALID_ARG;
    if (n == 0) { if (sq_err) *sq_err = 0.0; return CCQ_OK; }
    std::vector<double> errs(sq_err ? size_t(n) : 0);
    const int ng = k / group;
    parallel_rows(n, threads, [&](int r) {
        std::vector<float> sc(ng);
        std::vector<uint8_t> q(ng);
        encode_row(w + size_t(r) * k, k, group, flags, codes + size_t(r) * (k / 4), sc.data(), alpha + r, beta + r,
                   sq_err ? &errs[r] : nullptr, q.data(), super_scale + r);
        uint8_t *dst = scale_q4 + size_t(r) * (ng / 2);
        for (int b = 0; b < ng / 2; ++b) dst[b] = uint8_t(q[2 * b] | (q[2 * b + 1] << 4));
    });
    if (sq_err) {
        double e = 0.0;
        for (double v : errs) e += v;
        *sq_err = e;
    }
    return CCQ_OK;
}

extern "C" ccq_status ccq_quantize_w4_host(const float *w, int32_t n, int32_t k, int32_t threads,
                                           uint8_t *codes, float *scales) {
    if (!w || !codes || !scales || n < 0 || k <= 0 || k % 2) return CCQ_ERR_INVALID_ARG;
    if (n == 0) return CCQ_OK;
    parallel_rows(n, threads, [&](int r) {
        const float *wr = w + size_t(r) * k;
        double amax = 0.0;
        for (int i = 0; i < k; ++i) amax = std::max(amax, std::fabs(double(wr[i])));
        float s = to_bf16(float(amax / 7.0));
        scales[r] = s;
        for (int i = 0; i < k; i += 2) {
            int q[2];
            for (int h = 0; h < 2; ++h) {
                double v = s > 0.0f ? double(wr[i + h]) / double(s) : 0.0;
                double qr = std::nearbyint(v);
                q[h] = int(std::min(7.0, std::max(-8.0, qr)));
            }
            codes[size_t(r) * (k / 2) + i / 2] = uint8_t((q[0] & 0xF) | ((q[1] & 0xF) << 4));
        }
    });
    return CCQ_OK;
}
