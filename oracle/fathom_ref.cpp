/*
 * fathom_ref.cpp -- the ORACLE for the Fathom variable-depth bit-plane key scan.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is a plain, slow, single-threaded
 * restatement of what the method computes, written to be checked by eye
 * against the pages that describe it.  Only the tests, __graft_entry__.smoke()
 * and bench.py's CPU-baseline / reference arm may load it.  The product
 * (bit_plane_key_b200/) never links, imports or calls it, and it shares no
 * code with the CUDA path (no headers, tables, helpers or constants).
 *
 * Sources (page title, then the section the fact sits in):
 *   [ABS]  "Fathom: Per-Query Read Depth for Sparse Decoding over Offloaded KV
 *          Caches", arXiv 2609.17652 abstract (aiqbench.com mirror).
 *   [AIF]  "Fathom:面向卸载 KV Cache 的稀疏解码的逐查询读取深度" (ai-feeds.com
 *          summary), section 方法 (method): 输入 (inputs), 关键模块 (modules 1-5),
 *          输出 (output).
 *   [EVO]  evolve.pub review of the same paper: "Strengths" (citing the
 *          paper's Sec 3.2 shared block scale, Sec 3.3 depth rule, Sec 3.6
 *          contiguous runs, Appendix A) and "Frequently asked questions".
 *
 * Precision: fp64 throughout, except two places where the method's decision
 * is taken in a fixed narrower format so that the GPU can reach the same
 * integer result: the fp16 block scale (the store format) and the fp32
 * channel importance w = fl32(fl32(q*q) * sigma2).  Build with
 * -ffp-contract=off so that no fused multiply-add changes those roundings.
 *
 * Readings taken where the pages are silent (the same readings as the CUDA path):
 *   - mid-rise code: Delta = fp16_rn(amax/8), u = floor(x/Delta),
 *     code = clamp(u,-8,7)+8, offset binary, plane 0 = most significant bit;
 *   - basis rule: a t-plane prefix is rebuilt with the signed plane basis
 *     khat = Delta * sum_{j<t} (2 b_j - 1) 2^(2-j), which is the t-bit
 *     mid-rise quantizer value (t = 0 gives 0);
 *   - water-filling: candidates (c,t), value w_c 4^-t, ordered by value
 *     descending, then channel ascending, then t ascending; the first
 *     min(B,4d) are taken and t_c counts those on channel c;
 *   - fixed-r baselines: depth 4 on the r channels with the largest |q_c|
 *     (ties to the lower channel);
 *   - top-k: order (score descending, index ascending);
 *   - attention: softmax(q.K/sqrt(d)) V over the selected bf16 rows.
 *
 * Parity pins for every function live in tests/test_oracle_*.py.
 */
#include <stdint.h>
#include <math.h>
#include <string.h>
#include <stdlib.h>
#include <algorithm>
#include <vector>

typedef int64_t i64;

static const int BLOCK = 64;  /* tokens per shared block scale */
static const int PAD = 1024;  /* keys are padded to a multiple of this (a layout convention of the store) */

/* ------------------------------------------------------------------------ */
/* fp16 / bf16 conversions written from the IEEE 754 binary16 definition.    */
/* ------------------------------------------------------------------------ */

static uint32_t f32_bits(float x) { uint32_t u; memcpy(&u, &x, 4); return u; }
static float bits_f32(uint32_t u) { float x; memcpy(&x, &u, 4); return x; }

/* Round an fp32 value to the nearest binary16 value, ties to even.
 * Done in exact fp64 arithmetic on the value, not by bit tricks:
 * binary16 has 11 significant bits, exponents -14..15, subnormal
 * spacing 2^-24, largest finite 65504, and values at or beyond
 * 65520 (the midpoint to 2^16) round to infinity. */
extern "C" uint16_t oref_f32_to_f16(float xf) {
    double x = (double)xf;
    uint16_t sign = (f32_bits(xf) >> 31) ? 0x8000 : 0;
    double a = fabs(x);
    if (xf != xf) return 0x7E00; /* NaN */
    if (a >= 65520.0) return sign | 0x7C00;
    if (a == 0.0) return sign;
    int e; /* a = f * 2^e with f in [0.5, 1) */
    frexp(a, &e);
    int exp2 = e - 1;              /* a in [2^exp2, 2^(exp2+1)) */
    if (exp2 < -14) exp2 = -14;    /* subnormal range shares the 2^-24 spacing */
    double ulp = ldexp(1.0, exp2 - 10);
    double m = a / ulp;            /* exact: scaling by a power of two */
    double fl = floor(m);
    double frac = m - fl;
    double r;
    if (frac > 0.5) r = fl + 1.0;
    else if (frac < 0.5) r = fl;
    else r = (fmod(fl, 2.0) == 0.0) ? fl : fl + 1.0;
    double v = r * ulp;            /* rounded magnitude */
    if (v >= 65520.0) return sign | 0x7C00;
    /* encode v */
    if (v < ldexp(1.0, -14)) {     /* subnormal: v = k * 2^-24 */
        uint16_t k = (uint16_t)(v / ldexp(1.0, -24));
        return sign | k;
    }
    int ev;
    double fr = frexp(v, &ev);     /* v = fr * 2^ev, fr in [0.5,1) */
    int E = ev - 1;                /* v = (2 fr) * 2^E */
    uint16_t mant = (uint16_t)((2.0 * fr - 1.0) * 1024.0);
    return sign | (uint16_t)((E + 15) << 10) | mant;
}

extern "C" float oref_f16_to_f32(uint16_t h) {
    int s = (h >> 15) & 1;
    int E = (h >> 10) & 0x1F;
    int m = h & 0x3FF;
    double v;
    if (E == 0) v = ldexp((double)m, -24);
    else if (E == 31) v = m ? NAN : INFINITY;
    else v = ldexp(1.0 + m / 1024.0, E - 15);
    return (float)(s ? -v : v);
}

static float bf16_to_f32(uint16_t h) { return bits_f32(((uint32_t)h) << 16); }

/* ------------------------------------------------------------------------ */
/* Store geometry                                                            */
/* ------------------------------------------------------------------------ */

extern "C" i64 oref_n_pad(i64 n) { return ((n + PAD - 1) / PAD) * PAD; }

/* planes u32 [H][d][4][n_pad/32]: key i -> word i/32, bit i%32, plane 0 = MSB
 * scales u16 [H][d][n_pad/64]: fp16 bits of Delta for (head, channel, block) */
static i64 plane_word_index(int g, int c, int j, i64 i, int d, i64 npad) {
    return (((i64)g * d + c) * 4 + j) * (npad / 32) + i / 32;
}
static i64 scale_index(int g, int c, i64 b, int d, i64 npad) {
    return ((i64)g * d + c) * (npad / BLOCK) + b;
}

/* ------------------------------------------------------------------------ */
/* (1) 4-bit mid-rise quantizer with one shared fp16 scale per 64-token      */
/*     block per channel [AIF 关键模块 1; EVO Strengths, paper Sec 3.2;        */
/*     EVO FAQ "How does Fathom's bit-plane KV cache work?"]                 */
/* ------------------------------------------------------------------------ */

/* K f32 [H][n][d] -> scales (fp16 bits) [H][d][n_pad/64], codes u8 [H][n][d] */
extern "C" void oref_quantize(const float* K, int H, i64 n, int d,
                              uint16_t* scales, uint8_t* codes) {
    i64 npad = oref_n_pad(n);
    i64 nblk = npad / BLOCK;
    for (int g = 0; g < H; ++g)
        for (int c = 0; c < d; ++c)
            for (i64 b = 0; b < nblk; ++b) {
                i64 i0 = b * BLOCK, i1 = std::min(n, i0 + BLOCK);
                float amax = 0.0f;
                for (i64 i = i0; i < i1; ++i) {
                    float a = fabsf(K[((i64)g * n + i) * d + c]);
                    if (a > amax) amax = a;
                }
                uint16_t h = oref_f32_to_f16(amax / 8.0f);
                scales[scale_index(g, c, b, d, npad)] = h;
                double delta = (double)oref_f16_to_f32(h);
                for (i64 i = i0; i < i1; ++i) {
                    double x = (double)K[((i64)g * n + i) * d + c];
                    int code;
                    if (delta == 0.0) {
                        code = 8;
                    } else {
                        double u = floor(x / delta);  /* exact for fp32 x, fp16 delta */
                        if (u < -8.0) u = -8.0;
                        if (u > 7.0) u = 7.0;
                        code = (int)u + 8;
                    }
                    codes[((i64)g * n + i) * d + c] = (uint8_t)code;
                }
            }
}

/* (2) Channel-major bit planes [AIF 输入, 关键模块 1; ABS]: each bit position of
 *     the 4-bit code is its own plane and a channel's four planes are
 *     adjacent.  Bit j of plane j is bit (3-j) of the code. */
extern "C" void oref_pack_planes(const uint8_t* codes, int H, i64 n, int d, uint32_t* planes) {
    i64 npad = oref_n_pad(n);
    memset(planes, 0, sizeof(uint32_t) * (size_t)H * d * 4 * (npad / 32));
    for (int g = 0; g < H; ++g)
        for (i64 i = 0; i < n; ++i)
            for (int c = 0; c < d; ++c) {
                int code = codes[((i64)g * n + i) * d + c];
                for (int j = 0; j < 4; ++j) {
                    uint32_t bit = (uint32_t)((code >> (3 - j)) & 1);
                    planes[plane_word_index(g, c, j, i, d, npad)] |= bit << (i % 32);
                }
            }
}

extern "C" void oref_pack(const float* K, int H, i64 n, int d, uint32_t* planes, uint16_t* scales) {
    std::vector<uint8_t> codes((size_t)H * n * d);
    oref_quantize(K, H, n, d, scales, codes.data());
    oref_pack_planes(codes.data(), H, n, d, planes);
}

/* ------------------------------------------------------------------------ */
/* (3) Variance-weighted importance w_c = q_c^2 sigma_c^2 [ABS; AIF 输入]     */
/*     taken in fp32: w = fl32(fl32(q*q) * sigma2).                          */
/* ------------------------------------------------------------------------ */
extern "C" void oref_importance(const float* q, const float* sigma2, int d, float* w) {
    for (int c = 0; c < d; ++c) {
        volatile float qq = q[c] * q[c];
        volatile float wc = qq * sigma2[c];
        w[c] = wc;
    }
}

/* ------------------------------------------------------------------------ */
/* (4) Reverse water-filling over the 4x-per-bit error model                 */
/*     [ABS; AIF 关键模块 2; EVO Strengths, paper Sec 3.3].                     */
/*     Distortion of channel c at depth t is w_c 4^-t; reading plane t of     */
/*     channel c removes 3/4 of w_c 4^-t.  Greedy on the candidates          */
/*     v(c,t) = w_c 4^-t (t = 0..3) is optimal for this separable convex     */
/*     problem; the value of the last candidate taken is the water level.   */
/* ------------------------------------------------------------------------ */
struct Cand { double v; int c; int t; };

static bool cand_before(const Cand& a, const Cand& b) {
    if (a.v != b.v) return a.v > b.v;
    if (a.c != b.c) return a.c < b.c;
    return a.t < b.t;
}

/* returns 0, or -1 for B < 0 */
extern "C" int oref_depths(const float* w, int d, int B, uint8_t* t_out) {
    if (B < 0) return -1;
    std::vector<Cand> cands;
    for (int c = 0; c < d; ++c)
        for (int t = 0; t < 4; ++t) {
            Cand x;
            x.v = (double)w[c] * ldexp(1.0, -2 * t);
            x.c = c;
            x.t = t;
            cands.push_back(x);
        }
    std::sort(cands.begin(), cands.end(), cand_before);
    int take = std::min(B, 4 * d);
    for (int c = 0; c < d; ++c) t_out[c] = 0;
    for (int k = 0; k < take; ++k) {
        /* candidates of one channel come out in t order, so what is taken on
           a channel is always a prefix 0..t_c-1 of its planes */
        if (cands[k].t != t_out[cands[k].c]) return -2;
        t_out[cands[k].c] += 1;
    }
    return 0;
}

/* Fixed-depth comparison scans ("68-bit" r=16, "136-bit" r=32) [ABS; AIF
 * 与 Double Sparsity/Loki/SparQ 的差异]: depth 4 on the r channels with the
 * largest |q_c|, ties to the lower channel. */
extern "C" int oref_fixed_depths(const float* q, int d, int r, uint8_t* t_out) {
    if (r < 0) return -1;
    std::vector<int> order(d);
    for (int c = 0; c < d; ++c) order[c] = c;
    std::sort(order.begin(), order.end(), [&](int a, int b) {
        float qa = fabsf(q[a]), qb = fabsf(q[b]);
        if (qa != qb) return qa > qb;
        return a < b;
    });
    for (int c = 0; c < d; ++c) t_out[c] = 0;
    for (int k = 0; k < std::min(r, d); ++k) t_out[order[k]] = 4;
    return 0;
}

/* Per query head: importance from its own q and its KV head's sigma^2, then
 * the depth rule (fixed_r == 0) or the fixed-r baseline. q f32 [Hq][d],
 * sigma2 f32 [Hkv][d], depths u8 [Hq][d]. */
extern "C" int oref_alloc_depths(const float* q, const float* sigma2, int Hq, int Hkv, int d,
                                 int B, int fixed_r, uint8_t* depths) {
    if (Hkv <= 0 || Hq % Hkv) return -1;
    int G = Hq / Hkv;
    std::vector<float> w(d);
    for (int h = 0; h < Hq; ++h) {
        int rc;
        if (fixed_r == 0) {
            oref_importance(q + (i64)h * d, sigma2 + (i64)(h / G) * d, d, w.data());
            rc = oref_depths(w.data(), d, B, depths + (i64)h * d);
        } else {
            rc = oref_fixed_depths(q + (i64)h * d, d, fixed_r, depths + (i64)h * d);
        }
        if (rc) return rc;
    }
    return 0;
}

/* Group-pooled variant (not the pages' per-query rule): the importance of
 * channel c for KV head g is the fp32 sum, heads in order, of the group's
 * per-head importances; one water-filling per KV head, copied to every
 * query head of the group. */
extern "C" int oref_alloc_depths_pooled(const float* q, const float* sigma2, int Hq, int Hkv, int d, int B,
                                        uint8_t* depths) {
    if (Hkv <= 0 || Hq % Hkv) return -1;
    int G = Hq / Hkv;
    std::vector<float> w(d), wh(d);
    for (int g = 0; g < Hkv; ++g) {
        for (int c = 0; c < d; ++c) w[c] = 0.0f;
        for (int h = g * G; h < (g + 1) * G; ++h) {
            oref_importance(q + (i64)h * d, sigma2 + (i64)g * d, d, wh.data());
            for (int c = 0; c < d; ++c) {
                volatile float acc = w[c] + wh[c];
                w[c] = acc;
            }
        }
        int rc = oref_depths(w.data(), d, B, depths + (i64)g * G * d);
        if (rc) return rc;
        for (int h = g * G + 1; h < (g + 1) * G; ++h)
            for (int c = 0; c < d; ++c) depths[(i64)h * d + c] = depths[(i64)g * G * d + c];
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* (5) Basis rule on a read prefix [AIF 关键模块 4, paper Sec 3.5; ABS;       */
/*     EVO Strengths, paper Sec 3.2]: khat = Delta * sum_{j<t}(2b_j-1)2^(2-j) */
/* ------------------------------------------------------------------------ */
static double khat_from_planes(const uint32_t* planes, const uint16_t* scales, int g, int c,
                               i64 i, int t, int d, i64 npad) {
    double delta = (double)oref_f16_to_f32(scales[scale_index(g, c, i / BLOCK, d, npad)]);
    double sum = 0.0;
    for (int j = 0; j < t; ++j) {
        uint32_t word = planes[plane_word_index(g, c, j, i, d, npad)];
        int b = (int)((word >> (i % 32)) & 1u);
        sum += (2.0 * b - 1.0) * ldexp(1.0, 2 - j);
    }
    return delta * sum;
}

/* khat f64 [n][d] of KV head g, channel c read to depth t[c] */
extern "C" void oref_reconstruct(const uint32_t* planes, const uint16_t* scales, int H, i64 n, int d,
                                 int g, const uint8_t* t, double* khat) {
    (void)H;
    i64 npad = oref_n_pad(n);
    for (i64 i = 0; i < n; ++i)
        for (int c = 0; c < d; ++c)
            khat[i * d + c] = khat_from_planes(planes, scales, g, c, i, t[c], d, npad);
}

/* ------------------------------------------------------------------------ */
/* (6) Approximate scores s_{h,i} = sum_c q_{h,c} khat_{i,c} over every key  */
/*     [ABS: "the scan that ranks all n keys"; AIF 关键模块 5].                 */
/*     Query head h reads KV head h / (Hq/Hkv).  Keys [i0, i1) only.         */
/*     scores/absterm f64 [Hq][i1-i0]; absterm = sum_c |q_c khat_c|, the     */
/*     scale the score tolerance is stated against (may be NULL).           */
/* ------------------------------------------------------------------------ */
/* one query head q_h [d] with depths t_h [d] against KV head g */
extern "C" int oref_scores_head(const uint32_t* planes, const uint16_t* scales, int Hkv, i64 n, int d,
                                int g, const float* q_h, const uint8_t* t_h, i64 i0, i64 i1,
                                double* scores, double* absterm) {
    if (g < 0 || g >= Hkv || i0 < 0 || i1 > n || i0 > i1) return -1;
    for (int c = 0; c < d; ++c)
        if (t_h[c] > 4) return -1;
    i64 npad = oref_n_pad(n);
    for (i64 i = i0; i < i1; ++i) {
        double s = 0.0, a = 0.0;
        for (int c = 0; c < d; ++c) {
            double kh = khat_from_planes(planes, scales, g, c, i, t_h[c], d, npad);
            double term = (double)q_h[c] * kh;
            s += term;
            a += fabs(term);
        }
        scores[i - i0] = s;
        if (absterm) absterm[i - i0] = a;
    }
    return 0;
}

extern "C" int oref_scores(const uint32_t* planes, const uint16_t* scales, int Hkv, i64 n, int d,
                           const float* q, int Hq, const uint8_t* depths, i64 i0, i64 i1,
                           double* scores, double* absterm) {
    if (Hkv <= 0 || Hq % Hkv || i0 < 0 || i1 > n || i0 > i1) return -1;
    int G = Hq / Hkv;
    i64 m = i1 - i0;
    for (int h = 0; h < Hq; ++h) {
        int rc = oref_scores_head(planes, scales, Hkv, n, d, h / G, q + (i64)h * d, depths + (i64)h * d,
                                  i0, i1, scores + (i64)h * m, absterm ? absterm + (i64)h * m : NULL);
        if (rc) return rc;
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* (7) Top-k: the k keys with the largest score, ties to the lower index,    */
/*     listed in that order [AIF 关键模块 5, 输出; ABS].                         */
/* ------------------------------------------------------------------------ */
template <typename T>
static int topk_sorted(const T* s, i64 n, int k, int32_t* idx) {
    if (k < 0 || k > n) return -1;
    std::vector<int32_t> order((size_t)n);
    for (i64 i = 0; i < n; ++i) order[i] = (int32_t)i;
    std::sort(order.begin(), order.end(), [&](int32_t a, int32_t b) {
        if (s[a] != s[b]) return s[a] > s[b];
        return a < b;
    });
    for (int j = 0; j < k; ++j) idx[j] = order[j];
    return 0;
}
extern "C" int oref_topk_f64(const double* s, i64 n, int k, int32_t* idx) { return topk_sorted(s, n, k, idx); }
extern "C" int oref_topk_f32(const float* s, i64 n, int k, int32_t* idx) { return topk_sorted(s, n, k, idx); }

/* ------------------------------------------------------------------------ */
/* (8) Exact attention over the selected keys only [AIF 关键模块 5, 输出].     */
/*     o_h = softmax(q_h . K_idx / sqrt(d)) V_idx with bf16 rows            */
/*     K_rows, V_rows [Hkv][n][d] (bf16 bits), idx [Hq][k], out f64 [Hq][d] */
/* ------------------------------------------------------------------------ */
extern "C" int oref_attend(const float* q, const uint16_t* Krows, const uint16_t* Vrows,
                           const int32_t* idx, int Hq, int Hkv, i64 n, int d, int k, double* out) {
    if (Hkv <= 0 || Hq % Hkv || k < 1) return -1;
    int G = Hq / Hkv;
    std::vector<double> logit(k);
    for (int h = 0; h < Hq; ++h) {
        int g = h / G;
        double mx = -INFINITY;
        for (int j = 0; j < k; ++j) {
            i64 i = idx[(i64)h * k + j];
            if (i < 0 || i >= n) return -1;
            double dot = 0.0;
            for (int c = 0; c < d; ++c)
                dot += (double)q[(i64)h * d + c] * (double)bf16_to_f32(Krows[((i64)g * n + i) * d + c]);
            logit[j] = dot / sqrt((double)d);
            if (logit[j] > mx) mx = logit[j];
        }
        double z = 0.0;
        for (int j = 0; j < k; ++j) { logit[j] = exp(logit[j] - mx); z += logit[j]; }
        for (int c = 0; c < d; ++c) {
            double o = 0.0;
            for (int j = 0; j < k; ++j) {
                i64 i = idx[(i64)h * k + j];
                o += logit[j] * (double)bf16_to_f32(Vrows[((i64)g * n + i) * d + c]);
            }
            out[(i64)h * d + c] = o / z;
        }
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* One decode step of one layer over a packed store: depths, scores of all  */
/* keys, top-k, attention.  Used for whole-path parity and as the CPU       */
/* baseline.  depths u8 [Hq][d], idx [Hq][k], out f64 [Hq][d].              */
/* ------------------------------------------------------------------------ */
extern "C" int oref_decode(const uint32_t* planes, const uint16_t* scales, const uint16_t* Krows,
                           const uint16_t* Vrows, const float* q, const float* sigma2, int Hq, int Hkv,
                           i64 n, int d, int B, int fixed_r, int k, uint8_t* depths, int32_t* idx,
                           double* out) {
    int rc = oref_alloc_depths(q, sigma2, Hq, Hkv, d, B, fixed_r, depths);
    if (rc) return rc;
    std::vector<double> s((size_t)n);
    int G = Hq / Hkv;
    for (int h = 0; h < Hq; ++h) {
        rc = oref_scores_head(planes, scales, Hkv, n, d, h / G, q + (i64)h * d, depths + (i64)h * d,
                              0, n, s.data(), NULL);
        if (rc) return rc;
        rc = oref_topk_f64(s.data(), n, k, idx + (i64)h * k);
        if (rc) return rc;
    }
    if (Krows && Vrows && out) return oref_attend(q, Krows, Vrows, idx, Hq, Hkv, n, d, k, out);
    return 0;
}

/* elementwise fp32 -> fp16 (bits), for the rounding pin */
extern "C" void oref_f32_to_f16_array(const float* x, uint16_t* out, i64 m) {
    for (i64 i = 0; i < m; ++i) out[i] = oref_f32_to_f16(x[i]);
}
