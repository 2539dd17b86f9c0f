// K2: per-query read depths.
//
// Reverse water-filling over the variance-weighted channel importance
// w_c = q_c^2 sigma_c^2 (arXiv abstract; ai-feeds.com summary, 方法 · 关键模块 2;
// evolve.pub review, Strengths: depth rule from the 4x-per-bit error reduction,
// paper Sec 3.3).  Reading plane t of channel c removes three quarters of the
// remaining distortion w_c 4^-t, so spending B plane-bits optimally means
// taking the B largest candidates v(c,t) = w_c 4^-t, t = 0..3.  The water
// level theta is the value of the last candidate taken.
//
// One warp per query head.  Every candidate gets a distinct 64-bit key that
// orders exactly as (v descending, c ascending, t ascending):
//   the fp64 bit pattern of v = (double)w * 2^-2t (exact; a positive double's
//   bits are monotone in its value, and an fp32 w leaves the low 29 bits of
//   the pattern zero) OR-ed with ((255 - c) << 2 | (3 - t)).
// theta is found by a bitwise radix select of the N-th largest key (bisection
// on the threshold, 64 steps of one warp-wide count each); then
// t_c = #{t : key(c,t) >= theta}.  Because the keys are distinct exactly N
// candidates pass, so sum_c t_c = N = min(B, 4d).
//
// Group-pooled variant (not in the pages, which decide per query: arXiv
// abstract, "each query decides"): the importance of channel c for KV head g
// is the fp32 sum, in head order, of the group's per-head w_{h,c}; one water
// level per KV head; every head of the group gets the same depths, so the
// scan reads exactly min(B, 4d) plane bits per key and KV head.
//
// Fixed-r comparison scans (ai-feeds.com summary, 与 Double Sparsity / Loki /
// SparQ 的差异: a fixed 68 or 136 bits per key): depth 4 on the r channels with
// the largest |q_c|, ties to the lower channel, by the same select on the
// keys (bits(|q_c|) << 8 | (255 - c)).
#include "fathom_internal.cuh"

namespace fathom {
namespace {

constexpr int kWarpsPerCta = 4;
constexpr int kMaxChan = kMaxD / 32;  // channels per lane

__device__ __forceinline__ int warp_count_ge(const uint64_t* keys, int m, uint64_t thr) {
    int cnt = 0;
#pragma unroll
    for (int e = 0; e < 4 * kMaxChan; ++e)
        if (e < m && keys[e] >= thr) ++cnt;
    return __reduce_add_sync(0xffffffffu, cnt);
}

// Largest T with #{keys >= T} >= N (1 <= N <= total); exact N-th largest.
__device__ __forceinline__ uint64_t warp_select(const uint64_t* keys, int m, int N) {
    uint64_t T = 0;
    for (int bit = 63; bit >= 0; --bit) {
        uint64_t cand = T | (1ull << bit);
        if (warp_count_ge(keys, m, cand) >= N) T = cand;
    }
    return T;
}

__global__ void __launch_bounds__(kWarpsPerCta * 32)
depths_kernel(const void* __restrict__ q, int q_dtype, const float* __restrict__ sigma2, int Hq, int Hkv,
              int d, int budget, int fixed_r, int pooled, uint8_t* __restrict__ depths) {
    const int lane = threadIdx.x & 31;
    const int h = blockIdx.x * kWarpsPerCta + (threadIdx.x >> 5);
    if (h >= Hq) return;
    const int g = h / (Hq / Hkv);
    const int per_lane = d / 32;  // channel c = lane + 32 * e
    uint64_t keys[4 * kMaxChan];
    int m;
    int N;
    if (fixed_r == 0) {
        m = 4 * per_lane;
        N = min(budget, 4 * d);
#pragma unroll
        for (int e = 0; e < kMaxChan; ++e) {
            if (e < per_lane) {
                int c = lane + 32 * e;
                const float s2 = sigma2[(int64_t)g * d + c];
                float w;
                if (pooled) {   // sum of the group's per-head importances, in head order
                    const int G = Hq / Hkv;
                    w = 0.0f;
                    for (int hh = g * G; hh < (g + 1) * G; ++hh) {
                        const float qc = load_q(q, q_dtype, (int64_t)hh * d + c);
                        w = __fadd_rn(w, __fmul_rn(__fmul_rn(qc, qc), s2));
                    }
                } else {
                    const float qc = load_q(q, q_dtype, (int64_t)h * d + c);
                    w = __fmul_rn(__fmul_rn(qc, qc), s2);
                }
#pragma unroll
                for (int t = 0; t < 4; ++t) {
                    double v = (double)w * ((t == 0) ? 1.0 : (t == 1) ? 0.25 : (t == 2) ? 0.0625 : 0.015625);
                    keys[4 * e + t] = (uint64_t)__double_as_longlong(v) |
                                      ((uint64_t)(255 - c) << 2) | (uint64_t)(3 - t);
                }
            }
        }
    } else {
        m = per_lane;
        N = min(fixed_r, d);
#pragma unroll
        for (int e = 0; e < kMaxChan; ++e) {
            if (e < per_lane) {
                int c = lane + 32 * e;
                float qa = fabsf(load_q(q, q_dtype, (int64_t)h * d + c));
                keys[e] = ((uint64_t)__float_as_uint(qa) << 8) | (uint64_t)(255 - c);
            }
        }
    }
    uint64_t theta = ~0ull;  // N == 0: nothing passes
    if (N > 0) theta = warp_select(keys, m, N);
#pragma unroll
    for (int e = 0; e < kMaxChan; ++e) {
        if (e < per_lane) {
            int c = lane + 32 * e;
            int t;
            if (fixed_r == 0) {
                t = 0;
#pragma unroll
                for (int s = 0; s < 4; ++s) t += (N > 0 && keys[4 * e + s] >= theta) ? 1 : 0;
            } else {
                t = (N > 0 && keys[e] >= theta) ? 4 : 0;
            }
            depths[(int64_t)h * d + c] = (uint8_t)t;
        }
    }
}

}  // namespace

cudaError_t launch_depths(const void* q, int q_dtype, const float* sigma2, int Hq, int Hkv, int d,
                          int budget, int fixed_r, uint8_t* depths, cudaStream_t stream, int pooled) {
    dim3 grid((unsigned)((Hq + kWarpsPerCta - 1) / kWarpsPerCta));
    depths_kernel<<<grid, kWarpsPerCta * 32, 0, stream>>>(q, q_dtype, sigma2, Hq, Hkv, d, budget, fixed_r,
                                                         pooled, depths);
    return cudaGetLastError();
}

}  // namespace fathom
