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
// One CTA per query head, one thread per candidate (c, t) = (tid / 4, tid % 4).
// Each candidate gets a 32-bit key that orders exactly as v: v = (double)w 2^-2t
// is exact in fp64 (a subnormal fp32 w included), its biased exponent lies in
// [868, 1151] and its significand in the top 23 mantissa bits, so
//   key = (exponent - 860) << 23 | significand   (0 for w = 0, ~0 for inf)
// is monotone in v and equal only for equal v.  theta = the N-th largest key,
// N = min(B, 4d), found bit by bit from the top (32 block-wide counts); the
// candidates above theta are taken, and of those equal to theta the first
// N - #{key > theta} in (c, t) order, which is the tie rule (c ascending, then
// t ascending).  t_c = the number taken on channel c, so sum_c t_c = N.
//
// Group-pooled variant (not in the pages, which decide per query: arXiv
// abstract, "each query decides"): the importance of channel c for KV head g
// is the fp32 sum, in head order, of the group's per-head w_{h,c}; one water
// level per KV head; every head of the group gets the same depths, so the
// scan reads exactly min(B, 4d) plane bits per key and KV head.
//
// Fixed-r comparison scans (ai-feeds.com summary, 与 Double Sparsity / Loki /
// SparQ 的差异: a fixed 68 or 136 bits per key): depth 4 on the r channels with
// the largest |q_c|, ties to the lower channel, by the same select with one
// candidate per channel and key bits(|q_c|).
#include "fathom_internal.cuh"

namespace fathom {
namespace {

// key of v = w 2^-2t (w >= 0): monotone in v, equal only for equal v
__device__ __forceinline__ uint32_t cand_key(float w, int t) {
    if (!(w > 0.0f)) return 0u;
    if (isinf(w)) return 0xFFFFFFFFu;
    const uint64_t b = (uint64_t)__double_as_longlong((double)w);   // normal, exponent >= 874
    const uint32_t e = (uint32_t)(b >> 52) - 2u * (uint32_t)t;          // times 2^-2t, exactly
    return (e - 860u) << 23 | ((uint32_t)(b >> 29) & 0x7FFFFFu);
}

// blockDim = 4d: thread (c, t) = (tid / 4, tid % 4)
__global__ void __launch_bounds__(4 * kMaxD)
depths_kernel(const void* __restrict__ q, int q_dtype, const float* __restrict__ sigma2, int Hq, int Hkv,
              int d, int budget, int fixed_r, int pooled, uint8_t* __restrict__ depths) {
    pdl_wait();
    __shared__ int s_ties[4 * kMaxD / 32];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int h = blockIdx.x;
    const int g = h / (Hq / Hkv);
    const int c = tid >> 2, t = tid & 3;
    uint32_t key;
    bool valid;
    int N;
    if (fixed_r == 0) {
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
        key = cand_key(w, t);
        valid = true;
        N = min(budget, 4 * d);
    } else {   // one candidate per channel: |q_c|
        key = __float_as_uint(fabsf(load_q(q, q_dtype, (int64_t)h * d + c)));
        valid = t == 0;
        N = min(fixed_r, d);
    }
    // theta: the largest T with #{key >= T} >= N
    uint32_t T = 0;
    for (int bit = 31; bit >= 0 && N > 0; --bit) {
        const uint32_t cand = T | (1u << bit);
        if (__syncthreads_count(valid && key >= cand) >= N) T = cand;
    }
    const int above = __syncthreads_count(valid && key > T);
    const bool tie = valid && key == T;
    const unsigned tb = __ballot_sync(0xffffffffu, tie);
    if (lane == 0) s_ties[warp] = __popc(tb);
    __syncthreads();
    int rank = __popc(tb & ((1u << lane) - 1u));   // ties before this one, in (c, t) order
    for (int x = 0; x < warp; ++x) rank += s_ties[x];
    const bool take = N > 0 && valid && (key > T || (tie && rank < N - above));
    const unsigned taken = __ballot_sync(0xffffffffu, take);
    if (t == 0) {
        const int dep = (fixed_r == 0) ? __popc((taken >> (lane & ~3)) & 0xFu) : (take ? 4 : 0);
        depths[(int64_t)h * d + c] = (uint8_t)dep;
    }
}

}  // namespace

cudaError_t launch_depths(const void* q, int q_dtype, const float* sigma2, int Hq, int Hkv, int d,
                          int budget, int fixed_r, uint8_t* depths, cudaStream_t stream, int pooled) {
    depths_kernel<<<(unsigned)Hq, 4 * d, 0, stream>>>(q, q_dtype, sigma2, Hq, Hkv, d, budget, fixed_r,
                                                         pooled, depths);
    return cudaGetLastError();
}

}  // namespace fathom
