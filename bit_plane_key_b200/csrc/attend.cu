// K5: exact attention over the selected keys only.
//
// ai-feeds.com summary, 方法 · 输出: each query produces top-k key indices and
// true attention is then computed over those keys.
//   o_h = sum_j p_j V[g][idx_j],  p = softmax_j(q_h . K[g][idx_j] / sqrt(d)),
// g = h / (Hq/Hkv), K and V rows in bf16, fp32 accumulation, exp via exp2f.
//
// One thread-block cluster of kSplit CTAs per query head.  CTA r of the
// cluster takes every kSplit-th of the head's k selected keys.  Inside it a
// row is held by d/16 lanes of a warp (16 channels each, read as 16-byte
// pieces), so a warp works on 32/(d/16) rows at once, each group of lanes
// running its own online softmax; the groups merge by shuffles, the warps'
// partial (max, sum, o) in shared memory, then CTA 0 merges the kSplit CTA
// partials through distributed shared memory and writes o_h.  No workspace
// and no second kernel.  Products and sums use packed two-lane FMAs; the
// running maximum moves only when a score passes it by more than 2^8, so the
// per-row rescale of o is skipped on almost every row.
// With a key range split across GPUs, each rank runs the same kernel over
// the rows it holds (global indices shifted by its first key; the other
// ranks' indices skipped) and writes the CTA 0 merge unnormalised: o relative
// to the running maximum m, m and the sum l (log2 units, as below);
// attend_merge_kernel combines the ranks' partials the way CTA 0 combines
// its cluster's.
// Rows may live in device memory or in page-locked host memory.  Over the
// host link, gathering rows in address order is faster than in score order,
// so for host-resident rows every CTA first sorts the head's indices in
// shared memory; the head's 32 warps then sweep the sorted list together
// (the softmax sum does not depend on the order).  Rows are addressed with a
// row stride, so K and V may be two arrays or one interleaved [n][2][d]
// array; the latter keeps a key's two rows in one run on the host link.
#include <cooperative_groups.h>

#include "fathom_internal.cuh"

namespace cg = cooperative_groups;

namespace fathom {
namespace {

constexpr int kSplit = 8;      // CTAs per head (cluster size)
constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kSortCap = kMaxTopK;   // indices sorted in shared memory
constexpr int kIdxRegs = (kMaxTopK + kSplit * kWarps * 32 - 1) / (kSplit * kWarps * 32);   // row indices per lane
// A slot's running maximum is moved (and its sum and output rescaled) only
// when a score passes it by more than kTau (log2 units): exp2(score - m) then
// stays below 2^kTau, and the result is the same softmax up to rounding.
constexpr float kTau = 8.0f;

// Lane layout for head dimension D.  LPR = D / 16 lanes share a row ("a
// slot"), each holding 16 channels: lane j of a slot reads the 16-byte pieces
// t = 0, 1 of the K row and of the V row that start at channel t * D/2 + 8 j,
// so one warp load instruction reads D contiguous bytes of each of the RPW =
// 32 / LPR rows it covers.  A lane keeps R rows in flight: a warp loads RB =
// R * RPW rows before it uses any of them.
template <int D>
struct Lanes {
    static constexpr int LPR = D / 16;
    static constexpr int RPW = 32 / LPR;
    static constexpr int R = (D == 32) ? 2 : 4;
    static constexpr int RB = R * RPW;
    static_assert(32 % RB == 0, "a batch's row positions lie in one index register");
};

// a word of two bf16 values as two floats (bf16 -> f32 is a shift)
__device__ __forceinline__ float2 bf16x2_f2(uint32_t w) {
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}
__device__ __forceinline__ uint32_t word_of(const uint4& v, int w) {
    return w == 0 ? v.x : (w == 1 ? v.y : (w == 2 ? v.z : v.w));
}

template <int D>
__global__ void __cluster_dims__(kSplit, 1, 1) __launch_bounds__(kThreads)
attend_kernel(const void* __restrict__ q, int q_dtype, const uint16_t* __restrict__ Kr,
              const uint16_t* __restrict__ Vr, int64_t row_stride, const int32_t* __restrict__ idx, int Hq, int Hkv,
              int64_t n, int64_t key0, int k, int sort_rows, float* __restrict__ out, float* __restrict__ parts,
              unsigned int* status) {
    pdl_wait();
    using Ln = Lanes<D>;
    constexpr int d = D;
    __shared__ int32_t s_idx[kSortCap];
    __shared__ float s_m[kWarps], s_l[kWarps];
    __shared__ float s_o[kWarps][d];
    __shared__ float c_m, c_l;        // this CTA's merged partial (read by CTA 0)
    __shared__ float c_o[d];

    cg::cluster_group cluster = cg::this_cluster();
    const int r = (int)cluster.block_rank();
    const int h = blockIdx.x / kSplit;
    const int g = h / (Hq / Hkv);
    const int lane = threadIdx.x & 31, wp = threadIdx.x >> 5;
    const int slot = lane / Ln::LPR, j = lane % Ln::LPR;
    const float scale = 1.4426950408889634f / sqrtf((float)d);  // log2(e)/sqrt(d)

    // the query's channels of this lane, in pairs: piece t, word w holds
    // channels t * d/2 + 8 j + 2 w and the one after it
    float2 q2[2][4];
#pragma unroll
    for (int t = 0; t < 2; ++t)
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            const int64_t c = (int64_t)h * d + t * (d / 2) + 8 * j + 2 * w;
            q2[t][w] = make_float2(load_q(q, q_dtype, c) * scale, load_q(q, q_dtype, c + 1) * scale);
        }

    // the slot's online softmax: maximum m and sum l (log2 units), output o
    // for the lane's channels (same pairing as q2)
    float m = -INFINITY, l = 0.0f;
    float2 o2[2][4];
#pragma unroll
    for (int t = 0; t < 2; ++t)
#pragma unroll
        for (int w = 0; w < 4; ++w) o2[t][w] = make_float2(0.0f, 0.0f);

    const int32_t* ih = idx + (int64_t)h * k;
    const int64_t head_base = (int64_t)g * n * row_stride;
    if (sort_rows) {
        // bitonic sort (ascending) of the head's indices, padded to a power of two
        int P = 1;
        while (P < k) P <<= 1;
        for (int e = threadIdx.x; e < P; e += kThreads) s_idx[e] = (e < k) ? ih[e] : INT32_MAX;
        __syncthreads();
        for (int size = 2; size <= P; size <<= 1) {
            for (int stride = size >> 1; stride > 0; stride >>= 1) {
                for (int t = threadIdx.x; t < P / 2; t += kThreads) {
                    const int i = 2 * t - (t & (stride - 1)), j2 = i + stride;
                    const bool up = (i & size) == 0;
                    const int32_t a = s_idx[i], b2 = s_idx[j2];
                    if ((a > b2) == up) {
                        s_idx[i] = b2;
                        s_idx[j2] = a;
                    }
                }
                __syncthreads();
            }
        }
        ih = s_idx;
    }
    // rows of this warp: positions p = r + kSplit * (wp + kWarps * mm) of the (sorted) list,
    // so the head's warps sweep the list together, in address order when sorted.
    // The warp's row indices are read once, lane x holding those of mm = x + 32 e;
    // batch m0 takes mm = m0 + u * RPW + slot for u < R
    const int stride = kSplit * kWarps;
    const int rows_w = (k - (r + kSplit * wp) + stride - 1) / stride;   // rows of this warp (may be <= 0)
    int32_t my_idx[kIdxRegs];
#pragma unroll
    for (int e = 0; e < kIdxRegs; ++e) {
        const int mm = lane + 32 * e;
        my_idx[e] = (mm < rows_w) ? ih[r + kSplit * wp + stride * mm] : -1;
    }
    for (int m0 = 0; m0 < rows_w; m0 += Ln::RB) {
        int32_t reg = -1;   // the index register holding this batch (warp-uniform choice)
#pragma unroll
        for (int e = 0; e < kIdxRegs; ++e)
            if ((m0 >> 5) == e) reg = my_idx[e];
        uint4 kp[Ln::R][2], vp[Ln::R][2];
        bool ok[Ln::R];
#pragma unroll
        for (int u = 0; u < Ln::R; ++u) {
            const int mm = m0 + u * Ln::RPW + slot;
            const int32_t i = __shfl_sync(0xffffffffu, reg, (m0 & 31) + u * Ln::RPW + slot);
            ok[u] = false;
#pragma unroll
            for (int t = 0; t < 2; ++t) kp[u][t] = vp[u][t] = make_uint4(0u, 0u, 0u, 0u);
            if (mm < rows_w) {
                const int64_t il = (int64_t)i - key0;   // row in this array
                if (il >= 0 && il < n) {
                    ok[u] = true;
                    const int64_t off = head_base + il * row_stride + 8 * j;
#pragma unroll
                    for (int t = 0; t < 2; ++t) {
                        kp[u][t] = *reinterpret_cast<const uint4*>(Kr + off + t * (d / 2));
                        vp[u][t] = *reinterpret_cast<const uint4*>(Vr + off + t * (d / 2));
                    }
                } else if (!parts && j == 0) {   // a partial skips the other ranges' rows
                    atomicOr(status, (unsigned)FATHOM_DEV_BAD_INDEX);
                }
            }
        }
#pragma unroll
        for (int u = 0; u < Ln::R; ++u) {
            float2 acc = make_float2(0.0f, 0.0f);
#pragma unroll
            for (int t = 0; t < 2; ++t)
#pragma unroll
                for (int w = 0; w < 4; ++w) acc = __ffma2_rn(q2[t][w], bf16x2_f2(word_of(kp[u][t], w)), acc);
            float x = acc.x + acc.y;
#pragma unroll
            for (int off = Ln::LPR / 2; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
            if (!ok[u]) continue;   // uniform within the slot
            if (x > m + kTau) {     // also the slot's first row (m = -inf)
                const float a = exp2f(m - x);   // 0 when m = -inf
                l *= a;
#pragma unroll
                for (int t = 0; t < 2; ++t)
#pragma unroll
                    for (int w = 0; w < 4; ++w) o2[t][w] = make_float2(o2[t][w].x * a, o2[t][w].y * a);
                m = x;
            }
            const float p = exp2f(x - m);
            l += p;
            const float2 pp = make_float2(p, p);
#pragma unroll
            for (int t = 0; t < 2; ++t)
#pragma unroll
                for (int w = 0; w < 4; ++w) o2[t][w] = __ffma2_rn(pp, bf16x2_f2(word_of(vp[u][t], w)), o2[t][w]);
        }
    }

    // merge the warp's slots: lane j of every slot holds the same channels
#pragma unroll
    for (int off = Ln::LPR; off < 32; off <<= 1) {
        const float mo = __shfl_xor_sync(0xffffffffu, m, off);
        const float lo = __shfl_xor_sync(0xffffffffu, l, off);
        const float mn = fmaxf(m, mo);
        const float fa = (m == -INFINITY) ? 0.0f : exp2f(m - mn);
        const float fb = (mo == -INFINITY) ? 0.0f : exp2f(mo - mn);
        l = l * fa + lo * fb;
#pragma unroll
        for (int t = 0; t < 2; ++t)
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                const float ox = __shfl_xor_sync(0xffffffffu, o2[t][w].x, off);
                const float oy = __shfl_xor_sync(0xffffffffu, o2[t][w].y, off);
                o2[t][w] = make_float2(o2[t][w].x * fa + ox * fb, o2[t][w].y * fa + oy * fb);
            }
        m = mn;
    }

    // merge the warps of this CTA
    if (lane == 0) {
        s_m[wp] = m;
        s_l[wp] = l;
    }
    if (slot == 0) {
#pragma unroll
        for (int t = 0; t < 2; ++t)
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                s_o[wp][t * (d / 2) + 8 * j + 2 * w] = o2[t][w].x;
                s_o[wp][t * (d / 2) + 8 * j + 2 * w + 1] = o2[t][w].y;
            }
    }
    __syncthreads();
    {
        float M = -INFINITY;
        for (int x = 0; x < kWarps; ++x) M = fmaxf(M, s_m[x]);
        float f[kWarps];
        float L = 0.0f;
        for (int x = 0; x < kWarps; ++x) {
            f[x] = (s_m[x] == -INFINITY) ? 0.0f : exp2f(s_m[x] - M);
            L = fmaf(s_l[x], f[x], L);
        }
        for (int c = threadIdx.x; c < d; c += kThreads) {
            float O = 0.0f;
            for (int x = 0; x < kWarps; ++x) O = fmaf(s_o[x][c], f[x], O);
            c_o[c] = O;
        }
        if (threadIdx.x == 0) {
            c_m = M;
            c_l = L;
        }
    }
    cluster.sync();
    if (r == 0) {
        float f[kSplit];
        float M = -INFINITY, L = 0.0f;
#pragma unroll
        for (int x = 0; x < kSplit; ++x) M = fmaxf(M, *cluster.map_shared_rank(&c_m, x));
#pragma unroll
        for (int x = 0; x < kSplit; ++x) {
            float mx = *cluster.map_shared_rank(&c_m, x);
            f[x] = (mx == -INFINITY) ? 0.0f : exp2f(mx - M);
            L = fmaf(*cluster.map_shared_rank(&c_l, x), f[x], L);
        }
        float* ph = parts ? parts + (int64_t)h * (d + 2) : nullptr;
        for (int c = threadIdx.x; c < d; c += kThreads) {
            float O = 0.0f;
#pragma unroll
            for (int x = 0; x < kSplit; ++x) O = fmaf(cluster.map_shared_rank(c_o, x)[c], f[x], O);
            if (ph) ph[c] = O;
            else out[(int64_t)h * d + c] = (L > 0.0f) ? O / L : 0.0f;
        }
        if (ph && threadIdx.x == 0) {
            ph[d] = M;
            ph[d + 1] = L;
        }
    }
    cluster.sync();   // keep every CTA's shared memory alive until CTA 0 has read it
}

// Merge of per-range partials (o relative to m, m, l) of the same heads:
// M = max_r m_r, L = sum_r l_r 2^(m_r - M), out = sum_r o_r 2^(m_r - M) / L,
// ranges summed in order r = 0, 1, ...  One CTA per head.
__global__ void __launch_bounds__(128)
attend_merge_kernel(const float* __restrict__ parts, int world, int Hq, int d, float* __restrict__ out) {
    pdl_wait();
    const int h = blockIdx.x;
    const int64_t rs = (int64_t)Hq * (d + 2);   // one range's partials
    const float* p = parts + (int64_t)h * (d + 2);
    float M = -INFINITY;
    for (int r = 0; r < world; ++r) M = fmaxf(M, p[r * rs + d]);
    float L = 0.0f;
    for (int r = 0; r < world; ++r) {
        const float mr = p[r * rs + d];
        L = fmaf(p[r * rs + d + 1], (mr == -INFINITY) ? 0.0f : exp2f(mr - M), L);
    }
    for (int c = threadIdx.x; c < d; c += blockDim.x) {
        float O = 0.0f;
        for (int r = 0; r < world; ++r) {
            const float mr = p[r * rs + d];
            O = fmaf(p[r * rs + c], (mr == -INFINITY) ? 0.0f : exp2f(mr - M), O);
        }
        out[(int64_t)h * d + c] = (L > 0.0f) ? O / L : 0.0f;
    }
}

}  // namespace

cudaError_t launch_attend_merge(const float* parts, int world, int Hq, int d, float* out, cudaStream_t stream) {
    attend_merge_kernel<<<(unsigned)Hq, 128, 0, stream>>>(parts, world, Hq, d, out);
    return cudaGetLastError();
}

cudaError_t launch_attend(const void* q, int q_dtype, const uint16_t* K_rows, const uint16_t* V_rows,
                          int64_t row_stride, const int32_t* idx, int Hq, int Hkv, int64_t n, int d, int k,
                          int sort_rows, float* out, cudaStream_t stream, int64_t key0, float* parts, bool pdl) {
    dim3 grid((unsigned)(Hq * kSplit));
    unsigned int* st = device_status_ptr();
    const int sr = (sort_rows && k <= kSortCap) ? 1 : 0;
    auto go = [&](auto kern) {
        return launch_ex(kern, grid, dim3(kThreads), 0, stream, pdl, 1, q, q_dtype, K_rows, V_rows, row_stride, idx, Hq,
                         Hkv, n, key0, k, sr, out, parts, st);
    };
    switch (d) {
        case 32: return go(attend_kernel<32>);
        case 64: return go(attend_kernel<64>);
        case 128: return go(attend_kernel<128>);
        case 256: return go(attend_kernel<256>);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace fathom
