// K5: exact attention over the selected keys only.
//
// ai-feeds.com summary, 方法 · 输出: each query produces top-k key indices and
// true attention is then computed over those keys.
//   o_h = sum_j p_j V[g][idx_j],  p = softmax_j(q_h . K[g][idx_j] / sqrt(d)),
// g = h / (Hq/Hkv), K and V rows in bf16, fp32 accumulation, exp via exp2f.
//
// One thread-block cluster of kSplit CTAs per query head.  CTA r of the
// cluster takes every kSplit-th of the head's k selected keys; inside it each
// warp runs an online softmax over its rows (lane l holds channels
// [l*d/32, (l+1)*d/32)).  The warps' partial (max, sum, o) merge in shared
// memory, then CTA 0 merges the kSplit CTA partials through distributed
// shared memory and writes o_h.  No workspace and no second kernel.
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
// rows in flight per warp: all of a lane's row words are loaded before any is
// used; 16 rows (32 loads per lane) for d <= 128, 8 for d = 256
template <int V>
constexpr int unroll_of() { return V <= 4 ? 16 : 8; }
constexpr int kSortCap = kMaxTopK;   // indices sorted in shared memory
constexpr int kIdxRegs = (kMaxTopK + kSplit * kWarps * 32 - 1) / (kSplit * kWarps * 32);   // row indices per lane


// A lane's V bf16 values of a row, kept as raw 32-bit words until used: the
// loads of all rows in flight are issued before any value is converted.
template <int V>
struct RowWords {
    static constexpr int W = (V + 1) / 2;
    uint32_t w[W];
    __device__ __forceinline__ void load(const uint16_t* __restrict__ p) {
        if constexpr (V == 8) {
            const uint4 u = *reinterpret_cast<const uint4*>(p);
            w[0] = u.x; w[1] = u.y; w[2] = u.z; w[3] = u.w;
        } else if constexpr (V == 4) {
            const uint2 u = *reinterpret_cast<const uint2*>(p);
            w[0] = u.x; w[1] = u.y;
        } else if constexpr (V == 2) {
            w[0] = *reinterpret_cast<const uint32_t*>(p);
        } else {
            w[0] = p[0];
        }
    }
    __device__ __forceinline__ void clear() {
#pragma unroll
        for (int e = 0; e < W; ++e) w[e] = 0u;
    }
    __device__ __forceinline__ float at(int e) const {   // value e (bf16 -> f32 is a shift)
        const uint32_t x = w[e >> 1];
        return (V == 1) ? __uint_as_float(x << 16) : ((e & 1) ? __uint_as_float(x & 0xFFFF0000u)
                                                              : __uint_as_float(x << 16));
    }
};

template <int V>
__global__ void __cluster_dims__(kSplit, 1, 1) __launch_bounds__(kThreads)
attend_kernel(const void* __restrict__ q, int q_dtype, const uint16_t* __restrict__ Kr,
              const uint16_t* __restrict__ Vr, int64_t row_stride, const int32_t* __restrict__ idx, int Hq, int Hkv,
              int64_t n, int64_t key0, int k, int sort_rows, float* __restrict__ out, float* __restrict__ parts,
              unsigned int* status) {
    constexpr int d = V * 32;
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
    const float scale = 1.4426950408889634f / sqrtf((float)d);  // log2(e)/sqrt(d)

    float qv[V];
#pragma unroll
    for (int e = 0; e < V; ++e) qv[e] = load_q(q, q_dtype, (int64_t)h * d + lane * V + e) * scale;

    float m = -INFINITY, l = 0.0f, o[V];
#pragma unroll
    for (int e = 0; e < V; ++e) o[e] = 0.0f;

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
                    const int i = 2 * t - (t & (stride - 1)), j = i + stride;
                    const bool up = (i & size) == 0;
                    const int32_t a = s_idx[i], b2 = s_idx[j];
                    if ((a > b2) == up) {
                        s_idx[i] = b2;
                        s_idx[j] = a;
                    }
                }
                __syncthreads();
            }
        }
        ih = s_idx;
    }
    // rows of this warp: positions p = r + kSplit * (wp + kWarps * m) of the (sorted) list,
    // so the head's warps sweep the list together, in address order when sorted.
    // The warp's row indices are read once, lane j holding those of m = j + 32 e,
    // so every batch issues its row loads at once
    const int stride = kSplit * kWarps;
    const int rows_w = (k - (r + kSplit * wp) + stride - 1) / stride;   // rows of this warp (may be <= 0)
    int32_t my_idx[kIdxRegs];
#pragma unroll
    for (int e = 0; e < kIdxRegs; ++e) {
        const int mm = lane + 32 * e;
        my_idx[e] = (mm < rows_w) ? ih[r + kSplit * wp + stride * mm] : -1;
    }
    constexpr int kUnroll = unroll_of<V>();
    for (int m0 = 0; m0 < rows_w; m0 += kUnroll) {
        RowWords<V> kw[kUnroll], vw[kUnroll];
        bool ok[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int mm = m0 + u;
            ok[u] = false;
            kw[u].clear();
            vw[u].clear();
            int32_t i = -1;
#pragma unroll
            for (int e = 0; e < kIdxRegs; ++e)
                if ((mm >> 5) == e) i = __shfl_sync(0xffffffffu, my_idx[e], mm & 31);
            if (mm < rows_w) {
                const int64_t il = (int64_t)i - key0;   // row in this array
                if (il >= 0 && il < n) {
                    ok[u] = true;
                    const int64_t off = head_base + il * row_stride + lane * V;
                    kw[u].load(Kr + off);
                    vw[u].load(Vr + off);
                } else if (!parts && lane == 0) {   // a partial skips the other ranges' rows
                    atomicOr(status, (unsigned)FATHOM_DEV_BAD_INDEX);
                }
            }
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            float dot = 0.0f;
#pragma unroll
            for (int e = 0; e < V; ++e) dot = fmaf(qv[e], kw[u].at(e), dot);
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, off);
            if (!ok[u]) continue;   // warp-uniform
            float mn = fmaxf(m, dot);
            float a = exp2f(m - mn);     // 0 when m = -inf
            float p = exp2f(dot - mn);
            l = l * a + p;
#pragma unroll
            for (int e = 0; e < V; ++e) o[e] = fmaf(p, vw[u].at(e), o[e] * a);
            m = mn;
        }
    }

    // merge the warps of this CTA
    if (lane == 0) {
        s_m[wp] = m;
        s_l[wp] = l;
    }
#pragma unroll
    for (int e = 0; e < V; ++e) s_o[wp][lane * V + e] = o[e];
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
                          int sort_rows, float* out, cudaStream_t stream, int64_t key0, float* parts) {
    dim3 grid((unsigned)(Hq * kSplit));
    unsigned int* st = device_status_ptr();
    const int sr = (sort_rows && k <= kSortCap) ? 1 : 0;
    auto go = [&](auto kern) {
        kern<<<grid, kThreads, 0, stream>>>(q, q_dtype, K_rows, V_rows, row_stride, idx, Hq, Hkv, n, key0, k, sr, out,
                                            parts, st);
        return cudaGetLastError();
    };
    switch (d) {
        case 32: return go(attend_kernel<1>);
        case 64: return go(attend_kernel<2>);
        case 128: return go(attend_kernel<4>);
        case 256: return go(attend_kernel<8>);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace fathom
