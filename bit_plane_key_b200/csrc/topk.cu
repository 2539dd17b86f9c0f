// K4: top-k selection over score rows.
//
// The scan's output is a ranking of all n keys from which the top-k indices
// are taken (ai-feeds.com summary, 方法 · 关键模块 5 and 输出; arXiv abstract).
// Result: for each row, the k largest scores, ties to the lower index,
// listed in (score descending, index ascending) order.
//
// Scores are mapped to order-preserving u32 keys.  A radix select narrows
// each row to the bin holding the k-th key: level 0 histograms bits 31..20,
// level 1 bits 19..8 inside the chosen bin, level 2 bits 7..0; a row stops
// refining as soon as its chosen bin holds at most kCap keys.  Keys above the
// bin are certainly selected ("sure"), keys inside it are candidates.  A
// final CTA per row bitonic-sorts sure + candidates as 64-bit composites
// (key << 32 | ~index) and keeps the first k.  If even the exact 32-bit key
// is shared by more than kCap keys (e.g. every score equal), the ties are
// taken in index order by an ordered block scan instead, which keeps the
// lower-index rule exact.
//
// Kernels: init, (hist, select) x 3 levels, compact, finish.  Rows already
// resolved leave the later levels at once.
#include "fathom_internal.cuh"

namespace fathom {
namespace {

constexpr int kBins = 4096;
constexpr int kCap = 8192;          // candidate capacity per row
constexpr int kChunk = 4096;        // elements per CTA in the row passes
constexpr int kPassThreads = 256;
constexpr int kFinishThreads = 1024;
constexpr int kSortMax = 16384;     // >= next_pow2(kMaxTopK + kCap)

__constant__ int kLevelShift[3] = {20, 8, 0};
__constant__ int kLevelBits[3] = {12, 12, 8};

struct RowState {
    uint32_t prefix;   // resolved high bits of the threshold key
    int shift;         // low bits not yet resolved (32 = none resolved)
    int count_above;   // keys strictly above the prefix range (all selected)
    int cand;          // keys inside the prefix range
    int phase;         // 0 refining, 1 compact candidates, 2 ties overflow
    int n_sure;        // compaction counters
    int n_cand;
    int pad;
};

struct Workspace {
    RowState* state;
    uint32_t* hist;      // [3][rows][kBins]
    uint64_t* sure;      // [rows][k]
    uint64_t* cand;      // [rows][kCap]
};

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

Workspace carve(void* ws, int rows, int k) {
    Workspace w;
    char* p = static_cast<char*>(ws);
    w.state = reinterpret_cast<RowState*>(p);
    p += align256(sizeof(RowState) * rows);
    w.hist = reinterpret_cast<uint32_t*>(p);
    p += align256(sizeof(uint32_t) * 3 * (size_t)rows * kBins);
    w.sure = reinterpret_cast<uint64_t*>(p);
    p += align256(sizeof(uint64_t) * (size_t)rows * k);
    w.cand = reinterpret_cast<uint64_t*>(p);
    return w;
}

__device__ __forceinline__ void row_span(const RowMap& m, int row, int64_t* off, int64_t* n) {
    const int set = row / m.rows_per_set;
    *off = m.base[set] + (int64_t)(row - set * m.rows_per_set) * m.ld[set];
    *n = m.n[set];
}

__device__ __forceinline__ uint64_t composite(uint32_t key, int64_t i) {
    return ((uint64_t)key << 32) | (uint64_t)(0xFFFFFFFFu - (uint32_t)i);
}

__global__ void topk_init(Workspace w, const __grid_constant__ RowMap m, int rows) {
    const int row = blockIdx.x;
    int64_t off, n;
    row_span(m, row, &off, &n);
    uint32_t* h = w.hist + (size_t)row * kBins;
    for (int b = threadIdx.x; b < kBins; b += blockDim.x) {
        h[b] = 0;
        h[(size_t)rows * kBins + b] = 0;
        h[2 * (size_t)rows * kBins + b] = 0;
    }
    if (threadIdx.x == 0) {
        RowState s;
        s.prefix = 0;
        s.shift = 32;
        s.count_above = 0;
        s.cand = (int)n;
        s.phase = (n <= kCap) ? 1 : 0;
        s.n_sure = 0;
        s.n_cand = 0;
        s.pad = 0;
        w.state[row] = s;
    }
}

__global__ void __launch_bounds__(kPassThreads)
topk_hist(const float* __restrict__ scores, const __grid_constant__ RowMap m, int rows, Workspace w, int level) {
    __shared__ uint32_t h[kBins];
    const int row = blockIdx.y;
    const RowState st = w.state[row];
    if (st.phase != 0) return;
    int64_t off, n;
    row_span(m, row, &off, &n);
    if ((int64_t)blockIdx.x * kChunk >= n) return;
    for (int b = threadIdx.x; b < kBins; b += kPassThreads) h[b] = 0;
    __syncthreads();
    const int sh = kLevelShift[level];
    const uint32_t mask = (1u << kLevelBits[level]) - 1u;
    const int64_t i0 = (int64_t)blockIdx.x * kChunk;
    const int64_t i1 = min(n, i0 + kChunk);
    const float* s = scores + off;
    for (int64_t i = i0 + threadIdx.x; i < i1; i += kPassThreads) {
        uint32_t key = float_to_ordered(s[i]);
        bool in = (st.shift == 32) || ((key >> st.shift) == st.prefix);
        if (in) atomicAdd(&h[(key >> sh) & mask], 1u);
    }
    __syncthreads();
    uint32_t* gh = w.hist + ((size_t)level * rows + row) * kBins;
    for (int b = threadIdx.x; b < kBins; b += kPassThreads)
        if (h[b]) atomicAdd(&gh[b], h[b]);
}

// One CTA (1024 threads) per row: find the bin holding the need-th largest key.
__global__ void __launch_bounds__(1024)
topk_select(Workspace w, int rows, int k, int level) {
    __shared__ uint32_t warp_tot[32];
    const int row = blockIdx.x;
    RowState st = w.state[row];
    if (st.phase != 0) return;
    const uint32_t* gh = w.hist + ((size_t)level * rows + row) * kBins;
    const int t = threadIdx.x, lane = t & 31, wp = t >> 5;
    const int nb = 1 << kLevelBits[level];               // 4096 or 256 bins
    const int per = nb / 1024 > 0 ? nb / 1024 : 1;      // bins per thread
    // thread t owns bins [per*t, per*t + per); "above" counts bins of higher threads
    uint32_t mine = 0;
    if (per * t < nb)
        for (int e = 0; e < per; ++e) mine += gh[per * t + e];
    // suffix sum over threads: reverse the thread order
    const int rt = 1023 - t;  // reversed rank
    // inclusive prefix over reversed rank = sum of threads t' >= t
    uint32_t v = mine;
    // warp-level inclusive scan in reversed lane order
    const int rl = 31 - lane;
    (void)rt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        uint32_t y = __shfl_down_sync(0xffffffffu, v, o);
        if (rl >= o) v += y;   // lanes above me in the warp have higher bins
    }
    if (lane == 0) warp_tot[wp] = v;   // lane 0 holds the warp's total
    __syncthreads();
    uint32_t higher_warps = 0;
    for (int x = wp + 1; x < 32; ++x) higher_warps += warp_tot[x];
    const uint32_t incl = v + higher_warps;     // sum of my bins and all higher ones
    const uint32_t above = incl - mine;
    const uint32_t need = (uint32_t)(k - st.count_above);
    if (above < need && incl >= need && per * t < nb) {
        uint32_t acc = above;
        for (int e = per - 1; e >= 0; --e) {
            int b = per * t + e;
            uint32_t c = gh[b];
            if (acc + c >= need) {
                RowState ns = st;
                ns.count_above = st.count_above + (int)acc;
                ns.cand = (int)c;
                ns.prefix = (st.shift == 32) ? (uint32_t)b : ((st.prefix << kLevelBits[level]) | (uint32_t)b);
                ns.shift = kLevelShift[level];
                ns.phase = (c <= (uint32_t)kCap) ? 1 : (ns.shift == 0 ? 2 : 0);
                w.state[row] = ns;
                break;
            }
            acc += c;
        }
    }
}

__global__ void __launch_bounds__(kPassThreads)
topk_compact(const float* __restrict__ scores, const __grid_constant__ RowMap m, int k, Workspace w,
             unsigned int* status) {
    const int row = blockIdx.y;
    const RowState st = w.state[row];
    int64_t off, n;
    row_span(m, row, &off, &n);
    const int64_t i0 = (int64_t)blockIdx.x * kChunk;
    if (i0 >= n) return;
    const int64_t i1 = min(n, i0 + kChunk);
    const float* s = scores + off;
    const int lane = threadIdx.x & 31;
    RowState* gst = w.state + row;
    for (int64_t base = i0; base < i1; base += kPassThreads) {
        int64_t i = base + threadIdx.x;
        uint32_t key = 0;
        bool above = false, eq = false;
        if (i < i1) {
            key = float_to_ordered(s[i]);
            if (st.shift == 32) {
                eq = true;
            } else {
                uint32_t hi = key >> st.shift;
                above = hi > st.prefix;
                eq = hi == st.prefix;
            }
        }
        const bool take_c = eq && st.phase == 1;
        unsigned ma = __ballot_sync(0xffffffffu, above);
        unsigned mc = __ballot_sync(0xffffffffu, take_c);
        int base_a = 0, base_c = 0;
        if (lane == 0) {
            if (ma) base_a = atomicAdd(&gst->n_sure, __popc(ma));
            if (mc) base_c = atomicAdd(&gst->n_cand, __popc(mc));
        }
        base_a = __shfl_sync(0xffffffffu, base_a, 0);
        base_c = __shfl_sync(0xffffffffu, base_c, 0);
        const unsigned lower = (1u << lane) - 1u;
        if (above) {
            int slot = base_a + __popc(ma & lower);
            if (slot < k) w.sure[(size_t)row * k + slot] = composite(key, i);
            else atomicOr(status, (unsigned)FATHOM_DEV_TOPK_OVERFLOW);
        }
        if (take_c) {
            int slot = base_c + __popc(mc & lower);
            if (slot < kCap) w.cand[(size_t)row * kCap + slot] = composite(key, i);
            else atomicOr(status, (unsigned)FATHOM_DEV_TOPK_OVERFLOW);
        }
    }
}

__device__ void bitonic_desc(uint64_t* buf, int S) {
    for (int size = 2; size <= S; size <<= 1) {
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            for (int t = threadIdx.x; t < S / 2; t += blockDim.x) {
                int i = 2 * t - (t & (stride - 1));
                int j = i + stride;
                bool desc = (i & size) == 0;
                uint64_t a = buf[i], b = buf[j];
                if ((a < b) == desc) {
                    buf[i] = b;
                    buf[j] = a;
                }
            }
            __syncthreads();
        }
    }
}

__global__ void __launch_bounds__(kFinishThreads)
topk_finish(const float* __restrict__ scores, const __grid_constant__ RowMap m, int k, Workspace w,
            int32_t* __restrict__ idx, float* __restrict__ top_scores, unsigned int* status) {
    extern __shared__ uint64_t buf[];
    __shared__ int warp_cnt[32];
    __shared__ int s_got;
    const int row = blockIdx.x;
    const RowState st = w.state[row];
    int64_t off, n;
    row_span(m, row, &off, &n);
    const int ns = min(st.count_above, k);
    int total;
    if (st.phase == 1) {
        const int nc = min(st.cand, kCap);
        total = ns + nc;
        for (int e = threadIdx.x; e < ns; e += blockDim.x) buf[e] = w.sure[(size_t)row * k + e];
        for (int e = threadIdx.x; e < nc; e += blockDim.x) buf[ns + e] = w.cand[(size_t)row * kCap + e];
    } else {
        // ties at the exact threshold key: take the lowest indices, in order
        if (st.phase != 2) atomicOr(status, (unsigned)FATHOM_DEV_TOPK_OVERFLOW);
        const uint32_t T = st.prefix;
        const int r = k - ns;
        for (int e = threadIdx.x; e < ns; e += blockDim.x) buf[e] = w.sure[(size_t)row * k + e];
        if (threadIdx.x == 0) s_got = 0;
        __syncthreads();
        const float* s = scores + off;
        const int lane = threadIdx.x & 31, wp = threadIdx.x >> 5;
        for (int64_t base = 0; base < n; base += blockDim.x) {
            int got = s_got;
            if (got >= r) break;
            int64_t i = base + threadIdx.x;
            bool f = (i < n) && float_to_ordered(s[i]) == T;
            unsigned m = __ballot_sync(0xffffffffu, f);
            if (lane == 0) warp_cnt[wp] = __popc(m);
            __syncthreads();
            int before = 0;
            for (int x = 0; x < wp; ++x) before += warp_cnt[x];
            int rank = got + before + __popc(m & ((1u << lane) - 1u));
            if (f && rank < r) buf[ns + rank] = composite(T, i);
            __syncthreads();
            if (threadIdx.x == 0) {
                int add = 0;
                for (int x = 0; x < (int)(blockDim.x >> 5); ++x) add += warp_cnt[x];
                s_got = got + add;
            }
            __syncthreads();
        }
        total = k;
    }
    int S = 1;
    while (S < total) S <<= 1;
    for (int e = total + threadIdx.x; e < S; e += blockDim.x) buf[e] = 0ull;
    __syncthreads();
    bitonic_desc(buf, S);
    for (int e = threadIdx.x; e < k; e += blockDim.x) {
        uint64_t c = buf[e];
        idx[(int64_t)row * k + e] = (int32_t)(0xFFFFFFFFu - (uint32_t)c);
        if (top_scores) top_scores[(int64_t)row * k + e] = ordered_to_float((uint32_t)(c >> 32));
    }
}

}  // namespace

size_t topk_workspace_bytes(int64_t n, int rows, int k) {
    (void)n;
    return align256(sizeof(RowState) * rows) + align256(sizeof(uint32_t) * 3 * (size_t)rows * kBins) +
           align256(sizeof(uint64_t) * (size_t)rows * k) + align256(sizeof(uint64_t) * (size_t)rows * kCap);
}

cudaError_t launch_topk_map(const float* scores, const RowMap& map, int rows, int k, int32_t* idx,
                            float* top_scores, void* ws, cudaStream_t stream) {
    Workspace w = carve(ws, rows, k);
    unsigned int* status = device_status_ptr();
    const unsigned chunks = (unsigned)((map.max_n + kChunk - 1) / kChunk);
    topk_init<<<rows, 256, 0, stream>>>(w, map, rows);
    for (int level = 0; level < 3; ++level) {
        topk_hist<<<dim3(chunks, rows), kPassThreads, 0, stream>>>(scores, map, rows, w, level);
        topk_select<<<rows, 1024, 0, stream>>>(w, rows, k, level);
    }
    topk_compact<<<dim3(chunks, rows), kPassThreads, 0, stream>>>(scores, map, k, w, status);
    const size_t smem = sizeof(uint64_t) * kSortMax;
    cudaError_t e = cudaFuncSetAttribute(topk_finish, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    topk_finish<<<rows, kFinishThreads, smem, stream>>>(scores, map, k, w, idx, top_scores, status);
    return cudaGetLastError();
}

cudaError_t launch_topk(const float* scores, int64_t n, int64_t ld, int rows, int k, int32_t* idx,
                        float* top_scores, void* ws, cudaStream_t stream) {
    RowMap m;
    m.rows_per_set = rows;
    m.nsets = 1;
    m.max_n = n;
    m.base[0] = 0;
    m.ld[0] = ld;
    m.n[0] = n;
    return launch_topk_map(scores, m, rows, k, idx, top_scores, ws, stream);
}

}  // namespace fathom
