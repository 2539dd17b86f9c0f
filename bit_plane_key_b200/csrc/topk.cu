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
// bin are certainly selected ("sure"), keys inside it are candidates, and one
// pass over the row compacts both.  A final CTA per row finds the exact k-th
// key among its candidates by the same radix steps in shared memory, keeps
// the sure keys and the candidates at or above it, and bitonic-sorts them as
// 64-bit composites (key << 32 | ~index): about k entries.  If even the exact
// 32-bit key is shared by more than kCap keys (e.g. every score equal), the
// ties are taken in index order by an ordered block scan instead, which keeps
// the lower-index rule exact.
//
// Kernels: init, (hist, select) x 3 levels, compact, finish.  Level 0 always
// runs over every row; levels 1 and 2 run as small grid-stride launches that
// leave at once when no row is still refining (the common case).  Rows of at
// most kRowsMax keys skip all of this: one cluster kernel per launch holds a
// row in the shared memory of 1 to 8 CTAs and selects there (topk_rows).
// Rows with at least 8k blocks of 64 keys take the block-maximum path.
#include <cooperative_groups.h>

#include "fathom_internal.cuh"

namespace cg = cooperative_groups;

namespace fathom {
namespace {

constexpr int kBins = 4096;
constexpr int kCap = 8192;          // candidate capacity per row
constexpr int kChunk = 4096;        // elements per CTA in the row passes
constexpr int kPassThreads = 256;
constexpr int kFinishThreads = 1024;
constexpr int kSortMax = 16384;     // >= next_pow2(kMaxTopK + kCap)
constexpr int kPer = kChunk / kPassThreads;   // elements per thread in the row passes

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
    int* active;         // [4]: rows still refining after select level l
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
    w.active = reinterpret_cast<int*>(p);
    p += align256(sizeof(int) * 4);
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
    if (row == 0 && threadIdx.x < 4) w.active[threadIdx.x] = 0;
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

// The kPer elements of a row chunk that thread t handles, all loads in
// flight at once: with 16-byte aligned rows, four float4 loads (element
// (q, e) at i0 + 4 (q * kPassThreads + t) + e), else kPer scalar loads
// (element j at i0 + j * kPassThreads + t).  Out-of-range elements read 0.
template <bool kVec>
__device__ __forceinline__ int64_t chunk_index(int64_t i0, int j) {
    return kVec ? i0 + 4 * ((int64_t)(j >> 2) * kPassThreads + threadIdx.x) + (j & 3)
                : i0 + (int64_t)j * kPassThreads + threadIdx.x;
}
template <bool kVec>
__device__ __forceinline__ void load_chunk(const float* __restrict__ s, int64_t i0, int64_t i1, float (&v)[kPer]) {
    if constexpr (kVec) {
#pragma unroll
        for (int qd = 0; qd < kPer / 4; ++qd) {
            const int64_t b = chunk_index<true>(i0, 4 * qd);
            if (b + 3 < i1) {
                const float4 x = *reinterpret_cast<const float4*>(s + b);
                v[4 * qd] = x.x; v[4 * qd + 1] = x.y; v[4 * qd + 2] = x.z; v[4 * qd + 3] = x.w;
            } else {
#pragma unroll
                for (int e = 0; e < 4; ++e) v[4 * qd + e] = (b + e < i1) ? s[b + e] : 0.0f;
            }
        }
    } else {
#pragma unroll
        for (int j = 0; j < kPer; ++j) {
            const int64_t i = chunk_index<false>(i0, j);
            v[j] = (i < i1) ? s[i] : 0.0f;
        }
    }
}

// Histogram of one chunk of one row into the row's level histogram.
template <bool kVec>
__device__ __forceinline__ void hist_body(const float* __restrict__ s, int64_t i0, int64_t i1, RowState st, int sh,
                                          uint32_t mask, uint32_t* h) {
    float v[kPer];
    load_chunk<kVec>(s, i0, i1, v);
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
        const int64_t i = chunk_index<kVec>(i0, j);
        const uint32_t key = float_to_ordered(v[j]);
        const bool in = (i < i1) && ((st.shift == 32) || ((key >> st.shift) == st.prefix));
        if (in) atomicAdd(&h[(key >> sh) & mask], 1u);
    }
}

__device__ __forceinline__ void hist_chunk(const float* __restrict__ scores, const RowMap& m, int rows, Workspace w,
                                           int level, int row, int chunk, uint32_t* h) {
    const RowState st = w.state[row];
    if (st.phase != 0) return;   // uniform over the CTA
    int64_t off, n;
    row_span(m, row, &off, &n);
    const int64_t i0 = (int64_t)chunk * kChunk;
    if (i0 >= n) return;
    const int nb = 1 << kLevelBits[level];
    for (int b = threadIdx.x; b < nb; b += kPassThreads) h[b] = 0;
    __syncthreads();
    const int sh = kLevelShift[level];
    const uint32_t mask = (uint32_t)nb - 1u;
    const int64_t i1 = min(n, i0 + kChunk);
    const float* s = scores + off;
    if ((reinterpret_cast<uintptr_t>(s + i0) & 15) == 0) hist_body<true>(s, i0, i1, st, sh, mask, h);
    else hist_body<false>(s, i0, i1, st, sh, mask, h);
    __syncthreads();
    uint32_t* gh = w.hist + ((size_t)level * rows + row) * kBins;
    for (int b = threadIdx.x; b < nb; b += kPassThreads)
        if (h[b]) atomicAdd(&gh[b], h[b]);
    __syncthreads();   // h is reused by the CTA's next chunk
}

// Level 0: every (chunk, row).
__global__ void __launch_bounds__(kPassThreads)
topk_hist(const float* __restrict__ scores, const __grid_constant__ RowMap m, int rows, Workspace w) {
    __shared__ uint32_t h[kBins];
    hist_chunk(scores, m, rows, w, 0, (int)blockIdx.y, (int)blockIdx.x, h);
}

// Levels 1 and 2: a grid-stride pass over (row, chunk) that leaves at once
// when the previous select left no row refining.
__global__ void __launch_bounds__(kPassThreads)
topk_hist_refine(const float* __restrict__ scores, const __grid_constant__ RowMap m, int rows, int chunks,
                 Workspace w, int level) {
    __shared__ uint32_t h[kBins];
    if (w.active[level - 1] == 0) return;
    for (int64_t item = blockIdx.x; item < (int64_t)rows * chunks; item += gridDim.x)
        hist_chunk(scores, m, rows, w, level, (int)(item / chunks), (int)(item % chunks), h);
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
                if (ns.phase == 0) atomicAdd(&w.active[level], 1);
                break;
            }
            acc += c;
        }
    }
}

// Keys above the row's bin go to the sure buffer, keys inside it to the
// candidates.  A CTA counts its keepers, reserves its output ranges with one
// atomic per buffer, then writes them: no warp waits on a contended counter.
// The write pass reloads only the kept keys.
template <bool kVec>
__device__ __forceinline__ void compact_body(const float* __restrict__ s, int64_t i0, int64_t i1, RowState st, int row,
                                             int k, Workspace w, unsigned int* status) {
    constexpr int kWarpsPerCta = kPassThreads / 32;
    __shared__ int s_na[kWarpsPerCta], s_nc[kWarpsPerCta];
    __shared__ int s_base_a, s_base_c;
    const int lane = threadIdx.x & 31, wp = threadIdx.x >> 5;
    float v[kPer];
    load_chunk<kVec>(s, i0, i1, v);
    // classify: bit j of fa / fc = element j is sure / a candidate
    uint32_t fa = 0, fc = 0;
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
        const int64_t i = chunk_index<kVec>(i0, j);
        const uint32_t key = float_to_ordered(v[j]);
        bool above = false, eq = false;
        if (i < i1) {
            if (st.shift == 32) {
                eq = true;
            } else {
                const uint32_t hi = key >> st.shift;
                above = hi > st.prefix;
                eq = hi == st.prefix;
            }
        }
        fa |= (above ? 1u : 0u) << j;
        fc |= ((eq && st.phase == 1) ? 1u : 0u) << j;
    }
    const int na = (int)__reduce_add_sync(0xffffffffu, (unsigned)__popc(fa));   // this warp's keepers
    const int nc = (int)__reduce_add_sync(0xffffffffu, (unsigned)__popc(fc));
    if (lane == 0) {
        s_na[wp] = na;
        s_nc[wp] = nc;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        int ta = 0, tc = 0;
        for (int x = 0; x < kWarpsPerCta; ++x) {
            ta += s_na[x];
            tc += s_nc[x];
        }
        RowState* gst = w.state + row;
        s_base_a = ta ? atomicAdd(&gst->n_sure, ta) : 0;
        s_base_c = tc ? atomicAdd(&gst->n_cand, tc) : 0;
    }
    __syncthreads();
    if (na + nc == 0) return;   // warp-uniform
    int pa = s_base_a, pc = s_base_c;
    for (int x = 0; x < wp; ++x) {
        pa += s_na[x];
        pc += s_nc[x];
    }
    const unsigned lower = (1u << lane) - 1u;
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
        const bool above = (fa >> j) & 1u, take_c = (fc >> j) & 1u;
        const unsigned ma = __ballot_sync(0xffffffffu, above);
        const unsigned mc = __ballot_sync(0xffffffffu, take_c);
        if (!(ma | mc)) continue;   // warp-uniform
        const int64_t i = chunk_index<kVec>(i0, j);
        const uint32_t key = (above || take_c) ? float_to_ordered(s[i]) : 0u;
        if (above) {
            const int slot = pa + __popc(ma & lower);
            if (slot < k) w.sure[(size_t)row * k + slot] = composite(key, i);
            else atomicOr(status, (unsigned)FATHOM_DEV_TOPK_OVERFLOW);
        }
        if (take_c) {
            const int slot = pc + __popc(mc & lower);
            if (slot < kCap) w.cand[(size_t)row * kCap + slot] = composite(key, i);
            else atomicOr(status, (unsigned)FATHOM_DEV_TOPK_OVERFLOW);
        }
        pa += __popc(ma);
        pc += __popc(mc);
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
    if ((reinterpret_cast<uintptr_t>(s + i0) & 15) == 0) compact_body<true>(s, i0, i1, st, row, k, w, status);
    else compact_body<false>(s, i0, i1, st, row, k, w, status);
}

// Bitonic sort, descending, of buf[0..S), S a power of two.  Thread t
// compares elements i = 2t - t % stride and i + stride, so while stride <= 32
// a warp touches only its own 64-element ranges and a warp barrier suffices
// between two such stages; the block barrier is taken before and after every
// stage that crosses warps.
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
            // a stage that crosses warps (stride > 32) needs the block barrier
            // after it, and so does the stage before one
            const int next = stride > 1 ? stride >> 1 : size;   // stride of the next stage
            if (stride > 32 || next > 32 || (stride == 1 && size == S)) __syncthreads();
            else __syncwarp();
        }
    }
}

// Descending bitonic sort of buf[0..S) (S a power of two, 32 <= S <=
// blockDim.x) with one element per thread: thread e holds element e in a
// register; stages whose partner lies in the same warp (stride < 32) exchange
// by shuffles, the others through buf between two block barriers.  S is a
// template argument, so every stage is unrolled with its size and stride
// fixed.  Called by every thread of the block.
template <int S>
__device__ __forceinline__ void bitonic_desc_reg_t(uint64_t* buf) {
    const int e = threadIdx.x;
    uint64_t v = (e < S) ? buf[e] : 0ull;
#pragma unroll
    for (int size = 2; size <= S; size <<= 1) {
#pragma unroll
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            uint64_t w;
            if (stride >= 32) {
                __syncthreads();
                if (e < S) buf[e] = v;
                __syncthreads();
                w = (e < S) ? buf[e ^ stride] : 0ull;
            } else {
                const uint32_t lo = __shfl_xor_sync(0xffffffffu, (uint32_t)v, stride);
                const uint32_t hi = __shfl_xor_sync(0xffffffffu, (uint32_t)(v >> 32), stride);
                w = ((uint64_t)hi << 32) | lo;
            }
            // in a descending run the lower index of a pair keeps the larger
            const bool keep_max = (((e & stride) != 0) == ((e & size) != 0));
            const bool gt = v > w;
            v = (keep_max == gt) ? v : w;
        }
    }
    __syncthreads();
    if (e < S) buf[e] = v;
    __syncthreads();
}

// bitonic_desc_reg_t for a run-time S in [32, 512]
__device__ void bitonic_desc_reg(uint64_t* buf, int S) {
    switch (S) {
        case 32: bitonic_desc_reg_t<32>(buf); break;
        case 64: bitonic_desc_reg_t<64>(buf); break;
        case 128: bitonic_desc_reg_t<128>(buf); break;
        case 256: bitonic_desc_reg_t<256>(buf); break;
        default: bitonic_desc_reg_t<512>(buf); break;
    }
}

// Number of entries of the descending list ly[0..n) greater than v: a binary
// search whose steps depend only on n (the same for every thread that
// searches a list of that length).
__device__ __forceinline__ int count_above(const uint64_t* ly, int n, uint64_t v) {
    if (n == 0) return 0;
    int base = 0;
#pragma unroll
    for (int it = 0; it < 13; ++it) {   // n <= kMaxTopK = 2^12: at most 12 halvings
        if (n > 1) {
            const int half = n >> 1;
            base += (ly[base + half - 1] > v) ? half : 0;
            n -= half;
        }
    }
    return base + (ly[base] > v ? 1 : 0);
}

// With hist[0..nb) filled, finds the bin b holding the need-th largest key
// (bins ordered high to low): *above = keys in bins above b, *cnt = keys in b.
// Called by every thread of the block (a multiple of 32 threads, at most
// 1024); all get the result.
__device__ void block_pick_bin(const uint32_t* hist, int nb, uint32_t need, int* s_bin, uint32_t* s_above,
                               uint32_t* s_cnt, uint32_t* warp_tot) {
    const int t = threadIdx.x, lane = t & 31, wp = t >> 5, nt = (int)blockDim.x;
    const int per = nb / nt > 0 ? nb / nt : 1;   // bins per thread
    uint32_t mine = 0;
    if (per * t < nb)
        for (int e = 0; e < per; ++e) mine += hist[per * t + e];
    uint32_t v = mine;   // sum over this thread and the higher lanes of its warp
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_down_sync(0xffffffffu, v, o);
        if (31 - lane >= o) v += y;
    }
    if (lane == 0) warp_tot[wp] = v;
    __syncthreads();
    uint32_t higher = 0;
    for (int x = wp + 1; x < nt / 32; ++x) higher += warp_tot[x];
    const uint32_t incl = v + higher, above = incl - mine;
    if (above < need && incl >= need && per * t < nb) {
        uint32_t acc = above;
        for (int e = per - 1; e >= 0; --e) {
            const uint32_t c = hist[per * t + e];
            if (acc + c >= need) {
                *s_bin = per * t + e;
                *s_above = acc;
                *s_cnt = c;
                break;
            }
            acc += c;
        }
    }
    __syncthreads();
}

__global__ void __launch_bounds__(kFinishThreads)
topk_finish(const float* __restrict__ scores, const __grid_constant__ RowMap m, int k, Workspace w,
            int32_t* __restrict__ idx, float* __restrict__ top_scores, unsigned int* status) {
    extern __shared__ uint64_t buf[];
    __shared__ uint32_t hist[kBins];
    __shared__ uint32_t warp_tot[32];
    __shared__ int warp_cnt[32];
    __shared__ int s_got, s_bin, s_fill;
    __shared__ uint32_t s_above, s_cnt;
    const int row = blockIdx.x;
    const RowState st = w.state[row];
    int64_t off, n;
    row_span(m, row, &off, &n);
    const int ns = min(st.count_above, k);
    int total;
    if (st.phase == 1) {
        // the exact k-th key T among the candidates, by radix steps over the
        // bits the row passes left unresolved
        const int nc = min(st.cand, kCap);
        const uint64_t* cand = w.cand + (size_t)row * kCap;
        uint32_t need = (uint32_t)(k - ns);
        uint32_t prefix = st.prefix;
        int shift = st.shift;
        while (shift > 0) {
            const int nbits = shift >= 12 ? 12 : shift, sh = shift - nbits;
            const int nb = 1 << nbits;
            for (int b = threadIdx.x; b < nb; b += kFinishThreads) hist[b] = 0;
            __syncthreads();
            for (int e = threadIdx.x; e < nc; e += kFinishThreads) {
                const uint32_t key = (uint32_t)(cand[e] >> 32);
                if (shift == 32 || (key >> shift) == prefix) atomicAdd(&hist[(key >> sh) & (nb - 1)], 1u);
            }
            __syncthreads();
            block_pick_bin(hist, nb, need, &s_bin, &s_above, &s_cnt, warp_tot);
            need -= s_above;
            prefix = (shift == 32 ? 0u : (prefix << nbits)) | (uint32_t)s_bin;
            shift = sh;
            __syncthreads();   // s_bin / s_above are rewritten by the next step
        }
        const uint32_t T = prefix;
        // keep the sure keys, the candidates above T and the candidates at T
        for (int e = threadIdx.x; e < ns; e += kFinishThreads) buf[e] = w.sure[(size_t)row * k + e];
        if (threadIdx.x == 0) s_fill = ns;
        __syncthreads();
        for (int e = threadIdx.x; e < nc; e += kFinishThreads) {
            const uint64_t c = cand[e];
            if ((uint32_t)(c >> 32) >= T) buf[atomicAdd(&s_fill, 1)] = c;
        }
        __syncthreads();
        total = s_fill;
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
            unsigned msk = __ballot_sync(0xffffffffu, f);
            if (lane == 0) warp_cnt[wp] = __popc(msk);
            __syncthreads();
            int before = 0;
            for (int x = 0; x < wp; ++x) before += warp_cnt[x];
            int rank = got + before + __popc(msk & ((1u << lane) - 1u));
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

// ---------------------------------------------------------------------------
// Top-k from block maxima.  The scan also writes, for every 64-key block, the
// largest score of the block (as an ordered key).  With m = the k-th largest
// block maximum of a row, k distinct keys (each block's maximum) score at
// least m, so the k-th largest score T >= m, and every key at or above T lies
// in a block whose maximum is >= m: only those blocks (about k of them) are
// read.  Kernels: threshold (m per row), compact (the keys >= m of the
// surviving blocks), finish (the exact T among them, the sure keys and ties,
// sorted).  A row whose candidates overflow the buffer (e.g. all scores
// equal) is finished from its full row instead, with the same exact rules.
// ---------------------------------------------------------------------------
constexpr int kCapB = 16384;   // candidates per row on the block path

struct BlkWs {
    RowState* state;   // [rows]: prefix = m, n_cand, pad bit 0 = candidate overflow
    uint64_t* cand;    // [rows][kCapB]
};

BlkWs carve_blk(void* ws, int rows) {
    BlkWs w;
    char* p = static_cast<char*>(ws);
    w.state = reinterpret_cast<RowState*>(p);
    p += align256(sizeof(RowState) * rows);
    w.cand = reinterpret_cast<uint64_t*>(p);
    return w;
}

// The exact need-th largest of cnt ordered keys key_at(0..cnt) (1 <= need <=
// cnt): radix steps of 12, 12 and 8 bits with a shared-memory histogram.
// Returns T; *gt = keys above T, *eq = keys equal to T.  All threads of a
// kFinishThreads block call it and get the result.
template <class KeyAt>
__device__ uint32_t block_kth_key(KeyAt key_at, int64_t cnt, uint32_t need, uint32_t* hist, int* s_bin,
                                  uint32_t* s_above, uint32_t* s_cnt, uint32_t* warp_tot, uint32_t* gt, uint32_t* eq) {
    uint32_t prefix = 0, above = 0;
    int shift = 32;
    while (shift > 0) {
        const int nbits = shift >= 12 ? 12 : shift, sh = shift - nbits, nb = 1 << nbits;
        for (int b = threadIdx.x; b < nb; b += blockDim.x) hist[b] = 0;
        __syncthreads();
        for (int64_t e = threadIdx.x; e < cnt; e += blockDim.x) {
            const uint32_t key = key_at(e);
            if (shift == 32 || (key >> shift) == prefix) atomicAdd(&hist[(key >> sh) & (nb - 1)], 1u);
        }
        __syncthreads();
        block_pick_bin(hist, nb, need, s_bin, s_above, s_cnt, warp_tot);
        need -= *s_above;
        above += *s_above;
        prefix = (shift == 32 ? 0u : (prefix << nbits)) | (uint32_t)*s_bin;
        shift = sh;
        __syncthreads();   // s_bin / s_above are rewritten by the next step
    }
    *gt = above;
    *eq = *s_cnt;
    return prefix;
}

__global__ void __launch_bounds__(kFinishThreads)
topk_blk_threshold(const uint32_t* __restrict__ bmax, const __grid_constant__ RowMap m, int k, BlkWs w) {
    pdl_wait();
    __shared__ uint32_t hist[kBins];
    __shared__ uint32_t warp_tot[32];
    __shared__ int s_bin;
    __shared__ uint32_t s_above, s_cnt;
    const int row = blockIdx.x;
    int64_t off, n;
    row_span(m, row, &off, &n);
    const uint32_t* bm = bmax + off / kBlock;
    const int64_t nreal = (n + kBlock - 1) / kBlock;
    uint32_t mkey = 0;   // fewer blocks than k: every key is a candidate
    if (k <= nreal) {
        uint32_t gt, eq;
        mkey = block_kth_key([&](int64_t e) { return bm[e]; }, nreal, (uint32_t)k, hist, &s_bin, &s_above, &s_cnt,
                             warp_tot, &gt, &eq);
    }
    if (threadIdx.x == 0) {
        RowState s;
        s.prefix = mkey;
        s.shift = 0;
        s.count_above = 0;
        s.cand = 0;
        s.phase = 1;
        s.n_sure = 0;
        s.n_cand = 0;
        s.pad = 0;
        w.state[row] = s;
    }
}

// Thread t of CTA x looks at block j = 256 x + t; a warp then reads each of
// its surviving blocks (64 scores, two per lane) and keeps the keys >= m.
__global__ void __launch_bounds__(kPassThreads)
topk_blk_compact(const float* __restrict__ scores, const uint32_t* __restrict__ bmax, const __grid_constant__ RowMap m,
                 BlkWs w) {
    pdl_wait();
    const int row = blockIdx.y;
    int64_t off, n;
    row_span(m, row, &off, &n);
    const int64_t nreal = (n + kBlock - 1) / kBlock;
    const uint32_t mkey = w.state[row].prefix;
    const uint32_t* bm = bmax + off / kBlock;
    const float* s = scores + off;
    RowState* gst = w.state + row;
    const int lane = threadIdx.x & 31;
    const int64_t j = (int64_t)blockIdx.x * kPassThreads + threadIdx.x;
    const bool surv = j < nreal && bm[j] >= mkey;
    unsigned sm = __ballot_sync(0xffffffffu, surv);
    const unsigned lower = (1u << lane) - 1u;
    const int64_t j0 = j - lane;
    while (sm) {   // warp-uniform
        const int src = __ffs(sm) - 1;
        sm &= sm - 1;
        const int64_t i0 = (j0 + src) * kBlock;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            const int64_t i = i0 + half * 32 + lane;
            const uint32_t key = (i < n) ? float_to_ordered(s[i]) : 0u;
            const bool keep = i < n && key >= mkey;
            const unsigned km = __ballot_sync(0xffffffffu, keep);
            if (!km) continue;
            int base = 0;
            if (lane == 0) base = atomicAdd(&gst->n_cand, __popc(km));
            base = __shfl_sync(0xffffffffu, base, 0);
            if (keep) {
                const int slot = base + __popc(km & lower);
                if (slot < kCapB) w.cand[(size_t)row * kCapB + slot] = composite(key, i);
                else atomicOr(&gst->pad, 1);
            }
        }
    }
}

__global__ void __launch_bounds__(kFinishThreads)
topk_blk_finish(const float* __restrict__ scores, const __grid_constant__ RowMap m, int k, BlkWs w,
                int32_t* __restrict__ idx, float* __restrict__ top_scores) {
    pdl_wait();
    extern __shared__ uint64_t buf[];
    __shared__ uint32_t hist[kBins];
    __shared__ uint32_t warp_tot[32];
    __shared__ int warp_cnt[32];
    __shared__ int s_bin, s_fill, s_got;
    __shared__ uint32_t s_above, s_cnt;
    const int row = blockIdx.x;
    const RowState st = w.state[row];
    int64_t off, n;
    row_span(m, row, &off, &n);
    const float* s = scores + off;
    const uint64_t* cand = w.cand + (size_t)row * kCapB;
    const bool use_cand = !(st.pad & 1);   // else the candidates overflowed: use the full row
    const int64_t cnt = use_cand ? (int64_t)min(st.n_cand, kCapB) : n;
    auto key_at = [&](int64_t e) -> uint32_t {
        return use_cand ? (uint32_t)(cand[e] >> 32) : float_to_ordered(s[e]);
    };
    uint32_t gt, eq;
    const uint32_t T = block_kth_key(key_at, cnt, (uint32_t)k, hist, &s_bin, &s_above, &s_cnt, warp_tot, &gt, &eq);
    const bool ties_fit = gt + eq <= (uint32_t)kSortMax;
    if (threadIdx.x == 0) s_fill = 0;
    __syncthreads();
    for (int64_t e = threadIdx.x; e < cnt; e += blockDim.x) {
        const uint32_t key = key_at(e);
        if (key > T || (ties_fit && key == T)) buf[atomicAdd(&s_fill, 1)] = use_cand ? cand[e] : composite(key, e);
    }
    __syncthreads();
    int total = s_fill;
    if (!ties_fit) {
        // more keys tie at T than the sort holds: take the lowest indices, in order
        const int ns = (int)gt, r = k - ns;
        if (threadIdx.x == 0) s_got = 0;
        __syncthreads();
        const int lane = threadIdx.x & 31, wp = threadIdx.x >> 5;
        for (int64_t base = 0; base < n; base += blockDim.x) {
            const int got = s_got;
            if (got >= r) break;
            const int64_t i = base + threadIdx.x;
            const bool f = (i < n) && float_to_ordered(s[i]) == T;
            const unsigned msk = __ballot_sync(0xffffffffu, f);
            if (lane == 0) warp_cnt[wp] = __popc(msk);
            __syncthreads();
            int before = 0;
            for (int x = 0; x < wp; ++x) before += warp_cnt[x];
            const int rank = got + before + __popc(msk & ((1u << lane) - 1u));
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
        const uint64_t c = buf[e];
        idx[(int64_t)row * k + e] = (int32_t)(0xFFFFFFFFu - (uint32_t)c);
        if (top_scores) top_scores[(int64_t)row * k + e] = ordered_to_float((uint32_t)(c >> 32));
    }
}

// ---------------------------------------------------------------------------
// Short rows (n <= kRowsMax keys): one kernel, no workspace.  A cluster of CL
// CTAs takes a row; CTA x holds the ordered keys of its slice of the row
// in shared memory (thread t: keys 4 (t + 512 u) .. + 3, u < 8).  The first
// histogram (bits 31..20) is built while the keys load.  The CTAs' histograms
// are combined through distributed shared memory (cluster_pick).  When at
// most kMaxTopK keys lie at or above the k-th key's 12-bit bin - the usual
// case - those are the candidates: each CTA compacts its own (a block
// scan of per-thread counts), sorts them, copies the other CTAs' sorted lists
// into its shared memory, and ranks each of its candidates by binary searches
// in them.  Otherwise two more radix steps (12 and 8 bits) find the exact k-th
// key T; each CTA writes its keys above T, and its keys equal to T whose rank
// among the row's ties (CTA order, then index order) is below k - #{keys > T},
// into CTA 0's shared memory; CTA 0 sorts the k entries as 64-bit composites
// (key << 32 | ~index).
// ---------------------------------------------------------------------------
constexpr int kSliceKeys = 16384;   // keys per CTA
constexpr int kRowThreads = 512;
constexpr int kRowVec = kSliceKeys / (4 * kRowThreads);   // 4-key groups per thread
constexpr int kMaxCluster = 8;
constexpr int64_t kRowsMax = (int64_t)kMaxCluster * kSliceKeys;
// keys, histogram, candidate buffer (which also holds the cluster's range
// sums while a pick runs): 112 KB, so two CTAs share an SM
constexpr size_t kRowSmem = sizeof(uint32_t) * (kSliceKeys + kBins) + sizeof(uint64_t) * kMaxTopK;

__device__ __forceinline__ int block_sum_int(int v, int* warp_cnt) {
    const int lane = threadIdx.x & 31, wp = threadIdx.x >> 5;
    v = __reduce_add_sync(0xffffffffu, v);
    if (lane == 0) warp_cnt[wp] = v;
    __syncthreads();
    int t = 0;
    for (int x = 0; x < (int)(blockDim.x >> 5); ++x) t += warp_cnt[x];
    __syncthreads();
    return t;
}

template <int CL>
__device__ __forceinline__ void cluster_barrier() {
    if constexpr (CL > 1) cg::this_cluster().sync();
    else __syncthreads();
}

// With this CTA's keys added to hist[0..nb), picks the bin of the need-th
// largest key of the whole cluster, as block_pick_bin (every CTA gets the
// result).  The summed histogram is split: CTA x sums bins [x nb/CL,
// (x+1) nb/CL) over the cluster into hsum and publishes their total; every
// CTA then finds the range holding the need-th key from the totals and picks
// inside it from that range's sums.  Cluster barriers: after the first every
// histogram is complete, after the second every range sum (hist is read by
// other CTAs only between the two), after the third every CTA has read the
// range it needed (hsum shares memory with the candidate buffer, written next).
template <int CL>
__device__ __forceinline__ void cluster_pick(uint32_t* hist, uint32_t* hsum, int nb, uint32_t need, int* s_bin,
                                             uint32_t* s_above, uint32_t* s_cnt, uint32_t* warp_tot, int* warp_cnt,
                                             uint32_t* s_tot) {
    if constexpr (CL > 1) {
        cg::cluster_group cluster = cg::this_cluster();
        const int x = (int)cluster.block_rank(), per = nb / CL, tid = threadIdx.x;
        cluster.sync();   // every CTA's histogram is complete
        int mine = 0;
        for (int j = tid; j < per; j += kRowThreads) {
            uint32_t t = 0;
#pragma unroll
            for (int y = 0; y < CL; ++y) t += cluster.map_shared_rank(hist, y)[x * per + j];
            hsum[j] = t;
            mine += (int)t;
        }
        mine = block_sum_int(mine, warp_cnt);
        if (tid == 0) *s_tot = (uint32_t)mine;
        cluster.sync();   // range sums and totals are published; nobody reads hist any more
        uint32_t tot[CL];
#pragma unroll
        for (int y = 0; y < CL; ++y) tot[y] = *cluster.map_shared_rank(s_tot, y);
        uint32_t acc = 0;
        int ys = 0;
        for (int y = CL - 1; y >= 0; --y) {   // ranges from the highest bins down
            if (acc + tot[y] >= need) {
                ys = y;
                break;
            }
            acc += tot[y];
        }
        const uint32_t* hy = cluster.map_shared_rank(hsum, ys);
        for (int j = tid; j < per; j += kRowThreads) hist[j] = hy[j];
        __syncthreads();
        block_pick_bin(hist, per, need - acc, s_bin, s_above, s_cnt, warp_tot);
        if (tid == 0) {
            *s_bin += ys * per;
            *s_above += acc;
        }
        cluster.sync();   // the picks are visible, and every CTA has read the range it needed
    } else {
        __syncthreads();
        block_pick_bin(hist, nb, need, s_bin, s_above, s_cnt, warp_tot);
    }
}

// The candidates of a row (its keys at or above a threshold below the k-th
// key, at most kMaxTopK over the cluster) are sorted per CTA: buf[0..c) holds
// this CTA's, descending, and *s_fill their count.  Each CTA copies the other
// CTAs' lists into its own shared memory (the key slice is free by then); the
// rank of a candidate in the row is its position in its CTA's list plus, for
// every other CTA, the number of that CTA's candidates above it (a binary
// search in the copy); ranks below k are written out.  Composites are
// distinct (the index is part of them), so the ranks are a permutation and
// ties order by index.
template <int CL>
__device__ void rank_candidates(uint32_t* keys, const uint64_t* buf, int c, int* s_fill, int row, int k,
                                int32_t* __restrict__ idx, float* __restrict__ top_scores) {
    const int tid = threadIdx.x;
    cluster_barrier<CL>();   // every CTA's list is sorted and its count published
    int lo_of[CL], n_of[CL];
    uint64_t* lists = reinterpret_cast<uint64_t*>(keys);   // at most kMaxTopK composites, the slice holds kSliceKeys / 2
    if constexpr (CL > 1) {
        cg::cluster_group cluster = cg::this_cluster();
        const int x = (int)cluster.block_rank();
        int at = 0;
#pragma unroll
        for (int y = 0; y < CL; ++y) {
            n_of[y] = (y == x) ? 0 : *cluster.map_shared_rank(s_fill, y);
            lo_of[y] = at;
            at += n_of[y];
        }
        // the lists in rounds of kRowThreads entries, each round's remote
        // loads all issued before its stores
        int most = 0;
#pragma unroll
        for (int y = 0; y < CL; ++y) most = max(most, n_of[y]);
        for (int base = 0; base < most; base += kRowThreads) {
            const int e = base + tid;
            uint64_t v[CL];
#pragma unroll
            for (int y = 0; y < CL; ++y)
                if (e < n_of[y]) v[y] = cluster.map_shared_rank(buf, y)[e];
#pragma unroll
            for (int y = 0; y < CL; ++y)
                if (e < n_of[y]) lists[lo_of[y] + e] = v[y];
        }
        cluster_barrier<CL>();   // every CTA has its copies: no remote reads after this
    }
    for (int j = tid; j < c; j += kRowThreads) {
        const uint64_t v = buf[j];
        int r = j;
        if constexpr (CL > 1) {
#pragma unroll
            for (int y = 0; y < CL; ++y) r += count_above(lists + lo_of[y], n_of[y], v);
        }
        if (r < k) {
            idx[(int64_t)row * k + r] = (int32_t)(0xFFFFFFFFu - (uint32_t)v);
            if (top_scores) top_scores[(int64_t)row * k + r] = ordered_to_float((uint32_t)(v >> 32));
        }
    }
}

template <int CL>
__global__ void __launch_bounds__(kRowThreads, 2)
topk_rows(const float* __restrict__ scores, const __grid_constant__ RowMap m, int k, int32_t* __restrict__ idx,
          float* __restrict__ top_scores) {
    pdl_wait();
    extern __shared__ __align__(16) unsigned char row_sm[];
    uint32_t* keys = reinterpret_cast<uint32_t*>(row_sm);                        // [kSliceKeys]
    uint32_t* hist = keys + kSliceKeys;                                           // [kBins]
    uint64_t* buf = reinterpret_cast<uint64_t*>(hist + kBins);                    // [kMaxTopK]
    uint32_t* hsum = reinterpret_cast<uint32_t*>(buf);                            // [kBins / CL], CL > 1
    __shared__ uint32_t warp_tot[32];
    __shared__ int warp_cnt[32];
    __shared__ int s_bin, s_fill, s_gt, s_eq;
    __shared__ uint32_t s_above, s_cnt, s_tot;
    const int tid = threadIdx.x, lane = tid & 31, wp = tid >> 5;
    int rank = 0;
    if constexpr (CL > 1) rank = (int)cg::this_cluster().block_rank();
    const int row = blockIdx.x / CL;
    int64_t off, n;
    row_span(m, row, &off, &n);
    const int64_t L = ((n + CL - 1) / CL + 3) & ~int64_t(3);   // slice length, <= kSliceKeys
    const int64_t start = rank * L;
    const int cnt = (int)(n - start < 0 ? 0 : (n - start < L ? n - start : L));
    const float* s = scores + off + start;

    for (int b = tid; b < kBins; b += kRowThreads) hist[b] = 0;
    if (tid == 0) s_fill = 0;   // the candidate count (the fast path's reservations)
    __syncthreads();

    // the slice as ordered keys in shared memory (thread t: 4-key groups
    // t + 512 u), counted into the first histogram as they arrive
    const bool vec = (reinterpret_cast<uintptr_t>(s) & 15u) == 0;
    // a whole aligned slice (every CTA of a 131072-key row) takes the loop
    // without bounds checks
    const bool full = vec && cnt == kSliceKeys;
    if (full) {
#pragma unroll 4
        for (int u = 0; u < kRowVec; ++u) {
            const int e = 4 * (tid + kRowThreads * u);
            const float4 x = __ldg(reinterpret_cast<const float4*>(s + e));
            const uint32_t v[4] = {float_to_ordered(x.x), float_to_ordered(x.y), float_to_ordered(x.z),
                                   float_to_ordered(x.w)};
            *reinterpret_cast<uint4*>(keys + e) = make_uint4(v[0], v[1], v[2], v[3]);
#pragma unroll
            for (int c = 0; c < 4; ++c) atomicAdd(&hist[v[c] >> 20], 1u);
        }
    } else {
#pragma unroll 4
        for (int u = 0; u < kRowVec; ++u) {
            const int e = 4 * (tid + kRowThreads * u);
            uint32_t v[4];
            if (vec && e + 3 < cnt) {
                const float4 x = __ldg(reinterpret_cast<const float4*>(s + e));
                v[0] = float_to_ordered(x.x);
                v[1] = float_to_ordered(x.y);
                v[2] = float_to_ordered(x.z);
                v[3] = float_to_ordered(x.w);
                *reinterpret_cast<uint4*>(keys + e) = make_uint4(v[0], v[1], v[2], v[3]);
            } else {
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    v[c] = (e + c < cnt) ? float_to_ordered(__ldg(s + e + c)) : 0u;
                    if (e + c < cnt) keys[e + c] = v[c];
                }
            }
#pragma unroll
            for (int c = 0; c < 4; ++c)
                if (e + c < cnt) atomicAdd(&hist[v[c] >> 20], 1u);
        }
    }

    // the exact k-th largest key T of the row (the first step's histogram is built)
    uint32_t need = (uint32_t)k, prefix = 0, above = 0;
    int shift = 32;
    while (shift > 0) {
        const int nbits = shift >= 12 ? 12 : shift, sh = shift - nbits, nb = 1 << nbits;
        if (shift != 32) {
            for (int b = tid; b < nb; b += kRowThreads) hist[b] = 0;
            __syncthreads();
            for (int e = tid; e < cnt; e += kRowThreads) {
                const uint32_t key = keys[e];
                if ((key >> shift) == prefix) atomicAdd(&hist[(key >> sh) & (nb - 1)], 1u);
            }
        }
        cluster_pick<CL>(hist, hsum, nb, need, &s_bin, &s_above, &s_cnt, warp_tot, warp_cnt, &s_tot);
        need -= s_above;
        above += s_above;
        prefix = (shift == 32 ? 0u : (prefix << nbits)) | (uint32_t)s_bin;
        const uint32_t in_bin = s_cnt;   // keys of the row in the picked bin
        shift = sh;
        __syncthreads();   // s_bin / s_above are rewritten by the next step
        if (shift == 20 && above + in_bin <= (uint32_t)kMaxTopK) {
            // few keys at or above thr: they are the candidates, and an exact
            // sort of them gives the top k
            const uint32_t thr = prefix << 20;
            int mine = 0;
            if (full) {
#pragma unroll
                for (int u = 0; u < kRowVec; ++u) {
                    const uint4 v = *reinterpret_cast<const uint4*>(keys + 4 * (tid + kRowThreads * u));
                    mine += (v.x >= thr) + (v.y >= thr) + (v.z >= thr) + (v.w >= thr);
                }
            } else {
                for (int u = 0; u < kRowVec; ++u) {
                    const int e = 4 * (tid + kRowThreads * u);
                    if (e >= cnt) break;
                    const uint4 v = *reinterpret_cast<const uint4*>(keys + e);   // past cnt: never counted
                    mine += (v.x >= thr) + (e + 1 < cnt && v.y >= thr) + (e + 2 < cnt && v.z >= thr) +
                            (e + 3 < cnt && v.w >= thr);
                }
            }
            // one reservation per warp in the candidate buffer (any order: sorted next)
            int incl = mine;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += y;
            }
            const int wtot = __shfl_sync(0xffffffffu, incl, 31);
            int wbase = 0;
            if (lane == 0 && wtot > 0) wbase = atomicAdd(&s_fill, wtot);
            int at = __shfl_sync(0xffffffffu, wbase, 0) + incl - mine;
            for (int u = 0; u < kRowVec && mine > 0; ++u) {
                const int e = 4 * (tid + kRowThreads * u);
                if (e >= cnt) break;
                const uint4 v = *reinterpret_cast<const uint4*>(keys + e);
                const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    if (e + c < cnt && w[c] >= thr) {
                        buf[at++] = composite(w[c], start + e + c);
                        --mine;
                    }
            }
            __syncthreads();
            const int c_all = s_fill;
            int S = 32;
            while (S < c_all) S <<= 1;
            for (int e = c_all + tid; e < S; e += kRowThreads) buf[e] = 0ull;   // below every composite of the row
            __syncthreads();
            if (S <= kRowThreads) bitonic_desc_reg(buf, S);
            else bitonic_desc(buf, S);
            rank_candidates<CL>(keys, buf, c_all, &s_fill, row, k, idx, top_scores);
            return;
        }
    }
    const uint32_t T = prefix;
    const int gt_row = (int)above, take_eq = k - gt_row;   // keys above T; ties to take (>= 1)

    // this CTA's keys above T and at T, and those of the CTAs before it
    int my_gt = 0, my_eq = 0;
    for (int e = tid; e < cnt; e += kRowThreads) {
        my_gt += keys[e] > T;
        my_eq += keys[e] == T;
    }
    my_gt = block_sum_int(my_gt, warp_cnt);
    my_eq = block_sum_int(my_eq, warp_cnt);
    if (tid == 0) {
        s_gt = my_gt;
        s_eq = my_eq;
        s_fill = 0;
    }
    cluster_barrier<CL>();
    int gt_before = 0, eq_before = 0;
    uint64_t* dst = buf;
    if constexpr (CL > 1) {
        cg::cluster_group cluster = cg::this_cluster();
        for (int x = 0; x < rank; ++x) {
            gt_before += *cluster.map_shared_rank(&s_gt, x);
            eq_before += *cluster.map_shared_rank(&s_eq, x);
        }
        dst = cluster.map_shared_rank(buf, 0);
    }
    // keys above T, in any order (the sort orders them)
    for (int e = tid; e < cnt; e += kRowThreads)
        if (keys[e] > T) dst[gt_before + atomicAdd(&s_fill, 1)] = composite(keys[e], start + e);
    // keys at T with row tie rank < take_eq
    if (my_eq > 0 && eq_before < take_eq) {
        if (eq_before + my_eq <= take_eq) {   // all of this CTA's ties are taken: any order
            __syncthreads();
            if (tid == 0) s_fill = 0;
            __syncthreads();
            for (int e = tid; e < cnt; e += kRowThreads)
                if (keys[e] == T) dst[gt_row + eq_before + atomicAdd(&s_fill, 1)] = composite(T, start + e);
        } else {   // the cut falls inside this CTA: ordered scan
            int got = eq_before;
            for (int base = 0; base < cnt && got < take_eq; base += kRowThreads) {
                const int e = base + tid;
                const bool f = e < cnt && keys[e] == T;
                const unsigned msk = __ballot_sync(0xffffffffu, f);
                if (lane == 0) warp_cnt[wp] = __popc(msk);
                __syncthreads();
                int before = 0, all = 0;
                for (int x = 0; x < kRowThreads / 32; ++x) {
                    before += (x < wp) ? warp_cnt[x] : 0;
                    all += warp_cnt[x];
                }
                const int r = got + before + __popc(msk & ((1u << lane) - 1u));
                if (f && r < take_eq) dst[gt_row + r] = composite(T, start + e);
                got += all;
                __syncthreads();   // warp_cnt is rewritten by the next window
            }
        }
    }
    cluster_barrier<CL>();   // CTA 0 holds the row's k entries
    if (rank != 0) return;
    int S = 1;
    while (S < k) S <<= 1;
    for (int e = k + tid; e < S; e += kRowThreads) buf[e] = 0ull;
    __syncthreads();
    bitonic_desc(buf, S);
    for (int e = tid; e < k; e += kRowThreads) {
        const uint64_t c = buf[e];
        idx[(int64_t)row * k + e] = (int32_t)(0xFFFFFFFFu - (uint32_t)c);
        if (top_scores) top_scores[(int64_t)row * k + e] = ordered_to_float((uint32_t)(c >> 32));
    }
}

template <int CL>
cudaError_t launch_topk_rows_cl(const float* scores, const RowMap& map, int rows, int k, int32_t* idx,
                                float* top_scores, cudaStream_t stream, bool pdl) {
    auto kern = topk_rows<CL>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kRowSmem);
    if (e != cudaSuccess) return e;
    return launch_ex(kern, dim3((unsigned)(rows * CL)), dim3(kRowThreads), kRowSmem, stream, pdl, CL, scores, map, k,
                     idx, top_scores);
}

// ---------------------------------------------------------------------------
// Long rows with block maxima (at least k blocks of 64 keys, at most
// kMaxCluster * kSliceKeys blocks): one cluster kernel, no workspace.  A
// cluster of CL CTAs takes a row; CTA x holds the block maxima of its share of
// the row's blocks in shared memory.  Two radix steps over the maxima (10 and
// 10 bits, combined through distributed shared memory) give thr = the lower
// edge of the 20-bit bin of the k-th largest block maximum m.  Every block
// holds its maximum, so at least k keys are >= m >= thr, the row's k-th key is
// >= thr, and every key at or above it lies in a block whose maximum is >= thr:
// the keys >= thr of those blocks are the candidates (about k of them).  Each
// CTA reads its surviving blocks' scores, keeps the candidates, sorts them and
// ranks them across the cluster as the short-row kernel does.  A row with more
// than kMaxTopK candidates (many keys tied near the threshold) is selected
// exactly from all its keys instead (exact_topk_cluster).
// ---------------------------------------------------------------------------
struct RowShared {
    uint32_t warp_tot[32];
    int warp_cnt[32];
    int bin, fill, gt, eq;
    uint32_t above, cnt, tot;
};

// The exact top k of a row whose keys key_at(0..cnt) (global indices start +
// e) are split over the CL CTAs of a cluster, with no bound on the ties:
// radix steps (12, 12 and 8 bits) find the k-th largest key T; keys above T
// and the first ties at T (CTA order, then index order) go to CTA 0's buffer,
// which sorts the k entries as composites and writes them.  hist (kBins
// words) and buf (kMaxTopK composites; also the range sums) are this CTA's.
template <int CL, class KeyAt>
__device__ void exact_topk_cluster(KeyAt key_at, int cnt, int64_t start, int k, uint32_t* hist, uint64_t* buf,
                                   RowShared* sh, int row, int32_t* __restrict__ idx,
                                   float* __restrict__ top_scores) {
    const int tid = threadIdx.x, lane = tid & 31, wp = tid >> 5;
    int rank = 0;
    if constexpr (CL > 1) rank = (int)cg::this_cluster().block_rank();
    uint32_t* hsum = reinterpret_cast<uint32_t*>(buf);
    uint32_t need = (uint32_t)k, prefix = 0, above = 0;
    for (int shift = 32; shift > 0;) {
        const int nbits = shift >= 12 ? 12 : shift, sh_ = shift - nbits, nb = 1 << nbits;
        cluster_barrier<CL>();   // nobody reads this CTA's histogram or range sums any more
        for (int b = tid; b < nb; b += kRowThreads) hist[b] = 0;
        __syncthreads();
        for (int e = tid; e < cnt; e += kRowThreads) {
            const uint32_t key = key_at(e);
            if (shift == 32 || (key >> shift) == prefix) atomicAdd(&hist[(key >> sh_) & (nb - 1)], 1u);
        }
        cluster_pick<CL>(hist, hsum, nb, need, &sh->bin, &sh->above, &sh->cnt, sh->warp_tot, sh->warp_cnt, &sh->tot);
        need -= sh->above;
        above += sh->above;
        prefix = (shift == 32 ? 0u : (prefix << nbits)) | (uint32_t)sh->bin;
        shift = sh_;
        __syncthreads();   // bin / above are rewritten by the next step
    }
    const uint32_t T = prefix;
    const int gt_row = (int)above, take_eq = k - gt_row;   // keys above T; ties to take (>= 1)
    int my_gt = 0, my_eq = 0;
    for (int e = tid; e < cnt; e += kRowThreads) {
        const uint32_t key = key_at(e);
        my_gt += key > T;
        my_eq += key == T;
    }
    my_gt = block_sum_int(my_gt, sh->warp_cnt);
    my_eq = block_sum_int(my_eq, sh->warp_cnt);
    if (tid == 0) {
        sh->gt = my_gt;
        sh->eq = my_eq;
        sh->fill = 0;
    }
    cluster_barrier<CL>();
    int gt_before = 0, eq_before = 0;
    uint64_t* dst = buf;
    if constexpr (CL > 1) {
        cg::cluster_group cluster = cg::this_cluster();
        for (int x = 0; x < rank; ++x) {
            gt_before += cluster.map_shared_rank(sh, x)->gt;
            eq_before += cluster.map_shared_rank(sh, x)->eq;
        }
        dst = cluster.map_shared_rank(buf, 0);
    }
    for (int e = tid; e < cnt; e += kRowThreads) {
        const uint32_t key = key_at(e);
        if (key > T) dst[gt_before + atomicAdd(&sh->fill, 1)] = composite(key, start + e);
    }
    if (my_eq > 0 && eq_before < take_eq) {
        if (eq_before + my_eq <= take_eq) {   // all of this CTA's ties are taken: any order
            __syncthreads();
            if (tid == 0) sh->fill = 0;
            __syncthreads();
            for (int e = tid; e < cnt; e += kRowThreads)
                if (key_at(e) == T) dst[gt_row + eq_before + atomicAdd(&sh->fill, 1)] = composite(T, start + e);
        } else {   // the cut falls inside this CTA: ordered scan
            int got = eq_before;
            for (int base = 0; base < cnt && got < take_eq; base += kRowThreads) {
                const int e = base + tid;
                const bool f = e < cnt && key_at(e) == T;
                const unsigned msk = __ballot_sync(0xffffffffu, f);
                if (lane == 0) sh->warp_cnt[wp] = __popc(msk);
                __syncthreads();
                int before = 0, all = 0;
                for (int x = 0; x < kRowThreads / 32; ++x) {
                    before += (x < wp) ? sh->warp_cnt[x] : 0;
                    all += sh->warp_cnt[x];
                }
                const int r = got + before + __popc(msk & ((1u << lane) - 1u));
                if (f && r < take_eq) dst[gt_row + r] = composite(T, start + e);
                got += all;
                __syncthreads();   // warp_cnt is rewritten by the next window
            }
        }
    }
    cluster_barrier<CL>();   // CTA 0 holds the row's k entries
    if (rank != 0) return;
    int S = 1;
    while (S < k) S <<= 1;
    for (int e = k + tid; e < S; e += kRowThreads) buf[e] = 0ull;
    __syncthreads();
    bitonic_desc(buf, S);
    for (int e = tid; e < k; e += kRowThreads) {
        const uint64_t c = buf[e];
        idx[(int64_t)row * k + e] = (int32_t)(0xFFFFFFFFu - (uint32_t)c);
        if (top_scores) top_scores[(int64_t)row * k + e] = ordered_to_float((uint32_t)(c >> 32));
    }
}

constexpr int kGatherBlocks = 8;   // surviving blocks a half-warp reads at once

template <int CL>
__global__ void __launch_bounds__(kRowThreads, 2)
topk_bmax_rows(const float* __restrict__ scores, const uint32_t* __restrict__ bmax, const __grid_constant__ RowMap m,
               int k, int32_t* __restrict__ idx, float* __restrict__ top_scores) {
    pdl_wait();
    extern __shared__ __align__(16) unsigned char row_smem[];
    uint32_t* maxima = reinterpret_cast<uint32_t*>(row_smem);                    // [kSliceKeys]
    uint32_t* hist = maxima + kSliceKeys;                                         // [kBins]
    uint64_t* buf = reinterpret_cast<uint64_t*>(hist + kBins);                    // [kMaxTopK]
    uint32_t* hsum = reinterpret_cast<uint32_t*>(buf);                            // range sums, CL > 1
    __shared__ RowShared sh;
    const int tid = threadIdx.x, lane = tid & 31, wp = tid >> 5;
    int rank = 0;
    if constexpr (CL > 1) rank = (int)cg::this_cluster().block_rank();
    const int row = blockIdx.x / CL;
    int64_t off, n;
    row_span(m, row, &off, &n);
    const int64_t nbk = (n + kBlock - 1) / kBlock;
    const int64_t Lb = (nbk + CL - 1) / CL;   // blocks per CTA, <= kSliceKeys
    const int64_t b0 = rank * Lb;
    const int cntb = (int)(nbk - b0 < 0 ? 0 : (nbk - b0 < Lb ? nbk - b0 : Lb));
    const uint32_t* bm = bmax + off / kBlock + b0;
    const float* srow = scores + off;

    // this CTA's block maxima, counted into the first (10-bit) histogram as they load
    for (int b = tid; b < kBins; b += kRowThreads) hist[b] = 0;
    __syncthreads();
    for (int b = tid; b < cntb; b += kRowThreads) {
        const uint32_t v = __ldg(bm + b);
        maxima[b] = v;
        atomicAdd(&hist[v >> 22], 1u);
    }
    cluster_pick<CL>(hist, hsum, 1024, (uint32_t)k, &sh.bin, &sh.above, &sh.cnt, sh.warp_tot, sh.warp_cnt, &sh.tot);
    const uint32_t p1 = (uint32_t)sh.bin, need2 = (uint32_t)k - sh.above;
    __syncthreads();
    for (int b = tid; b < 1024; b += kRowThreads) hist[b] = 0;   // the pick ended with a cluster barrier
    __syncthreads();
    for (int b = tid; b < cntb; b += kRowThreads) {
        const uint32_t v = maxima[b];
        if ((v >> 22) == p1) atomicAdd(&hist[(v >> 12) & 1023u], 1u);
    }
    cluster_pick<CL>(hist, hsum, 1024, need2, &sh.bin, &sh.above, &sh.cnt, sh.warp_tot, sh.warp_cnt, &sh.tot);
    const uint32_t thr = ((p1 << 10) | (uint32_t)sh.bin) << 12;   // <= the k-th largest block maximum
    if (tid == 0) sh.fill = 0;
    __syncthreads();

    // the numbers of the blocks whose maximum is >= thr (any order) in hist,
    // which the picks no longer need; each of them holds at least one
    // candidate, so more than kBins of them means a candidate overflow
    const unsigned lower = (1u << lane) - 1u;
    if (tid == 0) sh.tot = 0;
    __syncthreads();
    for (int b0w = wp * 32; b0w < cntb; b0w += kRowThreads) {
        const int b = b0w + lane;
        const bool surv = b < cntb && maxima[b] >= thr;
        const unsigned sm = __ballot_sync(0xffffffffu, surv);
        if (!sm) continue;
        int base = 0;
        if (lane == 0) base = (int)atomicAdd(&sh.tot, (uint32_t)__popc(sm));
        base = __shfl_sync(0xffffffffu, base, 0);
        const int slot = base + __popc(sm & lower);
        if (surv && slot < kBins) hist[slot] = (uint32_t)b;
    }
    __syncthreads();
    const int nsurv = (int)sh.tot;
    // the keys >= thr of those blocks: a half-warp reads a block (16 lanes x 4
    // keys), a warp 2 * kGatherBlocks blocks at once
    const int hw = lane >> 4, hl = lane & 15;
    const bool vec = (reinterpret_cast<uintptr_t>(srow) & 15u) == 0;
    const int nlist = min(nsurv, kBins);
    for (int q0 = wp * 2 * kGatherBlocks; q0 < nlist; q0 += (kRowThreads / 32) * 2 * kGatherBlocks) {
        // the keys as ordered u32; a key past the row's end or past the list
        // reads as 0, below every threshold (thr > 0: the k-th block maximum
        // is a real score)
        uint4 x[kGatherBlocks];
#pragma unroll
        for (int j = 0; j < kGatherBlocks; ++j) {
            const int q = q0 + 2 * j + hw;
            x[j] = make_uint4(0u, 0u, 0u, 0u);
            if (q < nlist) {
                const int i = (int)((b0 + (int64_t)hist[q]) * kBlock) + 4 * hl;
                if (vec && i + 3 < n) {
                    const float4 f = __ldg(reinterpret_cast<const float4*>(srow + i));
                    x[j] = make_uint4(float_to_ordered(f.x), float_to_ordered(f.y), float_to_ordered(f.z),
                                      float_to_ordered(f.w));
                } else {
                    x[j].x = (i < n) ? float_to_ordered(__ldg(srow + i)) : 0u;
                    x[j].y = (i + 1 < n) ? float_to_ordered(__ldg(srow + i + 1)) : 0u;
                    x[j].z = (i + 2 < n) ? float_to_ordered(__ldg(srow + i + 2)) : 0u;
                    x[j].w = (i + 3 < n) ? float_to_ordered(__ldg(srow + i + 3)) : 0u;
                }
            }
        }
        // this lane's candidates, one reservation per warp
        int mine = 0;
#pragma unroll
        for (int j = 0; j < kGatherBlocks; ++j)
            mine += (x[j].x >= thr) + (x[j].y >= thr) + (x[j].z >= thr) + (x[j].w >= thr);
        int incl = mine;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        const int wtot = __shfl_sync(0xffffffffu, incl, 31);
        int base = 0;
        if (lane == 0 && wtot > 0) base = atomicAdd(&sh.fill, wtot);
        base = __shfl_sync(0xffffffffu, base, 0);
        int pos = base + incl - mine;
        if (mine > 0) {
#pragma unroll
            for (int j = 0; j < kGatherBlocks; ++j) {
                const int q = q0 + 2 * j + hw;
                const uint32_t w4[4] = {x[j].x, x[j].y, x[j].z, x[j].w};
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    if (w4[c] >= thr) {
                        const int i = (int)((b0 + (int64_t)hist[q]) * kBlock) + 4 * hl + c;
                        if (pos < kMaxTopK) buf[pos] = composite(w4[c], i);
                        ++pos;
                    }
            }
        }
    }
    __syncthreads();
    if (nsurv > kBins && tid == 0) sh.fill = kMaxTopK + 1;   // too many blocks: the exact selection below
    __syncthreads();
    const int c_all = sh.fill;   // may exceed kMaxTopK (then only the first kMaxTopK were kept)
    cluster_barrier<CL>();       // every CTA's count is published
    int total = 0;
    if constexpr (CL > 1) {
        cg::cluster_group cluster = cg::this_cluster();
#pragma unroll
        for (int y = 0; y < CL; ++y) total += cluster.map_shared_rank(&sh, y)->fill;
    } else {
        total = c_all;
    }
    if (total > kMaxTopK) {   // the same decision in every CTA of the row
        const int64_t L = (n + CL - 1) / CL;
        const int64_t start = rank * L;
        const int cnt = (int)(n - start < 0 ? 0 : (n - start < L ? n - start : L));
        exact_topk_cluster<CL>([&](int e) { return float_to_ordered(srow[start + e]); }, cnt, start, k, hist, buf, &sh,
                               row, idx, top_scores);
        return;
    }
    int S = 32;
    while (S < c_all) S <<= 1;
    for (int e = c_all + tid; e < S; e += kRowThreads) buf[e] = 0ull;   // below every composite of the row
    __syncthreads();
    if (S <= kRowThreads) bitonic_desc_reg(buf, S);
    else bitonic_desc(buf, S);
    rank_candidates<CL>(maxima, buf, c_all, &sh.fill, row, k, idx, top_scores);
}

template <int CL>
cudaError_t launch_topk_bmax_rows_cl(const float* scores, const uint32_t* bmax, const RowMap& map, int rows, int k,
                                     int32_t* idx, float* top_scores, cudaStream_t stream, bool pdl) {
    auto kern = topk_bmax_rows<CL>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kRowSmem);
    if (e != cudaSuccess) return e;
    return launch_ex(kern, dim3((unsigned)(rows * CL)), dim3(kRowThreads), kRowSmem, stream, pdl, CL, scores, bmax,
                     map, k, idx, top_scores);
}

// rows of at most kRowsMax keys and k <= kMaxTopK
cudaError_t launch_topk_rows(const float* scores, const RowMap& map, int rows, int k, int32_t* idx,
                             float* top_scores, cudaStream_t stream, bool pdl = false) {
    int cl = 1;
    while ((int64_t)cl * kSliceKeys < map.max_n) cl <<= 1;
    switch (cl) {
        case 1: return launch_topk_rows_cl<1>(scores, map, rows, k, idx, top_scores, stream, pdl);
        case 2: return launch_topk_rows_cl<2>(scores, map, rows, k, idx, top_scores, stream, pdl);
        case 4: return launch_topk_rows_cl<4>(scores, map, rows, k, idx, top_scores, stream, pdl);
        case 8: return launch_topk_rows_cl<8>(scores, map, rows, k, idx, top_scores, stream, pdl);
        default: return cudaErrorInvalidValue;
    }
}

// positions into the gathered candidate lists -> the candidates' global indices
__global__ void topk_map_positions(const int32_t* __restrict__ cand_idx, int n_cand, int k, int32_t* idx) {
    const int row = blockIdx.y;
    const int e = blockIdx.x * blockDim.x + threadIdx.x;
    if (e >= k) return;
    const int32_t p = idx[(int64_t)row * k + e];
    idx[(int64_t)row * k + e] = (p >= 0 && p < n_cand) ? cand_idx[(int64_t)row * n_cand + p] : -1;
}

}  // namespace

cudaError_t launch_topk_merge(const float* cand_scores, const int32_t* cand_idx, int rows, int n_cand, int k,
                              int32_t* idx, float* top_scores, void* ws, cudaStream_t stream) {
    cudaError_t e = launch_topk(cand_scores, n_cand, n_cand, rows, k, idx, top_scores, ws, stream);
    if (e != cudaSuccess) return e;
    topk_map_positions<<<dim3((unsigned)((k + 255) / 256), (unsigned)rows), 256, 0, stream>>>(cand_idx, n_cand, k,
                                                                                             idx);
    return cudaGetLastError();
}

size_t topk_blocks_workspace_bytes(int rows) {
    return align256(sizeof(RowState) * rows) + align256(sizeof(uint64_t) * (size_t)rows * kCapB);
}

cudaError_t launch_topk_blocks_map(const float* scores, const uint32_t* bmax, const RowMap& map, int rows, int k,
                                   int32_t* idx, float* top_scores, void* ws, cudaStream_t stream, bool pdl) {
    // The bound m is tight only when a row has many more blocks than k: with
    // at least 8k blocks, m lies in the top eighth of the block maxima and the
    // surviving blocks hold about k candidates.  Shorter rows take the
    // histogram path over the whole row.
    if (map.max_n <= kRowsMax && k <= kMaxTopK)
        return launch_topk_rows(scores, map, rows, k, idx, top_scores, stream, pdl);
    int64_t min_n = map.max_n;
    for (int s = 0; s < map.nsets; ++s) min_n = map.n[s] < min_n ? map.n[s] : min_n;
    // rows of at least k blocks and at most kMaxCluster * kSliceKeys blocks:
    // the one-kernel cluster path over the block maxima
    if (k <= kMaxTopK && (min_n + kBlock - 1) / kBlock >= k &&
        (map.max_n + kBlock - 1) / kBlock <= (int64_t)kMaxCluster * kSliceKeys)
        return launch_topk_bmax_rows_cl<kMaxCluster>(scores, bmax, map, rows, k, idx, top_scores, stream, pdl);
    if (min_n / kBlock < 8 * (int64_t)k) return launch_topk_map(scores, map, rows, k, idx, top_scores, ws, stream);
    BlkWs w = carve_blk(ws, rows);
    const size_t smem = sizeof(uint64_t) * kSortMax;
    cudaError_t e = cudaFuncSetAttribute(topk_blk_finish, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    // the second and third launches follow the path's own kernels
    e = launch_ex(topk_blk_threshold, dim3((unsigned)rows), dim3(kFinishThreads), 0, stream, pdl, 1, bmax, map, k, w);
    if (e != cudaSuccess) return e;
    const int64_t nbk = (map.max_n + kBlock - 1) / kBlock;
    e = launch_ex(topk_blk_compact, dim3((unsigned)((nbk + kPassThreads - 1) / kPassThreads), (unsigned)rows),
                  dim3(kPassThreads), 0, stream, true, 1, scores, bmax, map, w);
    if (e != cudaSuccess) return e;
    return launch_ex(topk_blk_finish, dim3((unsigned)rows), dim3(kFinishThreads), smem, stream, true, 1, scores, map, k,
                     w, idx, top_scores);
}

cudaError_t launch_topk_blocks(const float* scores, const uint32_t* bmax, int64_t n, int64_t ld, int rows, int k,
                               int32_t* idx, float* top_scores, void* ws, cudaStream_t stream, bool pdl) {
    RowMap m;
    m.rows_per_set = rows;
    m.nsets = 1;
    m.max_n = n;
    m.base[0] = 0;
    m.ld[0] = ld;
    m.n[0] = n;
    return launch_topk_blocks_map(scores, bmax, m, rows, k, idx, top_scores, ws, stream, pdl);
}

size_t topk_workspace_bytes(int64_t n, int rows, int k) {
    (void)n;
    return align256(sizeof(RowState) * rows) + align256(sizeof(int) * 4) +
           align256(sizeof(uint32_t) * 3 * (size_t)rows * kBins) +
           align256(sizeof(uint64_t) * (size_t)rows * k) + align256(sizeof(uint64_t) * (size_t)rows * kCap);
}

cudaError_t launch_topk_map(const float* scores, const RowMap& map, int rows, int k, int32_t* idx,
                            float* top_scores, void* ws, cudaStream_t stream) {
    if (map.max_n <= kRowsMax && k <= kMaxTopK)
        return launch_topk_rows(scores, map, rows, k, idx, top_scores, stream);
    Workspace w = carve(ws, rows, k);
    unsigned int* status = device_status_ptr();
    const unsigned chunks = (unsigned)((map.max_n + kChunk - 1) / kChunk);
    topk_init<<<rows, 256, 0, stream>>>(w, map, rows);
    topk_hist<<<dim3(chunks, rows), kPassThreads, 0, stream>>>(scores, map, rows, w);
    topk_select<<<rows, 1024, 0, stream>>>(w, rows, k, 0);
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const long long items = (long long)chunks * rows;
    const unsigned refine_grid = (unsigned)(items < 4LL * sms ? items : 4LL * sms);
    for (int level = 1; level < 3; ++level) {
        topk_hist_refine<<<refine_grid, kPassThreads, 0, stream>>>(scores, map, rows, (int)chunks, w, level);
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
