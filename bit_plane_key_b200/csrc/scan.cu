// K3: variable-depth scan over the bit-plane store.
//
// For query head h (KV head g = h / G) and key i in 64-token block b:
//   s[h][i] = sum_c q[h][c] * Delta[b][c] * sum_{j < t[h][c]} (2 b_{i,c,j} - 1) 2^(2-j)
// i.e. every channel contributes its t-bit mid-rise value rebuilt from the
// first t planes (basis rule; ai-feeds.com summary, 方法 · 关键模块 4, paper
// Sec 3.5; a t-plane prefix is exactly the t-bit quantizer: arXiv abstract,
// evolve.pub review Strengths, paper Sec 3.2).  The scan reads only the first
// U_c = max_{h in group} t[h][c] planes of each channel (ai-feeds.com summary,
// 关键模块 5: only the budgeted planes are pulled); channels nobody reads are
// never touched, nor are their scales.
//
// Arithmetic.  Let code be the channel's 4-bit code with the unread planes
// as zero bits and P_t = code with its low 4-t bits cleared (the t-bit prefix
// in place).  With F_t = 1/2 (1 + P_t/16), an fp32 number whose mantissa bits
// 22..19 are exactly P_t,
//   v_t = 2^(3-t)(2m + 1) - 8 = 32 F_t - 24 + 2^(3-t),
// so a (channel, head) pair adds (32 q Delta) F_t per key, and
// Delta q (2^(3-t) - 24) per (block, head) once.
//
// Work.  One CTA per (tile of 1024 keys, KV head).  A channel's codes in a
// tile are 8 x 32 words: word (s, w) holds the codes of keys 32w + s + 8k,
// k = 0..3, one per byte at bits 6..3.  The tile's active channels
// (U_c > 0) are streamed in chunks of 16:
//   stage: thread (channel group, plane word w) loads the U_c plane words of
//     its channels (row pointers prepared once per tile) and transposes them
//     to the 8 code words (s, w) (planes paired, then merged to nibbles, one
//     rotate + mask per word), stored with conflict-free 32-bit stores.  Thread (channel, block) pairs form
//     the coefficients 32 q Delta of every head and add Delta q (2^(3-t) - 24)
//     into a per-(block, head) constant kept in registers.
//   compute: warp (head h, key split) walks head h's item list of the chunk:
//     the channels h reads, first those read to the union depth, then those
//     read to fewer planes (their code bytes masked to t planes).  Lane
//     (block b, variant half) owns 32 / S keys of block b: per item one
//     coefficient load, 64-bit loads of its code words, and per key one byte
//     permute building F and one FMA.  No per-head branch, no unread channel.
//   The next chunk's plane words and scales are loaded into registers before
//   the current chunk is computed, so the loads overlap the arithmetic.
// The same kernel serves a host-resident store: its loads then cross the host
// link as 128-byte runs per (channel, plane) and tile.
#include "fathom_internal.cuh"

namespace fathom {
namespace {

constexpr int kTileKeys = 1024;
constexpr int kTileWords = kTileKeys / 32;   // 32 plane words per tile row
constexpr int kTileBlocks = kTileKeys / kBlock;
constexpr int kChanWords = 8 * kTileWords;   // code words of one channel in a tile
constexpr int kChunk = 16;                   // active channels per stage
constexpr uint32_t kHalfExp = 0x3F000000u;   // bits of 0.5f: exponent byte of F

// Launch geometry for G query heads per KV head.
template <int G>
struct Geo {
    static constexpr int S = G >= 4 ? 1 : 4 / G;    // warps per query head (key splits)
    static constexpr int NW = G * S;                // warps per CTA
    static constexpr int T = 32 * NW;               // threads per CTA
    static constexpr int NSV = 4 / S;               // code variants per compute thread
    static constexpr int CPT = kChunk / NW;         // staged channels per thread
    static constexpr int DPT = kChunk * kTileBlocks / T;   // staged (channel, block) scales per thread
    static constexpr int MinBlocks = T <= 128 ? 4 : 2;
    static_assert(CPT >= 1 && DPT >= 1 && NSV >= 1, "geometry");
};

// Shared memory of one CTA (byte offsets; every region 16-byte aligned for d % 32 == 0).
struct ScanSmem {
    int d, G;
    __host__ __device__ size_t codes() const { return 0; }   // [2][kChunk][8][32] u32
    __host__ __device__ size_t coef() const { return codes() + 2u * kChunk * kChanWords * 4; }   // [2][G][kChunk][16] f32
    __host__ __device__ size_t prow() const { return coef() + 2u * G * kChunk * kTileBlocks * 4; }   // [d] plane-0 row ptr
    __host__ __device__ size_t srow() const { return prow() + (size_t)d * 8; }      // [d] scale row ptr
    __host__ __device__ size_t items() const { return srow() + (size_t)d * 8; }     // [G][d] u32
    __host__ __device__ size_t q32() const { return items() + (size_t)G * d * 4; }   // [d][G] f32
    __host__ __device__ size_t qk() const { return q32() + (size_t)G * d * 4; }      // [d][G] f32
    __host__ __device__ size_t off() const { return qk() + (size_t)G * d * 4; }      // [G][d/8 + 4] i32
    __host__ __device__ size_t act() const { return off() + (size_t)G * (d / 8 + 4) * 4; }   // [d] i32
    __host__ __device__ size_t uni() const { return act() + (size_t)d * 4; }         // [d] u8
    __host__ __device__ size_t tdep() const { return uni() + (size_t)d; }            // [G][d] u8
    __host__ __device__ size_t bytes() const { return (tdep() + (size_t)G * d + 15) & ~size_t(15); }
};

__device__ __forceinline__ uint32_t rotr(uint32_t x, int sft) { return __funnelshift_r(x, x, (uint32_t)sft & 31u); }

// The 8 code words of 32 keys of one channel from its first U plane words p
// (p[j] = 0 for j >= U): word sv holds keys sv + 8k, k = 0..3, plane j of key
// sv + 8k at bit 8k + 6 - j.  Planes are first paired, and for U >= 3 the two
// pairs merged into nibbles (key 4m + c in nibble m of a word per class c),
// so that one rotate and one mask place several planes at once.
__device__ __forceinline__ void codes_of(const uint32_t (&p)[4], int U, uint32_t (&x)[8]) {
    if (U >= 2) {
        // even keys 2m: bit 2m = plane 1, bit 2m+1 = plane 0; odd keys 2m+1 likewise
        const uint32_t e01 = (p[1] & 0x55555555u) | ((p[0] << 1) & 0xAAAAAAAAu);
        const uint32_t o01 = ((p[1] >> 1) & 0x55555555u) | (p[0] & 0xAAAAAAAAu);
        if (U == 2) {
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                x[2 * r] = rotr(e01, 2 * r - 5) & 0x60606060u;
                x[2 * r + 1] = rotr(o01, 2 * r - 5) & 0x60606060u;
            }
        } else {
            const uint32_t e23 = (p[3] & 0x55555555u) | ((p[2] << 1) & 0xAAAAAAAAu);
            const uint32_t o23 = ((p[3] >> 1) & 0x55555555u) | (p[2] & 0xAAAAAAAAu);
            // key 4m + c: nibble m of q[c], planes 3..0 in its bits 0..3
            const uint32_t q[4] = {(e23 & 0x33333333u) | ((e01 << 2) & 0xCCCCCCCCu),
                                   (o23 & 0x33333333u) | ((o01 << 2) & 0xCCCCCCCCu),
                                   ((e23 >> 2) & 0x33333333u) | (e01 & 0xCCCCCCCCu),
                                   ((o23 >> 2) & 0x33333333u) | (o01 & 0xCCCCCCCCu)};
#pragma unroll
            for (int sv = 0; sv < 8; ++sv) x[sv] = rotr(q[sv & 3], 4 * (sv >> 2) - 3) & 0x78787878u;
        }
    } else {
#pragma unroll
        for (int sv = 0; sv < 8; ++sv) x[sv] = (U == 1) ? (rotr(p[0], sv - 6) & 0x40404040u) : 0u;
    }
}

// F of byte k of a code word (he = kHalfExp)
__device__ __forceinline__ float f_of(uint32_t x, uint32_t he, uint32_t k) {
    return __uint_as_float(__byte_perm(x, he, 0x7044u | (k << 8)));
}

// G consecutive floats of shared memory (16-byte aligned when G >= 4)
template <int G>
__device__ __forceinline__ void load_g(const float* p, float (&v)[G]) {
    if constexpr (G % 4 == 0) {
#pragma unroll
        for (int i = 0; i < G; i += 4) {
            const float4 t = *reinterpret_cast<const float4*>(p + i);
            v[i] = t.x; v[i + 1] = t.y; v[i + 2] = t.z; v[i + 3] = t.w;
        }
    } else {
#pragma unroll
        for (int i = 0; i < G; ++i) v[i] = p[i];
    }
}

// One (tile of 1024 keys, KV head g) of one store; q, depths and scores are
// the store's own [Hq][d], [Hq][d] and [Hq][n_pad_of(n)] arrays; n_pad is the
// store's row stride (its capacity, >= n_pad_of(n)).
template <int G>
__device__ __forceinline__ void scan_tile(const uint32_t* __restrict__ planes, const uint16_t* __restrict__ scales,
                                          int d, int64_t n, int64_t n_pad, int tile, int g,
                                          const void* __restrict__ q, int q_dtype,
                                          const uint8_t* __restrict__ depths, float* __restrict__ scores,
                                          uint32_t* __restrict__ bmax, unsigned int* status) {
    using Z = Geo<G>;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const ScanSmem lay{d, G};
    uint32_t* s_codes = reinterpret_cast<uint32_t*>(smem_raw + lay.codes());
    float* s_coef = reinterpret_cast<float*>(smem_raw + lay.coef());
    const uint32_t** s_prow = reinterpret_cast<const uint32_t**>(smem_raw + lay.prow());
    const uint16_t** s_srow = reinterpret_cast<const uint16_t**>(smem_raw + lay.srow());
    uint32_t* s_items = reinterpret_cast<uint32_t*>(smem_raw + lay.items());
    float* s_q32 = reinterpret_cast<float*>(smem_raw + lay.q32());
    float* s_qk = reinterpret_cast<float*>(smem_raw + lay.qk());
    int* s_off = reinterpret_cast<int*>(smem_raw + lay.off());
    int* s_act = reinterpret_cast<int*>(smem_raw + lay.act());
    uint8_t* s_U = smem_raw + lay.uni();
    uint8_t* s_t = smem_raw + lay.tdep();
    __shared__ int s_L;
    __shared__ uint32_t s_bmax[8 * kTileBlocks];   // per (head, block) max score as an ordered key; G <= 8
    const int off_stride = d / 8 + 4;

    const int64_t tile0 = (int64_t)tile * kTileKeys;
    const int64_t words_total = n_pad / 32;
    const int64_t nblk_total = n_pad / kBlock;
    const int64_t wrem = words_total - tile0 / 32;
    const int nwords = wrem < kTileWords ? (int)wrem : kTileWords;   // multiple of 4
    const int nblocks = nwords / 2;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    // ---- plan: depths, union list, row pointers, per-head item lists, per-(channel, head) factors ----
    for (int e = tid; e < G * kTileBlocks; e += Z::T) s_bmax[e] = 0u;   // below every ordered key
    for (int e = tid; e < G * d; e += Z::T) {
        int t = depths[(int64_t)g * G * d + e];
        if (t > 4) {
            atomicOr(status, (unsigned)FATHOM_DEV_BAD_DEPTH);
            t = 0;
        }
        s_t[e] = (uint8_t)t;
    }
    __syncthreads();
    if (warp == 0) {
        int base = 0;
        for (int c0 = 0; c0 < d; c0 += 32) {
            const int c = c0 + lane;
            int U = 0;
#pragma unroll
            for (int hh = 0; hh < G; ++hh) U = max(U, (int)s_t[hh * d + c]);
            const unsigned m = __ballot_sync(0xffffffffu, U > 0);
            if (U > 0) {
                const int pos = base + __popc(m & ((1u << lane) - 1u));
                s_act[pos] = c;
                s_U[pos] = (uint8_t)U;
            }
            base += __popc(m);
        }
        if (lane == 0) s_L = base;
    }
    __syncthreads();
    const int L = s_L;
    const int nchunks = (L + kChunk - 1) / kChunk;
    for (int a = tid; a < nchunks * kChunk; a += Z::T) {   // slots past the list: nothing to read
        const bool live = a < L;
        const int64_t row = (int64_t)g * d + (live ? s_act[a] : 0);
        s_prow[a] = planes + row * 4 * words_total + tile0 / 32;
        s_srow[a] = scales + row * nblk_total + tile0 / kBlock;
        if (!live) s_U[a] = 0;
    }
    for (int e = tid; e < L * G; e += Z::T) {
        const int a = e / G, hh = e - a * G;
        const int c = s_act[a];
        const int t = s_t[hh * d + c];
        const float qv = load_q(q, q_dtype, ((int64_t)g * G + hh) * d + c);
        s_q32[e] = (t > 0) ? 32.0f * qv : 0.0f;
        s_qk[e] = (t > 0) ? qv * (__uint_as_float((uint32_t)(130 - t) << 23) - 24.0f) : 0.0f;
    }
    for (int e = L * G + tid; e < nchunks * kChunk * G; e += Z::T) {   // the last chunk's unused slots
        s_q32[e] = 0.0f;
        s_qk[e] = 0.0f;
    }
    if (warp < G) {
        // item list of head h = warp, chunk by chunk: channels read to the
        // union depth, then channels read to fewer planes.  An item holds the
        // word offset of the channel's codes in a chunk buffer (slot *
        // kChanWords, bits 0..11) and, for a shallower read, the byte mask
        // (bits 16..23)
        const int h = warp;
        uint32_t* items = s_items + h * d;
        int* off = s_off + h * off_stride;
        int base = 0;
        for (int a0 = 0; a0 < L; a0 += 32) {
            const int a = a0 + lane;
            const int t = (a < L) ? (int)s_t[h * d + s_act[a]] : 0;
            const int U = (a < L) ? (int)s_U[a] : 0;
            const bool full = t > 0 && t == U, part = t > 0 && t < U;
            const unsigned mf = __ballot_sync(0xffffffffu, full);
            const unsigned mp = __ballot_sync(0xffffffffu, part);
            const int nf0 = __popc(mf & 0xFFFFu), np0 = __popc(mp & 0xFFFFu);
            const int nf1 = __popc(mf >> 16), np1 = __popc(mp >> 16);
            const int start0 = base, start1 = base + nf0 + np0;
            const bool upper = lane >= 16;
            const unsigned below = ((1u << lane) - 1u) & (upper ? 0xFFFF0000u : 0x0000FFFFu);
            const int cstart = upper ? start1 : start0, cnf = upper ? nf1 : nf0;
            const uint32_t slot = (uint32_t)(a & 15) * kChanWords;
            if (full) items[cstart + __popc(mf & below)] = slot;
            if (part) items[cstart + cnf + __popc(mp & below)] = slot | (((0x780u >> t) & 0x78u) << 16);
            if (lane == 0) {
                const int ch = a0 / 16;
                off[2 * ch] = start0;
                off[2 * ch + 1] = start0 + nf0;
                off[2 * ch + 2] = start1;
                off[2 * ch + 3] = start1 + nf1;
            }
            base = start1 + nf1 + np1;
        }
        if (lane == 0) off[2 * nchunks] = base;
    }
    __syncthreads();

    // ---- stage role: channels cg*CPT + i of a chunk at plane word w; scales (al, bb) ----
    const int cg = warp, w = lane;
    const bool wok = w < nwords;
    const int bb = tid & 15;   // block of this thread's scales (the same for every u: T is a multiple of 16)
    uint32_t pw[Z::CPT][4];
    float pd[Z::DPT];
    float cstp[G];
#pragma unroll
    for (int hh = 0; hh < G; ++hh) cstp[hh] = 0.0f;

    auto load_chunk = [&](int ch) {
#pragma unroll
        for (int i = 0; i < Z::CPT; ++i) {
            const int a = ch * kChunk + cg * Z::CPT + i;   // warp-uniform
            const int U = wok ? s_U[a] : 0;
            const uint32_t* p = s_prow[a] + w;
#pragma unroll
            for (int j = 0; j < 4; ++j) pw[i][j] = (j < U) ? __ldg(p + j * words_total) : 0u;
        }
#pragma unroll
        for (int u = 0; u < Z::DPT; ++u) {
            const int a = ch * kChunk + ((tid + u * Z::T) >> 4);
            pd[u] = (a < L && bb < nblocks) ? __half2float(__ushort_as_half(__ldg(s_srow[a] + bb))) : 0.0f;
        }
    };
    auto store_chunk = [&](int ch, int buf) {
        uint32_t* cbase = s_codes + (size_t)buf * kChunk * kChanWords + w;
#pragma unroll
        for (int i = 0; i < Z::CPT; ++i) {
            const int al = cg * Z::CPT + i, a = ch * kChunk + al;
            const int U = s_U[a];   // warp-uniform; 0 past the list
            uint32_t x[8];
            codes_of(pw[i], U, x);
#pragma unroll
            for (int sv = 0; sv < 8; ++sv) cbase[al * kChanWords + sv * kTileWords] = x[sv];
        }
        float* cf = s_coef + (size_t)buf * G * kChunk * kTileBlocks;
#pragma unroll
        for (int u = 0; u < Z::DPT; ++u) {
            const int al = (tid + u * Z::T) >> 4, a = ch * kChunk + al;   // a < d: nchunks * 16 <= d
            float qv[G], kv[G];
            load_g<G>(s_q32 + a * G, qv);   // zero past the union list
            load_g<G>(s_qk + a * G, kv);
#pragma unroll
            for (int hh = 0; hh < G; ++hh) {
                cf[(hh * kChunk + al) * kTileBlocks + bb] = qv[hh] * pd[u];
                cstp[hh] = fmaf(kv[hh], pd[u], cstp[hh]);
            }
        }
    };

    // ---- compute role: head h; lane (block b, variant half) ----
    const int h = warp / Z::S, sp = warp % Z::S;
    const int b = lane & 15, sv0 = Z::NSV * (2 * sp + (lane >> 4));
    // key of acc[i][wd][k]: 64 b + 32 wd + sv0 + i + 8 k
    float acc[Z::NSV][2][4];
#pragma unroll
    for (int i = 0; i < Z::NSV; ++i)
#pragma unroll
        for (int k = 0; k < 4; ++k) acc[i][0][k] = acc[i][1][k] = 0.0f;
    const uint32_t he = kHalfExp;
    const uint32_t* cth = s_codes + sv0 * kTileWords + 2 * b;                  // + buffer + slot + i * 32
    const float* cfth = s_coef + (size_t)h * kChunk * kTileBlocks + b;         // + buffer + slot * 16

    auto item = [&](const uint32_t* cb, const float* cfb, uint32_t it, bool masked) {
        const uint32_t slot = it & 0xFFFu;
        const uint32_t* rp = cb + slot;
        const float c = cfb[slot >> 4];                       // slot / kChanWords * kTileBlocks
        const uint32_t mk = __byte_perm(it, 0u, 0x2222u);     // byte 2 in all four bytes
#pragma unroll
        for (int i = 0; i < Z::NSV; ++i) {
            const uint2 X = *reinterpret_cast<const uint2*>(rp + i * kTileWords);
            const uint32_t x0 = masked ? (X.x & mk) : X.x, x1 = masked ? (X.y & mk) : X.y;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                acc[i][0][k] = fmaf(c, f_of(x0, he, (uint32_t)k), acc[i][0][k]);
                acc[i][1][k] = fmaf(c, f_of(x1, he, (uint32_t)k), acc[i][1][k]);
            }
        }
    };

    if (nchunks > 0) {
        load_chunk(0);
        store_chunk(0, 0);
    }
    __syncthreads();
    const uint32_t* items = s_items + h * d;
    const int* off = s_off + h * off_stride;
    for (int ch = 0; ch < nchunks; ++ch) {
        const int buf = ch & 1;
        if (ch + 1 < nchunks) load_chunk(ch + 1);
        const uint32_t* cb = cth + (size_t)buf * kChunk * kChanWords;
        const float* cfb = cfth + (size_t)buf * G * kChunk * kTileBlocks;
        const int f0 = off[2 * ch], p0 = off[2 * ch + 1], e0 = off[2 * ch + 2];
        for (int k = f0; k < p0; ++k) item(cb, cfb, items[k], false);
        for (int k = p0; k < e0; ++k) item(cb, cfb, items[k], true);
        if (ch + 1 < nchunks) store_chunk(ch + 1, buf ^ 1);
        __syncthreads();
    }

    // ---- constants: the per-thread partials of each (block, head), summed in a fixed order ----
    float* s_cred = reinterpret_cast<float*>(smem_raw + lay.codes());   // [NW][16][G]; the codes are dead now
    float* s_cst = s_cred + Z::NW * 16 * G;                              // [G][16]
#pragma unroll
    for (int hh = 0; hh < G; ++hh) {
        const float v = cstp[hh] + __shfl_xor_sync(0xffffffffu, cstp[hh], 16);
        if (lane < 16) s_cred[(warp * 16 + lane) * G + hh] = v;
    }
    __syncthreads();
    if (tid < 16 * G) {
        const int hh = tid >> 4, b16 = tid & 15;
        float v = 0.0f;
        for (int wv = 0; wv < Z::NW; ++wv) v += s_cred[(wv * 16 + b16) * G + hh];
        s_cst[hh * 16 + b16] = v;
    }
    __syncthreads();

    // ---- epilogue ----
    if (b < nblocks) {
        const int64_t k0 = tile0 + 64 * b + sv0;   // key of acc[0][0][0]
        float* out = scores + ((int64_t)g * G + h) * n_pad_of(n) + k0;
        const float cst = s_cst[h * 16 + b];
        const bool whole = tile0 + kTileKeys <= n;
        uint32_t kmax = 0u;
#pragma unroll
        for (int i = 0; i < Z::NSV; ++i)
#pragma unroll
            for (int wd = 0; wd < 2; ++wd)
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int o = 32 * wd + i + 8 * k;
                    const float v = (whole || k0 + o < n) ? acc[i][wd][k] + cst : -INFINITY;
                    out[o] = v;
                    kmax = max(kmax, float_to_ordered(v));
                }
        atomicMax(&s_bmax[h * kTileBlocks + b], kmax);
    }
    // the maximum of every 64-key block, for the top-k that reads only the
    // blocks that can hold a selected key
    __syncthreads();
    if (bmax && tid < G * kTileBlocks) {
        const int hh = tid / kTileBlocks, bb = tid % kTileBlocks;
        bmax[((int64_t)g * G + hh) * (n_pad_of(n) / kBlock) + tile0 / kBlock + bb] = s_bmax[tid];
    }
}

template <int G>
__global__ void __launch_bounds__(Geo<G>::T, Geo<G>::MinBlocks)
scan_kernel(const uint32_t* __restrict__ planes, const uint16_t* __restrict__ scales, int d, int64_t n,
            int64_t n_pad, const void* __restrict__ q, int q_dtype, const uint8_t* __restrict__ depths,
            float* __restrict__ scores, uint32_t* __restrict__ bmax, unsigned int* status) {
    scan_tile<G>(planes, scales, d, n, n_pad, (int)blockIdx.x, (int)blockIdx.y, q, q_dtype, depths, scores, bmax,
                 status);
}

// Batched sessions: blockIdx.x runs over the tiles of all sessions.
template <int G>
__global__ void __launch_bounds__(Geo<G>::T, Geo<G>::MinBlocks)
scan_batched_kernel(const __grid_constant__ SessionMap map, int d, int Hq, const void* __restrict__ q, int q_dtype,
                    const uint8_t* __restrict__ depths, float* __restrict__ scores, uint32_t* __restrict__ bmax,
                    unsigned int* status) {
    const int t = (int)blockIdx.x;
    int lo = 0, hi = map.nsess - 1;   // last session with tile0 <= t
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (map.tile0[mid] <= t) lo = mid;
        else hi = mid - 1;
    }
    const int sidx = lo;
    const size_t qstride = (size_t)Hq * d;
    const void* qs = (q_dtype == FATHOM_BF16)
                         ? static_cast<const void*>(static_cast<const uint16_t*>(q) + sidx * qstride)
                         : static_cast<const void*>(static_cast<const float*>(q) + sidx * qstride);
    scan_tile<G>(map.planes[sidx], map.scales[sidx], d, map.n[sidx], map.n_pad[sidx], t - map.tile0[sidx],
                 (int)blockIdx.y, qs, q_dtype, depths + sidx * qstride, scores + map.score_base[sidx],
                 bmax ? bmax + map.score_base[sidx] / kBlock : nullptr, status);
}

template <int G>
cudaError_t launch_scan_g(const uint32_t* planes, const uint16_t* scales, int Hkv, int d, int64_t n,
                          int64_t n_pad, const void* q, int q_dtype, const uint8_t* depths, float* scores,
                          uint32_t* bmax, cudaStream_t stream) {
    const size_t smem = ScanSmem{d, G}.bytes();
    auto kern = scan_kernel<G>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)(n_pad_of(n) / kTileKeys), (unsigned)Hkv);   // the tiles holding keys; n_pad is the stride
    kern<<<grid, Geo<G>::T, smem, stream>>>(planes, scales, d, n, n_pad, q, q_dtype, depths, scores, bmax,
                                            device_status_ptr());
    return cudaGetLastError();
}

template <int G>
cudaError_t launch_scan_batched_g(const SessionMap& map, int Hkv, int d, const void* q, int q_dtype,
                                  const uint8_t* depths, int Hq, float* scores, uint32_t* bmax, cudaStream_t stream) {
    const size_t smem = ScanSmem{d, G}.bytes();
    auto kern = scan_batched_kernel<G>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)map.tile0[map.nsess], (unsigned)Hkv);
    kern<<<grid, Geo<G>::T, smem, stream>>>(map, d, Hq, q, q_dtype, depths, scores, bmax, device_status_ptr());
    return cudaGetLastError();
}

}  // namespace

size_t scan_smem_bytes(int d, int G) { return ScanSmem{d, G}.bytes(); }

cudaError_t launch_scan(const uint32_t* planes, const uint16_t* scales, int Hkv, int d, int64_t n, int64_t n_pad,
                        const void* q, int q_dtype, const uint8_t* depths, int Hq, float* scores,
                        cudaStream_t stream, uint32_t* bmax) {
    switch (Hq / Hkv) {
        case 1: return launch_scan_g<1>(planes, scales, Hkv, d, n, n_pad, q, q_dtype, depths, scores, bmax, stream);
        case 2: return launch_scan_g<2>(planes, scales, Hkv, d, n, n_pad, q, q_dtype, depths, scores, bmax, stream);
        case 4: return launch_scan_g<4>(planes, scales, Hkv, d, n, n_pad, q, q_dtype, depths, scores, bmax, stream);
        case 8: return launch_scan_g<8>(planes, scales, Hkv, d, n, n_pad, q, q_dtype, depths, scores, bmax, stream);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_scan_batched(const SessionMap& map, int Hkv, int d, const void* q, int q_dtype,
                                const uint8_t* depths, int Hq, float* scores, cudaStream_t stream, uint32_t* bmax) {
    switch (Hq / Hkv) {
        case 1: return launch_scan_batched_g<1>(map, Hkv, d, q, q_dtype, depths, Hq, scores, bmax, stream);
        case 2: return launch_scan_batched_g<2>(map, Hkv, d, q, q_dtype, depths, Hq, scores, bmax, stream);
        case 4: return launch_scan_batched_g<4>(map, Hkv, d, q, q_dtype, depths, Hq, scores, bmax, stream);
        case 8: return launch_scan_batched_g<8>(map, Hkv, d, q, q_dtype, depths, Hq, scores, bmax, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace fathom
