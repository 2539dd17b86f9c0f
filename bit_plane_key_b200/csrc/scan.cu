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
// Arithmetic.  Let P_t be the channel's 4-bit code with its low 4-t bits
// cleared (the t-bit prefix in place).  With F_t = 1/2 (1 + P_t/16), an fp32
// number whose mantissa bits 22..19 are exactly P_t,
//   v_t = 2^(3-t)(2m + 1) - 8 = 32 F_t - 24 + 2^(3-t),
// so a (channel, head) pair adds W F_t per key with W = 32 q Delta, and
// Delta q (2^(3-t) - 24) per (block, head) once.  One byte permute builds F_t
// from a code byte; W F_t products are exact in fp32 for bf16 q.
//
// Work.  One CTA per (tile of 2048 keys, KV head); the G query heads of the
// KV head form groups of up to 4 heads, and each group has 128 threads.  A
// thread owns 16 keys of one 64-key block (4 threads per block) and the
// accumulators of every head of its group, so a code value F_t is built once
// per key and shared by all heads of the group that read the channel to depth
// t.  The tile's active channels (U_c > 0) are streamed in chunks of 8:
//   load:  the chunk's U_c plane rows (256 bytes each in the tile) and scale
//          rows go to shared memory one chunk ahead of use: by cp.async from a
//          device-resident store; by 16-byte loads held in registers until
//          the current chunk is computed from a host-resident one (over the
//          host link each warp's loads are then runs of whole lines);
//   stage: thread (channel, block) transposes its 2 x U_c plane words into 16
//          code words (4 keys each, code at bits 6..3 of a byte) with a few
//          shifts and masks; thread (block, head) forms the head's
//          coefficients W (stored twice, for paired FMAs) of every channel of
//          the chunk and adds Delta q (2^(3-t) - 24) to the block's constant;
//   compute: the group's items, one per (channel, distinct depth), in channel
//          order: per item one 128-bit load of the thread's 16 code bytes,
//          masked to the item's depth, 16 byte permutes, and for each head
//          that reads the channel to that depth (a uniform branch) 8 paired
//          FMAs (fma.rn.f32x2) over 2 keys each.
#include "fathom_internal.cuh"

namespace fathom {
namespace {

constexpr int kTile = kScanTile;             // keys per CTA
constexpr int kNB = kTile / kBlock;          // 64-key blocks per tile
constexpr int kTW = kTile / 32;              // plane words per row in a tile
constexpr int kCH = 8;                       // active channels per chunk
constexpr int kMaxItems = 4 * kCH;           // items per (head group, chunk)
constexpr uint32_t kHalfExp = 0x3F000000u;   // bits of 0.5f: exponent byte of F

// Launch geometry for G query heads per KV head.
template <int G>
struct Geo {
    static constexpr int HG = G < 4 ? G : 4;   // heads per head group
    static constexpr int NHG = G / HG;         // head groups
    static constexpr int TPG = kNB * 4;        // threads per head group (4 per block)
    static constexpr int T = TPG * NHG;        // threads per CTA
    // host-resident stores hold the next chunk's rows in registers (see scan_tile)
    template <bool HOST>
    static constexpr int min_blocks() { return HOST ? (T <= 128 ? 3 : 1) : (T <= 128 ? 4 : 2); }
};

// Shared memory of one CTA (byte offsets; every region 16-byte aligned).
struct ScanSmem {
    int d, G;
    __host__ __device__ int hg() const { return G < 4 ? G : 4; }
    __host__ __device__ int nhg() const { return G / hg(); }
    __host__ __device__ int maxchunks() const { return (d + kCH - 1) / kCH; }
    __host__ __device__ size_t raw() const { return 0; }                                   // [2][kCH][4][kTW] u32
    __host__ __device__ size_t rawsc() const { return raw() + 2u * kCH * 4 * kTW * 4; }    // [2][kCH][kNB] u16
    __host__ __device__ size_t codes() const { return rawsc() + 2u * kCH * kNB * 2; }      // [kCH][kNB][8][2] u32
    __host__ __device__ size_t w2() const { return codes() + (size_t)kCH * kNB * 16 * 4; } // [nhg][kCH][kNB][hg][2] f32
    __host__ __device__ size_t qq() const { return w2() + (size_t)nhg() * kCH * kNB * hg() * 8; }   // [d][G] (32q, qk) f32x2
    __host__ __device__ size_t prow() const { return qq() + (size_t)d * G * 8; }          // [d] plane-0 row of the tile
    __host__ __device__ size_t srow() const { return prow() + (size_t)d * 8; }           // [d] scale row of the tile
    __host__ __device__ size_t items() const { return srow() + (size_t)d * 8; }          // [nhg*maxchunks][kMaxItems] u32
    __host__ __device__ size_t act() const { return items() + (size_t)nhg() * maxchunks() * kMaxItems * 4; }   // [d] i32
    __host__ __device__ size_t nitems() const { return act() + (size_t)d * 4; }            // [nhg*maxchunks] u8
    __host__ __device__ size_t uni() const { return nitems() + (size_t)nhg() * maxchunks(); }   // [d] u8
    __host__ __device__ size_t tdep() const { return uni() + (size_t)d; }                  // [G][d] u8
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

// F of byte k of a code word
__device__ __forceinline__ float f_of(uint32_t x, uint32_t k) {
    return __uint_as_float(__byte_perm(x, kHalfExp, 0x7044u | (k << 8)));
}

// acc += w * f on both halves (one paired instruction: two correctly rounded FMAs)
__device__ __forceinline__ void ffma2(float2& acc, const float2& w, const float2& f) { acc = __ffma2_rn(w, f, acc); }

// Code words of (slot, block): 64 bytes, four 16-byte pieces; piece v sits at
// position v ^ swz(block), so that the 32 stores of a warp staging 32 blocks
// and the loads of a warp computing 8 blocks both hit every bank once.
__device__ __forceinline__ int swz(int block) { return (block >> 1) & 3; }

__device__ __forceinline__ uint4 ldg16(const void* p) { return __ldg(reinterpret_cast<const uint4*>(p)); }

__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gmem_src) {
    const unsigned s = (unsigned)__cvta_generic_to_shared(smem_dst);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(s), "l"(gmem_src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// One item for the thread's 16 keys: an item is a channel slot of the chunk,
// a depth t and the set M of the group's heads that read the slot's channel to
// exactly depth t (desc bits 0..2: slot, 4..7: M, 8..15: the byte mask of t
// planes).  The 16 code bytes X are masked to depth t, 16 byte permutes build
// F_t, and each head of M adds its coefficient pair times F with 8 paired
// FMAs.  acc[h][2w + r] holds keys (byte 2r, byte 2r + 1) of code word w.
template <int HG>
__device__ __forceinline__ void item_fma(uint32_t desc, uint4 X, const float* __restrict__ wth,
                                         float2 (&acc)[HG][8]) {
    constexpr int kSlotW = kNB * HG * 2;   // floats of one slot's coefficients
    const uint32_t bm = __byte_perm(desc, 0u, 0x1111u);   // byte 1 in all four bytes
    X.x &= bm;
    X.y &= bm;
    X.z &= bm;
    X.w &= bm;
    const uint32_t xs[4] = {X.x, X.y, X.z, X.w};
    float2 F[8];
#pragma unroll
    for (int w = 0; w < 4; ++w) {
        F[2 * w] = make_float2(f_of(xs[w], 0), f_of(xs[w], 1));
        F[2 * w + 1] = make_float2(f_of(xs[w], 2), f_of(xs[w], 3));
    }
    const float* wa = wth + (desc & 7) * kSlotW;
#pragma unroll
    for (int h = 0; h < HG; ++h) {
        if (desc & (16u << h)) {
            const float2 W = *reinterpret_cast<const float2*>(wa + 2 * h);
#pragma unroll
            for (int i = 0; i < 8; ++i) ffma2(acc[h][i], W, F[i]);
        }
    }
}

// The items of one (head group, chunk), two per turn: both items' words and
// code bytes are loaded before either is computed.  Every lane reads the same
// item words; a warp reduction of each gives the compiler values it knows to
// be warp-uniform, so the per-head tests are uniform branches.
template <int HG>
__device__ __forceinline__ void chunk_items(const uint32_t* __restrict__ items, int nit,
                                            const unsigned char* __restrict__ cth, const float* __restrict__ wth,
                                            float2 (&acc)[HG][8]) {
    constexpr int kSlotCode = kNB * 16 * 4;   // bytes of one slot's code words
#pragma unroll 1
    for (int it = 0; it < nit; it += 2) {
        const bool two = it + 1 < nit;
        const uint32_t d0 = __reduce_or_sync(0xffffffffu, items[it]);
        const uint32_t d1 = two ? __reduce_or_sync(0xffffffffu, items[it + 1]) : 0u;
        const uint4 X0 = *reinterpret_cast<const uint4*>(cth + (d0 & 7) * kSlotCode);
        const uint4 X1 = *reinterpret_cast<const uint4*>(cth + (d1 & 7) * kSlotCode);
        item_fma<HG>(d0, X0, wth, acc);
        if (two) item_fma<HG>(d1, X1, wth, acc);
    }
}

// The tiles tile_begin, tile_begin + tile_step, ... (below the store's tile
// count) of KV head g of one store: the plan (depths, union list, per-(slot,
// head) factors, items) is made once for the head, then every tile is loaded,
// staged and computed in turn.  The kernels give every CTA one tile.
template <int G, bool HOST>
__device__ __forceinline__ void scan_head_tiles(const uint32_t* __restrict__ planes, const uint16_t* __restrict__ scales,
                                           int d, int64_t n, int64_t n_pad, int tile_begin, int tile_step, int g,
                                          const void* __restrict__ q, int q_dtype,
                                          const uint8_t* __restrict__ depths, float* __restrict__ scores,
                                          uint32_t* __restrict__ bmax, unsigned int* status) {
    using Z = Geo<G>;
    constexpr int HG = Z::HG, NHG = Z::NHG, T = Z::T;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const ScanSmem lay{d, G};
    uint32_t* s_raw = reinterpret_cast<uint32_t*>(smem_raw + lay.raw());
    uint16_t* s_rawsc = reinterpret_cast<uint16_t*>(smem_raw + lay.rawsc());
    uint32_t* s_codes = reinterpret_cast<uint32_t*>(smem_raw + lay.codes());
    float* s_w2 = reinterpret_cast<float*>(smem_raw + lay.w2());
    float2* s_qq = reinterpret_cast<float2*>(smem_raw + lay.qq());
    const uint32_t** s_prow = reinterpret_cast<const uint32_t**>(smem_raw + lay.prow());
    const uint16_t** s_srow = reinterpret_cast<const uint16_t**>(smem_raw + lay.srow());
    uint32_t* s_items = reinterpret_cast<uint32_t*>(smem_raw + lay.items());
    int* s_act = reinterpret_cast<int*>(smem_raw + lay.act());
    uint8_t* s_nitems = smem_raw + lay.nitems();
    uint8_t* s_U = smem_raw + lay.uni();
    uint8_t* s_t = smem_raw + lay.tdep();
    __shared__ int s_L;

    const int64_t words_total = n_pad / 32;   // plane row stride
    const int64_t nblk_total = n_pad / kBlock;
    const int64_t len = n_pad_of(n);          // keys covered by tiles
    const int ntiles = (int)scan_tiles(n);
    // the current tile (set at the top of each tile's turn; the loaders read them)
    int64_t tile0 = 0;
    int keys_here = 0, nw = 0, nblocks = 0;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    // ---- plan: depths, union list, per-(slot, head) factors, item runs ----
    // the group's depths and queries are read together (the queries parked in
    // the chunk staging buffer, which the first chunk's loads overwrite only
    // after the plan)
    float* s_qraw = reinterpret_cast<float*>(s_raw);   // [G][d]
    for (int e = tid; e < G * d; e += T) {
        int t = depths[(int64_t)g * G * d + e];
        s_qraw[e] = load_q(q, q_dtype, (int64_t)g * G * d + e);
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
    const int L = (int)__reduce_or_sync(0xffffffffu, (unsigned)s_L);   // warp-uniform to the compiler
    const int nchunks = (L + kCH - 1) / kCH;
    for (int e = tid; e < L * G; e += T) {
        const int a = e / G, hh = e - a * G;
        const int c = s_act[a];
        const int t = s_t[hh * d + c];
        const float qv = s_qraw[hh * d + c];
        s_qq[e] = (t > 0) ? make_float2(32.0f * qv, qv * (__uint_as_float((uint32_t)(130 - t) << 23) - 24.0f))
                          : make_float2(0.0f, 0.0f);
    }
    // items of (head group, chunk): lane (slot, depth) -> an item when some head
    // of the group reads the slot's channel to exactly that depth; kept in
    // lane order (slot, then depth)
    for (int task = warp; task < NHG * nchunks; task += T / 32) {
        const int hg = task % NHG, ch = task / NHG;
        const int al = lane >> 2, tt = (lane & 3) + 1, a = ch * kCH + al;
        uint32_t m = 0;
        if (a < L) {
            const int c = s_act[a];
#pragma unroll
            for (int hh = 0; hh < HG; ++hh) m |= (uint32_t)(s_t[(hg * HG + hh) * d + c] == tt) << hh;
        }
        const unsigned v = __ballot_sync(0xffffffffu, m != 0);
        if (m) {
            const uint32_t bm = (0x780u >> tt) & 0x78u;   // the first tt of the code's bits 6..3
            s_items[task * kMaxItems + __popc(v & ((1u << lane) - 1u))] = (uint32_t)al | (m << 4) | (bm << 8);
        }
        if (lane == 0) s_nitems[task] = (uint8_t)__popc(v);
    }

    // ---- roles ----
    const int hg = tid / Z::TPG, lt = tid % Z::TPG;
    const int b = lt >> 2, p = lt & 3;   // compute / coefficient thread: block b, word pair p
    const unsigned char* cth = reinterpret_cast<const unsigned char*>(s_codes) + b * 64 + 16 * (p ^ swz(b));
    const float* wth = s_w2 + ((size_t)hg * kCH * kNB + b) * HG * 2;

    __syncthreads();   // plan complete

    // The rows of chunk ch in 16-byte pieces: thread tid copies piece lp of
    // plane lj of slots la0 + kSlotStep * i (i < kPlaneIters), and threads
    // tid < kScalePieces piece tid & 3 of the scale row of slot tid >> 2.
    constexpr int kRowPieces = kTW / 4;                          // 16-byte pieces of a tile's plane row
    constexpr int kPlaneIters = kCH * 4 * kRowPieces / T;        // plane pieces per thread
    constexpr int kSlotStep = T / (4 * kRowPieces);              // slots apart for one thread
    constexpr int kScalePieces = kCH * (kNB / 8);
    static_assert(kCH * 4 * kRowPieces % T == 0 && kScalePieces <= T, "loader geometry");
    const int lp = tid % kRowPieces, lj = (tid / kRowPieces) & 3, la0 = tid / (4 * kRowPieces);
    const int64_t ljw = (int64_t)lj * words_total;
    auto plane_src = [&](int ch, int i) -> const uint32_t* {
        const int a = ch * kCH + la0 + kSlotStep * i;
        return (lp * 4 < nw && a < L && lj < (int)s_U[a]) ? s_prow[a] + ljw + lp * 4 : nullptr;
    };
    auto plane_dst = [&](int buf, int i) {
        return s_raw + ((size_t)(buf * kCH + la0 + kSlotStep * i) * 4 + lj) * kTW + lp * 4;
    };
    auto scale_src = [&](int ch) -> const uint16_t* {
        const int a = ch * kCH + (tid >> 2);
        return (tid < kScalePieces && a < L && (tid & 3) * 8 < nblocks) ? s_srow[a] + (tid & 3) * 8 : nullptr;
    };
    auto scale_dst = [&](int buf) { return s_rawsc + (size_t)(buf * kCH + (tid >> 2)) * kNB + (tid & 3) * 8; };
    // device-resident store: cp.async, one chunk ahead
    auto load_chunk = [&](int ch, int buf) {
#pragma unroll
        for (int i = 0; i < kPlaneIters; ++i)
            if (const uint32_t* src = plane_src(ch, i)) cp_async16(plane_dst(buf, i), src);
        if (const uint16_t* src = scale_src(ch)) cp_async16(scale_dst(buf), src);
        cp_async_commit();
    };
    // host-resident store: plain 16-byte loads into registers, one chunk ahead
    // (over the host link each load of a warp is one run of whole lines;
    // cp.async of page-locked memory carried 2.5x the bytes)
    uint4 pf[HOST ? kPlaneIters + 1 : 1];
    auto fetch_chunk = [&](int ch) {
#pragma unroll
        for (int i = 0; i < kPlaneIters; ++i) {
            const uint32_t* src = plane_src(ch, i);
            pf[i] = src ? ldg16(src) : make_uint4(0u, 0u, 0u, 0u);
        }
        const uint16_t* ss = scale_src(ch);
        pf[kPlaneIters] = ss ? ldg16(ss) : make_uint4(0u, 0u, 0u, 0u);
    };
    auto put_chunk = [&](int ch, int buf) {
#pragma unroll
        for (int i = 0; i < kPlaneIters; ++i)
            if (plane_src(ch, i)) *reinterpret_cast<uint4*>(plane_dst(buf, i)) = pf[i];
        if (scale_src(ch)) *reinterpret_cast<uint4*>(scale_dst(buf)) = pf[kPlaneIters];
    };

  for (int tile = tile_begin; tile < ntiles; tile += tile_step) {
    tile0 = (int64_t)tile * kTile;
    keys_here = (int)(len - tile0 < kTile ? len - tile0 : kTile);   // a multiple of 1024
    nw = keys_here / 32;
    nblocks = keys_here / kBlock;
    float2 acc[HG][8];
#pragma unroll
    for (int h = 0; h < HG; ++h)
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[h][i] = make_float2(0.0f, 0.0f);
    float cst_own = 0.0f;   // constant of (block b, head p of the group), summed over the slots in order
    for (int a = tid; a < L; a += T) {   // the tile's rows of every active channel
        const int64_t row = (int64_t)g * d + s_act[a];
        s_prow[a] = planes + row * 4 * words_total + tile0 / 32;
        s_srow[a] = scales + row * nblk_total + tile0 / kBlock;
    }
    __syncthreads();   // the rows are set; the previous tile's loads and stages are done
    if (nchunks > 0) {
        if constexpr (HOST) {
            fetch_chunk(0);
            put_chunk(0, 0);
        } else {
            load_chunk(0, 0);
        }
    }
    for (int ch = 0; ch < nchunks; ++ch) {
        const int buf = ch & 1;
        if constexpr (HOST) {
            if (ch + 1 < nchunks) fetch_chunk(ch + 1);   // in flight during this chunk's stage and compute
        } else {
            if (ch + 1 < nchunks) {
                load_chunk(ch + 1, buf ^ 1);
                cp_async_wait<1>();
            } else {
                cp_async_wait<0>();
            }
        }
        __syncthreads();   // chunk ch's rows are in; the previous chunk's compute is done

        // stage: (slot, block) -> 16 code words
        for (int u = tid; u < kCH * kNB; u += T) {
            const int al = u / kNB, bb = u % kNB, a = ch * kCH + al;
            // a warp stages one slot: its depth made warp-uniform to the compiler
            const int U = (int)__reduce_or_sync(0xffffffffu, (a < L) ? (unsigned)s_U[a] : 0u);
            if (U == 0 || bb >= nblocks) continue;
            const uint32_t* r = s_raw + (size_t)(buf * kCH + al) * 4 * kTW + 2 * bb;
            uint32_t p0[4], p1[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                if (j < U) {
                    const uint2 v = *reinterpret_cast<const uint2*>(r + j * kTW);
                    p0[j] = v.x;
                    p1[j] = v.y;
                } else {
                    p0[j] = p1[j] = 0u;
                }
            }
            uint32_t x0[8], x1[8];
            codes_of(p0, U, x0);
            codes_of(p1, U, x1);
            uint4* dst = reinterpret_cast<uint4*>(s_codes + (size_t)(al * kNB + bb) * 16);
            const int sw = swz(bb);
#pragma unroll
            for (int v = 0; v < 4; ++v) dst[v ^ sw] = make_uint4(x0[2 * v], x1[2 * v], x0[2 * v + 1], x1[2 * v + 1]);
        }
        // coefficients: thread (b, p) those of head p of its group, block b, every slot
        if (p < HG) {
            const int hq = hg * HG + p, nal = L - ch * kCH;   // slots of this chunk: min(nal, kCH)
            const uint16_t* dsc = s_rawsc + (size_t)buf * kCH * kNB + b;
            float* wd = s_w2 + (((size_t)hg * kCH) * kNB + b) * HG * 2 + 2 * p;
#pragma unroll
            for (int al = 0; al < kCH; ++al) {
                if (al < nal) {
                    const float D = __half2float(__ushort_as_half(dsc[al * kNB]));
                    const float2 qq = s_qq[(ch * kCH + al) * G + hq];
                    const float w = qq.x * D;
                    *reinterpret_cast<float2*>(wd + (size_t)al * kNB * HG * 2) = make_float2(w, w);
                    cst_own = fmaf(qq.y, D, cst_own);
                }
            }
        }
        __syncthreads();   // codes and coefficients of chunk ch are ready

        const int task = ch * NHG + hg;
        chunk_items<HG>(s_items + task * kMaxItems, (int)__reduce_or_sync(0xffffffffu, s_nitems[task]), cth, wth,
                        acc);
        if constexpr (HOST) {
            // raw buffer buf ^ 1 was last read by chunk ch - 1's stage, before this chunk's first barrier
            if (ch + 1 < nchunks) put_chunk(ch + 1, buf ^ 1);
        }
    }

    // ---- epilogue: the block's constants (head h's is held by thread p = h of
    // the block), scores, and the maximum of every 64-key block for the top-k ----
    float cst[HG];
#pragma unroll
    for (int h = 0; h < HG; ++h) cst[h] = __shfl_sync(0xffffffffu, cst_own, (lane & ~3) | h);
    if (b < nblocks) {   // uniform per warp: a warp covers 8 blocks and nblocks is a multiple of 16
        const int64_t ld = len;
        const int64_t kb = tile0 + 64 * b + 2 * p;   // key of (word 2p, half 0, byte 0)
        const bool whole = tile0 + keys_here <= n;
#pragma unroll
        for (int h = 0; h < HG; ++h) {
            const int hq = g * G + hg * HG + h;
            float* out = scores + (int64_t)hq * ld + kb;
            float fmax_ = -INFINITY;   // the block's largest score (ordered once: the order is monotone)
#pragma unroll
            for (int wd = 0; wd < 2; ++wd)
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const float2 a0 = acc[h][2 * wd + (k >> 1)];       // word 2p: keys kb + 32 wd + 8k
                    const float2 a1 = acc[h][2 * (2 + wd) + (k >> 1)]; // word 2p + 1: one key later
                    const int o = 32 * wd + 8 * k;
                    float v0 = ((k & 1) ? a0.y : a0.x) + cst[h];
                    float v1 = ((k & 1) ? a1.y : a1.x) + cst[h];
                    if (!whole) {
                        if (kb + o >= n) v0 = -INFINITY;
                        if (kb + o + 1 >= n) v1 = -INFINITY;
                    }
                    *reinterpret_cast<float2*>(out + o) = make_float2(v0, v1);
                    fmax_ = fmaxf(fmax_, fmaxf(v0, v1));
                }
            uint32_t kmax = float_to_ordered(fmax_);
            kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, 1));
            kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, 2));
            if (bmax && p == 0) bmax[(int64_t)hq * (ld / kBlock) + tile0 / kBlock + b] = kmax;
        }
    }
  }
}

// One tile per CTA: blockIdx.x = KV head * tiles + tile (head major).
template <int G, bool HOST>
__global__ void __launch_bounds__(Geo<G>::T, Geo<G>::template min_blocks<HOST>())
scan_kernel(const uint32_t* __restrict__ planes, const uint16_t* __restrict__ scales, int d, int64_t n,
            int64_t n_pad, const void* __restrict__ q, int q_dtype, const uint8_t* __restrict__ depths,
            float* __restrict__ scores, uint32_t* __restrict__ bmax, unsigned int* status) {
    pdl_wait();
    const int b = (int)blockIdx.x, tiles = (int)scan_tiles(n);
    scan_head_tiles<G, HOST>(planes, scales, d, n, n_pad, b % tiles, tiles, b / tiles, q, q_dtype, depths, scores,
                             bmax, status);
}

// Batched sessions: blockIdx.x runs over the tiles of all sessions.
template <int G, bool HOST>
__global__ void __launch_bounds__(Geo<G>::T, Geo<G>::template min_blocks<HOST>())
scan_batched_kernel(const __grid_constant__ SessionMap map, int d, int Hq, const void* __restrict__ q, int q_dtype,
                    const uint8_t* __restrict__ depths, float* __restrict__ scores, uint32_t* __restrict__ bmax,
                    unsigned int* status) {
    pdl_wait();
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
    const int tile = t - map.tile0[sidx];
    scan_head_tiles<G, HOST>(map.planes[sidx], map.scales[sidx], d, map.n[sidx], map.n_pad[sidx], tile, INT32_MAX - tile,
                        (int)blockIdx.y, qs, q_dtype, depths + sidx * qstride, scores + map.score_base[sidx],
                        bmax ? bmax + map.score_base[sidx] / kBlock : nullptr, status);
}

template <int G, bool HOST>
cudaError_t launch_scan_g(const uint32_t* planes, const uint16_t* scales, int Hkv, int d, int64_t n,
                          int64_t n_pad, const void* q, int q_dtype, const uint8_t* depths, float* scores,
                          uint32_t* bmax, cudaStream_t stream, bool pdl) {
    const size_t smem = ScanSmem{d, G}.bytes();
    auto kern = scan_kernel<G, HOST>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    // One CTA per (tile, KV head), head major: the resident CTAs read about
    // 600 consecutive tiles of one or two heads at a time, which the host link
    // serves best.  (A persistent grid that plans each head once per CTA and
    // walks its tiles was bit-identical but slower on a device-resident store
    // too: 0.40 against 0.35 ms at n = 2^20, its CTAs ending unevenly.)
    const int64_t ctas = scan_tiles(n) * Hkv;
    if (ctas > INT32_MAX) return cudaErrorInvalidValue;
    return launch_ex(kern, dim3((unsigned)ctas), dim3(Geo<G>::T), smem, stream, pdl, 1, planes, scales, d, n, n_pad, q,
                     q_dtype, depths, scores, bmax, device_status_ptr());
}

template <int G, bool HOST>
cudaError_t launch_scan_batched_g(const SessionMap& map, int Hkv, int d, const void* q, int q_dtype,
                                  const uint8_t* depths, int Hq, float* scores, uint32_t* bmax, cudaStream_t stream) {
    const size_t smem = ScanSmem{d, G}.bytes();
    auto kern = scan_batched_kernel<G, HOST>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)map.tile0[map.nsess], (unsigned)Hkv);
    kern<<<grid, Geo<G>::T, smem, stream>>>(map, d, Hq, q, q_dtype, depths, scores, bmax, device_status_ptr());
    return cudaGetLastError();
}

template <int G>
cudaError_t launch_scan_r(bool host, const uint32_t* planes, const uint16_t* scales, int Hkv, int d, int64_t n,
                          int64_t n_pad, const void* q, int q_dtype, const uint8_t* depths, float* scores,
                          uint32_t* bmax, cudaStream_t stream, bool pdl) {
    return host ? launch_scan_g<G, true>(planes, scales, Hkv, d, n, n_pad, q, q_dtype, depths, scores, bmax, stream, pdl)
                : launch_scan_g<G, false>(planes, scales, Hkv, d, n, n_pad, q, q_dtype, depths, scores, bmax, stream,
                                          pdl);
}

template <int G>
cudaError_t launch_scan_batched_r(bool host, const SessionMap& map, int Hkv, int d, const void* q, int q_dtype,
                                  const uint8_t* depths, int Hq, float* scores, uint32_t* bmax, cudaStream_t stream) {
    return host ? launch_scan_batched_g<G, true>(map, Hkv, d, q, q_dtype, depths, Hq, scores, bmax, stream)
                : launch_scan_batched_g<G, false>(map, Hkv, d, q, q_dtype, depths, Hq, scores, bmax, stream);
}

}  // namespace

size_t scan_smem_bytes(int d, int G) { return ScanSmem{d, G}.bytes(); }

cudaError_t launch_scan(const uint32_t* planes, const uint16_t* scales, int Hkv, int d, int64_t n, int64_t n_pad,
                        const void* q, int q_dtype, const uint8_t* depths, int Hq, float* scores,
                        cudaStream_t stream, uint32_t* bmax, bool host, bool pdl) {
    switch (Hq / Hkv) {
        case 1: return launch_scan_r<1>(host, planes, scales, Hkv, d, n, n_pad, q, q_dtype, depths, scores, bmax, stream, pdl);
        case 2: return launch_scan_r<2>(host, planes, scales, Hkv, d, n, n_pad, q, q_dtype, depths, scores, bmax, stream, pdl);
        case 4: return launch_scan_r<4>(host, planes, scales, Hkv, d, n, n_pad, q, q_dtype, depths, scores, bmax, stream, pdl);
        case 8: return launch_scan_r<8>(host, planes, scales, Hkv, d, n, n_pad, q, q_dtype, depths, scores, bmax, stream, pdl);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_scan_batched(const SessionMap& map, int Hkv, int d, const void* q, int q_dtype,
                                const uint8_t* depths, int Hq, float* scores, cudaStream_t stream, uint32_t* bmax,
                                bool host) {
    switch (Hq / Hkv) {
        case 1: return launch_scan_batched_r<1>(host, map, Hkv, d, q, q_dtype, depths, Hq, scores, bmax, stream);
        case 2: return launch_scan_batched_r<2>(host, map, Hkv, d, q, q_dtype, depths, Hq, scores, bmax, stream);
        case 4: return launch_scan_batched_r<4>(host, map, Hkv, d, q, q_dtype, depths, Hq, scores, bmax, stream);
        case 8: return launch_scan_batched_r<8>(host, map, Hkv, d, q, q_dtype, depths, Hq, scores, bmax, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace fathom
