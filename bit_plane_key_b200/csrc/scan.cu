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
// so a channel adds (32 q Delta) F_t per key and head, and q Delta (2^(3-t) - 24)
// per (block, head) once.
//
// Work.  One CTA of 128 threads per (tile of 1024 keys, KV head).  The tile's
// active channels are streamed in chunks of 16:
//   stage: thread (channel group of 4, plane word w) loads the U_c plane
//     words of its channels and transposes them to byte codes: variant word
//     s (s = 0..7) holds the codes of keys s, s+8, s+16, s+24 of the word,
//     one byte each, bits 6..3 = planes 0..3 (rotate + mask per plane and
//     variant, i.e. half an operation per plane bit), stored to a double
//     buffer in shared memory with conflict-free 16-byte stores;
//   compute: thread (block b, variant s) owns the 8 keys s + 8k of words 2b
//     and 2b+1.  Per channel one byte permute builds F for a key, heads that
//     read the channel add coef*F with packed fp32x2 FMAs (two keys of the
//     same block share the coefficient), heads that read fewer planes than
//     the union mask F first, heads that read nothing cost nothing.
//   The next chunk's plane words are loaded into registers before the
//   current chunk is computed, so the loads overlap the arithmetic.
// The same kernel serves a host-resident store: its loads then cross the host
// link as 128-byte runs per (channel, plane) and tile.
#include "fathom_internal.cuh"

namespace fathom {
namespace {

constexpr int kTileKeys = 1024;
constexpr int kTileWords = kTileKeys / 32;   // 32 plane words per tile row
constexpr int kTileBlocks = kTileKeys / kBlock;
constexpr int kThreads = 128;                // (16 blocks) x (8 variants)
constexpr int kChunk = 16;                   // active channels per stage
constexpr int kCPad = 20;                    // words per (word, variant) code row; 20 = 4 mod 8
constexpr uint32_t kHalfExp = 0x3F000000u;   // bits of 0.5f: exponent byte of F
constexpr bool kScanPacked = true;           // fp32x2 FMAs: two keys of a block per instruction

struct ScanSmem {
    static size_t bytes(int d, int G) {
        size_t s = sizeof(uint32_t) * 2 * kTileWords * 8 * kCPad;   // codes, double-buffered
        s += sizeof(float) * 2 * kChunk * kTileBlocks * G;          // coefficients, double-buffered
        s += sizeof(float) * (size_t)d * G * 2;                     // 32 q, constant factor
        s += sizeof(uint32_t) * (size_t)d * G;                      // masks
        s += sizeof(uint32_t) * (size_t)d * 3;                      // meta, channel, U
        s += (size_t)G * d + 64;                                    // t [G][d]
        return s;
    }
};

__device__ __forceinline__ uint64_t pack2(uint32_t lo, uint32_t hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "r"(lo), "r"(hi));
    return r;
}
__device__ __forceinline__ void fma2(uint64_t& acc, uint64_t a, uint64_t b) {
    asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(acc) : "l"(a), "l"(b));
}
__device__ __forceinline__ float2 unpack2(uint64_t v) {
    uint32_t lo, hi;
    asm("mov.b64 {%0, %1}, %2;" : "=r"(lo), "=r"(hi) : "l"(v));
    return make_float2(__uint_as_float(lo), __uint_as_float(hi));
}
// fp32 mask keeping sign, exponent and the top t code bits (mantissa 22..19)
__device__ __forceinline__ uint32_t depth_mask(uint32_t t) {
    return 0xFF800000u | ((((0xFu << (4u - t)) & 0xFu)) << 19);
}

// Transposes one 32-key plane word column of a channel (U planes) into the
// byte-code variant `sv`: byte k = code of key sv + 8k, planes at bits 6..3.
template <int U>
__device__ __forceinline__ uint32_t code_variant(const uint32_t* p, int sv) {
    uint32_t x = 0;
#pragma unroll
    for (int j = 0; j < U; ++j)
        x |= __funnelshift_r(p[j], p[j], (uint32_t)(sv + j - 6) & 31u) & (0x01010101u << (6 - j));
    return x;
}

// One (tile of 1024 keys, KV head g) of one store; q, depths and scores are
// the store's own [Hq][d], [Hq][d] and [Hq][n_pad] arrays.
template <int G, bool kPacked>
__device__ __forceinline__ void scan_tile(const uint32_t* __restrict__ planes, const uint16_t* __restrict__ scales,
                                          int d, int64_t n, int64_t n_pad, int tile, int g,
                                          const void* __restrict__ q, int q_dtype,
                                          const uint8_t* __restrict__ depths, float* __restrict__ scores,
                                          unsigned int* status) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const int64_t tile0 = (int64_t)tile * kTileKeys;
    const int64_t words_total = n_pad / 32;
    const int64_t nblk_total = n_pad / kBlock;
    const int64_t wrem = words_total - tile0 / 32;
    const int nwords = wrem < kTileWords ? (int)wrem : kTileWords;   // multiple of 4
    const int nblocks = nwords / 2;

    uint32_t* s_codes = reinterpret_cast<uint32_t*>(smem_raw);                 // [2][32][8][kCPad]
    float* s_coef = reinterpret_cast<float*>(s_codes + 2 * kTileWords * 8 * kCPad);   // [2][kChunk][16][G]
    float* s_q32 = s_coef + 2 * kChunk * kTileBlocks * G;                        // [L][G]: 32 q (0 if t = 0)
    float* s_kc = s_q32 + (size_t)d * G;                                         // [L][G]: (2^(3-t) - 24) / 32
    uint32_t* s_mask = reinterpret_cast<uint32_t*>(s_kc + (size_t)d * G);        // [L][G]
    uint32_t* s_meta = s_mask + (size_t)d * G;                                   // [L]: act | part << 8
    int* s_act = reinterpret_cast<int*>(s_meta + d);                             // [L]: channel
    int* s_U = s_act + d;                                                        // [L]: union depth
    uint8_t* s_t = reinterpret_cast<uint8_t*>(s_U + d);                          // [G][d]
    __shared__ int s_L;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    // ---- plan: depths, union, active channels, per (channel, head) factors ----
    for (int e = tid; e < G * d; e += kThreads) {
        int hh = e / d, c = e - hh * d;
        int t = depths[((int64_t)g * G + hh) * d + c];
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
            uint32_t act = 0;
#pragma unroll
            for (int hh = 0; hh < G; ++hh) {
                const int t = s_t[hh * d + c];
                U = max(U, t);
                act |= (t > 0 ? 1u : 0u) << hh;
            }
            uint32_t part = 0;
#pragma unroll
            for (int hh = 0; hh < G; ++hh) {
                const int t = s_t[hh * d + c];
                part |= (t > 0 && t < U ? 1u : 0u) << hh;
            }
            const unsigned m = __ballot_sync(0xffffffffu, U > 0);
            if (U > 0) {
                const int pos = base + __popc(m & ((1u << lane) - 1u));
                s_act[pos] = c;
                s_U[pos] = U;
                s_meta[pos] = act | (part << 8);
            }
            base += __popc(m);
        }
        if (lane == 0) s_L = base;
    }
    __syncthreads();
    const int L = s_L;
    const int nchunks = (L + kChunk - 1) / kChunk;
    for (int e = tid; e < L * G; e += kThreads) {
        const int a = e / G, hh = e - a * G;
        const int c = s_act[a];
        const int t = s_t[hh * d + c];
        const float qv = load_q(q, q_dtype, ((int64_t)g * G + hh) * d + c);
        s_q32[e] = (t > 0) ? 32.0f * qv : 0.0f;
        s_kc[e] = (t > 0) ? (__uint_as_float((uint32_t)(130 - t) << 23) - 24.0f) * 0.03125f : 0.0f;
        s_mask[e] = (t > 0) ? depth_mask((uint32_t)t) : 0u;
    }
    __syncthreads();

    // ---- stage / compute roles ----
    const int cg = warp, w = lane;               // stage: channel group of 4, plane word
    const int b = tid >> 3, s = tid & 7;         // compute: block (words 2b, 2b+1), variant

    uint32_t pw[4][4];   // prefetched plane words: [channel in group][plane]
    float pd[2];         // prefetched scales of (channel, block) items tid and tid + 128
    auto load_chunk = [&](int ch) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int a = ch * kChunk + cg * 4 + i;
            const int U = (a < L) ? s_U[a] : 0;
            const uint32_t* row = planes + ((int64_t)g * d + ((a < L) ? s_act[a] : 0)) * 4 * words_total +
                                  tile0 / 32 + w;
#pragma unroll
            for (int j = 0; j < 4; ++j)
                pw[i][j] = (j < U && w < nwords) ? __ldg(row + (int64_t)j * words_total) : 0u;
        }
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int e = tid + u * kThreads, al = e >> 4, bb = e & 15;
            const int a = ch * kChunk + al;
            pd[u] = (a < L && bb < nblocks)
                        ? __half2float(__ushort_as_half(__ldg(scales + ((int64_t)g * d + s_act[a]) * nblk_total +
                                                              tile0 / kBlock + bb)))
                        : 0.0f;
        }
    };
    auto store_chunk = [&](int ch, int buf) {
        uint32_t x[4][8];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int a = ch * kChunk + cg * 4 + i;
            const int U = (a < L) ? s_U[a] : 0;
            switch (U) {
                case 4:
#pragma unroll
                    for (int sv = 0; sv < 8; ++sv) x[i][sv] = code_variant<4>(pw[i], sv);
                    break;
                case 3:
#pragma unroll
                    for (int sv = 0; sv < 8; ++sv) x[i][sv] = code_variant<3>(pw[i], sv);
                    break;
                case 2:
#pragma unroll
                    for (int sv = 0; sv < 8; ++sv) x[i][sv] = code_variant<2>(pw[i], sv);
                    break;
                case 1:
#pragma unroll
                    for (int sv = 0; sv < 8; ++sv) x[i][sv] = code_variant<1>(pw[i], sv);
                    break;
                default:
#pragma unroll
                    for (int sv = 0; sv < 8; ++sv) x[i][sv] = 0u;
            }
        }
        uint32_t* base = s_codes + (size_t)buf * kTileWords * 8 * kCPad;
#pragma unroll
        for (int sv = 0; sv < 8; ++sv) {
            // XOR swizzle of the variant row keeps both these stores and the
            // compute-phase loads free of bank conflicts
            const int prow = w * 8 + (sv ^ (w & 7));
            *reinterpret_cast<uint4*>(base + (size_t)prow * kCPad + cg * 4) = make_uint4(x[0][sv], x[1][sv], x[2][sv], x[3][sv]);
        }
        float* cbuf = s_coef + (size_t)buf * kChunk * kTileBlocks * G;
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int e = tid + u * kThreads, al = e >> 4, bb = e & 15;
            const int a = min(ch * kChunk + al, max(L - 1, 0));
#pragma unroll
            for (int hh = 0; hh < G; ++hh) cbuf[(al * kTileBlocks + bb) * G + hh] = s_q32[a * G + hh] * pd[u];
        }
    };

    float acc[G][8];
    float cst[G];
#pragma unroll
    for (int hh = 0; hh < G; ++hh) {
        cst[hh] = 0.0f;
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[hh][e] = 0.0f;
    }

    if (nchunks > 0) {
        load_chunk(0);
        store_chunk(0, 0);
    }
    __syncthreads();
    for (int ch = 0; ch < nchunks; ++ch) {
        const int buf = ch & 1;
        if (ch + 1 < nchunks) load_chunk(ch + 1);
        if (b < nblocks) {
            const uint32_t* cbase = s_codes + (size_t)buf * kTileWords * 8 * kCPad;
            const uint32_t* row0 = cbase + ((size_t)(2 * b) * 8 + (s ^ ((2 * b) & 7))) * kCPad;
            const uint32_t* row1 = cbase + ((size_t)(2 * b + 1) * 8 + (s ^ ((2 * b + 1) & 7))) * kCPad;
            const float* cbuf = s_coef + (size_t)buf * kChunk * kTileBlocks * G;
            const int nloc = min(kChunk, L - ch * kChunk);
            for (int i4 = 0; i4 < nloc; i4 += 4) {
                const uint4 X0 = *reinterpret_cast<const uint4*>(row0 + i4);
                const uint4 X1 = *reinterpret_cast<const uint4*>(row1 + i4);
                const uint32_t xs0[4] = {X0.x, X0.y, X0.z, X0.w};
                const uint32_t xs1[4] = {X1.x, X1.y, X1.z, X1.w};
#pragma unroll
                for (int ii = 0; ii < 4; ++ii) {
                    if (i4 + ii >= nloc) break;
                    const int al = i4 + ii, a = ch * kChunk + al;
                    const uint32_t meta = s_meta[a];
                    float cf[G], kc[G];
                    uint32_t mk[G];
#pragma unroll
                    for (int hh = 0; hh < G; ++hh) {
                        cf[hh] = cbuf[(al * kTileBlocks + b) * G + hh];
                        kc[hh] = s_kc[a * G + hh];
                        mk[hh] = s_mask[a * G + hh];
                    }
                    uint32_t F[8];
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        F[k] = __byte_perm(xs0[ii], kHalfExp, 0x7044u | ((uint32_t)k << 8));
                        F[4 + k] = __byte_perm(xs1[ii], kHalfExp, 0x7044u | ((uint32_t)k << 8));
                    }
#pragma unroll
                    for (int hh = 0; hh < G; ++hh) {
                        if (!(meta & (1u << hh))) continue;
                        cst[hh] = fmaf(cf[hh], kc[hh], cst[hh]);
                        uint32_t Fm[8];
                        if (meta & (0x100u << hh)) {
#pragma unroll
                            for (int e = 0; e < 8; ++e) Fm[e] = F[e] & mk[hh];
                        } else {
#pragma unroll
                            for (int e = 0; e < 8; ++e) Fm[e] = F[e];
                        }
                        if constexpr (kPacked) {
                            const uint64_t c2 = pack2(__float_as_uint(cf[hh]), __float_as_uint(cf[hh]));
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                uint64_t a2 = pack2(__float_as_uint(acc[hh][2 * e]), __float_as_uint(acc[hh][2 * e + 1]));
                                fma2(a2, c2, pack2(Fm[2 * e], Fm[2 * e + 1]));
                                const float2 r = unpack2(a2);
                                acc[hh][2 * e] = r.x;
                                acc[hh][2 * e + 1] = r.y;
                            }
                        } else {
#pragma unroll
                            for (int e = 0; e < 8; ++e) acc[hh][e] = fmaf(cf[hh], __uint_as_float(Fm[e]), acc[hh][e]);
                        }
                    }
                }
            }
        }
        if (ch + 1 < nchunks) store_chunk(ch + 1, buf ^ 1);
        __syncthreads();
    }

    // ---- epilogue: F[k] / F[4+k] are keys s + 8k of words 2b / 2b+1 ----
    if (b < nblocks) {
#pragma unroll
        for (int hh = 0; hh < G; ++hh) {
            float* out = scores + ((int64_t)g * G + hh) * n_pad + tile0;
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const int64_t i = 32 * (2 * b + (e >> 2)) + s + 8 * (e & 3);
                out[i] = (tile0 + i < n) ? acc[hh][e] + cst[hh] : -INFINITY;
            }
        }
    }
}

template <int G>
__global__ void __launch_bounds__(kThreads)
scan_kernel(const uint32_t* __restrict__ planes, const uint16_t* __restrict__ scales, int d, int64_t n,
            int64_t n_pad, const void* __restrict__ q, int q_dtype, const uint8_t* __restrict__ depths,
            float* __restrict__ scores, unsigned int* status) {
    scan_tile<G, kScanPacked>(planes, scales, d, n, n_pad, (int)blockIdx.x, (int)blockIdx.y, q, q_dtype, depths,
                              scores, status);
}

// Batched sessions: blockIdx.x runs over the tiles of all sessions.
template <int G>
__global__ void __launch_bounds__(kThreads)
scan_batched_kernel(const __grid_constant__ SessionMap map, int d, int Hq, const void* __restrict__ q, int q_dtype,
                    const uint8_t* __restrict__ depths, float* __restrict__ scores, unsigned int* status) {
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
    scan_tile<G, kScanPacked>(map.planes[sidx], map.scales[sidx], d, map.n[sidx], map.n_pad[sidx],
                              t - map.tile0[sidx], (int)blockIdx.y, qs, q_dtype, depths + sidx * qstride,
                              scores + map.score_base[sidx], status);
}

template <int G>
cudaError_t launch_scan_g(const uint32_t* planes, const uint16_t* scales, int Hkv, int d, int64_t n,
                          int64_t n_pad, const void* q, int q_dtype, const uint8_t* depths, float* scores,
                          cudaStream_t stream) {
    size_t smem = ScanSmem::bytes(d, G);
    auto kern = scan_kernel<G>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)((n_pad + kTileKeys - 1) / kTileKeys), (unsigned)Hkv);
    kern<<<grid, kThreads, smem, stream>>>(planes, scales, d, n, n_pad, q, q_dtype, depths, scores,
                                           device_status_ptr());
    return cudaGetLastError();
}

template <int G>
cudaError_t launch_scan_batched_g(const SessionMap& map, int Hkv, int d, const void* q, int q_dtype,
                                  const uint8_t* depths, int Hq, float* scores, cudaStream_t stream) {
    size_t smem = ScanSmem::bytes(d, G);
    auto kern = scan_batched_kernel<G>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)map.tile0[map.nsess], (unsigned)Hkv);
    kern<<<grid, kThreads, smem, stream>>>(map, d, Hq, q, q_dtype, depths, scores, device_status_ptr());
    return cudaGetLastError();
}

}  // namespace

size_t scan_smem_bytes(int d, int G) { return ScanSmem::bytes(d, G); }

cudaError_t launch_scan(const uint32_t* planes, const uint16_t* scales, int Hkv, int d, int64_t n, int64_t n_pad,
                        const void* q, int q_dtype, const uint8_t* depths, int Hq, float* scores,
                        cudaStream_t stream) {
    switch (Hq / Hkv) {
        case 1: return launch_scan_g<1>(planes, scales, Hkv, d, n, n_pad, q, q_dtype, depths, scores, stream);
        case 2: return launch_scan_g<2>(planes, scales, Hkv, d, n, n_pad, q, q_dtype, depths, scores, stream);
        case 4: return launch_scan_g<4>(planes, scales, Hkv, d, n, n_pad, q, q_dtype, depths, scores, stream);
        case 8: return launch_scan_g<8>(planes, scales, Hkv, d, n, n_pad, q, q_dtype, depths, scores, stream);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_scan_batched(const SessionMap& map, int Hkv, int d, const void* q, int q_dtype,
                                const uint8_t* depths, int Hq, float* scores, cudaStream_t stream) {
    switch (Hq / Hkv) {
        case 1: return launch_scan_batched_g<1>(map, Hkv, d, q, q_dtype, depths, Hq, scores, stream);
        case 2: return launch_scan_batched_g<2>(map, Hkv, d, q, q_dtype, depths, Hq, scores, stream);
        case 4: return launch_scan_batched_g<4>(map, Hkv, d, q, q_dtype, depths, Hq, scores, stream);
        case 8: return launch_scan_batched_g<8>(map, Hkv, d, q, q_dtype, depths, Hq, scores, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace fathom
