// K3: variable-depth scan over the bit-plane store.
//
// For query head h (KV head g = h / G) and key i in 64-token block b:
//   s[h][i] = sum_c q[h][c] * Delta[b][c] * sum_{j < t[h][c]} (2 b_{i,c,j} - 1) 2^(2-j)
// i.e. every channel contributes its t-bit mid-rise value rebuilt from the
// first t planes (basis rule; ai-feeds.com summary, 方法 · 关键模块 4, paper
// Sec 3.5; a t-plane prefix is exactly the t-bit quantizer: arXiv abstract,
// evolve.pub review Strengths, paper Sec 3.2).  The scan reads only the first
// U_c = max_{h in group} t[h][c] planes of each channel (ai-feeds.com summary,
// 关键模块 5: only the budgeted planes are pulled); a channel nobody reads is
// never touched, nor is its scale row.
//
// Arithmetic.  With m = the t-bit prefix of the code, the rebuilt value is
//   v = 2^(3-t) (2m + 1) - 8 = 16 F - 24 + 2^(3-t),   F = 1 + m / 2^t,
// and F is an fp32 number whose mantissa holds exactly the prefix bits.  So
// per (key, head, channel) the scan does one AND (keep the head's t bits of
// the union prefix) and one FFMA with the coefficient 16 q Delta; the
// constant q Delta (2^(3-t) - 24) is summed once per (block, head).
//
// Layout of work.  One CTA per (tile of 1024 keys, KV head); 256 threads,
// thread = 4 keys (key = 32 w + lane, words w = warp + 8 r), so a warp's
// lanes take the 32 bits of one plane word.  The tile's plane words of the
// active channels are staged in shared memory as [channel][word][4 planes]
// (unread planes as zero) with 16-byte loads; each lane then rotates its bit
// into the mantissa position.  The same kernel serves a host-resident store:
// its loads then cross the host link, and only the budgeted runs are read.
#include "fathom_internal.cuh"

namespace fathom {
namespace {

constexpr int kTileKeys = 1024;
constexpr int kTileWords = kTileKeys / 32;   // 32 plane words per tile row
constexpr int kTileBlocks = kTileKeys / kBlock;
constexpr int kThreads = 256;

struct ScanSmem {
    // sized at launch for (d, G); offsets in bytes
    static size_t bytes(int d, int G) {
        size_t s = 0;
        s += (size_t)d * kTileWords * 4 * sizeof(uint32_t);      // planes [L][32][4]
        s += (size_t)d * kTileBlocks * G * sizeof(float);        // coef  [L][16][G]
        s += (size_t)d * G * sizeof(uint32_t);                   // mask  [L][G]
        s += (size_t)G * kTileBlocks * sizeof(float);            // const [G][16]
        s += (size_t)G * d * sizeof(float);                      // q     [G][d]
        s += (size_t)G * d;                                      // t     [G][d]
        s += (size_t)d * sizeof(int) * 2 + 64;                   // active list, U
        return s;
    }
};

template <int G>
__global__ void __launch_bounds__(kThreads)
scan_kernel(const uint32_t* __restrict__ planes, const uint16_t* __restrict__ scales, int d, int64_t n,
            int64_t n_pad, const void* __restrict__ q, int q_dtype, const uint8_t* __restrict__ depths,
            float* __restrict__ scores, unsigned int* status) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const int g = blockIdx.y;
    const int64_t tile0 = (int64_t)blockIdx.x * kTileKeys;
    const int64_t words_total = n_pad / 32;
    const int64_t nblk_total = n_pad / kBlock;
    const int64_t wrem = words_total - tile0 / 32;
    const int nwords = wrem < kTileWords ? (int)wrem : kTileWords;
    const int nblocks = (nwords + 1) / 2;

    uint32_t* s_planes = reinterpret_cast<uint32_t*>(smem_raw);
    float* s_coef = reinterpret_cast<float*>(s_planes + (size_t)d * kTileWords * 4);
    uint32_t* s_mask = reinterpret_cast<uint32_t*>(s_coef + (size_t)d * kTileBlocks * G);
    float* s_const = reinterpret_cast<float*>(s_mask + (size_t)d * G);
    float* s_q = s_const + G * kTileBlocks;
    uint8_t* s_t = reinterpret_cast<uint8_t*>(s_q + G * d);
    int* s_act = reinterpret_cast<int*>(s_t + ((G * d + 15) & ~15));
    int* s_U = s_act + d;
    __shared__ int s_L;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    // 1. depths and queries of the group; union depth per channel.
    for (int e = tid; e < G * d; e += kThreads) {
        int hh = e / d, c = e - hh * d;
        int64_t h = (int64_t)g * G + hh;
        int t = depths[h * d + c];
        if (t > 4) {
            atomicOr(status, (unsigned)FATHOM_DEV_BAD_DEPTH);
            t = 0;
        }
        s_t[e] = (uint8_t)t;
        s_q[e] = load_q(q, q_dtype, h * d + c);
    }
    __syncthreads();
    if (warp == 0) {
        // ordered compaction of channels with U_c > 0
        int base = 0;
        for (int c0 = 0; c0 < d; c0 += 32) {
            int c = c0 + lane;
            int U = 0;
#pragma unroll
            for (int hh = 0; hh < G; ++hh) U = max(U, (int)s_t[hh * d + c]);
            unsigned act = __ballot_sync(0xffffffffu, U > 0);
            if (U > 0) {
                int pos = base + __popc(act & ((1u << lane) - 1u));
                s_act[pos] = c;
                s_U[pos] = U;
            }
            base += __popc(act);
        }
        if (lane == 0) s_L = base;
    }
    __syncthreads();
    const int L = s_L;

    // 2. stage the plane words of the active channels: [a][w][j], zero beyond U.
    //    Each (a, j) row segment is nwords contiguous words; 16-byte loads.
    {
        const int chunks = (nwords + 3) / 4;   // nwords is a multiple of 4 (n_pad % 128 == 0)
        const int items = L * 4 * chunks;
        constexpr int kBatch = 8;
        for (int base = tid; base < items; base += kThreads * kBatch) {
            uint4 v[kBatch];
#pragma unroll
            for (int u = 0; u < kBatch; ++u) {
                int it = base + u * kThreads;
                v[u] = make_uint4(0u, 0u, 0u, 0u);
                if (it < items) {
                    int a = it / (4 * chunks);
                    int r = it - a * 4 * chunks;
                    int j = r / chunks, ch = r - j * chunks;
                    if (j < s_U[a]) {
                        int c = s_act[a];
                        const uint4* src = reinterpret_cast<const uint4*>(
                            planes + (((int64_t)g * d + c) * 4 + j) * words_total + tile0 / 32) + ch;
                        v[u] = __ldg(src);
                    }
                }
            }
#pragma unroll
            for (int u = 0; u < kBatch; ++u) {
                int it = base + u * kThreads;
                if (it < items) {
                    int a = it / (4 * chunks);
                    int r = it - a * 4 * chunks;
                    int j = r / chunks, ch = r - j * chunks;
                    uint32_t* dst = s_planes + ((size_t)a * kTileWords + ch * 4) * 4 + j;
                    dst[0] = v[u].x;
                    dst[4] = v[u].y;
                    dst[8] = v[u].z;
                    dst[12] = v[u].w;
                }
            }
        }
    }

    // 3. per (active channel, head): mask of the head's depth; per (channel,
    //    block, head): coefficient 16 q Delta.
    for (int e = tid; e < L * G; e += kThreads) {
        int a = e / G, hh = e - a * G;
        int t = s_t[hh * d + s_act[a]];
        s_mask[e] = (t == 0) ? 0u : (0xFF800000u | (((1u << t) - 1u) << (23 - t)));
    }
    for (int e = tid; e < L * kTileBlocks; e += kThreads) {
        int a = e / kTileBlocks, bb = e - a * kTileBlocks;
        int c = s_act[a];
        float delta = 0.0f;
        if (bb < nblocks)
            delta = __half2float(__ushort_as_half(
                __ldg(scales + ((int64_t)g * d + c) * nblk_total + tile0 / kBlock + bb)));
#pragma unroll
        for (int hh = 0; hh < G; ++hh) {
            int t = s_t[hh * d + c];
            s_coef[((size_t)a * kTileBlocks + bb) * G + hh] = (t == 0) ? 0.0f : 16.0f * s_q[hh * d + c] * delta;
        }
    }
    __syncthreads();
    // constants per (head, block): sum_c q Delta (2^(3-t) - 24), from the coefficients
    for (int e = tid; e < G * kTileBlocks; e += kThreads) {
        int hh = e / kTileBlocks, bb = e - hh * kTileBlocks;
        float acc = 0.0f;
        for (int a = 0; a < L; ++a) {
            int t = s_t[hh * d + s_act[a]];
            if (t == 0) continue;
            float qd = s_coef[((size_t)a * kTileBlocks + bb) * G + hh] * 0.0625f;   // q Delta
            acc = fmaf(qd, ldexpf(1.0f, 3 - t) - 24.0f, acc);   // q Delta (2^(3-t) - 24)
        }
        s_const[e] = acc;
    }
    __syncthreads();

    // 4. scan: thread keys 32 w + lane, w = warp + 8 r.
    uint32_t sh[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) sh[j] = (uint32_t)(22 - j - lane) & 31u;

    float acc[4][G];
    int wv[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        wv[r] = warp + 8 * r;
        int bb = wv[r] >> 1;
#pragma unroll
        for (int hh = 0; hh < G; ++hh) acc[r][hh] = (wv[r] < nwords) ? s_const[hh * kTileBlocks + bb] : 0.0f;
    }

    for (int a = 0; a < L; ++a) {
        uint32_t mk[G];
#pragma unroll
        for (int hh = 0; hh < G; ++hh) mk[hh] = s_mask[a * G + hh];
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            if (wv[r] >= nwords) continue;
            const uint4 p = *reinterpret_cast<const uint4*>(s_planes + ((size_t)a * kTileWords + wv[r]) * 4);
            uint32_t r0 = __funnelshift_l(p.x, p.x, sh[0]);
            uint32_t r1 = __funnelshift_l(p.y, p.y, sh[1]);
            uint32_t r2 = __funnelshift_l(p.z, p.z, sh[2]);
            uint32_t r3 = __funnelshift_l(p.w, p.w, sh[3]);
            uint32_t F = 0x3F800000u | (r0 & 0x400000u) | (r1 & 0x200000u) | (r2 & 0x100000u) | (r3 & 0x80000u);
            const float* cf = s_coef + ((size_t)a * kTileBlocks + (wv[r] >> 1)) * G;
#pragma unroll
            for (int hh = 0; hh < G; ++hh) acc[r][hh] = fmaf(cf[hh], __uint_as_float(F & mk[hh]), acc[r][hh]);
        }
    }

    // 5. write scores [Hq][n_pad]; padding keys get -inf.
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        if (wv[r] >= nwords) continue;
        int64_t i = tile0 + 32 * wv[r] + lane;
#pragma unroll
        for (int hh = 0; hh < G; ++hh) {
            int64_t h = (int64_t)g * G + hh;
            scores[h * n_pad + i] = (i < n) ? acc[r][hh] : -INFINITY;
        }
    }
}

template <int G>
cudaError_t launch_scan_g(const uint32_t* planes, const uint16_t* scales, int Hkv, int d, int64_t n,
                          int64_t n_pad, const void* q, int q_dtype, const uint8_t* depths, float* scores,
                          cudaStream_t stream) {
    size_t smem = ScanSmem::bytes(d, G);
    cudaError_t e = cudaFuncSetAttribute(scan_kernel<G>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)((n_pad + kTileKeys - 1) / kTileKeys), (unsigned)Hkv);
    scan_kernel<G><<<grid, kThreads, smem, stream>>>(planes, scales, d, n, n_pad, q, q_dtype, depths, scores,
                                                    device_status_ptr());
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

}  // namespace fathom
