// K1: bit-plane packer.
//
// Quantizes a K cache to 4-bit mid-rise codes under one fp16 scale per
// (KV head, channel, 64-token block) and writes the codes channel-major as
// four bit planes.  Sources: ai-feeds.com summary, 方法 · 关键模块 1 (bit-plane
// store: each channel kept as 4 planes, reading the first t gives the t-bit
// quantized value); evolve.pub review, Strengths (one shared block scale,
// paper Sec 3.2) and FAQ "How does Fathom's bit-plane KV cache work?"
// (uniform per-channel codes, each bit position a contiguous plane).
//
// One CTA per (64-token block, KV head).  The block's 64 x d tile is staged
// in shared memory with coalesced loads; each warp then owns channels
// c = warp, warp + 4, ...: lane l quantizes keys l and 32 + l, and a warp
// ballot per plane yields the two 32-key plane words directly.
//
// A block is self-contained (its scale, its two words per plane row), so the
// same kernel packs a whole store or re-packs a range of blocks: decode-time
// append re-packs the last partial block (its scale changes when keys join
// it) and the blocks after it, from a buffer holding the keys from that
// block's first key on.
#include "fathom_internal.cuh"

namespace fathom {
namespace {

constexpr int kWarps = 4;

__global__ void __launch_bounds__(kWarps * 32)
pack_kernel(const void* __restrict__ K, int k_dtype, int64_t rows, int64_t key0, int64_t blk0, int64_t n, int d,
            int64_t n_pad, uint32_t* __restrict__ planes, uint16_t* __restrict__ scales) {
    // K holds keys [key0, key0 + rows) of every KV head: [Hkv][rows][d];
    // n = keys of the store after this pack; n_pad = the store's row stride
    extern __shared__ float tile[];  // [64][d + 1]
    const int g = blockIdx.y;
    const int64_t blk = blk0 + blockIdx.x;
    const int64_t i0 = blk * kBlock;
    const int ld = d + 1;
    const int64_t rem = n - i0;
    const int keys = rem <= 0 ? 0 : (rem < kBlock ? (int)rem : kBlock);  // real keys in this block

    // Stage the tile: rows [i0, i0 + keys) are contiguous in K.
    const int64_t base = ((int64_t)g * rows + (i0 - key0)) * d;
    for (int e = threadIdx.x; e < kBlock * d; e += blockDim.x) {
        int r = e / d, c = e - r * d;
        float x = 0.0f;
        if (r < keys) {
            if (k_dtype == FATHOM_BF16)
                x = __uint_as_float((uint32_t)static_cast<const uint16_t*>(K)[base + e] << 16);
            else
                x = static_cast<const float*>(K)[base + e];
        }
        tile[r * ld + c] = x;
    }
    __syncthreads();

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t words = n_pad / 32, nblk = n_pad / kBlock;
    const bool v0 = lane < keys, v1 = lane + 32 < keys;
    for (int c = warp; c < d; c += kWarps) {
        float x0 = tile[lane * ld + c], x1 = tile[(lane + 32) * ld + c];
        float amax = fmaxf(v0 ? fabsf(x0) : 0.0f, v1 ? fabsf(x1) : 0.0f);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        const __half dh = __float2half_rn(amax * 0.125f);   // amax/8, exact scaling then one rounding
        const double delta = (double)__half2float(dh);
        int code0 = 8, code1 = 8;
        if (delta != 0.0) {
            // floor of the exact quotient: the fp64 quotient of an fp32 and an
            // fp16 value never rounds across an integer.
            double u0 = floor((double)x0 / delta), u1 = floor((double)x1 / delta);
            code0 = (int)fmin(fmax(u0, -8.0), 7.0) + 8;
            code1 = (int)fmin(fmax(u1, -8.0), 7.0) + 8;
        }
        if (!v0) code0 = 0;   // padding keys: all plane bits 0
        if (!v1) code1 = 0;
        uint32_t w[8];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            w[2 * j] = __ballot_sync(0xffffffffu, (code0 >> (3 - j)) & 1);
            w[2 * j + 1] = __ballot_sync(0xffffffffu, (code1 >> (3 - j)) & 1);
        }
        if (lane < 8) {
            int j = lane >> 1, h = lane & 1;
            uint32_t word = w[0];
#pragma unroll
            for (int e = 1; e < 8; ++e)
                if (lane == e) word = w[e];
            planes[(((int64_t)g * d + c) * 4 + j) * words + blk * 2 + h] = word;
        }
        if (lane == 0) scales[((int64_t)g * d + c) * nblk + blk] = __half_as_ushort(dh);
    }
}

}  // namespace

cudaError_t launch_pack_blocks(const void* K, int k_dtype, int Hkv, int64_t rows, int64_t key0, int64_t blk0,
                               int64_t blk1, int64_t n, int d, int64_t n_pad, uint32_t* planes, uint16_t* scales,
                               cudaStream_t stream) {
    if (blk1 <= blk0) return cudaSuccess;
    dim3 grid((unsigned)(blk1 - blk0), (unsigned)Hkv);
    size_t smem = sizeof(float) * kBlock * (d + 1);
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(pack_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    pack_kernel<<<grid, kWarps * 32, smem, stream>>>(K, k_dtype, rows, key0, blk0, n, d, n_pad, planes, scales);
    return cudaGetLastError();
}

cudaError_t launch_pack(const void* K, int k_dtype, int Hkv, int64_t n, int d, uint32_t* planes,
                        uint16_t* scales, cudaStream_t stream) {
    const int64_t n_pad = n_pad_of(n);
    return launch_pack_blocks(K, k_dtype, Hkv, n, 0, 0, n_pad / kBlock, n, d, n_pad, planes, scales, stream);
}

}  // namespace fathom
