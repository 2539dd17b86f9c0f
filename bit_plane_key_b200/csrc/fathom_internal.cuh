// Internal declarations shared by the CUDA translation units of libfathom.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "fathom.h"

namespace fathom {

constexpr int kBlock = 64;     // tokens per shared block scale
constexpr int kPad = 1024;     // key padding granule of the store: plane rows start 128-byte aligned
constexpr int kMaxD = 256;     // largest supported head dimension
constexpr int kMaxTopK = 4096; // largest supported k
constexpr size_t kMaxSmem = 227 * 1024;  // opt-in shared memory per CTA on sm_100

__host__ __device__ inline int64_t n_pad_of(int64_t n) { return ((n + kPad - 1) / kPad) * kPad; }

// Keys per CTA of the scan; the last tile of a store may hold kScanTile / 2
// keys (n_pad_of(n) is a multiple of 1024).
constexpr int kScanTile = 2048;
__host__ __device__ inline int64_t scan_tiles(int64_t n) { return (n_pad_of(n) + kScanTile - 1) / kScanTile; }

// Per-device status word (FATHOM_DEV_* bits); its device address is passed
// to every kernel that can set a bit.
unsigned int* device_status_ptr();

// Unique id of the calling thread's current CUDA context (the driver's
// cuCtxGetId), 0 when there is none or the driver cannot say.  A device reset
// ends the context, and the next one has a new id.
unsigned long long current_context_id();

// The device address of a __device__ variable, looked up once per context:
// cached with the id of the context it was looked up in, and looked up again
// when the current context differs (after cudaDeviceReset the module is
// loaded anew and the variable may move).  Callers hold their own lock.
struct CtxCache {
    unsigned long long ctx = 0;
    void* ptr = nullptr;
    void* get(const void* symbol);
};

// Programmatic dependent launch.  A kernel of the path launched with the
// attribute is scheduled as the CTAs of the kernel before it in the stream
// exit, instead of after that whole grid has completed; every kernel of the
// path calls pdl_wait() before its first access to global memory (it returns
// once the kernel before has completed and its writes are visible, at once
// for a launch without the attribute).  The kernels release their dependents
// only by exiting: an early release (griddepcontrol.launch_dependents at a
// kernel's start) let the next grid's CTAs take SM space during the scan and
// made the n = 131072 decode step slower (114 against 109 us on B200).
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// cudaLaunchKernelEx with the programmatic-serialization attribute when pdl,
// and a cluster of `cluster` CTAs along x when cluster > 1 (kernels whose
// cluster size is fixed at compile time pass 1).
template <typename... KArgs, typename... Args>
cudaError_t launch_ex(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream, bool pdl,
                      int cluster, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    int na = 0;
    if (pdl) {
        attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[na].val.programmaticStreamSerializationAllowed = 1;
        ++na;
    }
    if (cluster > 1) {
        attr[na].id = cudaLaunchAttributeClusterDimension;
        attr[na].val.clusterDim.x = (unsigned)cluster;
        attr[na].val.clusterDim.y = 1;
        attr[na].val.clusterDim.z = 1;
        ++na;
    }
    cfg.attrs = attr;
    cfg.numAttrs = (unsigned)na;
    return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

// Host-side argument checks shared by the entry points (api.cu).
enum class Where { kDevice, kHostPinned, kOther };
Where classify(const void* p, const void** dev);
bool is_device(const void* p);
bool dims_ok(int Hkv, int d);
bool heads_ok(int Hq, int Hkv);
bool scan_fits(int d, int Hq, int Hkv);
int to_status(cudaError_t e);
int resolve_store(const fathom_store* s, const uint32_t** planes, const uint16_t** scales);

// Host launchers (each enqueues on `stream`; arguments already validated).
cudaError_t launch_pack(const void* K, int k_dtype, int Hkv, int64_t n, int d, uint32_t* planes,
                        uint16_t* scales, cudaStream_t stream);
// (re)packs blocks [blk0, blk1) of a store of row stride n_pad holding n keys,
// from K = keys [key0, key0 + rows) of every KV head
cudaError_t launch_pack_blocks(const void* K, int k_dtype, int Hkv, int64_t rows, int64_t key0, int64_t blk0,
                               int64_t blk1, int64_t n, int d, int64_t n_pad, uint32_t* planes, uint16_t* scales,
                               cudaStream_t stream);
cudaError_t launch_depths(const void* q, int q_dtype, const float* sigma2, int Hq, int Hkv, int d,
                          int budget, int fixed_r, uint8_t* depths, cudaStream_t stream, int pooled = 0);
size_t scan_smem_bytes(int d, int G);
// bmax (optional): the max score of every 64-key block as an ordered key,
// [Hq][n_pad_of(n)/64], for launch_topk_blocks; host: the store is in
// page-locked host memory (planes and scales are its device-mapped addresses)
cudaError_t launch_scan(const uint32_t* planes, const uint16_t* scales, int Hkv, int d, int64_t n,
                        int64_t n_pad, const void* q, int q_dtype, const uint8_t* depths, int Hq,
                        float* scores, cudaStream_t stream, uint32_t* bmax, bool host, bool pdl = false);
size_t topk_workspace_bytes(int64_t n, int rows, int k);

// Where the score rows are: rows are grouped in sets of `rows_per_set`
// (the query heads of one session); row r of set s starts at
// base[s] + (r % rows_per_set) * ld[s] and has n[s] valid scores.
constexpr int kMaxSets = 64;
struct RowMap {
    int rows_per_set;
    int nsets;
    int64_t max_n;
    int64_t base[kMaxSets];
    int64_t ld[kMaxSets];
    int64_t n[kMaxSets];
};
cudaError_t launch_topk(const float* scores, int64_t n, int64_t ld, int rows, int k, int32_t* idx,
                        float* top_scores, void* ws, cudaStream_t stream);
// top-k of score rows whose 64-key block maxima (ordered keys, [row][ld/64])
// the scan wrote alongside; ld a multiple of 64 and base offsets too
size_t topk_blocks_workspace_bytes(int rows);

// top-k buffers for either path of launch_topk_blocks
inline size_t topk_any_workspace_bytes(int64_t n, int rows, int k) {
    const size_t a = topk_workspace_bytes(n, rows, k), b = topk_blocks_workspace_bytes(rows);
    return a > b ? a : b;
}

// Workspace of a scan followed by top-k: scores f32 [Hq][n_pad_of(n)], block
// maxima u32 [Hq][n_pad_of(n)/64], the top-k buffers for `topk_rows` rows;
// each part 256-byte aligned.
struct ScanTopkLayout {
    size_t bmax_off, topk_off, total;
};
inline ScanTopkLayout scan_topk_layout(int64_t n, int Hq, int topk_rows, int k) {
    const size_t ld = (size_t)n_pad_of(n);
    const size_t sb = (sizeof(float) * (size_t)Hq * ld + 255) & ~size_t(255);
    const size_t bb = (sizeof(uint32_t) * (size_t)Hq * (ld / kBlock) + 255) & ~size_t(255);
    return {sb, sb + bb, sb + bb + topk_any_workspace_bytes(n, topk_rows, k)};
}
// pdl: launch the first kernel with programmatic serialization (the kernel
// before it in the stream is one of the path's)
cudaError_t launch_topk_blocks(const float* scores, const uint32_t* bmax, int64_t n, int64_t ld, int rows, int k,
                               int32_t* idx, float* top_scores, void* ws, cudaStream_t stream, bool pdl = false);
cudaError_t launch_topk_blocks_map(const float* scores, const uint32_t* bmax, const RowMap& map, int rows, int k,
                                   int32_t* idx, float* top_scores, void* ws, cudaStream_t stream, bool pdl = false);
cudaError_t launch_topk_merge(const float* cand_scores, const int32_t* cand_idx, int rows, int n_cand, int k,
                              int32_t* idx, float* top_scores, void* ws, cudaStream_t stream);
cudaError_t launch_topk_map(const float* scores, const RowMap& map, int rows, int k, int32_t* idx,
                            float* top_scores, void* ws, cudaStream_t stream);

// Sessions of a batched scan: session s owns tiles [tile0[s], tile0[s+1]) of
// the flattened grid and writes scores [Hq][n_pad[s]] at score_base[s].
struct SessionMap {
    int nsess;
    const uint32_t* planes[kMaxSets];
    const uint16_t* scales[kMaxSets];
    int64_t n[kMaxSets];
    int64_t n_pad[kMaxSets];
    int64_t score_base[kMaxSets];
    int tile0[kMaxSets + 1];
};
// host: some session's store is in page-locked host memory
cudaError_t launch_scan_batched(const SessionMap& map, int Hkv, int d, const void* q, int q_dtype,
                                const uint8_t* depths, int Hq, float* scores, cudaStream_t stream,
                                uint32_t* bmax, bool host);
size_t decode_workspace_bytes(int64_t n, int Hq, int groups, int k);
cudaError_t launch_decode(const uint32_t* planes, const uint16_t* scales, int store_host, int Hkv, int d, int64_t n,
                          int64_t n_pad, const void* q, int q_dtype, const float* sigma2, int Hq, int budget, int fixed_r, int k,
                          const uint16_t* K_rows, const uint16_t* V_rows, int64_t row_stride, int64_t rows_n,
                          int rows_host, int groups, uint8_t* depths, int32_t* idx, float* top_scores, float* out,
                          void* workspace, cudaStream_t stream);
// key0 / parts: the rows hold keys [key0, key0 + n) of a key range split
// across GPUs; with parts non-null the kernel writes per-head partials
// [Hq][d + 2] (o relative to m, then m, l) instead of out.
cudaError_t launch_attend(const void* q, int q_dtype, const uint16_t* K_rows, const uint16_t* V_rows,
                          int64_t row_stride, const int32_t* idx, int Hq, int Hkv, int64_t n, int d, int k, int sort_rows, float* out,
                          cudaStream_t stream, int64_t key0 = 0, float* parts = nullptr, bool pdl = false);
cudaError_t launch_attend_merge(const float* parts, int world, int Hq, int d, float* out, cudaStream_t stream);

cudaError_t launch_probe(const void* src, size_t bytes, unsigned long long* sink, int ctas,
                         cudaStream_t stream);

// fp32 <-> order-preserving u32: a > b as real numbers  <=>  key(a) > key(b),
// and a == b  <=>  key(a) == key(b) (-0 and +0 share the key of +0).
__device__ __forceinline__ uint32_t float_to_ordered(float f) {
    uint32_t u = __float_as_uint(f);
    if (u == 0x80000000u) u = 0u;
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float ordered_to_float(uint32_t k) {
    uint32_t u = (k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k;
    return __uint_as_float(u);
}

__device__ __forceinline__ float load_q(const void* q, int dtype, int64_t i) {
    if (dtype == FATHOM_BF16) {
        uint16_t b = static_cast<const uint16_t*>(q)[i];
        return __uint_as_float(static_cast<uint32_t>(b) << 16);
    }
    return static_cast<const float*>(q)[i];
}

}  // namespace fathom
