// Scan + top-k for callers that cannot allocate device memory.
//
// fathom_scan_topk needs a workspace (the fp32 scores of every key and the
// top-k buffers) that the caller allocates.  Some callers cannot do that:
// an inference engine whose device memory is all handed out up front to its
// own pool, a plug-in that runs inside a host program which forbids
// cudaMalloc/cudaFree on its serving path (they synchronise the device and
// stall every stream), or a decode step issued from a context where
// allocation is simply not available.  For them, fathom_scan_topk_noalloc
// runs the same kernels with the workspace taken from one fixed-size array
// that lives in this library's own device memory.
//
// The array is a file-scope __device__ variable, so every GPU on which the
// library is loaded holds its kNoallocScratchBytes until the process exits.
// Host code must not pass the array's name to a kernel: on the host that
// name is only a stand-in, not a device address.  The first call on a device
// looks the device address up with cudaGetSymbolAddress (with that device
// current) and caches it together with the id of the current context; a later
// call in another context (after cudaDeviceReset) looks it up again.  Make the
// first call on a device, and the first after a reset, before any stream
// capture.
// All calls share the one array and it keeps the previous call's contents:
// the top-k clears its own counters and histograms at the start of every
// call, and the scan overwrites every score it later reads.  Calls whose
// work overlaps on the GPU (two streams, or two host threads) race on the
// array; serialise them.
#include <mutex>

#include "fathom_internal.cuh"

namespace fathom {
namespace {

constexpr size_t kNoallocScratchBytes = size_t(24) << 20;   // 24 MiB
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];

CtxCache g_scratch_dev[kMaxDevices];
std::mutex g_scratch_mu;

// Device address of the scratch array on the current device: looked up with
// cudaGetSymbolAddress, with that device current, on the first call in each
// context, and cached with the context's id.
void* scratch_address() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    return g_scratch_dev[dev].get(g_noalloc_scratch);
}

}  // namespace
}  // namespace fathom

using namespace fathom;

extern "C" {

size_t fathom_noalloc_scratch_bytes(void) { return kNoallocScratchBytes; }

int fathom_scan_topk_noalloc(const fathom_store* store, const void* q, int q_dtype, const uint8_t* depths,
                             int n_q_heads, int k, int32_t* idx, float* top_scores, fathom_stream_t stream) {
    if (!store || !q || !depths || !idx || !heads_ok(n_q_heads, store->n_kv_heads)) return FATHOM_EINVAL;
    if (q_dtype != FATHOM_F32 && q_dtype != FATHOM_BF16) return FATHOM_EINVAL;
    if (k < 1 || k > store->n || k > kMaxTopK || store->n > INT32_MAX) return FATHOM_EINVAL;
    const size_t need = fathom_scan_workspace_bytes(store, n_q_heads, k);
    if (need == 0) return FATHOM_EINVAL;
    if (need > kNoallocScratchBytes) return FATHOM_ENOMEM;   // beyond the fixed scratch array
    const uint32_t* planes;
    const uint16_t* scales;
    int rc = resolve_store(store, &planes, &scales);
    if (rc) return rc;
    if (!is_device(q) || !is_device(depths) || !is_device(idx) || (top_scores && !is_device(top_scores)))
        return FATHOM_EINVAL;
    if (!scan_fits(store->d, n_q_heads, store->n_kv_heads)) return FATHOM_EUNSUPPORTED;
    if (!device_status_ptr()) return FATHOM_ECUDA;
    char* scratch = static_cast<char*>(scratch_address());
    if (!scratch) return FATHOM_ECUDA;
    // same split as fathom_scan_topk: scores [Hq][n_pad_of(n)], block maxima, then the top-k buffers
    float* scores = reinterpret_cast<float*>(scratch);
    const int64_t ld = n_pad_of(store->n);
    const ScanTopkLayout lay = scan_topk_layout(store->n, n_q_heads, n_q_heads, k);
    uint32_t* bmax = reinterpret_cast<uint32_t*>(scratch + lay.bmax_off);
    cudaStream_t s = (cudaStream_t)stream;
    cudaError_t e = launch_scan(planes, scales, store->n_kv_heads, store->d, store->n, store->n_pad, q, q_dtype,
                                depths, n_q_heads, scores, s, bmax, store->host_resident != 0);
    if (e != cudaSuccess) return FATHOM_ECUDA;
    return to_status(launch_topk_blocks(scores, bmax, store->n, ld, n_q_heads, k, idx, top_scores,
                                        scratch + lay.topk_off, s, true));
}

}  // extern "C"
