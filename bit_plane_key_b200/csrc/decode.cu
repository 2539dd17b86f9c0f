// One decode step of one layer as a single call: depths, scan, top-k and
// exact attention (the whole method of the ai-feeds.com summary, 方法:
// 输入 -> 关键模块 2-5 -> 输出), pipelined over groups of KV heads.
//
// The KV heads of a layer are independent problems.  The scan of group i+1
// runs on the caller's stream while the top-k and attention of group i run on
// an auxiliary stream of the library, so the host-link-bound scan, the
// HBM-bound top-k and the link-bound row gather overlap instead of queueing.
// The auxiliary stream is forked from and joined back to the caller's stream
// with events, so the whole step is ordered on the caller's stream and can be
// captured into a CUDA graph.  With one group the step is the plain sequence
// depths -> scan -> top-k -> attention on the caller's stream, each launch
// made with programmatic serialization, so that it is scheduled while the
// kernel before it finishes (every kernel waits for its predecessor's
// results before it reads anything).
//
// Every kernel is one of the separate entry points' kernels, launched on a
// slice of the same arrays, so the results equal fathom_alloc_depths +
// fathom_scan_topk + fathom_sparse_attend bit for bit.
#include <mutex>

#include "fathom_internal.cuh"

namespace fathom {
namespace {

constexpr int kMaxDevices = 64;
constexpr int kMaxGroups = 64;

struct Aux {
    unsigned long long ctx = 0;             // id of the context the handles belong to
    cudaStream_t stream = nullptr;
    cudaEvent_t scanned[kMaxGroups] = {};   // group i's scores are written
    cudaEvent_t done = nullptr;             // the auxiliary stream's work is finished
};
Aux g_aux[kMaxDevices];
std::mutex g_aux_mu;

// The current device's auxiliary stream and events, created on first use in
// each context (after cudaDeviceReset the old handles are gone with their
// context, and new ones are made).  Calls on one device share them: steps
// issued concurrently from several host threads serialise their top-k and
// attention on the one auxiliary stream.
Aux* aux_for_device() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(g_aux_mu);
    Aux& a = g_aux[dev];
    const unsigned long long id = current_context_id();
    // a new set on first use, and when the context is known to have changed
    // (when the driver cannot name the context, the first set is kept)
    if (!a.stream || (id != 0 && id != a.ctx)) {
        Aux fresh;
        cudaStream_t s = nullptr;
        if (cudaStreamCreateWithFlags(&s, cudaStreamNonBlocking) != cudaSuccess) return nullptr;
        for (int i = 0; i < kMaxGroups; ++i)
            if (cudaEventCreateWithFlags(&fresh.scanned[i], cudaEventDisableTiming) != cudaSuccess) return nullptr;
        if (cudaEventCreateWithFlags(&fresh.done, cudaEventDisableTiming) != cudaSuccess) return nullptr;
        fresh.stream = s;
        fresh.ctx = current_context_id();   // creating the stream made the context if there was none
        a = fresh;
    }
    return &a;
}

}  // namespace

size_t decode_workspace_bytes(int64_t n, int Hq, int groups, int k) {
    return scan_topk_layout(n, Hq, Hq / groups, k).total;
}

cudaError_t launch_decode(const uint32_t* planes, const uint16_t* scales, int store_host, int Hkv, int d, int64_t n,
                          int64_t n_pad, const void* q, int q_dtype, const float* sigma2, int Hq, int budget, int fixed_r, int k,
                          const uint16_t* K_rows, const uint16_t* V_rows, int64_t row_stride, int64_t rows_n,
                          int rows_host, int groups, uint8_t* depths, int32_t* idx, float* top_scores, float* out,
                          void* workspace, cudaStream_t stream) {
    const int hkv_g = Hkv / groups, hq_g = Hq / groups;
    const size_t q_elt = (q_dtype == FATHOM_BF16) ? 2 : 4;
    float* scores = static_cast<float*>(workspace);
    const int64_t ld = n_pad_of(n);   // score row stride; n_pad is the store's row stride
    const ScanTopkLayout lay = scan_topk_layout(n, Hq, hq_g, k);
    uint32_t* bmax = reinterpret_cast<uint32_t*>(static_cast<char*>(workspace) + lay.bmax_off);
    void* topk_ws = static_cast<char*>(workspace) + lay.topk_off;

    cudaError_t e = launch_depths(q, q_dtype, sigma2, Hq, Hkv, d, budget, fixed_r, depths, stream);
    if (e != cudaSuccess) return e;
    if (groups == 1) {
        e = launch_scan(planes, scales, Hkv, d, n, n_pad, q, q_dtype, depths, Hq, scores, stream, bmax,
                        store_host != 0, true);
        if (e == cudaSuccess)
            e = launch_topk_blocks(scores, bmax, n, ld, Hq, k, idx, top_scores, topk_ws, stream, true);
        if (e == cudaSuccess)
            e = launch_attend(q, q_dtype, K_rows, V_rows, row_stride, idx, Hq, Hkv, rows_n, d, k, rows_host, out,
                              stream, 0, nullptr, true);
        return e;
    }
    Aux* aux = aux_for_device();
    if (!aux) return cudaErrorUnknown;
    cudaError_t first = cudaSuccess;
    for (int i = 0; i < groups; ++i) {
        const int g0 = i * hkv_g, h0 = i * hq_g;
        const void* qi = static_cast<const char*>(q) + q_elt * (size_t)h0 * d;
        float* si = scores + (size_t)h0 * ld;
        uint32_t* bi = bmax + (size_t)h0 * (ld / kBlock);
        e = launch_scan(planes + (size_t)g0 * d * 4 * (n_pad / 32), scales + (size_t)g0 * d * (n_pad / kBlock),
                        hkv_g, d, n, n_pad, qi, q_dtype, depths + (size_t)h0 * d, hq_g, si, stream, bi,
                        store_host != 0);
        if (e == cudaSuccess) e = cudaEventRecord(aux->scanned[i], stream);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(aux->stream, aux->scanned[i], 0);
        int32_t* ii = idx + (size_t)h0 * k;
        float* ti = top_scores ? top_scores + (size_t)h0 * k : nullptr;
        const size_t rows_off = (size_t)g0 * rows_n * row_stride;
        if (e == cudaSuccess) e = launch_topk_blocks(si, bi, n, ld, hq_g, k, ii, ti, topk_ws, aux->stream);
        if (e == cudaSuccess)
            e = launch_attend(qi, q_dtype, K_rows + rows_off, V_rows + rows_off, row_stride, ii, hq_g, hkv_g, rows_n,
                              d, k, rows_host, out + (size_t)h0 * d, aux->stream, 0, nullptr, true);
        if (e != cudaSuccess) {
            first = e;
            break;
        }
    }
    // join the auxiliary stream back, also after a failed launch, so that the
    // caller's stream (or its capture) is left whole
    cudaError_t j = cudaEventRecord(aux->done, aux->stream);
    if (j == cudaSuccess) j = cudaStreamWaitEvent(stream, aux->done, 0);
    return first != cudaSuccess ? first : j;
}

}  // namespace fathom
