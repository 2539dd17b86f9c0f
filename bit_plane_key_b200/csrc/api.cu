// C-ABI entry points of libfathom: argument checks, pointer classification,
// kernel launches.  Declarations and contracts: include/fathom.h.
#include <cuda.h>

#include <mutex>

#include "fathom_internal.cuh"

namespace fathom {
namespace {

// Status word written by kernels (FATHOM_DEV_* bits); one per device.
__device__ unsigned int g_status;

constexpr int kMaxDevices = 64;
CtxCache g_status_ptr[kMaxDevices];
std::mutex g_status_mu;

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);
CtxGetCurrentFn g_ctx_get_current = nullptr;
CtxGetIdFn g_ctx_get_id = nullptr;
std::once_flag g_ctx_fn_once;

}  // namespace

unsigned long long current_context_id() {
    // the driver's functions through the runtime, so that the library needs
    // no link to libcuda (it loads on machines without a GPU driver)
    std::call_once(g_ctx_fn_once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult r;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &r) == cudaSuccess &&
            r == cudaDriverEntryPointSuccess)
            g_ctx_get_current = reinterpret_cast<CtxGetCurrentFn>(f);
        f = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &f, cudaEnableDefault, &r) == cudaSuccess &&
            r == cudaDriverEntryPointSuccess)
            g_ctx_get_id = reinterpret_cast<CtxGetIdFn>(f);
        cudaGetLastError();
    });
    if (!g_ctx_get_current || !g_ctx_get_id) return 0;
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (g_ctx_get_current(&ctx) != CUDA_SUCCESS || !ctx) return 0;
    if (g_ctx_get_id(ctx, &id) != CUDA_SUCCESS) return 0;
    return id;
}

void* CtxCache::get(const void* symbol) {
    const unsigned long long id = current_context_id();
    if (ptr && id != 0 && id == ctx) return ptr;
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, symbol) != cudaSuccess) {
        cudaGetLastError();
        return nullptr;
    }
    ptr = p;
    ctx = current_context_id();   // the look-up creates the context if there was none
    return ptr;
}

// Where a pointer lives.  Returns the device-usable address through `dev`.
Where classify(const void* p, const void** dev) {
    cudaPointerAttributes a;
    cudaError_t e = cudaPointerGetAttributes(&a, p);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return Where::kOther;
    }
    if (a.type == cudaMemoryTypeDevice || a.type == cudaMemoryTypeManaged) {
        if (dev) *dev = p;
        return Where::kDevice;
    }
    if (a.type == cudaMemoryTypeHost && a.devicePointer != nullptr) {
        if (dev) *dev = a.devicePointer;
        return Where::kHostPinned;
    }
    return Where::kOther;
}

bool is_device(const void* p) { return p != nullptr && classify(p, nullptr) == Where::kDevice; }

bool dims_ok(int Hkv, int d) { return Hkv >= 1 && d >= 32 && d <= kMaxD && d % 32 == 0; }

bool heads_ok(int Hq, int Hkv) {
    if (Hq < 1 || Hkv < 1 || Hq % Hkv) return false;
    int G = Hq / Hkv;
    return G == 1 || G == 2 || G == 4 || G == 8;
}

bool scan_fits(int d, int Hq, int Hkv) { return scan_smem_bytes(d, Hq / Hkv) <= kMaxSmem; }

int to_status(cudaError_t e) { return e == cudaSuccess ? FATHOM_OK : FATHOM_ECUDA; }

// Resolve a store's arrays to device-usable addresses, checking residency.
int resolve_store(const fathom_store* s, const uint32_t** planes, const uint16_t** scales) {
    if (!s || !s->planes || !s->scales) return FATHOM_EINVAL;
    if (!dims_ok(s->n_kv_heads, s->d) || s->n < 1 || s->n_pad < n_pad_of(s->n) || s->n_pad % kPad)
        return FATHOM_EINVAL;
    if ((reinterpret_cast<uintptr_t>(s->planes) & 15) || (reinterpret_cast<uintptr_t>(s->scales) & 15))
        return FATHOM_EINVAL;
    const void* dp = nullptr;
    const void* ds = nullptr;
    Where wp = classify(s->planes, &dp), ws = classify(s->scales, &ds);
    Where want = s->host_resident ? Where::kHostPinned : Where::kDevice;
    if (wp != want || ws != want) return FATHOM_EINVAL;
    *planes = static_cast<const uint32_t*>(dp);
    *scales = static_cast<const uint16_t*>(ds);
    return FATHOM_OK;
}

unsigned int* device_status_ptr() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(g_status_mu);
    return static_cast<unsigned int*>(g_status_ptr[dev].get(&g_status));
}

}  // namespace fathom

using namespace fathom;

extern "C" {

int64_t fathom_n_pad(int64_t n) { return n < 0 ? 0 : n_pad_of(n); }

size_t fathom_planes_bytes(int n_kv_heads, int d, int64_t n) {
    if (!dims_ok(n_kv_heads, d) || n < 1) return 0;
    return (size_t)n_kv_heads * d * 4 * (size_t)(n_pad_of(n) / 8);
}

size_t fathom_scales_bytes(int n_kv_heads, int d, int64_t n) {
    if (!dims_ok(n_kv_heads, d) || n < 1) return 0;
    return (size_t)n_kv_heads * d * (size_t)(n_pad_of(n) / kBlock) * sizeof(uint16_t);
}

int fathom_pack_bitplanes(const void* K, int k_dtype, int n_kv_heads, int64_t n, int d, uint32_t* planes,
                          uint16_t* scales, fathom_stream_t stream) {
    if (!K || !planes || !scales || n < 1 || !dims_ok(n_kv_heads, d)) return FATHOM_EINVAL;
    if (k_dtype != FATHOM_F32 && k_dtype != FATHOM_BF16) return FATHOM_EINVAL;
    if (!is_device(K) || !is_device(planes) || !is_device(scales)) return FATHOM_EINVAL;
    if (!device_status_ptr()) return FATHOM_ECUDA;
    return to_status(launch_pack(K, k_dtype, n_kv_heads, n, d, planes, scales, (cudaStream_t)stream));
}

int fathom_append_keys(fathom_store* store, const void* K_tail, int k_dtype, int64_t n_new, fathom_stream_t stream) {
    if (!store || !K_tail || !store->planes || !store->scales) return FATHOM_EINVAL;
    if (k_dtype != FATHOM_F32 && k_dtype != FATHOM_BF16) return FATHOM_EINVAL;
    const int64_t n_old = store->n;
    if (!dims_ok(store->n_kv_heads, store->d) || n_old < 0 || n_new <= n_old || store->n_pad % kPad ||
        n_pad_of(n_new) > store->n_pad)
        return FATHOM_EINVAL;
    if ((reinterpret_cast<uintptr_t>(store->planes) & 15) || (reinterpret_cast<uintptr_t>(store->scales) & 1))
        return FATHOM_EINVAL;
    const void* dp = nullptr;
    const void* ds = nullptr;
    Where want = store->host_resident ? Where::kHostPinned : Where::kDevice;
    if (classify(store->planes, &dp) != want || classify(store->scales, &ds) != want) return FATHOM_EINVAL;
    if (!is_device(K_tail)) return FATHOM_EINVAL;
    const int64_t tail = (n_old / kBlock) * kBlock;   // first key of the last partial block
    cudaError_t e = launch_pack_blocks(K_tail, k_dtype, store->n_kv_heads, n_new - tail, tail, tail / kBlock,
                                       (n_new + kBlock - 1) / kBlock, n_new, store->d, store->n_pad,
                                       const_cast<uint32_t*>(static_cast<const uint32_t*>(dp)),
                                       const_cast<uint16_t*>(static_cast<const uint16_t*>(ds)), (cudaStream_t)stream);
    if (e != cudaSuccess) return FATHOM_ECUDA;
    store->n = n_new;
    return FATHOM_OK;
}

int fathom_alloc_depths(const void* q, int q_dtype, const float* sigma2, int n_q_heads, int n_kv_heads, int d,
                        int budget_bits, int fixed_r, uint8_t* depths, fathom_stream_t stream) {
    if (!q || !sigma2 || !depths || !dims_ok(n_kv_heads, d) || n_q_heads < 1 || n_q_heads % n_kv_heads)
        return FATHOM_EINVAL;
    if (q_dtype != FATHOM_F32 && q_dtype != FATHOM_BF16) return FATHOM_EINVAL;
    if (budget_bits < 0 || fixed_r < 0 || fixed_r > d) return FATHOM_EINVAL;
    if (!is_device(q) || !is_device(sigma2) || !is_device(depths)) return FATHOM_EINVAL;
    return to_status(launch_depths(q, q_dtype, sigma2, n_q_heads, n_kv_heads, d, budget_bits, fixed_r, depths,
                                   (cudaStream_t)stream));
}

int fathom_alloc_depths_pooled(const void* q, int q_dtype, const float* sigma2, int n_q_heads, int n_kv_heads,
                               int d, int budget_bits, uint8_t* depths, fathom_stream_t stream) {
    if (!q || !sigma2 || !depths || !dims_ok(n_kv_heads, d) || n_q_heads < 1 || n_q_heads % n_kv_heads)
        return FATHOM_EINVAL;
    if (q_dtype != FATHOM_F32 && q_dtype != FATHOM_BF16) return FATHOM_EINVAL;
    if (budget_bits < 0) return FATHOM_EINVAL;
    if (!is_device(q) || !is_device(sigma2) || !is_device(depths)) return FATHOM_EINVAL;
    return to_status(launch_depths(q, q_dtype, sigma2, n_q_heads, n_kv_heads, d, budget_bits, 0, depths,
                                   (cudaStream_t)stream, 1));
}

int fathom_scan_scores(const fathom_store* store, const void* q, int q_dtype, const uint8_t* depths,
                       int n_q_heads, float* scores, uint32_t* block_max, fathom_stream_t stream) {
    const uint32_t* planes;
    const uint16_t* scales;
    int rc = resolve_store(store, &planes, &scales);
    if (rc) return rc;
    if (!q || !depths || !scores || !heads_ok(n_q_heads, store->n_kv_heads)) return FATHOM_EINVAL;
    if (q_dtype != FATHOM_F32 && q_dtype != FATHOM_BF16) return FATHOM_EINVAL;
    if (!is_device(q) || !is_device(depths) || !is_device(scores) || (block_max && !is_device(block_max)))
        return FATHOM_EINVAL;
    if (!scan_fits(store->d, n_q_heads, store->n_kv_heads)) return FATHOM_EUNSUPPORTED;
    if (!device_status_ptr()) return FATHOM_ECUDA;
    return to_status(launch_scan(planes, scales, store->n_kv_heads, store->d, store->n, store->n_pad, q, q_dtype,
                                 depths, n_q_heads, scores, (cudaStream_t)stream, block_max,
                                 store->host_resident != 0));
}

size_t fathom_topk_workspace_bytes(int64_t n, int n_rows, int k) {
    if (n < 1 || n_rows < 1 || k < 1 || k > kMaxTopK) return 0;
    return topk_any_workspace_bytes(n, n_rows, k);   // either path
}

int fathom_topk(const float* scores, const uint32_t* block_max, int64_t n, int64_t ld, int n_rows, int k,
                int32_t* idx, float* top_scores, void* workspace, size_t workspace_bytes, fathom_stream_t stream) {
    if (!scores || !idx || !workspace || n < 1 || ld < n || n_rows < 1 || k < 1 || k > n || k > kMaxTopK ||
        n > INT32_MAX)
        return FATHOM_EINVAL;
    if (block_max && ld % kBlock) return FATHOM_EINVAL;
    if (reinterpret_cast<uintptr_t>(workspace) & 255) return FATHOM_EINVAL;
    if (workspace_bytes < fathom_topk_workspace_bytes(n, n_rows, k)) return FATHOM_ENOMEM;
    if (!is_device(scores) || !is_device(idx) || !is_device(workspace) || (top_scores && !is_device(top_scores)) ||
        (block_max && !is_device(block_max)))
        return FATHOM_EINVAL;
    if (!device_status_ptr()) return FATHOM_ECUDA;
    cudaStream_t s = (cudaStream_t)stream;
    if (block_max)
        return to_status(launch_topk_blocks(scores, block_max, n, ld, n_rows, k, idx, top_scores, workspace, s));
    return to_status(launch_topk(scores, n, ld, n_rows, k, idx, top_scores, workspace, s));
}

int fathom_topk_merge(const float* cand_scores, const int32_t* cand_idx, int n_rows, int n_cand, int k, int32_t* idx,
                      float* top_scores, void* workspace, size_t workspace_bytes, fathom_stream_t stream) {
    if (!cand_scores || !cand_idx || !idx || !workspace || n_rows < 1 || n_cand < 1 || k < 1 || k > n_cand ||
        k > kMaxTopK)
        return FATHOM_EINVAL;
    if (reinterpret_cast<uintptr_t>(workspace) & 255) return FATHOM_EINVAL;
    if (workspace_bytes < topk_workspace_bytes(n_cand, n_rows, k)) return FATHOM_ENOMEM;
    if (!is_device(cand_scores) || !is_device(cand_idx) || !is_device(idx) || !is_device(workspace) ||
        (top_scores && !is_device(top_scores)))
        return FATHOM_EINVAL;
    if (!device_status_ptr()) return FATHOM_ECUDA;
    return to_status(launch_topk_merge(cand_scores, cand_idx, n_rows, n_cand, k, idx, top_scores, workspace,
                                       (cudaStream_t)stream));
}

size_t fathom_scan_workspace_bytes(const fathom_store* store, int n_q_heads, int k) {
    if (!store || n_q_heads < 1 || k < 1 || k > kMaxTopK || store->n < 1) return 0;
    return scan_topk_layout(store->n, n_q_heads, n_q_heads, k).total;
}

int fathom_scan_topk(const fathom_store* store, const void* q, int q_dtype, const uint8_t* depths, int n_q_heads,
                     int k, int32_t* idx, float* top_scores, void* workspace, size_t workspace_bytes,
                     fathom_stream_t stream) {
    const uint32_t* planes;
    const uint16_t* scales;
    int rc = resolve_store(store, &planes, &scales);
    if (rc) return rc;
    if (!q || !depths || !idx || !workspace || !heads_ok(n_q_heads, store->n_kv_heads)) return FATHOM_EINVAL;
    if (q_dtype != FATHOM_F32 && q_dtype != FATHOM_BF16) return FATHOM_EINVAL;
    if (k < 1 || k > store->n || k > kMaxTopK || store->n > INT32_MAX) return FATHOM_EINVAL;
    if (reinterpret_cast<uintptr_t>(workspace) & 255) return FATHOM_EINVAL;
    if (workspace_bytes < fathom_scan_workspace_bytes(store, n_q_heads, k)) return FATHOM_ENOMEM;
    if (!scan_fits(store->d, n_q_heads, store->n_kv_heads)) return FATHOM_EUNSUPPORTED;
    if (!is_device(q) || !is_device(depths) || !is_device(idx) || !is_device(workspace) ||
        (top_scores && !is_device(top_scores)))
        return FATHOM_EINVAL;
    if (!device_status_ptr()) return FATHOM_ECUDA;
    float* scores = static_cast<float*>(workspace);
    const int64_t ld = n_pad_of(store->n);   // score row stride
    const ScanTopkLayout lay = scan_topk_layout(store->n, n_q_heads, n_q_heads, k);
    uint32_t* bmax = reinterpret_cast<uint32_t*>(static_cast<char*>(workspace) + lay.bmax_off);
    cudaStream_t s = (cudaStream_t)stream;
    cudaError_t e = launch_scan(planes, scales, store->n_kv_heads, store->d, store->n, store->n_pad, q, q_dtype,
                                depths, n_q_heads, scores, s, bmax, store->host_resident != 0);
    if (e != cudaSuccess) return FATHOM_ECUDA;
    e = launch_topk_blocks(scores, bmax, store->n, ld, n_q_heads, k, idx, top_scores,
                           static_cast<char*>(workspace) + lay.topk_off, s, true);
    return to_status(e);
}

namespace {
inline size_t a256(size_t x) { return (x + 255) & ~size_t(255); }

// Checks a batch of stores and returns the bytes of all sessions' scores
// (0 on an invalid batch).
size_t batched_score_bytes(const fathom_store* stores, int S, int Hq) {
    if (!stores || S < 1 || S > kMaxSets) return 0;
    size_t total = 0;
    for (int s = 0; s < S; ++s) {
        const fathom_store& st = stores[s];
        if (st.n < 1 || st.n_kv_heads != stores[0].n_kv_heads || st.d != stores[0].d) return 0;
        total += a256(sizeof(float) * (size_t)Hq * (size_t)n_pad_of(st.n));
    }
    return total;
}
}  // namespace

size_t fathom_scan_batched_workspace_bytes(const fathom_store* stores, int n_sessions, int n_q_heads, int k) {
    if (n_q_heads < 1 || k < 1 || k > kMaxTopK) return 0;
    const size_t sb = batched_score_bytes(stores, n_sessions, n_q_heads);
    if (sb == 0) return 0;
    int64_t max_n = 0;
    for (int s = 0; s < n_sessions; ++s) max_n = stores[s].n > max_n ? stores[s].n : max_n;
    return sb + a256(sb / kBlock) + topk_any_workspace_bytes(max_n, n_sessions * n_q_heads, k);
}

int fathom_scan_topk_batched(const fathom_store* stores, int n_sessions, const void* q, int q_dtype,
                             const uint8_t* depths, int n_q_heads, int k, int32_t* idx, float* top_scores,
                             void* workspace, size_t workspace_bytes, fathom_stream_t stream) {
    if (!stores || n_sessions < 1 || n_sessions > kMaxSets || !q || !depths || !idx || !workspace)
        return FATHOM_EINVAL;
    if (q_dtype != FATHOM_F32 && q_dtype != FATHOM_BF16) return FATHOM_EINVAL;
    if (k < 1 || k > kMaxTopK || !heads_ok(n_q_heads, stores[0].n_kv_heads)) return FATHOM_EINVAL;
    if (reinterpret_cast<uintptr_t>(workspace) & 255) return FATHOM_EINVAL;
    const size_t need = fathom_scan_batched_workspace_bytes(stores, n_sessions, n_q_heads, k);
    if (need == 0) return FATHOM_EINVAL;
    if (workspace_bytes < need) return FATHOM_ENOMEM;
    SessionMap sm;
    RowMap rm;
    sm.nsess = n_sessions;
    rm.nsets = n_sessions;
    rm.rows_per_set = n_q_heads;
    rm.max_n = 0;
    int tiles = 0;
    size_t off = 0;
    bool any_host = false;
    for (int s = 0; s < n_sessions; ++s) {
        const fathom_store& st = stores[s];
        any_host = any_host || st.host_resident != 0;
        if (k > st.n || st.n > INT32_MAX) return FATHOM_EINVAL;
        int rc = resolve_store(&st, &sm.planes[s], &sm.scales[s]);
        if (rc) return rc;
        sm.n[s] = st.n;
        sm.n_pad[s] = st.n_pad;
        sm.score_base[s] = (int64_t)(off / sizeof(float));
        sm.tile0[s] = tiles;
        const int64_t t = scan_tiles(st.n);
        if (t > INT32_MAX - tiles) return FATHOM_EINVAL;
        tiles += (int)t;
        rm.base[s] = sm.score_base[s];
        rm.ld[s] = n_pad_of(st.n);
        rm.n[s] = st.n;
        rm.max_n = st.n > rm.max_n ? st.n : rm.max_n;
        off += a256(sizeof(float) * (size_t)n_q_heads * (size_t)n_pad_of(st.n));
    }
    sm.tile0[n_sessions] = tiles;
    if (!is_device(q) || !is_device(depths) || !is_device(idx) || !is_device(workspace) ||
        (top_scores && !is_device(top_scores)))
        return FATHOM_EINVAL;
    if (!scan_fits(stores[0].d, n_q_heads, stores[0].n_kv_heads)) return FATHOM_EUNSUPPORTED;
    if (!device_status_ptr()) return FATHOM_ECUDA;
    float* scores = static_cast<float*>(workspace);
    // block maxima after all sessions' scores: session s's rows at score_base[s] / 64
    uint32_t* bmax = reinterpret_cast<uint32_t*>(static_cast<char*>(workspace) + off);
    cudaStream_t cs = (cudaStream_t)stream;
    cudaError_t e = launch_scan_batched(sm, stores[0].n_kv_heads, stores[0].d, q, q_dtype, depths, n_q_heads, scores,
                                        cs, bmax, any_host);
    if (e != cudaSuccess) return FATHOM_ECUDA;
    return to_status(launch_topk_blocks_map(scores, bmax, rm, n_sessions * n_q_heads, k, idx, top_scores,
                                            static_cast<char*>(workspace) + off + a256(off / kBlock), cs, true));
}

int fathom_sparse_attend(const void* q, int q_dtype, const uint16_t* K_rows, const uint16_t* V_rows,
                         int64_t row_stride, int rows_host_resident, const int32_t* idx, int n_q_heads, int n_kv_heads, int64_t n,
                         int d, int k, float* out, fathom_stream_t stream) {
    if (!q || !K_rows || !V_rows || !idx || !out || n < 1 || k < 1 || !dims_ok(n_kv_heads, d) ||
        !heads_ok(n_q_heads, n_kv_heads))
        return FATHOM_EINVAL;
    if (q_dtype != FATHOM_F32 && q_dtype != FATHOM_BF16) return FATHOM_EINVAL;
    if (d != 32 && d != 64 && d != 128 && d != 256) return FATHOM_EUNSUPPORTED;
    if (row_stride < d || row_stride % 8) return FATHOM_EINVAL;
    if ((reinterpret_cast<uintptr_t>(K_rows) & 15) || (reinterpret_cast<uintptr_t>(V_rows) & 15))
        return FATHOM_EINVAL;
    const void* kd = nullptr;
    const void* vd = nullptr;
    Where want = rows_host_resident ? Where::kHostPinned : Where::kDevice;
    if (classify(K_rows, &kd) != want || classify(V_rows, &vd) != want) return FATHOM_EINVAL;
    if (!is_device(q) || !is_device(idx) || !is_device(out)) return FATHOM_EINVAL;
    if (!device_status_ptr()) return FATHOM_ECUDA;
    return to_status(launch_attend(q, q_dtype, static_cast<const uint16_t*>(kd), static_cast<const uint16_t*>(vd),
                                   row_stride, idx, n_q_heads, n_kv_heads, n, d, k, rows_host_resident, out,
                                   (cudaStream_t)stream));
}

int fathom_sparse_attend_partial(const void* q, int q_dtype, const uint16_t* K_rows, const uint16_t* V_rows,
                                 int64_t row_stride, int rows_host_resident, int64_t key0, const int32_t* idx,
                                 int n_q_heads, int n_kv_heads, int64_t n, int d, int k, float* parts,
                                 fathom_stream_t stream) {
    if (!q || !K_rows || !V_rows || !idx || !parts || n < 1 || key0 < 0 || k < 1 || !dims_ok(n_kv_heads, d) ||
        !heads_ok(n_q_heads, n_kv_heads))
        return FATHOM_EINVAL;
    if (q_dtype != FATHOM_F32 && q_dtype != FATHOM_BF16) return FATHOM_EINVAL;
    if (d != 32 && d != 64 && d != 128 && d != 256) return FATHOM_EUNSUPPORTED;
    if (row_stride < d || row_stride % 8) return FATHOM_EINVAL;
    if ((reinterpret_cast<uintptr_t>(K_rows) & 15) || (reinterpret_cast<uintptr_t>(V_rows) & 15))
        return FATHOM_EINVAL;
    const void* kd = nullptr;
    const void* vd = nullptr;
    Where want = rows_host_resident ? Where::kHostPinned : Where::kDevice;
    if (classify(K_rows, &kd) != want || classify(V_rows, &vd) != want) return FATHOM_EINVAL;
    if (!is_device(q) || !is_device(idx) || !is_device(parts)) return FATHOM_EINVAL;
    if (!device_status_ptr()) return FATHOM_ECUDA;
    return to_status(launch_attend(q, q_dtype, static_cast<const uint16_t*>(kd), static_cast<const uint16_t*>(vd),
                                   row_stride, idx, n_q_heads, n_kv_heads, n, d, k, rows_host_resident, nullptr,
                                   (cudaStream_t)stream, key0, parts));
}

int fathom_attend_merge(const float* parts, int world, int n_q_heads, int d, float* out, fathom_stream_t stream) {
    if (!parts || !out || world < 1 || n_q_heads < 1 || d < 1 || d > kMaxD) return FATHOM_EINVAL;
    if (!is_device(parts) || !is_device(out)) return FATHOM_EINVAL;
    return to_status(launch_attend_merge(parts, world, n_q_heads, d, out, (cudaStream_t)stream));
}

size_t fathom_decode_workspace_bytes(const fathom_store* store, int n_q_heads, int k, int kv_groups) {
    if (!store || store->n < 1 || n_q_heads < 1 || k < 1 || k > kMaxTopK || kv_groups < 1 || kv_groups > 64 ||
        store->n_kv_heads < 1 || store->n_kv_heads % kv_groups || n_q_heads % store->n_kv_heads)
        return 0;
    return decode_workspace_bytes(store->n, n_q_heads, kv_groups, k);
}

int fathom_decode_step(const fathom_store* store, const void* q, int q_dtype, const float* sigma2, int n_q_heads,
                       int budget_bits, int fixed_r, int k, const uint16_t* K_rows, const uint16_t* V_rows,
                       int64_t rows_n, int64_t row_stride, int rows_host_resident, int kv_groups, uint8_t* depths,
                       int32_t* idx, float* top_scores, float* out, void* workspace, size_t workspace_bytes,
                       fathom_stream_t stream) {
    const uint32_t* planes;
    const uint16_t* scales;
    int rc = resolve_store(store, &planes, &scales);
    if (rc) return rc;
    const int Hkv = store->n_kv_heads, d = store->d;
    const int64_t n = store->n;
    if (!q || !sigma2 || !depths || !idx || !out || !K_rows || !V_rows || !workspace) return FATHOM_EINVAL;
    if (!heads_ok(n_q_heads, Hkv) || kv_groups < 1 || kv_groups > 64 || Hkv % kv_groups) return FATHOM_EINVAL;
    if (q_dtype != FATHOM_F32 && q_dtype != FATHOM_BF16) return FATHOM_EINVAL;
    if (budget_bits < 0 || fixed_r < 0 || fixed_r > d) return FATHOM_EINVAL;
    if (k < 1 || k > n || k > kMaxTopK || n > INT32_MAX) return FATHOM_EINVAL;
    if (d != 32 && d != 64 && d != 128 && d != 256) return FATHOM_EUNSUPPORTED;
    if (row_stride < d || row_stride % 8 || rows_n < n) return FATHOM_EINVAL;
    if ((reinterpret_cast<uintptr_t>(K_rows) & 15) || (reinterpret_cast<uintptr_t>(V_rows) & 15) ||
        (reinterpret_cast<uintptr_t>(workspace) & 255))
        return FATHOM_EINVAL;
    if (workspace_bytes < decode_workspace_bytes(n, n_q_heads, kv_groups, k)) return FATHOM_ENOMEM;
    if (!scan_fits(d, n_q_heads, Hkv)) return FATHOM_EUNSUPPORTED;
    const void* kd = nullptr;
    const void* vd = nullptr;
    Where want = rows_host_resident ? Where::kHostPinned : Where::kDevice;
    if (classify(K_rows, &kd) != want || classify(V_rows, &vd) != want) return FATHOM_EINVAL;
    if (!is_device(q) || !is_device(sigma2) || !is_device(depths) || !is_device(idx) || !is_device(out) ||
        !is_device(workspace) || (top_scores && !is_device(top_scores)))
        return FATHOM_EINVAL;
    if (!device_status_ptr()) return FATHOM_ECUDA;
    return to_status(launch_decode(planes, scales, store->host_resident, Hkv, d, n, store->n_pad, q, q_dtype, sigma2,
                                   n_q_heads,
                                   budget_bits, fixed_r, k, static_cast<const uint16_t*>(kd),
                                   static_cast<const uint16_t*>(vd), row_stride, rows_n, rows_host_resident, kv_groups,
                                   depths, idx, top_scores, out, workspace, (cudaStream_t)stream));
}

int fathom_last_device_status(fathom_stream_t stream) {
    unsigned int* p = device_status_ptr();
    if (!p) return -FATHOM_ECUDA;
    unsigned int v = 0;
    cudaStream_t s = (cudaStream_t)stream;
    if (cudaMemcpyAsync(&v, p, sizeof(v), cudaMemcpyDeviceToHost, s) != cudaSuccess) return -FATHOM_ECUDA;
    if (cudaMemsetAsync(p, 0, sizeof(v), s) != cudaSuccess) return -FATHOM_ECUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return -FATHOM_ECUDA;
    return (int)v;
}

int fathom_read_probe(const void* src, size_t bytes, int host_resident, uint64_t* sink, int ctas,
                      fathom_stream_t stream) {
    if (!src || !sink || bytes < 16 || (bytes & 15) || (reinterpret_cast<uintptr_t>(src) & 15) || ctas < 1)
        return FATHOM_EINVAL;
    const void* d = nullptr;
    Where want = host_resident ? Where::kHostPinned : Where::kDevice;
    if (classify(src, &d) != want || !is_device(sink)) return FATHOM_EINVAL;
    return to_status(launch_probe(d, bytes, reinterpret_cast<unsigned long long*>(sink), ctas, (cudaStream_t)stream));
}

const char* fathom_status_string(int status) {
    switch (status) {
        case FATHOM_OK: return "ok";
        case FATHOM_EINVAL: return "invalid argument";
        case FATHOM_ENOMEM: return "workspace or buffer too small";
        case FATHOM_ECUDA: return "CUDA error";
        case FATHOM_ETIMEOUT: return "bounded device wait timed out";
        case FATHOM_EUNSUPPORTED: return "unsupported shape or dtype";
        default: return "unknown status";
    }
}

}  // extern "C"
