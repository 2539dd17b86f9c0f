/*
 * fathom.h -- C ABI of the Fathom variable-depth bit-plane key scan for
 * NVIDIA B200 (sm_100a).
 *
 * What the method computes (page title, then section):
 *   "Fathom: Per-Query Read Depth for Sparse Decoding over Offloaded KV Caches"
 *   (arXiv 2609.17652 abstract): a 4-bit K cache stored channel-major as bit
 *   planes, so that a prefix of t planes is exactly the channel's t-bit
 *   quantizer; each query spends a bit budget by reverse water-filling over the
 *   variance-weighted importance of its channels; the scan ranks all n keys
 *   for a top-k step.
 *   "Fathom:面向卸载 KV Cache 的稀疏解码的逐查询读取深度" (ai-feeds.com summary),
 *   方法 · 关键模块 1-5: bit-plane store, per-query read depth by reverse
 *   water-filling, per-layer budgets, basis rule (paper Sec 3.5), scan kernel
 *   that pulls only budgeted planes and outputs top-k indices; 输出: true
 *   attention over the selected keys.
 *   evolve.pub review, Strengths: one shared block scale (paper Sec 3.2),
 *   depth rule from the 4x-per-bit error reduction (Sec 3.3), contiguous
 *   host-link runs (Sec 3.6).
 *
 * Conventions for every entry point:
 *   - The caller owns all memory it passes; no call allocates device
 *     memory for it.  The library keeps this state of its own, per device:
 *       . one status word (see below), a __device__ variable;
 *       . for fathom_decode_step with kv_groups > 1, one auxiliary stream
 *         and 65 events, made on the first such call in a context;
 *       . for fathom_scan_topk_noalloc, a fixed scratch array of
 *         fathom_noalloc_scratch_bytes(), a __device__ variable that every GPU
 *         which loads the library holds until the process exits.
 *     The host-side handles and the device addresses of these variables are
 *     cached with the id of the CUDA context they belong to, and made or
 *     looked up again when a call runs in another context (e.g. after
 *     cudaDeviceReset).
 *   - Device pointers must be cudaMalloc'd (or equivalent) on the current
 *     device.  "Host-resident" pointers must be page-locked host memory
 *     (cudaHostAlloc / cudaHostRegister), mapped into the device address space
 *     (always true with unified addressing on 64-bit Linux).
 *   - Calls are asynchronous on `stream` (NULL = legacy default stream) and
 *     return after enqueueing.  Argument errors are detected on the host
 *     before any launch and return FATHOM_EINVAL; nothing has been enqueued.
 *     FATHOM_ECUDA means a CUDA API or launch error (cudaGetLastError is
 *     left set for the caller to inspect).
 *   - Kernels never trap or assert.  Problems only the device can see (a
 *     depth above 4, an out-of-range index) are recorded in a per-device
 *     status word that fathom_last_device_status() reads and clears; the
 *     offending element is skipped.
 *   - Layouts are row-major C arrays; the shapes below use the names
 *     Hkv = number of KV heads, Hq = number of query heads (a multiple of
 *     Hkv, query head h reads KV head h / (Hq/Hkv)), d = head dimension
 *     (a multiple of 32, at most 256), n = number of keys,
 *     n_pad = n rounded up to a multiple of 1024 (so that every plane row,
 *     n_pad/8 bytes, starts on a 128-byte boundary and the 128-byte run
 *     that a 1024-key tile reads from it is one aligned line).
 */
#ifndef FATHOM_H
#define FATHOM_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t. */
typedef struct CUstream_st* fathom_stream_t;

enum {
    FATHOM_OK = 0,
    FATHOM_EINVAL = 1,       /* bad argument (null pointer, size, alignment, pinning) */
    FATHOM_ENOMEM = 2,       /* caller-provided workspace or buffer too small */
    FATHOM_ECUDA = 3,        /* CUDA runtime or launch error */
    FATHOM_ETIMEOUT = 4,     /* a bounded device wait gave up (device status only) */
    FATHOM_EUNSUPPORTED = 5  /* valid but unsupported shape or dtype */
};

typedef enum { FATHOM_F32 = 0, FATHOM_BF16 = 1 } fathom_dtype;

/* Bits of the device status word (fathom_last_device_status). */
enum {
    FATHOM_DEV_BAD_DEPTH = 1u << 0,   /* a depth above 4 was read; that channel was skipped */
    FATHOM_DEV_BAD_INDEX = 1u << 1,   /* an index outside [0,n) reached sparse attention; skipped */
    FATHOM_DEV_TOPK_OVERFLOW = 1u << 2 /* internal: a top-k buffer overflowed (never expected) */
};

/*
 * The packed K index of one layer (bit-plane store).
 *   planes  u32 [Hkv][d][4][n_pad/32]: bit (i % 32) of word (i / 32) of plane j
 *           holds bit (3-j) of key i's 4-bit code (plane 0 = most significant);
 *           padding keys hold 0.  A channel's four planes are contiguous, so the
 *           first t planes of a channel are one contiguous run of t*n_pad/8
 *           bytes.
 *   scales  u16 [Hkv][d][n_pad/64]: fp16 bit pattern of the block scale Delta
 *           of (KV head, channel, 64-token block); 0 for all-padding blocks.
 *   Both arrays start on a 16-byte boundary (the scan copies their rows to
 *           shared memory in 16-byte pieces); a store that violates this is
 *           rejected with FATHOM_EINVAL.
 *   host_resident: 0 = both arrays in device memory, 1 = both in page-locked
 *           host memory (the scan then streams only the budgeted planes over
 *           the host link).
 *   n       keys in the store; n_pad = its capacity and row stride in keys:
 *           a multiple of 1024, at least fathom_n_pad(n) (equal for a store
 *           packed once; larger for a cache that grows by fathom_append_keys).
 *           Scans cover the keys [0, fathom_n_pad(n)) only, and score rows
 *           have length fathom_n_pad(n) whatever the capacity.
 */
typedef struct {
    int32_t n_kv_heads;
    int32_t d;
    int64_t n;
    int64_t n_pad;
    int32_t host_resident;
    int32_t reserved;
    const uint32_t* planes;
    const uint16_t* scales;
} fathom_store;

/* n rounded up to a multiple of 1024; the padded key count of a store. */
int64_t fathom_n_pad(int64_t n);
/* Bytes of the planes / scales arrays of a store; 0 for invalid sizes. */
size_t fathom_planes_bytes(int n_kv_heads, int d, int64_t n);
size_t fathom_scales_bytes(int n_kv_heads, int d, int64_t n);

/*
 * Pack a K cache into the bit-plane store (quantize + plane layout).
 * [ai-feeds summary 关键模块 1; evolve.pub Strengths (Sec 3.2); FAQ "How does
 *  Fathom's bit-plane KV cache work?"]
 * For each (KV head, channel, 64-token block): amax = max |x| over the
 * block's real keys, Delta = fp16_rn(amax/8), code = clamp(floor(x/Delta),
 * -8, 7) + 8 (code 8 when Delta = 0; floor taken on the exact quotient).
 *   K       device, [Hkv][n][d], dtype FATHOM_F32 or FATHOM_BF16; finite values.
 *   planes  device, fathom_planes_bytes() bytes, fully overwritten.
 *   scales  device, fathom_scales_bytes() bytes, fully overwritten.
 * To build a host-resident store, pack into device buffers and copy them to
 * page-locked host memory.
 * Errors: EINVAL for null pointers, n < 1, Hkv < 1, d not a multiple of 32
 * or d > 256, unknown dtype.
 */
int fathom_pack_bitplanes(const void* K, int k_dtype, int n_kv_heads, int64_t n, int d,
                          uint32_t* planes, uint16_t* scales, fathom_stream_t stream);

/*
 * Decode-time append: adds keys [store->n, n_new) to a store that has the
 * capacity for them (not on the pages, which pack a cache once; a serving
 * cache grows by a key per decoded token).  The block scale of the last
 * partial 64-token block changes when keys join it, so that block is packed
 * again, from its first key on, together with the new blocks; blocks before
 * it are untouched.  The result equals fathom_pack_bitplanes of all n_new keys
 * (bit for bit, over the first fathom_n_pad(n_new) keys of every row).
 *   store   its planes/scales (device, or page-locked host memory written
 *           through the mapping) sized for capacity store->n_pad; n may be 0
 *           (an empty store).  On success store->n becomes n_new.
 *   K_tail  device, [Hkv][n_new - t][d] with t = (store->n / 64) * 64: the keys
 *           from the first key of the last partial block to n_new - 1 (keys
 *           before n keep their values), dtype FATHOM_F32 or FATHOM_BF16.
 *   Capacity outside [0, n_new] beyond fathom_n_pad(n_new) is never read.
 * Errors: EINVAL for null pointers, n_new <= store->n, n_pad not a multiple of
 * 1024 or below fathom_n_pad(n_new), arrays not where host_resident says.
 */
int fathom_append_keys(fathom_store* store, const void* K_tail, int k_dtype, int64_t n_new, fathom_stream_t stream);

/*
 * Per-query read depths.
 * [arXiv abstract; ai-feeds summary 关键模块 2-3; evolve.pub Strengths (Sec 3.3)]
 * fixed_r == 0: reverse water-filling.  w_c = fl32(fl32(q_c*q_c)*sigma2_c)
 *   (IEEE fp32, no fused multiply-add); the candidates (c,t), t = 0..3,
 *   valued w_c 4^-t, are ordered by value descending, then c ascending, then
 *   t ascending; the first min(budget_bits, 4d) are taken and depth t_c is
 *   the number taken on channel c.  So sum_c t_c = min(B, 4d).
 * fixed_r > 0: comparison scans at a fixed depth: 4 planes on the fixed_r
 *   channels with the largest |q_c| (ties to the lower channel), 0 elsewhere
 *   (r = 16 is the "68-bit" scan, r = 32 the "136-bit" one).
 *   q       device, [Hq][d], FATHOM_F32 or FATHOM_BF16.
 *   sigma2  device, f32 [Hkv][d], the per-channel key statistic (>= 0).
 *   depths  device, u8 [Hq][d], overwritten.
 * Errors: EINVAL for null pointers, budget_bits < 0, fixed_r < 0 or > d,
 * Hq not a multiple of Hkv, d not a multiple of 32 or d > 256.
 */
int fathom_alloc_depths(const void* q, int q_dtype, const float* sigma2, int n_q_heads,
                        int n_kv_heads, int d, int budget_bits, int fixed_r, uint8_t* depths,
                        fathom_stream_t stream);

/*
 * Group-pooled depths: a variant for comparison, not the pages' rule (which
 * decides per query: arXiv abstract, "each query decides").  For KV head g
 * the importance of channel c is the fp32 sum, in head order, of the group's
 * per-head importances q_{h,c}^2 sigma2_{g,c} (each product rounded as in
 * fathom_alloc_depths); one reverse water-filling over it with budget B; every
 * query head of the group receives the same depths, so the scan reads exactly
 * min(B, 4d) plane bits per key and KV head.
 * Arguments and errors as fathom_alloc_depths (no fixed_r).
 */
int fathom_alloc_depths_pooled(const void* q, int q_dtype, const float* sigma2, int n_q_heads, int n_kv_heads,
                               int d, int budget_bits, uint8_t* depths, fathom_stream_t stream);

/*
 * Variable-depth scan: approximate scores of every key for every query head.
 * [ai-feeds summary 关键模块 4 (basis rule, paper Sec 3.5) and 5; arXiv abstract]
 * s[h][i] = sum_c q[h][c] * Delta[b(i)][c] * sum_{j < t[h][c]} (2 b_{i,c,j} - 1) 2^(2-j)
 * Only the first U_c = max over the KV group of t[h][c] planes of channel c
 * are read; planes beyond are never touched.
 *   store   a packed store (device or host-resident).
 *   q       device, [Hq][d], FATHOM_F32 or FATHOM_BF16.
 *   depths  device, u8 [Hq][d], values 0..4.
 *   scores  device, f32 [Hq][fathom_n_pad(store->n)]; keys >= n are written -inf.
 *   block_max  NULL, or device u32 [Hq][fathom_n_pad(store->n)/64]: the largest
 *           score of every 64-key block as an order-preserving key, for
 *           fathom_topk to read only the blocks that can hold a selected key.
 * Errors: EINVAL as above, or a host-resident store whose pointers are not
 * page-locked, or a device store whose pointers are not device memory.
 */
int fathom_scan_scores(const fathom_store* store, const void* q, int q_dtype, const uint8_t* depths,
                       int n_q_heads, float* scores, uint32_t* block_max, fathom_stream_t stream);

/*
 * Top-k of score rows: the k largest of scores[r][0..n), ties to the lower
 * index, listed in that order.  [ai-feeds summary 关键模块 5, 输出]
 *   scores      device, f32 [n_rows][ld] (ld >= n); NaN is not allowed.
 *   block_max   NULL (select from the scores alone), or the block maxima
 *               that fathom_scan_scores wrote with these scores (ld a
 *               multiple of 64): with m = the k-th largest block maximum of a
 *               row, k keys score at least m, so only the blocks whose
 *               maximum is >= m are read.  Rows of at most 131072 keys are
 *               selected in on-chip memory by one kernel; longer rows with
 *               block maxima and at least k blocks (up to 2^23 keys) by one
 *               cluster kernel over the maxima and the surviving blocks; the
 *               rest by histogram passes over the whole row.  The result is
 *               the same on every path.
 *   idx         device, i32 [n_rows][k].
 *   top_scores  device, f32 [n_rows][k], or NULL.
 *   workspace   device, at least fathom_topk_workspace_bytes(n, n_rows, k) bytes,
 *               256-byte aligned; contents need not be initialised.
 * Errors: EINVAL for k < 1, k > n, k > 4096, n_rows < 1; ENOMEM for a short
 * workspace.
 */
size_t fathom_topk_workspace_bytes(int64_t n, int n_rows, int k);
int fathom_topk(const float* scores, const uint32_t* block_max, int64_t n, int64_t ld, int n_rows, int k,
                int32_t* idx, float* top_scores, void* workspace, size_t workspace_bytes, fathom_stream_t stream);

/*
 * Merge of per-shard top-k lists, for a key range split across GPUs (not on
 * the pages, whose system runs on one GPU): every GPU scans a contiguous,
 * 1024-aligned key range and takes its local top-k; the lists are gathered
 * (one all-gather of (score, index) pairs per query head) and merged here
 * into the top-k of all keys.
 *   cand_scores  device, f32 [n_rows][n_cand]: the gathered lists, shard by
 *                shard in ascending key-range order, each list in (score
 *                descending, index ascending) order; padding entries -inf.
 *   cand_idx     device, i32 [n_rows][n_cand]: the candidates' global key
 *                indices.
 *   idx, top_scores (or NULL), workspace (fathom_topk_workspace_bytes(n_cand,
 *                n_rows, k) bytes)  as fathom_topk.
 * Equal scores go to the candidate listed first, which is the lower global
 * index under the ordering above, so the result equals the top-k of the
 * unsplit scores.  Errors as fathom_topk with n = n_cand.
 */
int fathom_topk_merge(const float* cand_scores, const int32_t* cand_idx, int n_rows, int n_cand, int k, int32_t* idx,
                      float* top_scores, void* workspace, size_t workspace_bytes, fathom_stream_t stream);

/*
 * Scan + top-k of one decode step of one layer (fathom_scan_scores followed
 * by fathom_topk on the scores, which live in the workspace).
 *   idx         device, i32 [Hq][k].
 *   top_scores  device, f32 [Hq][k], or NULL.
 *   workspace   device, fathom_scan_workspace_bytes(store, Hq, k) bytes,
 *               256-byte aligned.
 */
size_t fathom_scan_workspace_bytes(const fathom_store* store, int n_q_heads, int k);
int fathom_scan_topk(const fathom_store* store, const void* q, int q_dtype, const uint8_t* depths,
                     int n_q_heads, int k, int32_t* idx, float* top_scores, void* workspace,
                     size_t workspace_bytes, fathom_stream_t stream);

/*
 * Scan + top-k of several sessions in one pass (many sessions resident at
 * once; arXiv abstract).  Session s has its own store stores[s] (all with
 * the same Hkv and d, each device- or host-resident, lengths may differ) and
 * its own queries; one launch scans the tiles of every session, then one
 * top-k pass serves all S x Hq rows.  Results equal S separate
 * fathom_scan_topk calls.
 *   stores      host array of n_sessions (1..64) store descriptors.
 *   q           device, [S][Hq][d], FATHOM_F32 or FATHOM_BF16.
 *   depths      device, u8 [S][Hq][d] (fathom_alloc_depths with S*Hq query heads
 *               and S*Hkv KV heads fills it in one call).
 *   idx         device, i32 [S][Hq][k];  top_scores f32 [S][Hq][k] or NULL.
 *   workspace   device, fathom_scan_batched_workspace_bytes() bytes, 256-byte aligned;
 *               session s's scores start at the s-th 256-byte-aligned slice.
 * Errors: EINVAL for bad sessions (count, mismatched Hkv/d, k > some n,
 * residency), ENOMEM for a short workspace.
 */
size_t fathom_scan_batched_workspace_bytes(const fathom_store* stores, int n_sessions, int n_q_heads, int k);
int fathom_scan_topk_batched(const fathom_store* stores, int n_sessions, const void* q, int q_dtype,
                             const uint8_t* depths, int n_q_heads, int k, int32_t* idx, float* top_scores,
                             void* workspace, size_t workspace_bytes, fathom_stream_t stream);

/*
 * Scan + top-k without any caller-provided workspace.  The paper has no
 * counterpart: this is a service to callers that cannot allocate device
 * memory (an engine whose memory is all handed to its own pool, a plug-in
 * inside a host program that forbids cudaMalloc/cudaFree on its serving
 * path).  Same inputs, outputs and results as fathom_scan_topk; the scratch
 * comes from one fixed array of fathom_noalloc_scratch_bytes() bytes (24 MiB)
 * in the library's own device memory, which every GPU that loads the library
 * holds until the process exits.  No call allocates or frees anything.
 *   - A step needing more than that (fathom_scan_workspace_bytes(store, Hq, k)
 *     above the maximum) returns FATHOM_ENOMEM before any work is enqueued.
 *     Example that fits: Hq = 32, n = 131072, k = 2048 (about 20 MB).
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress, with that device current) and keeps it; make
 *     that first call before any stream capture.
 *   - Every call shares the array, which keeps the previous call's contents
 *     (each call re-initialises what it needs).  Calls that overlap on the
 *     GPU (different streams or host threads) race on it: serialise them.
 * Other errors as fathom_scan_topk.
 */
size_t fathom_noalloc_scratch_bytes(void);
int fathom_scan_topk_noalloc(const fathom_store* store, const void* q, int q_dtype, const uint8_t* depths,
                             int n_q_heads, int k, int32_t* idx, float* top_scores, fathom_stream_t stream);

/*
 * Exact attention over the selected keys only.  [ai-feeds summary 输出]
 * out[h] = softmax_j(q[h] . K[g][idx[h][j]] / sqrt(d)) V[g][idx[h][j]],
 * g = h / (Hq/Hkv), fp32 accumulation.
 *   q       device, [Hq][d], FATHOM_F32 or FATHOM_BF16.
 *   K_rows, V_rows  bf16 bit patterns: the row of key i of KV head g starts
 *           at element (g * n + i) * row_stride; device memory, or page-locked
 *           host memory when rows_host_resident = 1.  row_stride = d for two
 *           plain [Hkv][n][d] arrays; row_stride = 2d with V_rows = K_rows + d
 *           for one interleaved [Hkv][n][2][d] array, the layout to use for
 *           host-resident rows: a key's K and V rows then cross the host link
 *           as one 4d-byte run (on B200 over PCIe, K and V rows gathered from
 *           two arrays gigabytes apart ran at about half the rate).
 *           row_stride >= d and a multiple of 8; rows 16-byte aligned.
 *   idx     device, i32 [Hq][k], each in [0, n) (others are skipped and
 *           flagged FATHOM_DEV_BAD_INDEX).
 *   out     device, f32 [Hq][d].
 * Errors: EINVAL for null pointers, k < 1, bad head counts, d not a
 * multiple of 32 or d > 256, a bad row_stride, rows not where
 * rows_host_resident says.
 */
int fathom_sparse_attend(const void* q, int q_dtype, const uint16_t* K_rows, const uint16_t* V_rows,
                         int64_t row_stride, int rows_host_resident, const int32_t* idx, int n_q_heads,
                         int n_kv_heads, int64_t n, int d, int k, float* out, fathom_stream_t stream);

/*
 * Attention over a key range split across GPUs (not on the pages, whose
 * system runs on one GPU).  Each rank holds the rows of keys [key0, key0 + n)
 * and runs fathom_sparse_attend_partial with the merged global indices (see
 * fathom_topk_merge): indices outside its range, and -1 padding, are skipped.
 * It writes per-head partials instead of the output:
 *   parts   device, f32 [Hq][d + 2]: o[0..d) = sum_j 2^(s_j - m) V_j over this
 *           range's selected rows, then m = max_j s_j and l = sum_j 2^(s_j - m),
 *           with s_j = q . K_j log2(e) / sqrt(d); a head with no row here has
 *           m = -inf, l = 0.
 * Other arguments as fathom_sparse_attend (K_rows / V_rows hold this range's
 * n rows per KV head; key0 >= 0).  The ranks' partials are gathered (one
 * all-gather of Hq (d + 2) floats per rank) and combined by
 * fathom_attend_merge:
 *   parts   device, f32 [world][Hq][d + 2], the ranks' partials.
 *   out     device, f32 [Hq][d] = sum_r o_r 2^(m_r - M) / sum_r l_r 2^(m_r - M),
 *           M = max_r m_r, ranks summed in order; 0 for a head with no rows.
 * The result equals fathom_sparse_attend over all rows up to fp32 rounding
 * (the partials are merged in a different order).
 * Errors: as fathom_sparse_attend; EINVAL for key0 < 0, world < 1.
 */
int fathom_sparse_attend_partial(const void* q, int q_dtype, const uint16_t* K_rows, const uint16_t* V_rows,
                                 int64_t row_stride, int rows_host_resident, int64_t key0, const int32_t* idx,
                                 int n_q_heads, int n_kv_heads, int64_t n, int d, int k, float* parts,
                                 fathom_stream_t stream);
int fathom_attend_merge(const float* parts, int world, int n_q_heads, int d, float* out, fathom_stream_t stream);

/*
 * One decode step of one layer in one call: per-query depths, the scan, top-k
 * and exact attention over the selected rows.  [ai-feeds summary 方法: 输入,
 * 关键模块 2-5, 输出]  The results equal fathom_alloc_depths, then
 * fathom_scan_topk, then fathom_sparse_attend on the same arguments, bit for
 * bit.
 *
 * The KV heads are split into kv_groups groups of equal size.  The scan of a
 * group runs on `stream` while the top-k and attention of the previous group
 * run on an auxiliary stream that the library creates per device on first
 * use; the two are forked and joined with events, so all work is ordered on
 * `stream` and the call may be captured into a CUDA graph.  kv_groups = 1
 * runs the plain sequence on `stream` alone, each kernel launched with
 * programmatic serialization (scheduled while the one before it finishes; it
 * waits for that kernel's results before reading them).  Steps issued at the
 * same time from several host threads on one device share the auxiliary
 * stream (they stay correct; their top-k and attention serialise).
 *   store        device- or host-resident store, as fathom_scan_topk.
 *   q, q_dtype, sigma2, budget_bits, fixed_r  as fathom_alloc_depths.
 *   k            as fathom_scan_topk (1 <= k <= min(n, 4096)).
 *   K_rows, V_rows, row_stride, rows_host_resident  as fathom_sparse_attend;
 *   rows_n       keys per KV head in the row arrays (>= store->n; a growing
 *                cache keeps its rows at a capacity: the head stride is
 *                rows_n * row_stride).
 *   kv_groups    1 <= kv_groups <= 64, dividing the store's n_kv_heads.
 *   depths       device, u8 [Hq][d], written.
 *   idx          device, i32 [Hq][k]; top_scores device f32 [Hq][k] or NULL.
 *   out          device, f32 [Hq][d].
 *   workspace    device, 256-byte aligned, at least
 *                fathom_decode_workspace_bytes(store, Hq, k, kv_groups) bytes
 *                (the scores of all heads and one top-k workspace).
 * Errors: as the three separate calls; EINVAL for a bad kv_groups.
 */
size_t fathom_decode_workspace_bytes(const fathom_store* store, int n_q_heads, int k, int kv_groups);
int fathom_decode_step(const fathom_store* store, const void* q, int q_dtype, const float* sigma2, int n_q_heads,
                       int budget_bits, int fixed_r, int k, const uint16_t* K_rows, const uint16_t* V_rows,
                       int64_t rows_n, int64_t row_stride, int rows_host_resident, int kv_groups, uint8_t* depths,
                       int32_t* idx, float* top_scores, float* out, void* workspace, size_t workspace_bytes,
                       fathom_stream_t stream);

/*
 * Reads and clears this device's status word (FATHOM_DEV_* bits) after
 * synchronising `stream`.  Returns the bits (>= 0), or -FATHOM_ECUDA.
 */
int fathom_last_device_status(fathom_stream_t stream);

/*
 * Measurement utility (not part of the method): streams `bytes` from `src`
 * with 16-byte loads from `ctas` CTAs of 256 threads and XORs a checksum into
 * *sink (device u64).  With host_resident = 1, `src` is page-locked host
 * memory and the kernel measures the host link as the scan's loads use it;
 * with 0, device memory (HBM read bandwidth).  Time it with CUDA events.
 * Errors: EINVAL for null or misaligned pointers, bytes not a multiple of 16,
 * or `src` not where host_resident says.
 */
int fathom_read_probe(const void* src, size_t bytes, int host_resident, uint64_t* sink, int ctas,
                      fathom_stream_t stream);

/* Static description of a status code. */
const char* fathom_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* FATHOM_H */
