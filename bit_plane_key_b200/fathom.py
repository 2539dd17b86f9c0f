"""Python binding of libfathom (the C ABI in include/fathom.h).

Argument marshalling only: every step of the scan runs in the library's CUDA
kernels.  Tensors are torch tensors (device memory, or page-locked host memory
for host-resident stores and rows); torch is used for allocation and streams.
If libfathom.so is missing this module raises at import: there is no CPU or
fallback path.
"""
import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfathom.so")

if not os.path.exists(LIB_PATH):
    raise ImportError("libfathom.so is not built; run `python -m bit_plane_key_b200.build` (needs nvcc)")

_lib = ctypes.CDLL(LIB_PATH)

OK, EINVAL, ENOMEM, ECUDA, ETIMEOUT, EUNSUPPORTED = range(6)
F32, BF16 = 0, 1
DEV_BAD_DEPTH, DEV_BAD_INDEX, DEV_TOPK_OVERFLOW = 1, 2, 4
MAX_TOPK = 4096


class FathomError(RuntimeError):
    def __init__(self, status, what):
        self.status = status
        msg = _lib.fathom_status_string(status).decode()
        super().__init__("%s: %s (status %d)" % (what, msg, status))


class fathom_store(ctypes.Structure):
    _fields_ = [("n_kv_heads", ctypes.c_int32), ("d", ctypes.c_int32), ("n", ctypes.c_int64),
                ("n_pad", ctypes.c_int64), ("host_resident", ctypes.c_int32), ("reserved", ctypes.c_int32),
                ("planes", ctypes.c_void_p), ("scales", ctypes.c_void_p)]


_P, _I, _L, _Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
_SP = ctypes.POINTER(fathom_store)


def _sig(name, res, args):
    f = getattr(_lib, name)
    f.restype = res
    f.argtypes = args
    return f


_sig("fathom_n_pad", _L, [_L])
_sig("fathom_planes_bytes", _Z, [_I, _I, _L])
_sig("fathom_scales_bytes", _Z, [_I, _I, _L])
_sig("fathom_pack_bitplanes", _I, [_P, _I, _I, _L, _I, _P, _P, _P])
_sig("fathom_alloc_depths", _I, [_P, _I, _P, _I, _I, _I, _I, _I, _P, _P])
_sig("fathom_alloc_depths_pooled", _I, [_P, _I, _P, _I, _I, _I, _I, _P, _P])
_sig("fathom_append_keys", _I, [_SP, _P, _I, _L, _P])
_sig("fathom_topk_merge", _I, [_P, _P, _I, _I, _I, _P, _P, _P, _Z, _P])
_sig("fathom_scan_scores", _I, [_SP, _P, _I, _P, _I, _P, _P, _P])
_sig("fathom_topk_workspace_bytes", _Z, [_L, _I, _I])
_sig("fathom_topk", _I, [_P, _P, _L, _L, _I, _I, _P, _P, _P, _Z, _P])
_sig("fathom_scan_workspace_bytes", _Z, [_SP, _I, _I])
_sig("fathom_scan_topk", _I, [_SP, _P, _I, _P, _I, _I, _P, _P, _P, _Z, _P])
_sig("fathom_sparse_attend", _I, [_P, _I, _P, _P, _L, _I, _P, _I, _I, _L, _I, _I, _P, _P])
_sig("fathom_sparse_attend_partial", _I, [_P, _I, _P, _P, _L, _I, _L, _P, _I, _I, _L, _I, _I, _P, _P])
_sig("fathom_attend_merge", _I, [_P, _I, _I, _I, _P, _P])
_sig("fathom_last_device_status", _I, [_P])
_sig("fathom_status_string", ctypes.c_char_p, [_I])
_sig("fathom_read_probe", _I, [_P, _Z, _I, _P, _I, _P])
_sig("fathom_noalloc_scratch_bytes", _Z, [])
_sig("fathom_scan_batched_workspace_bytes", _Z, [_SP, _I, _I, _I])
_sig("fathom_scan_topk_batched", _I, [_SP, _I, _P, _I, _P, _I, _I, _P, _P, _P, _Z, _P])
_sig("fathom_scan_topk_noalloc", _I, [_SP, _P, _I, _P, _I, _I, _P, _P, _P])
_sig("fathom_decode_workspace_bytes", _Z, [_SP, _I, _I, _I])
_sig("fathom_decode_step", _I, [_SP, _P, _I, _P, _I, _I, _I, _I, _P, _P, _L, _L, _I, _I, _P, _P, _P, _P, _P, _Z, _P])


def lib():
    """The loaded ctypes library (for calls with raw pointers)."""
    return _lib


def _check(rc, what):
    if rc != OK:
        raise FathomError(rc, what)


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def _dtype_code(t):
    if t.dtype == torch.float32:
        return F32
    if t.dtype in (torch.bfloat16, torch.int16, torch.uint16):
        return BF16
    raise TypeError("expected float32 or bfloat16, got %s" % t.dtype)


def n_pad(n):
    return int(_lib.fathom_n_pad(int(n)))


class Store:
    """A packed bit-plane store: planes u32 [Hkv][d][4][n_pad/32], scales u16 [Hkv][d][n_pad/64].
    n = keys held; n_pad = capacity (the row stride, from the arrays' shape)."""

    def __init__(self, planes, scales, n, host_resident=None):
        self.planes, self.scales, self.n = planes, scales, int(n)
        self.n_kv_heads, self.d = int(planes.shape[0]), int(planes.shape[1])
        self.n_pad = int(planes.shape[-1]) * 32
        self.host_resident = (not planes.is_cuda) if host_resident is None else bool(host_resident)
        self._c = fathom_store(self.n_kv_heads, self.d, self.n, self.n_pad, int(self.host_resident), 0,
                               planes.data_ptr(), scales.data_ptr())

    @property
    def c(self):
        return ctypes.byref(self._c)

    @classmethod
    def empty(cls, n_kv_heads, d, capacity, device=None, host_resident=False):
        """An empty store (n = 0) with room for `capacity` keys, zero-filled,
        in device memory or page-locked host memory; grow it with append_keys."""
        cap = n_pad(capacity)
        kw = dict(pin_memory=True) if host_resident else dict(device=device)
        planes = torch.zeros((n_kv_heads, d, 4, cap // 32), dtype=torch.int32, **kw)
        scales = torch.zeros((n_kv_heads, d, cap // 64), dtype=torch.int16, **kw)
        return cls(planes, scales, 0, host_resident=host_resident)

    def to_host(self):
        """Copy of this store in page-locked host memory (host-resident)."""
        return Store(self.planes.cpu().pin_memory(), self.scales.cpu().pin_memory(), self.n, host_resident=True)

    def plane_bytes_read(self, union_depths):
        """Plane + scale bytes a scan reads for union depths U [Hkv][d] (over the
        first n_pad(n) keys, the range a scan covers)."""
        U = union_depths.to(torch.int64)
        npad = n_pad(self.n)
        return int(U.sum()) * npad // 8 + int((U > 0).sum()) * (npad // 64) * 2


def pack_bitplanes(K, planes=None, scales=None, stream=None):
    """K [Hkv][n][d] (float32 or bfloat16, cuda) -> Store."""
    Hkv, n, d = K.shape
    npad = n_pad(n)
    if planes is None:
        planes = torch.empty((Hkv, d, 4, npad // 32), dtype=torch.int32, device=K.device)
    if scales is None:
        scales = torch.empty((Hkv, d, npad // 64), dtype=torch.int16, device=K.device)
    _check(_lib.fathom_pack_bitplanes(_ptr(K), _dtype_code(K), Hkv, n, d, _ptr(planes), _ptr(scales),
                                      _stream(stream)), "fathom_pack_bitplanes")
    return Store(planes, scales, n, host_resident=False)


def append_keys(store, K_tail, n_new, stream=None):
    """Decode-time append: keys [store.n, n_new) into a store with the capacity.
    K_tail [Hkv][n_new - t][d] (cuda, float32 or bfloat16) holds the keys from
    t = (store.n // 64) * 64 on.  Updates store.n."""
    _check(_lib.fathom_append_keys(store.c, _ptr(K_tail), _dtype_code(K_tail), int(n_new), _stream(stream)),
           "fathom_append_keys")
    store.n = int(store._c.n)
    return store


def alloc_depths(q, sigma2, budget_bits, fixed_r=0, out=None, stream=None):
    """q [Hq][d], sigma2 f32 [Hkv][d] -> depths u8 [Hq][d]."""
    Hq, d = q.shape
    Hkv = sigma2.shape[0]
    if out is None:
        out = torch.empty((Hq, d), dtype=torch.uint8, device=q.device)
    _check(_lib.fathom_alloc_depths(_ptr(q), _dtype_code(q), _ptr(sigma2), Hq, Hkv, d, int(budget_bits),
                                    int(fixed_r), _ptr(out), _stream(stream)), "fathom_alloc_depths")
    return out


def alloc_depths_pooled(q, sigma2, budget_bits, out=None, stream=None):
    """Group-pooled depths (one depth vector per KV head, repeated for its query
    heads): q [Hq][d], sigma2 f32 [Hkv][d] -> depths u8 [Hq][d]."""
    Hq, d = q.shape
    Hkv = sigma2.shape[0]
    if out is None:
        out = torch.empty((Hq, d), dtype=torch.uint8, device=q.device)
    _check(_lib.fathom_alloc_depths_pooled(_ptr(q), _dtype_code(q), _ptr(sigma2), Hq, Hkv, d, int(budget_bits),
                                           _ptr(out), _stream(stream)), "fathom_alloc_depths_pooled")
    return out


def scan_scores(store, q, depths, out=None, block_max=None, stream=None):
    """Scores f32 [Hq][n_pad(n)] (padding keys -inf); block_max (optional) u32
    [Hq][n_pad(n)/64] receives the block maxima that topk() can use."""
    Hq = q.shape[0]
    if out is None:
        out = torch.empty((Hq, n_pad(store.n)), dtype=torch.float32, device=q.device)
    _check(_lib.fathom_scan_scores(store.c, _ptr(q), _dtype_code(q), _ptr(depths), Hq, _ptr(out), _ptr(block_max),
                                   _stream(stream)), "fathom_scan_scores")
    return out


def block_max_buffer(n_rows, n, device):
    """A block-maxima buffer for scan_scores / topk: u32 (as int32) [rows][n_pad(n)/64]."""
    return torch.empty((n_rows, n_pad(n) // 64), dtype=torch.int32, device=device)


def topk_workspace_bytes(n, rows, k):
    return int(_lib.fathom_topk_workspace_bytes(int(n), int(rows), int(k)))


def topk(scores, n, k, idx=None, top_scores=None, workspace=None, block_max=None, stream=None):
    """Top-k of score rows [rows][ld] over the first n columns (block_max: the
    block maxima the scan wrote with these scores, or None)."""
    rows, ld = scores.shape
    if idx is None:
        idx = torch.empty((rows, k), dtype=torch.int32, device=scores.device)
    if top_scores is None:
        top_scores = torch.empty((rows, k), dtype=torch.float32, device=scores.device)
    nb = topk_workspace_bytes(n, rows, k)
    if workspace is None:
        workspace = torch.empty(max(nb, 1), dtype=torch.uint8, device=scores.device)
    _check(_lib.fathom_topk(_ptr(scores), _ptr(block_max), int(n), int(ld), rows, int(k), _ptr(idx),
                            _ptr(top_scores), _ptr(workspace), workspace.numel(), _stream(stream)), "fathom_topk")
    return idx, top_scores


def topk_merge(cand_scores, cand_idx, k, idx=None, top_scores=None, workspace=None, stream=None):
    """Top-k of gathered per-shard lists: cand_scores f32 / cand_idx i32 [rows][n_cand]
    (shards in ascending key-range order, each list in top-k order) -> idx, scores [rows][k]."""
    rows, n_cand = cand_scores.shape
    if idx is None:
        idx = torch.empty((rows, k), dtype=torch.int32, device=cand_scores.device)
    if top_scores is None:
        top_scores = torch.empty((rows, k), dtype=torch.float32, device=cand_scores.device)
    nb = topk_workspace_bytes(n_cand, rows, k)
    if workspace is None:
        workspace = torch.empty(max(nb, 1), dtype=torch.uint8, device=cand_scores.device)
    _check(_lib.fathom_topk_merge(_ptr(cand_scores), _ptr(cand_idx), rows, n_cand, int(k), _ptr(idx),
                                  _ptr(top_scores), _ptr(workspace), workspace.numel(), _stream(stream)),
           "fathom_topk_merge")
    return idx, top_scores


def scan_workspace_bytes(store, n_q_heads, k):
    return int(_lib.fathom_scan_workspace_bytes(store.c, int(n_q_heads), int(k)))


def scan_topk(store, q, depths, k, idx=None, top_scores=None, workspace=None, stream=None):
    """idx i32 [Hq][k] and top scores f32 [Hq][k]."""
    Hq = q.shape[0]
    if idx is None:
        idx = torch.empty((Hq, k), dtype=torch.int32, device=q.device)
    if top_scores is None:
        top_scores = torch.empty((Hq, k), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = torch.empty(max(scan_workspace_bytes(store, Hq, k), 1), dtype=torch.uint8, device=q.device)
    _check(_lib.fathom_scan_topk(store.c, _ptr(q), _dtype_code(q), _ptr(depths), Hq, int(k), _ptr(idx),
                                 _ptr(top_scores), _ptr(workspace), workspace.numel(), _stream(stream)),
           "fathom_scan_topk")
    return idx, top_scores


def _store_array(stores):
    arr = (fathom_store * len(stores))()
    for i, st in enumerate(stores):
        arr[i] = st._c
    return arr


def scan_batched_workspace_bytes(stores, n_q_heads, k):
    arr = _store_array(stores)
    return int(_lib.fathom_scan_batched_workspace_bytes(arr, len(stores), int(n_q_heads), int(k)))


def scan_topk_batched(stores, q, depths, k, idx=None, top_scores=None, workspace=None, stream=None):
    """Sessions `stores` (list of Store), q [S][Hq][d], depths [S][Hq][d] -> idx, top scores [S][Hq][k]."""
    S, Hq = q.shape[0], q.shape[1]
    arr = _store_array(stores)
    if idx is None:
        idx = torch.empty((S, Hq, k), dtype=torch.int32, device=q.device)
    if top_scores is None:
        top_scores = torch.empty((S, Hq, k), dtype=torch.float32, device=q.device)
    if workspace is None:
        nb = int(_lib.fathom_scan_batched_workspace_bytes(arr, S, Hq, int(k)))
        workspace = torch.empty(max(nb, 1), dtype=torch.uint8, device=q.device)
    _check(_lib.fathom_scan_topk_batched(arr, S, _ptr(q), _dtype_code(q), _ptr(depths), Hq, int(k), _ptr(idx),
                                         _ptr(top_scores), _ptr(workspace), workspace.numel(), _stream(stream)),
           "fathom_scan_topk_batched")
    return idx, top_scores


def scan_scores_view(workspace, n_q_heads, n_pad_keys):
    """The scan's scores inside a fathom_scan_topk workspace: f32 [Hq][n_pad]."""
    return workspace[: 4 * n_q_heads * n_pad_keys].view(torch.float32).view(n_q_heads, n_pad_keys)


def kv_rows(n_kv_heads, n, d, device=None, pin_memory=False):
    """K and V row views [Hkv][n][d] (bf16) of one interleaved [Hkv][n][2][d]
    buffer: a key's K and V rows are adjacent, which is the layout to use for
    rows kept in page-locked host memory."""
    kv = torch.empty((n_kv_heads, n, 2, d), dtype=torch.bfloat16, device=device, pin_memory=pin_memory)
    return kv[:, :, 0, :], kv[:, :, 1, :]


def sparse_attend(q, K_rows, V_rows, idx, n_kv_heads=None, out=None, stream=None):
    """o f32 [Hq][d]; K_rows/V_rows bf16 [Hkv][n][d] views with unit channel
    stride and equal strides (two arrays, or the views of kv_rows()), on the
    device or in page-locked host memory."""
    Hq, d = q.shape
    Hkv, n, _ = K_rows.shape
    k = idx.shape[1]
    host = not K_rows.is_cuda
    if K_rows.stride() != V_rows.stride() or K_rows.stride(2) != 1 or K_rows.stride(0) != n * K_rows.stride(1):
        raise ValueError("K_rows and V_rows need strides (n*s, s, 1), the same for both")
    if out is None:
        out = torch.empty((Hq, d), dtype=torch.float32, device=q.device)
    _check(_lib.fathom_sparse_attend(_ptr(q), _dtype_code(q), _ptr(K_rows), _ptr(V_rows), int(K_rows.stride(1)),
                                     int(host), _ptr(idx), Hq, Hkv, n, d, int(k), _ptr(out), _stream(stream)),
           "fathom_sparse_attend")
    return out


def sparse_attend_partial(q, K_rows, V_rows, idx, key0, n_kv_heads=None, parts=None, stream=None):
    """Partials f32 [Hq][d + 2] (o relative to m, then m, l) of attention over
    the rows this rank holds: K_rows/V_rows as sparse_attend, holding keys
    [key0, key0 + n); idx are global key indices (others and -1 skipped)."""
    Hq, d = q.shape
    Hkv, n, _ = K_rows.shape
    k = idx.shape[1]
    host = not K_rows.is_cuda
    if K_rows.stride() != V_rows.stride() or K_rows.stride(2) != 1 or K_rows.stride(0) != n * K_rows.stride(1):
        raise ValueError("K_rows and V_rows need strides (n*s, s, 1), the same for both")
    if parts is None:
        parts = torch.empty((Hq, d + 2), dtype=torch.float32, device=q.device)
    _check(_lib.fathom_sparse_attend_partial(_ptr(q), _dtype_code(q), _ptr(K_rows), _ptr(V_rows),
                                             int(K_rows.stride(1)), int(host), int(key0), _ptr(idx), Hq, Hkv, n, d,
                                             int(k), _ptr(parts), _stream(stream)),
           "fathom_sparse_attend_partial")
    return parts


def attend_merge(parts, out=None, stream=None):
    """o f32 [Hq][d] from the ranks' partials f32 [world][Hq][d + 2]."""
    world, Hq, d2 = parts.shape
    if out is None:
        out = torch.empty((Hq, d2 - 2), dtype=torch.float32, device=parts.device)
    _check(_lib.fathom_attend_merge(_ptr(parts.contiguous()), world, Hq, d2 - 2, _ptr(out), _stream(stream)),
           "fathom_attend_merge")
    return out


def last_device_status(stream=None):
    v = _lib.fathom_last_device_status(_stream(stream))
    if v < 0:
        raise FathomError(-v, "fathom_last_device_status")
    return v


def read_probe(src, sink, ctas=None, stream=None):
    """Stream all of `src` (device or page-locked host tensor) through the SMs."""
    host = not src.is_cuda
    if ctas is None:
        ctas = torch.cuda.get_device_properties(sink.device).multi_processor_count * 8
    _check(_lib.fathom_read_probe(_ptr(src), src.numel() * src.element_size(), int(host), _ptr(sink), int(ctas),
                                  _stream(stream)), "fathom_read_probe")


def noalloc_scratch_bytes():
    return int(_lib.fathom_noalloc_scratch_bytes())


def scan_topk_noalloc(store, q, depths, k, idx, top_scores=None, stream=None):
    """fathom_scan_topk on the library's fixed scratch array (no workspace; idx preallocated)."""
    _check(_lib.fathom_scan_topk_noalloc(store.c, _ptr(q), _dtype_code(q), _ptr(depths), q.shape[0], int(k),
                                         _ptr(idx), _ptr(top_scores), _stream(stream)), "fathom_scan_topk_noalloc")
    return idx, top_scores


def decode_workspace_bytes(store, n_q_heads, k, kv_groups):
    return int(_lib.fathom_decode_workspace_bytes(store.c, int(n_q_heads), int(k), int(kv_groups)))


def decode_step(store, q, sigma2, budget_bits, k, K_rows, V_rows, fixed_r=0, kv_groups=1, depths=None, idx=None,
                top_scores=None, out=None, workspace=None, stream=None, want_top_scores=True):
    """One decode step (depths, scan, top-k, attention) in one C-ABI call,
    pipelined over kv_groups groups of KV heads.  Returns (depths, idx,
    top_scores or None, out)."""
    Hq, d = q.shape
    dev = q.device
    rows_n = K_rows.shape[1]
    if K_rows.stride() != V_rows.stride() or K_rows.stride(2) != 1 or K_rows.stride(0) != rows_n * K_rows.stride(1):
        raise ValueError("K_rows and V_rows need strides (rows*s, s, 1), the same for both")
    if depths is None:
        depths = torch.empty((Hq, d), dtype=torch.uint8, device=dev)
    if idx is None:
        idx = torch.empty((Hq, k), dtype=torch.int32, device=dev)
    if top_scores is None and want_top_scores:
        top_scores = torch.empty((Hq, k), dtype=torch.float32, device=dev)
    if out is None:
        out = torch.empty((Hq, d), dtype=torch.float32, device=dev)
    need = decode_workspace_bytes(store, Hq, k, kv_groups)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    _check(_lib.fathom_decode_step(store.c, _ptr(q), _dtype_code(q), _ptr(sigma2), Hq, int(budget_bits), int(fixed_r),
                                   int(k), _ptr(K_rows), _ptr(V_rows), int(rows_n), int(K_rows.stride(1)),
                                   int(not K_rows.is_cuda), int(kv_groups), _ptr(depths), _ptr(idx),
                                   _ptr(top_scores), _ptr(out), _ptr(workspace), workspace.numel(), _stream(stream)),
           "fathom_decode_step")
    return depths, idx, top_scores, out
