"""Oracle for the Fathom bit-plane key scan -- TEST INFRASTRUCTURE ONLY.

A plain, single-threaded fp64 C++ restatement of the method (fathom_ref.cpp),
loaded with ctypes.  Only tests/, __graft_entry__.smoke() and bench.py's CPU
baseline / reference arm may import this package.  The product package
(bit_plane_key_b200) never imports it, and the two share no code.

Every wrapper takes and returns numpy arrays in the store's layouts:
  K        f32  [H][n][d]
  planes   u32  [H][d][4][n_pad/32]   key i -> word i/32, bit i%32, plane 0 = MSB
  scales   u16  [H][d][n_pad/64]      fp16 bits of the block scale
  q        f32  [Hq][d]               (bf16 queries are widened exactly first)
  sigma2   f32  [Hkv][d]
  depths   u8   [Hq][d]
  K_rows, V_rows  u16 (bf16 bits) [Hkv][n][d]
"""
import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "fathom_ref.cpp")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None

CXXFLAGS = ["-O2", "-std=c++17", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared"]


def build(force=False):
    """Compile fathom_ref.cpp into liboracle.so (g++, host only)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + ".tmp%d" % os.getpid()
    subprocess.check_call(["g++"] + CXXFLAGS + ["-o", tmp, _SRC])
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def lib():
    global _lib
    if _lib is None:
        build()
        _lib = ctypes.CDLL(_LIB_PATH)
        _declare(_lib)
    return _lib


_P = ctypes.c_void_p
_I = ctypes.c_int
_L = ctypes.c_int64


def _declare(L):
    L.oref_f32_to_f16.restype = ctypes.c_uint16
    L.oref_f32_to_f16.argtypes = [ctypes.c_float]
    L.oref_f16_to_f32.restype = ctypes.c_float
    L.oref_f16_to_f32.argtypes = [ctypes.c_uint16]
    L.oref_f32_to_f16_array.argtypes = [_P, _P, _L]
    L.oref_n_pad.restype = _L
    L.oref_n_pad.argtypes = [_L]
    L.oref_quantize.argtypes = [_P, _I, _L, _I, _P, _P]
    L.oref_pack_planes.argtypes = [_P, _I, _L, _I, _P]
    L.oref_pack.argtypes = [_P, _I, _L, _I, _P, _P]
    L.oref_importance.argtypes = [_P, _P, _I, _P]
    L.oref_depths.restype = _I
    L.oref_depths.argtypes = [_P, _I, _I, _P]
    L.oref_fixed_depths.restype = _I
    L.oref_fixed_depths.argtypes = [_P, _I, _I, _P]
    L.oref_alloc_depths.restype = _I
    L.oref_alloc_depths.argtypes = [_P, _P, _I, _I, _I, _I, _I, _P]
    L.oref_alloc_depths_pooled.restype = _I
    L.oref_alloc_depths_pooled.argtypes = [_P, _P, _I, _I, _I, _I, _P]
    L.oref_reconstruct.argtypes = [_P, _P, _I, _L, _I, _I, _P, _P]
    L.oref_scores_head.restype = _I
    L.oref_scores_head.argtypes = [_P, _P, _I, _L, _I, _I, _P, _P, _L, _L, _P, _P]
    L.oref_scores.restype = _I
    L.oref_scores.argtypes = [_P, _P, _I, _L, _I, _P, _I, _P, _L, _L, _P, _P]
    L.oref_topk_f64.restype = _I
    L.oref_topk_f64.argtypes = [_P, _L, _I, _P]
    L.oref_topk_f32.restype = _I
    L.oref_topk_f32.argtypes = [_P, _L, _I, _P]
    L.oref_attend.restype = _I
    L.oref_attend.argtypes = [_P, _P, _P, _P, _I, _I, _L, _I, _I, _P]
    L.oref_decode.restype = _I
    L.oref_decode.argtypes = [_P, _P, _P, _P, _P, _P, _I, _I, _L, _I, _I, _I, _I, _P, _P, _P]


def _c(a, dtype):
    a = np.ascontiguousarray(a, dtype=dtype)
    return a


def _ptr(a):
    return ctypes.c_void_p(a.ctypes.data) if a is not None else None


def _check(rc, what):
    if rc != 0:
        raise ValueError("oracle %s failed (rc=%d)" % (what, rc))


def n_pad(n):
    return int(lib().oref_n_pad(int(n)))


def f32_to_f16_bits(x):
    x = _c(x, np.float32).ravel()
    out = np.empty(x.size, np.uint16)
    lib().oref_f32_to_f16_array(_ptr(x), _ptr(out), x.size)
    return out


def f16_bits_to_f32(h):
    return np.array([lib().oref_f16_to_f32(int(v)) for v in np.ravel(h)], np.float32)


def quantize(K):
    K = _c(K, np.float32)
    H, n, d = K.shape
    npad = n_pad(n)
    scales = np.empty((H, d, npad // 64), np.uint16)
    codes = np.empty((H, n, d), np.uint8)
    lib().oref_quantize(_ptr(K), H, n, d, _ptr(scales), _ptr(codes))
    return scales, codes


def pack_planes(codes):
    codes = _c(codes, np.uint8)
    H, n, d = codes.shape
    planes = np.empty((H, d, 4, n_pad(n) // 32), np.uint32)
    lib().oref_pack_planes(_ptr(codes), H, n, d, _ptr(planes))
    return planes


def pack(K):
    K = _c(K, np.float32)
    H, n, d = K.shape
    npad = n_pad(n)
    planes = np.empty((H, d, 4, npad // 32), np.uint32)
    scales = np.empty((H, d, npad // 64), np.uint16)
    lib().oref_pack(_ptr(K), H, n, d, _ptr(planes), _ptr(scales))
    return planes, scales


def importance(q, sigma2):
    q = _c(q, np.float32)
    s = _c(sigma2, np.float32)
    w = np.empty(q.size, np.float32)
    lib().oref_importance(_ptr(q), _ptr(s), q.size, _ptr(w))
    return w


def depths(w, B):
    w = _c(w, np.float32)
    t = np.empty(w.size, np.uint8)
    _check(lib().oref_depths(_ptr(w), w.size, int(B), _ptr(t)), "depths")
    return t


def fixed_depths(q, r):
    q = _c(q, np.float32)
    t = np.empty(q.size, np.uint8)
    _check(lib().oref_fixed_depths(_ptr(q), q.size, int(r), _ptr(t)), "fixed_depths")
    return t


def alloc_depths_pooled(q, sigma2, B):
    """Group-pooled depths (a variant, not the pages' per-query rule)."""
    q = _c(q, np.float32)
    s = _c(sigma2, np.float32)
    Hq, d = q.shape
    Hkv = s.shape[0]
    out = np.empty((Hq, d), np.uint8)
    _check(lib().oref_alloc_depths_pooled(_ptr(q), _ptr(s), Hq, Hkv, d, int(B), _ptr(out)), "alloc_depths_pooled")
    return out


def alloc_depths(q, sigma2, B, fixed_r=0):
    q = _c(q, np.float32)
    s = _c(sigma2, np.float32)
    Hq, d = q.shape
    Hkv = s.shape[0]
    out = np.empty((Hq, d), np.uint8)
    _check(lib().oref_alloc_depths(_ptr(q), _ptr(s), Hq, Hkv, d, int(B), int(fixed_r), _ptr(out)),
           "alloc_depths")
    return out


def reconstruct(planes, scales, n, g, t):
    planes = _c(planes, np.uint32)
    scales = _c(scales, np.uint16)
    H, d = planes.shape[0], planes.shape[1]
    t = _c(t, np.uint8)
    out = np.empty((n, d), np.float64)
    lib().oref_reconstruct(_ptr(planes), _ptr(scales), H, n, d, int(g), _ptr(t), _ptr(out))
    return out


def scores(planes, scales, n, q, dep, i0=0, i1=None, with_abs=False):
    """fp64 scores [Hq][i1-i0] (and sum_c |q_c khat_c| if with_abs)."""
    planes = _c(planes, np.uint32)
    scales = _c(scales, np.uint16)
    q = _c(q, np.float32)
    dep = _c(dep, np.uint8)
    Hkv, d = planes.shape[0], planes.shape[1]
    Hq = q.shape[0]
    i1 = n if i1 is None else i1
    m = i1 - i0
    s = np.empty((Hq, m), np.float64)
    a = np.empty((Hq, m), np.float64) if with_abs else None
    _check(lib().oref_scores(_ptr(planes), _ptr(scales), Hkv, n, d, _ptr(q), Hq, _ptr(dep), i0, i1,
                             _ptr(s), _ptr(a)), "scores")
    return (s, a) if with_abs else s


def scores_head(planes, scales, n, g, q_h, t_h, i0=0, i1=None, with_abs=False):
    planes = _c(planes, np.uint32)
    scales = _c(scales, np.uint16)
    q_h = _c(q_h, np.float32)
    t_h = _c(t_h, np.uint8)
    Hkv, d = planes.shape[0], planes.shape[1]
    i1 = n if i1 is None else i1
    s = np.empty(i1 - i0, np.float64)
    a = np.empty(i1 - i0, np.float64) if with_abs else None
    _check(lib().oref_scores_head(_ptr(planes), _ptr(scales), Hkv, n, d, int(g), _ptr(q_h), _ptr(t_h),
                                  i0, i1, _ptr(s), _ptr(a)), "scores_head")
    return (s, a) if with_abs else s


def topk(s, k):
    """Indices of the k largest entries of a 1-D array, ties to the lower index."""
    s = np.ascontiguousarray(s)
    idx = np.empty(k, np.int32)
    if s.dtype == np.float64:
        rc = lib().oref_topk_f64(_ptr(s), s.size, int(k), _ptr(idx))
    elif s.dtype == np.float32:
        rc = lib().oref_topk_f32(_ptr(s), s.size, int(k), _ptr(idx))
    else:
        raise TypeError(s.dtype)
    _check(rc, "topk")
    return idx


def attend(q, K_rows, V_rows, idx):
    q = _c(q, np.float32)
    K_rows = _c(K_rows, np.uint16)
    V_rows = _c(V_rows, np.uint16)
    idx = _c(idx, np.int32)
    Hq, d = q.shape
    Hkv, n = K_rows.shape[0], K_rows.shape[1]
    k = idx.shape[1]
    out = np.empty((Hq, d), np.float64)
    _check(lib().oref_attend(_ptr(q), _ptr(K_rows), _ptr(V_rows), _ptr(idx), Hq, Hkv, n, d, k, _ptr(out)),
           "attend")
    return out


def decode(planes, scales, n, q, sigma2, B, k, fixed_r=0, K_rows=None, V_rows=None):
    """depths, top-k indices and (if rows are given) attention output of one layer."""
    planes = _c(planes, np.uint32)
    scales = _c(scales, np.uint16)
    q = _c(q, np.float32)
    s2 = _c(sigma2, np.float32)
    Hkv, d = planes.shape[0], planes.shape[1]
    Hq = q.shape[0]
    dep = np.empty((Hq, d), np.uint8)
    idx = np.empty((Hq, k), np.int32)
    out = np.empty((Hq, d), np.float64) if K_rows is not None else None
    Kr = _c(K_rows, np.uint16) if K_rows is not None else None
    Vr = _c(V_rows, np.uint16) if V_rows is not None else None
    _check(lib().oref_decode(_ptr(planes), _ptr(scales), _ptr(Kr), _ptr(Vr), _ptr(q), _ptr(s2), Hq, Hkv, n, d,
                             int(B), int(fixed_r), int(k), _ptr(dep), _ptr(idx), _ptr(out)), "decode")
    return dep, idx, out
