"""ctypes wrapper around dsa_oracle.c (argument marshalling only).

TEST INFRASTRUCTURE: the tests, the smoke check and the benchmark's
CPU-baseline leg use this module; the CUDA product path never does.  Every
numeric step lives in dsa_oracle.c; this file only converts numpy arrays to
pointers.
"""
import ctypes
import os
import subprocess

import numpy as np

F32, BF16, E4M3 = 0, 1, 2
_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "dsa_oracle.c")
_LIB = os.path.join(_HERE, "liborc.so")
_lib = None


def lib_path():
    return _LIB


def build(force=False):
    """Compile dsa_oracle.c into oracle/liborc.so with gcc (-O2 -fopenmp)."""
    if not force and os.path.exists(_LIB) and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC):
        return _LIB
    cmd = ["gcc", "-O2", "-std=c99", "-fopenmp", "-fPIC", "-shared", "-Wall", "-o", _LIB, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        P, I64, I32, I = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_int
        L.orc_e4m3_decode.restype = ctypes.c_double
        L.orc_e4m3_decode.argtypes = [ctypes.c_uint8]
        L.orc_e4m3_encode.restype = ctypes.c_uint8
        L.orc_e4m3_encode.argtypes = [ctypes.c_float]
        L.orc_bf16_decode.restype = ctypes.c_double
        L.orc_bf16_decode.argtypes = [ctypes.c_uint16]
        L.orc_fold.argtypes = [I64, I, P, P, I, P, P, P]
        L.orc_scores.argtypes = [I64, I, P, P, P, P, P, P, I64, P]
        L.orc_topk.argtypes = [I64, P, I64, P, I32, P, I64]
        L.orc_topk_dyn.argtypes = [I64, P, I64, P, P, I32, P, I64]
        L.orc_attention.argtypes = [I64, I, I, I, I, P, P, I64, P, I64, P, P, I64, I32,
                                    ctypes.c_double, P, P]
        L.orc_forward_rows.argtypes = [I64, I, P, P, I, P, P, P, P, P, I64, I32,
                                       I, I, I, I, P, P, I64, P, I64, ctypes.c_double, P, P, P]
        L.orc_num_threads.restype = I
        _lib = L
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return None if a is None else np.ascontiguousarray(a, dtype=dtype)


def _dt(arr):
    """Oracle dtype code of a numpy array holding raw elements."""
    if arr.dtype == np.float32:
        return F32
    if arr.dtype == np.uint16:
        return BF16
    if arr.dtype == np.uint8:
        return E4M3
    raise TypeError(f"unsupported raw dtype {arr.dtype}")


def num_threads():
    return _load().orc_num_threads()


def e4m3_decode(code):
    return _load().orc_e4m3_decode(int(code))


def e4m3_encode(x):
    return int(_load().orc_e4m3_encode(float(x)))


def bf16_decode(bits):
    return _load().orc_bf16_decode(int(bits))


def fold(q_idx, q_scale, W):
    """q_idx: float32 [n,128] or uint8 e4m3 codes [n,128]; W: float32 or
    uint16 (bf16 bits) [128,128].  Returns (u, s_row)."""
    q_idx = np.ascontiguousarray(q_idx)
    W = np.ascontiguousarray(W)
    n = q_idx.shape[0]
    idt = _dt(q_idx)
    u = np.empty((n, 128), dtype=np.float32 if idt == F32 else np.uint8)
    s_row = np.empty(n, dtype=np.float32)
    _load().orc_fold(n, idt, _p(q_idx), _p(_c(q_scale, np.float32)), _dt(W), _p(W), _p(u), _p(s_row))
    return u, s_row


def scores(u, s_row, k_idx, k_scale, key_base, ncand, ld):
    """Scores of n folded query rows against their causal key prefixes."""
    u = np.ascontiguousarray(u)
    k_idx = np.ascontiguousarray(k_idx)
    n = u.shape[0]
    out = np.empty((n, ld), dtype=np.float32)
    _load().orc_scores(n, _dt(u), _p(u), _p(_c(s_row, np.float32)), _p(k_idx),
                       _p(_c(k_scale, np.float32)), _p(_c(key_base, np.int64)),
                       _p(_c(ncand, np.int64)), ld, _p(out))
    return out


def topk(scores_arr, ncand, k):
    s = np.ascontiguousarray(scores_arr, dtype=np.float32)
    n, ld = s.shape
    idx = np.empty((n, k), dtype=np.int32)
    _load().orc_topk(n, _p(s), ld, _p(_c(ncand, np.int64)), int(k), _p(idx), k)
    return idx


def topk_dyn(scores_arr, ncand, k_rows, k):
    """Dynamic k: row r keeps min(clamp(k_rows[r], 0, k), ncand[r]) keys (same
    order as topk), in a row of width k padded with -1."""
    s = np.ascontiguousarray(scores_arr, dtype=np.float32)
    n, ld = s.shape
    idx = np.empty((n, k), dtype=np.int32)
    _load().orc_topk_dyn(n, _p(s), ld, _p(_c(ncand, np.int64)), _p(_c(k_rows, np.int32)), int(k), _p(idx), k)
    return idx


def attention(q, K, k_stride, V, v_stride, key_base, idx, scale, dv):
    """q: [n,H,dk] float32 or uint16 (bf16 bits); K/V: flat arrays of the
    same dtype with the given row strides (elements)."""
    q = np.ascontiguousarray(q)
    n, H, dk = q.shape
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    out = np.empty((n, H, dv), dtype=np.float64)
    lse = np.empty((n, H), dtype=np.float64)
    _load().orc_attention(n, _dt(q), H, dk, dv, _p(q), _p(K), k_stride, _p(V), v_stride,
                          _p(_c(key_base, np.int64)), _p(idx), idx.shape[1], idx.shape[1],
                          float(scale), _p(out), _p(lse))
    return out, lse


def forward_rows(q_idx, q_scale, W, k_idx, k_scale, key_base, pos, k, q, K, k_stride, V, v_stride,
                 scale, dv):
    """Whole path (fold, scores, top-k, attention) for n gathered query rows."""
    q_idx = np.ascontiguousarray(q_idx)
    W = np.ascontiguousarray(W)
    q = np.ascontiguousarray(q)
    n, H, dk = q.shape
    pos = _c(pos, np.int64)
    idx = np.empty((n, k), dtype=np.int32)
    out = np.empty((n, H, dv), dtype=np.float64)
    lse = np.empty((n, H), dtype=np.float64)
    max_nc = int(pos.max()) + 1 if n else 1
    _load().orc_forward_rows(n, _dt(q_idx), _p(q_idx), _p(_c(q_scale, np.float32)), _dt(W), _p(W),
                             _p(k_idx), _p(_c(k_scale, np.float32)), _p(_c(key_base, np.int64)),
                             _p(pos), max_nc, int(k), _dt(q), H, dk, dv, _p(q), _p(K), k_stride,
                             _p(V), v_stride, float(scale), _p(idx), _p(out), _p(lse))
    return idx, out, lse
