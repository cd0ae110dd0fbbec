"""Python binding of libdsa (include/dsa.h): argument marshalling only.

Every function here has the name of the C entry point it calls, takes torch
tensors (device memory owned by torch) and passes their pointers, sizes and
the current CUDA stream.  No step of the DSA path runs in Python: if the
shared library is missing, importing this module raises.
"""
import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdsa.so")

DSA_OK, DSA_ERR_INVALID_ARG, DSA_ERR_UNSUPPORTED, DSA_ERR_WORKSPACE, DSA_ERR_CUDA, DSA_ERR_TIMEOUT, DSA_ERR_INDEX = range(7)
DSA_F32, DSA_BF16, DSA_E4M3 = 0, 1, 2
DSA_OP_FOLD, DSA_OP_INDEX_SCORES, DSA_OP_TOPK, DSA_OP_SPARSE_ATTN, DSA_OP_FORWARD, DSA_OP_FORWARD_HOST = range(6)

if not os.path.exists(LIB_PATH):
    raise ImportError(f"libdsa.so not built ({LIB_PATH}); run python -m sparse_attention_11_b200.build")
_lib = ctypes.CDLL(LIB_PATH)

_P, _I32, _I64, _SZ, _F = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t, ctypes.c_float


class dsa_seqs(ctypes.Structure):
    _fields_ = [("batch", _I32), ("total_q", _I64), ("total_k", _I64), ("max_seqlen_q", _I64),
                ("max_seqlen_k", _I64), ("cu_seqlens_q", _P), ("cu_seqlens_k", _P)]


class dsa_indexer_args(ctypes.Structure):
    _fields_ = [("dtype", _I32), ("q_idx", _P), ("q_idx_scale", _P), ("w_dtype", _I32), ("w_index", _P),
                ("k_idx", _P), ("k_idx_scale", _P), ("k_per_row", _P)]


class dsa_attn_args(ctypes.Structure):
    _fields_ = [("dtype", _I32), ("heads", _I32), ("dk", _I32), ("dv", _I32), ("q", _P), ("q_stride_tok", _I64),
                ("q_stride_head", _I64), ("k", _P), ("k_stride", _I64), ("v", _P), ("v_stride", _I64),
                ("scale", _F), ("out", _P), ("out_stride_tok", _I64), ("out_stride_head", _I64), ("lse", _P)]


_S, _IA, _AA = ctypes.POINTER(dsa_seqs), ctypes.POINTER(dsa_indexer_args), ctypes.POINTER(dsa_attn_args)
_lib.dsa_status_string.restype = ctypes.c_char_p
_lib.dsa_status_string.argtypes = [ctypes.c_int]
_lib.dsa_version.restype = ctypes.c_int
_lib.dsa_workspace_size.argtypes = [ctypes.c_int, _S, _I32, _IA, _AA, ctypes.POINTER(_SZ)]
_lib.dsa_fold.argtypes = [_S, _IA, _P, _P, _P, _SZ, _P]
_lib.dsa_index_scores.argtypes = [_S, _IA, _I64, _I64, _P, _I64, _P, _SZ, _P]
_lib.dsa_topk.argtypes = [_S, _P, _I64, _I64, _I64, _I32, _P, _I64, _P, _SZ, _P]
_lib.dsa_sparse_attn.argtypes = [_S, _AA, _P, _I64, _I32, _P, _SZ, _P]
_lib.dsa_attn_target.argtypes = [_S, _AA, _P, _I64, _I32, _P, _I64, _P, _SZ, _P]
_lib.dsa_indexer_kl.argtypes = [_S, _P, _I64, _P, _P, _I64, _P, _I64, _I32, _P, _I64, _P, _P, _I64, _P, _P, _I64, _P,
                                _SZ, _P]
_lib.dsa_sparse_attn_bwd.argtypes = [_S, _AA, _P, _I64, _I32, _P, _I64, _I64, _P, _I64, _I64, _P, _I64, _P, _I64,
                                     _P, _SZ, _P]
_lib.dsa_forward.argtypes = [_S, _IA, _AA, _I32, _P, _I64, _P, _SZ, _P]
_lib.dsa_forward_host.argtypes = [_S, _IA, _AA, _I32, _P, _I64, _P, _SZ, _P, _P, _P]
_lib.dsa_select.argtypes = [_S, _IA, _I32, _P, _I64, _P, _SZ, _P]
_lib.dsa_select_noalloc.argtypes = [_S, _IA, _I32, _P, _I64, _P]
_lib.dsa_sync_status.argtypes = [_P, _P, ctypes.POINTER(_I64)]
_lib.dsa_selftest_wait_timeout.argtypes = [_P, _SZ, _I64, _P]
for _f in ("dsa_workspace_size", "dsa_fold", "dsa_index_scores", "dsa_topk", "dsa_sparse_attn", "dsa_sparse_attn_bwd",
           "dsa_attn_target", "dsa_indexer_kl",
           "dsa_forward",
           "dsa_forward_host",
           "dsa_select", "dsa_select_noalloc",
           "dsa_sync_status", "dsa_selftest_wait_timeout"):
    getattr(_lib, _f).restype = ctypes.c_int

EXPORTED = ("dsa_status_string", "dsa_version", "dsa_workspace_size", "dsa_fold", "dsa_index_scores", "dsa_topk",
            "dsa_sparse_attn", "dsa_sparse_attn_bwd", "dsa_attn_target", "dsa_indexer_kl", "dsa_forward",
            "dsa_forward_host", "dsa_select",
            "dsa_select_noalloc", "dsa_sync_status",
            "dsa_selftest_wait_timeout")


class DsaError(RuntimeError):
    def __init__(self, code, where, detail=None):
        msg = f"{where}: {_lib.dsa_status_string(code).decode()} (status {code})"
        if detail is not None:
            msg += f", detail {detail}"
        super().__init__(msg)
        self.code = code
        self.detail = detail


def _check(code, where):
    if code != DSA_OK:
        raise DsaError(code, where)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def status_string(code):
    return _lib.dsa_status_string(code).decode()


def version():
    return _lib.dsa_version()


class Seqs:
    """Packed batch description; keeps the device cu_seqlens tensors alive."""

    def __init__(self, cu_q, cu_k, device="cuda"):
        cq = torch.as_tensor(cu_q, dtype=torch.int64)
        ck = torch.as_tensor(cu_k, dtype=torch.int64)
        lq, lk = (cq[1:] - cq[:-1]), (ck[1:] - ck[:-1])
        self.cu_q = cq.to(device)
        self.cu_k = ck.to(device)
        self.c = dsa_seqs(len(cq) - 1, int(cq[-1]), int(ck[-1]), int(lq.max()) if len(lq) else 0,
                          int(lk.max()) if len(lk) else 0, self.cu_q.data_ptr(), self.cu_k.data_ptr())

    @property
    def total_q(self):
        return self.c.total_q

    @property
    def total_k(self):
        return self.c.total_k

    @property
    def max_seqlen_k(self):
        return self.c.max_seqlen_k


def indexer_args(q_idx, q_idx_scale, w_index, k_idx, k_idx_scale, k_per_row=None):
    """Indexer operands: float32 tensors (fp32 path) or uint8 e4m3 codes +
    float32 scales with a bfloat16 W (FP8 path); k_per_row: optional int32
    device tensor [total_q] of per-query k (dynamic k)."""
    fp8 = q_idx.dtype == torch.uint8
    a = dsa_indexer_args(DSA_E4M3 if fp8 else DSA_F32, q_idx.data_ptr(),
                         q_idx_scale.data_ptr() if q_idx_scale is not None else None,
                         DSA_BF16 if w_index.dtype == torch.bfloat16 else DSA_F32, w_index.data_ptr(),
                         k_idx.data_ptr(), k_idx_scale.data_ptr() if k_idx_scale is not None else None,
                         k_per_row.data_ptr() if k_per_row is not None else None)
    a._keep = (q_idx, q_idx_scale, w_index, k_idx, k_idx_scale, k_per_row)
    return a


def attn_args(q, k, v, scale, out, lse=None):
    """q [T,H,dk]; k [Tk,>=dk] (row stride k.stride(0)); v [Tk,>=dv] (may be a
    view of k's first columns); out [T,H,dv]; lse [T,H] or None."""
    dt = DSA_BF16 if q.dtype == torch.bfloat16 else DSA_F32
    a = dsa_attn_args(dt, q.shape[1], q.shape[2], out.shape[2], q.data_ptr(), q.stride(0), q.stride(1), k.data_ptr(),
                      k.stride(0), v.data_ptr(), v.stride(0), float(scale), out.data_ptr(), out.stride(0),
                      out.stride(1), lse.data_ptr() if lse is not None else None)
    a._keep = (q, k, v, out, lse)
    return a


def dsa_workspace_size(op, seqs, k=0, ia=None, aa=None):
    n = _SZ(0)
    _check(_lib.dsa_workspace_size(op, ctypes.byref(seqs.c), k, ctypes.byref(ia) if ia is not None else None,
                                   ctypes.byref(aa) if aa is not None else None, ctypes.byref(n)), "dsa_workspace_size")
    return n.value


def workspace(nbytes, device="cuda"):
    """A zeroed workspace (its status header starts cleared)."""
    return torch.zeros(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def dsa_fold(seqs, ia, u_out, s_row_out, ws):
    _check(_lib.dsa_fold(ctypes.byref(seqs.c), ctypes.byref(ia), _ptr(u_out), _ptr(s_row_out), _ptr(ws), ws.numel(),
                         _stream()), "dsa_fold")


def dsa_index_scores(seqs, ia, row_begin, row_count, scores, ws):
    _check(_lib.dsa_index_scores(ctypes.byref(seqs.c), ctypes.byref(ia), row_begin, row_count, _ptr(scores),
                                 scores.stride(0), _ptr(ws), ws.numel(), _stream()), "dsa_index_scores")


def dsa_topk(seqs, scores, row_begin, row_count, k, idx, ws):
    _check(_lib.dsa_topk(ctypes.byref(seqs.c), _ptr(scores), scores.stride(0), row_begin, row_count, k, _ptr(idx),
                         idx.stride(0), _ptr(ws), ws.numel(), _stream()), "dsa_topk")


def dsa_sparse_attn(seqs, aa, idx, k_sel, ws):
    _check(_lib.dsa_sparse_attn(ctypes.byref(seqs.c), ctypes.byref(aa), _ptr(idx), idx.stride(0), k_sel, _ptr(ws),
                                ws.numel(), _stream()), "dsa_sparse_attn")


def dsa_sparse_attn_bwd(seqs, aa, idx, k_sel, d_out, d_q, d_k, d_v, ws):
    """Backward of dsa_sparse_attn.  aa is the forward's attn_args (its out
    and lse hold the forward's results; lse is required).  d_out [T,H,dv]
    has q's dtype; d_q [T,H,dk] float32 is written; d_k [Tk,>=dk] and d_v
    [Tk,>=dv] float32 accumulate (zero them first; d_v may be a view of d_k's
    first dv columns for the MLA-tied gradient)."""
    _check(_lib.dsa_sparse_attn_bwd(ctypes.byref(seqs.c), ctypes.byref(aa), _ptr(idx), idx.stride(0), k_sel,
                                    _ptr(d_out), d_out.stride(0), d_out.stride(1), _ptr(d_q), d_q.stride(0),
                                    d_q.stride(1), _ptr(d_k), d_k.stride(0), _ptr(d_v), d_v.stride(0), _ptr(ws),
                                    ws.numel(), _stream()), "dsa_sparse_attn_bwd")


def dsa_attn_target(seqs, aa, idx, k_sel, p, ws):
    """Head-averaged attention probabilities of the selected keys (the
    indexer's KL target).  aa is the forward's attn_args (lse required);
    p float32 [T, >= k_sel] is zeroed and written."""
    _check(_lib.dsa_attn_target(ctypes.byref(seqs.c), ctypes.byref(aa), _ptr(idx), idx.stride(0), k_sel, _ptr(p),
                                p.stride(0), _ptr(ws), ws.numel(), _stream()), "dsa_attn_target")


def dsa_indexer_kl(seqs, q_idx, W, k_idx, idx, k_sel, p, loss, d_q, d_W, d_k, ws):
    """The indexer's KL loss over the selection and its gradients (float32
    tensors: q_idx [T,128], W [128,128], k_idx [Tk,128], p [T,>=k_sel];
    loss [T] or None; d_q written; d_W, d_k accumulated)."""
    _check(_lib.dsa_indexer_kl(ctypes.byref(seqs.c), _ptr(q_idx), q_idx.stride(0), _ptr(W), _ptr(k_idx),
                               k_idx.stride(0), _ptr(idx), idx.stride(0), k_sel, _ptr(p), p.stride(0), _ptr(loss),
                               _ptr(d_q), d_q.stride(0), _ptr(d_W), _ptr(d_k), d_k.stride(0), _ptr(ws), ws.numel(),
                               _stream()), "dsa_indexer_kl")


def dsa_forward_host(seqs, ia, aa, k, idx_out, ws, h2d_stream=None, d2h_stream=None):
    """dsa_forward with aa's q and out in pinned host memory (see attn_args);
    the copies run on h2d_stream / d2h_stream (torch.cuda.Stream or None for
    the current stream), the compute on the current stream."""
    cur = _stream()
    sh = ctypes.c_void_p(h2d_stream.cuda_stream) if h2d_stream is not None else cur
    sd = ctypes.c_void_p(d2h_stream.cuda_stream) if d2h_stream is not None else cur
    _check(_lib.dsa_forward_host(ctypes.byref(seqs.c), ctypes.byref(ia), ctypes.byref(aa), k, _ptr(idx_out),
                                 idx_out.stride(0) if idx_out is not None else 0, _ptr(ws), ws.numel(), cur, sh, sd),
           "dsa_forward_host")


def dsa_forward(seqs, ia, aa, k, idx_out, ws):
    _check(_lib.dsa_forward(ctypes.byref(seqs.c), ctypes.byref(ia), ctypes.byref(aa), k, _ptr(idx_out),
                            idx_out.stride(0) if idx_out is not None else 0, _ptr(ws), ws.numel(), _stream()),
           "dsa_forward")


def dsa_select(seqs, ia, k, idx, ws):
    _check(_lib.dsa_select(ctypes.byref(seqs.c), ctypes.byref(ia), k, _ptr(idx), idx.stride(0), _ptr(ws), ws.numel(),
                           _stream()), "dsa_select")


def dsa_select_noalloc(seqs, ia, k, idx):
    """dsa_select without a workspace (for callers that cannot allocate device
    memory): synchronous, returns nothing, raises DsaError on any status."""
    _check(_lib.dsa_select_noalloc(ctypes.byref(seqs.c), ctypes.byref(ia), k, _ptr(idx), idx.stride(0), _stream()),
           "dsa_select_noalloc")


def dsa_sync_status(ws):
    """Synchronise the current stream; return (status, detail) recorded on the
    device since the last call, and clear it."""
    d = _I64(0)
    code = _lib.dsa_sync_status(_ptr(ws), _stream(), ctypes.byref(d))
    return code, d.value


def check_device_status(ws, where="device"):
    code, detail = dsa_sync_status(ws)
    if code != DSA_OK:
        raise DsaError(code, where, detail)


def dsa_selftest_wait_timeout(ws, budget_cycles):
    _check(_lib.dsa_selftest_wait_timeout(_ptr(ws), ws.numel(), budget_cycles, _stream()), "dsa_selftest_wait_timeout")


def raw_call(name, *args):
    """Call a C entry point with raw ctypes arguments (tests of the ABI)."""
    return getattr(_lib, name)(*args)
