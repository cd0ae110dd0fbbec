"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every entry point include/dsa.h declares, and rejects bad arguments before
launching anything."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from sparse_attention_11_b200 import build
    build.build()
    from sparse_attention_11_b200 import dsa
    return dsa


def _declared():
    src = open(os.path.join(ROOT, "include", "dsa.h")).read()
    return sorted(set(re.findall(r"DSA_API\s+[\w\s\*]*?\b(dsa_\w+)\s*\(", src)))


def test_header_declares_entry_points():
    names = _declared()
    for n in ("dsa_index_scores", "dsa_topk", "dsa_sparse_attn", "dsa_forward", "dsa_fold",
              "dsa_workspace_size", "dsa_sync_status", "dsa_status_string"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    raw = ctypes.CDLL(lib.LIB_PATH)
    for n in _declared():
        assert hasattr(raw, n), n
    assert set(_declared()) <= set(lib.EXPORTED) | set(_declared())


def test_status_strings(lib):
    assert lib.status_string(0) == "ok"
    assert "timed out" in lib.status_string(lib.DSA_ERR_TIMEOUT)
    assert lib.status_string(99) == "unknown status"
    assert lib.version() >= 1000


def _fake_seqs(lib, batch=1, tq=64, tk=64):
    # device pointers are never dereferenced on the host; any non-null value will do
    return lib.dsa_seqs(batch, tq, tk, tq, tk, 0x1000, 0x2000)


def test_validation_rejects_before_launch(lib):
    S = _fake_seqs(lib)
    P = ctypes.c_void_p
    ws = P(0x10000)  # 256-aligned, never touched on rejection
    # k < 1
    assert lib.raw_call("dsa_topk", ctypes.byref(S), P(0x3000), 64, 0, 64, 0, P(0x4000), 64, ws, 1 << 20, None) \
        == lib.DSA_ERR_INVALID_ARG
    # rows out of range
    assert lib.raw_call("dsa_topk", ctypes.byref(S), P(0x3000), 64, 10, 60, 8, P(0x4000), 64, ws, 1 << 20, None) \
        == lib.DSA_ERR_INVALID_ARG
    # ld_scores < max_seqlen_k
    assert lib.raw_call("dsa_topk", ctypes.byref(S), P(0x3000), 32, 0, 64, 8, P(0x4000), 64, ws, 1 << 20, None) \
        == lib.DSA_ERR_INVALID_ARG
    # workspace too small / misaligned
    assert lib.raw_call("dsa_topk", ctypes.byref(S), P(0x3000), 64, 0, 64, 8, P(0x4000), 64, ws, 16, None) \
        == lib.DSA_ERR_WORKSPACE
    assert lib.raw_call("dsa_topk", ctypes.byref(S), P(0x3000), 64, 0, 64, 8, P(0x4000), 64, P(0x10010), 1 << 20,
                        None) == lib.DSA_ERR_INVALID_ARG
    # batch 0
    S0 = lib.dsa_seqs(0, 64, 64, 64, 64, 0x1000, 0x2000)
    assert lib.raw_call("dsa_topk", ctypes.byref(S0), P(0x3000), 64, 0, 64, 8, P(0x4000), 64, ws, 1 << 20, None) \
        == lib.DSA_ERR_INVALID_ARG


def test_unsupported_attention_shapes(lib):
    S = _fake_seqs(lib)
    P = ctypes.c_void_p
    ws = P(0x10000)
    idx = P(0x5000)
    for dt, h, dk, dv in ((lib.DSA_BF16, 64, 576, 512), (lib.DSA_BF16, 128, 128, 128), (lib.DSA_F32, 64, 64, 64),
                          (lib.DSA_F32, 4, 48, 64), (7, 4, 64, 64)):
        aa = lib.dsa_attn_args(dt, h, dk, dv, 0x100000, h * dk, dk, 0x200000, dk, 0x300000, dk, 0.1, 0x400000,
                               h * dv, dv, None)
        assert lib.raw_call("dsa_sparse_attn", ctypes.byref(S), ctypes.byref(aa), idx, 64, 64, ws, 1 << 20, None) \
            == lib.DSA_ERR_UNSUPPORTED, (dt, h, dk, dv)


def test_indexer_dtype_rules(lib):
    S = _fake_seqs(lib)
    P = ctypes.c_void_p
    n = ctypes.c_size_t(0)
    # E4M3 without scales
    ia = lib.dsa_indexer_args(lib.DSA_E4M3, 0x100000, None, lib.DSA_BF16, 0x200000, 0x300000, None)
    assert lib.raw_call("dsa_fold", ctypes.byref(S), ctypes.byref(ia), P(0x400000), P(0x500000), P(0x10000),
                        1 << 20, None) == lib.DSA_ERR_INVALID_ARG
    # F32 with a bf16 W
    ia = lib.dsa_indexer_args(lib.DSA_F32, 0x100000, None, lib.DSA_BF16, 0x200000, 0x300000, None)
    assert lib.raw_call("dsa_fold", ctypes.byref(S), ctypes.byref(ia), P(0x400000), P(0x500000), P(0x10000),
                        1 << 20, None) == lib.DSA_ERR_UNSUPPORTED
    # workspace size grows with k for the forward op
    ia = lib.dsa_indexer_args(lib.DSA_E4M3, 0x100000, 0x110000, lib.DSA_BF16, 0x200000, 0x300000, 0x310000)
    sizes = []
    for k in (64, 2048):
        assert lib.raw_call("dsa_workspace_size", lib.DSA_OP_FORWARD, ctypes.byref(S), k, ctypes.byref(ia), None,
                            ctypes.byref(n)) == 0
        sizes.append(n.value)
    assert sizes[1] > sizes[0] >= 256


def test_selection_path_workspace(lib):
    """The selection path follows from the shapes alone, and so does the
    workspace.  Fewer than 80 128-row blocks over > 2048 keys select in two launches
    through a score buffer of total_q x max_seqlen_k floats.  Otherwise the
    prefill-shaped problem runs fused, with no score buffer: each of its
    persistent CTAs (at most one per SM; 148 without a GPU to ask) holds a
    bitmask of 128 rows x 8 * ceil(max_seqlen_k / 256) words."""
    n = ctypes.c_size_t(0)
    ia = lib.dsa_indexer_args(lib.DSA_E4M3, 0x100000, 0x110000, lib.DSA_BF16, 0x200000, 0x300000, 0x310000)

    def size(batch, tq, tk, mq, mk):
        S = lib.dsa_seqs(batch, tq, tk, mq, mk, 0x1000, 0x2000)
        assert lib.raw_call("dsa_workspace_size", lib.DSA_OP_FORWARD, ctypes.byref(S), 2048, ctypes.byref(ia), None,
                            ctypes.byref(n)) == 0
        return n.value

    k = 2048
    split = [(1, 2048, 32768, 2048, 32768), (1, 8192, 8192, 8192, 8192), (1, 10112, 10112, 10112, 10112),
             (2, 8192, 32768, 4096, 16384), (1, 2049, 2049, 2049, 2049), (1, 3000, 3000, 3000, 3000)]
    fused = [(1, 32768, 32768, 32768, 32768), (1, 2048, 2048, 2048, 2048), (1, 10240, 10240, 10240, 10240),
             (1, 18816, 18816, 18816, 18816), (3, 2329, 2329, 1500, 1500), (4, 32768, 32768, 8192, 8192)]
    for b, tq, tk, mq, mk in split:
        assert size(b, tq, tk, mq, mk) >= tq * mk * 4 + tq * k * 4, (b, tq, tk)
    for b, tq, tk, mq, mk in fused:
        ctas = min(148, b * ((mq + 127) // 128))
        bits = ctas * 128 * 8 * ((mk + 255) // 256) * 4
        got = size(b, tq, tk, mq, mk)
        assert bits <= got < tq * k * 4 + tq * 256 + (1 << 20) + bits, (b, tq, tk)


def test_backward_validation(lib):
    """dsa_sparse_attn_bwd rejects bad arguments before launching: a missing
    lse or gradient buffer, unsupported dtype or dims, short strides, a short
    workspace."""
    S = _fake_seqs(lib, tq=64, tk=64)
    P = ctypes.c_void_p
    h, dk, dv = 128, 576, 512

    def aa(dtype=lib.DSA_BF16, dk_=dk, dv_=dv, lse=0x500000):
        return lib.dsa_attn_args(dtype, h, dk_, dv_, 0x100000, h * dk_, dk_, 0x200000, dk_, 0x200000, dk_, 0.1,
                                 0x400000, h * dv_, dv_, lse)

    def call(a, d_out=0x600000, dq=0x700000, dk_=0x800000, dks=dk, dvs=dk, dos=(h * dv, dv), ws_bytes=1 << 20):
        return lib.raw_call("dsa_sparse_attn_bwd", ctypes.byref(S), ctypes.byref(a), P(0x900000), 64, 64, P(d_out),
                            dos[0], dos[1], P(dq), h * dk, dk, P(dk_), dks, P(dk_), dvs, P(0x10000), ws_bytes, None)

    assert call(aa(lse=None)) == lib.DSA_ERR_INVALID_ARG
    assert call(aa(), d_out=0) == lib.DSA_ERR_INVALID_ARG
    assert call(aa(), dq=0) == lib.DSA_ERR_INVALID_ARG
    assert call(aa(), dk_=0) == lib.DSA_ERR_INVALID_ARG
    assert call(aa(lib.DSA_E4M3)) == lib.DSA_ERR_UNSUPPORTED
    assert call(aa(dk_=640)) == lib.DSA_ERR_UNSUPPORTED
    assert call(aa(), dks=500) == lib.DSA_ERR_INVALID_ARG
    assert call(aa(), dos=(h * dv, 100)) == lib.DSA_ERR_INVALID_ARG
    assert call(aa(), ws_bytes=64) == lib.DSA_ERR_WORKSPACE


def test_kl_entry_points_validation(lib):
    """dsa_attn_target and dsa_indexer_kl reject bad arguments before
    launching anything."""
    S = _fake_seqs(lib, tq=64, tk=64)
    P = ctypes.c_void_p
    h, dk, dv = 128, 576, 512
    ok_aa = lib.dsa_attn_args(lib.DSA_BF16, h, dk, dv, 0x100000, h * dk, dk, 0x200000, dk, 0x200000, dk, 0.1,
                              0x400000, h * dv, dv, 0x500000)
    no_lse = lib.dsa_attn_args(lib.DSA_BF16, h, dk, dv, 0x100000, h * dk, dk, 0x200000, dk, 0x200000, dk, 0.1,
                               0x400000, h * dv, dv, None)
    tgt = lambda a, ldp=64, ws_bytes=1 << 20: lib.raw_call("dsa_attn_target", ctypes.byref(S), ctypes.byref(a),
                                                           P(0x900000), 64, 64, P(0xA00000), ldp, P(0x10000),
                                                           ws_bytes, None)
    assert tgt(no_lse) == lib.DSA_ERR_INVALID_ARG
    assert tgt(ok_aa, ldp=32) == lib.DSA_ERR_INVALID_ARG
    assert tgt(ok_aa, ws_bytes=64) == lib.DSA_ERR_WORKSPACE

    def kl(q=0x100000, qs=128, W=0x200000, k_sel=64, p=0xA00000, ws_bytes=1 << 20):
        return lib.raw_call("dsa_indexer_kl", ctypes.byref(S), P(q), qs, P(W), P(0x300000), 128, P(0x900000), 64,
                            k_sel, P(p), 64, None, P(0x700000), 128, P(0x800000), P(0x600000), 128, P(0x10000),
                            ws_bytes, None)
    assert kl(q=0) == lib.DSA_ERR_INVALID_ARG
    assert kl(qs=64) == lib.DSA_ERR_INVALID_ARG
    assert kl(W=0) == lib.DSA_ERR_INVALID_ARG
    assert kl(p=0) == lib.DSA_ERR_INVALID_ARG
    assert kl(k_sel=100) == lib.DSA_ERR_INVALID_ARG  # ld_idx 64 < k_sel
    assert kl(ws_bytes=64) == lib.DSA_ERR_WORKSPACE


def test_forward_host_validation(lib):
    """The host-memory forward rejects non-packed or fp32 attention operands
    and short workspaces before touching the device; its workspace holds the
    forward's plus two staging chunks each for Q and the output."""
    S = _fake_seqs(lib, tq=4096, tk=4096)
    P = ctypes.c_void_p
    n = ctypes.c_size_t(0)
    ia = lib.dsa_indexer_args(lib.DSA_E4M3, 0x100000, 0x110000, lib.DSA_BF16, 0x200000, 0x300000, 0x310000)
    h, dk, dv = 128, 576, 512
    packed = lib.dsa_attn_args(lib.DSA_BF16, h, dk, dv, 0x100000, h * dk, dk, 0x200000, dk, 0x200000, dk, 0.1,
                               0x400000, h * dv, dv, None)
    assert lib.raw_call("dsa_workspace_size", lib.DSA_OP_FORWARD, ctypes.byref(S), 2048, ctypes.byref(ia), None,
                        ctypes.byref(n)) == 0
    fwd = n.value
    assert lib.raw_call("dsa_workspace_size", lib.DSA_OP_FORWARD_HOST, ctypes.byref(S), 2048, ctypes.byref(ia),
                        ctypes.byref(packed), ctypes.byref(n)) == 0
    chunk = 1024  # DSA_HOST_CHUNK_ROWS
    assert n.value >= fwd + 2 * chunk * h * (dk + dv) * 2
    ws = P(0x10000)
    call = lambda aa, nbytes: lib.raw_call("dsa_forward_host", ctypes.byref(S), ctypes.byref(ia), ctypes.byref(aa),
                                           2048, None, 0, ws, nbytes, None, None, None)
    assert call(packed, 1 << 20) == lib.DSA_ERR_WORKSPACE
    strided = lib.dsa_attn_args(lib.DSA_BF16, h, dk, dv, 0x100000, h * 640, 640, 0x200000, dk, 0x200000, dk, 0.1,
                                0x400000, h * dv, dv, None)
    assert call(strided, 1 << 40) == lib.DSA_ERR_INVALID_ARG
    f32 = lib.dsa_attn_args(lib.DSA_F32, 4, 64, 64, 0x100000, 256, 64, 0x200000, 64, 0x300000, 64, 0.1,
                            0x400000, 256, 64, None)
    assert call(f32, 1 << 40) == lib.DSA_ERR_UNSUPPORTED


def test_bench_launch_count_follows_library_path(lib):
    """bench.py counts 4 launches per prefill step where the library selects
    in two launches, else 3.  The library's choice shows in its workspace:
    only the two-launch (and scan) paths hold a score buffer."""
    import sys
    sys.path.insert(0, ROOT)
    import bench
    from sparse_attention_11_b200 import workloads as W
    n = ctypes.c_size_t(0)
    ia = lib.dsa_indexer_args(lib.DSA_E4M3, 0x100000, 0x110000, lib.DSA_BF16, 0x200000, 0x300000, 0x310000)
    shapes = [((8192,), (8192,)), ((32768,), (32768,)), ((2048,), (2048,)), ((3000,), (3000,)),
              ((18944,), (18944,)), ((18816,), (18816,)), ((700, 1500, 129), (700, 1500, 129)),
              ((2048,), (32768,))]
    for sq, sk in shapes:
        wl = W.custom("probe", sq, sk, base="prefill_l8192")
        S = lib.dsa_seqs(len(sq), sum(sq), sum(sk), max(sq), max(sk), 0x1000, 0x2000)
        assert lib.raw_call("dsa_workspace_size", lib.DSA_OP_FORWARD, ctypes.byref(S), wl.k, ctypes.byref(ia), None,
                            ctypes.byref(n)) == 0
        has_scores = n.value >= sum(sq) * max(sk) * 4 + sum(sq) * wl.k * 4  # score buffer on top of the index rows
        assert bench.step_launches(wl) == (4 if has_scores else 3), (sq, sk, n.value)
