"""Pins for the oracle's whole path on the tiny workload.

The composition must equal the separately pinned steps; with k >= L the
path must reduce to dense causal attention; every query with pos+1 <= k
keeps all of its causal keys ("DeepSeek-V3.2与稀疏注意力技术革新", §2.3).
"""
import numpy as np

import oracle
from sparse_attention_11_b200 import workloads as W
from test_oracle_topk_attn import _dense_causal


def _tiny():
    return W.generate(W.WORKLOADS["tiny_l512"], q_on_device=False)


def test_forward_rows_equals_composition():
    inp = _tiny()
    wl = inp.wl
    rows = np.array([0, 1, 63, 64, 65, 200, 511])
    kb, pos = inp.key_base_pos(rows)
    idx, out, lse = oracle.forward_rows(inp.q_idx[rows], None, inp.W, inp.k_idx, None, kb, pos, wl.k,
                                        inp.q_rows(rows), inp.K.ravel(), wl.dk, inp.K.ravel() if inp.V is None else inp.V.ravel(),
                                        wl.dk if inp.V is None else wl.dv, wl.scale, wl.dv)
    u, s_row = oracle.fold(inp.q_idx[rows], None, inp.W)
    sc = oracle.scores(u, s_row, inp.k_idx, None, kb, pos + 1, 512)
    idx2 = oracle.topk(sc, pos + 1, wl.k)
    assert np.array_equal(idx, idx2)
    out2, lse2 = oracle.attention(inp.q_rows(rows), inp.K.ravel(), wl.dk, inp.V.ravel(), wl.dv, kb, idx2, wl.scale, wl.dv)
    assert np.array_equal(out, out2) and np.array_equal(lse, lse2)
    for r, p in enumerate(pos):
        if p + 1 <= wl.k:
            assert sorted(idx[r, : p + 1]) == list(range(p + 1))
        assert np.all(sc[r, : p + 1] >= 0)


def test_forward_k_at_least_L_is_dense_causal():
    inp = _tiny()
    wl = inp.wl
    L = 96
    rows = np.arange(L)
    kb, pos = np.zeros(L, np.int64), rows.astype(np.int64)
    idx, out, lse = oracle.forward_rows(inp.q_idx[rows], None, inp.W, inp.k_idx, None, kb, pos, L,
                                        inp.q_rows(rows), inp.K.ravel(), wl.dk, inp.V.ravel(), wl.dv, wl.scale, wl.dv)
    ref, rlse = _dense_causal(inp.q_rows(rows), inp.K[:L], inp.V[:L], wl.scale)
    assert np.allclose(out, ref, atol=1e-12)
    assert np.allclose(lse, rlse, atol=1e-12)


def test_workload_generator_is_deterministic():
    a, b = _tiny(), _tiny()
    for name in ("q_idx", "k_idx", "W", "K", "V", "q_host"):
        assert np.array_equal(getattr(a, name), getattr(b, name))
    wl = W.WORKLOADS["decode_b64"]
    assert len(wl.seqlens_k) == 64 and all(16384 <= x <= 65536 for x in wl.seqlens_k)
