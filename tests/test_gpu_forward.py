"""End-to-end parity of dsa_forward on the five workloads.

The selection runs fused (one tensor-core indexer / top-k kernel) at 32K and
128K and on the batched case (sequences of at most 2048 keys).  prefill_l8192
and the 3000-token case (fewer than 80 128-row blocks over more than 2048
keys) take the two-launch path: a key-split score sweep, then the
histogram top-k.
For every checked row: the selection equals dsa_topk applied to the
scores of dsa_index_scores (same arithmetic, bit-exact), its overlap with
the oracle's own selection is >= 0.999, and the attention output matches the
oracle run on the GPU's selected indices (2e-2 abs bf16, 1e-5 abs fp32).
Large workloads are checked on stratified row samples in the launch
configuration the benchmark times."""
import numpy as np
import pytest
import torch

import oracle
from sparse_attention_11_b200 import dsa, workloads as W

from gpu_util import (ATOL, OVERLAP_MIN, gpu_out_rows, make, oracle_attention_rows, overlap, sets_equal,
                      stratified_rows)

pytestmark = pytest.mark.gpu


def _oracle_select(inp, rows):
    """Oracle fold -> scores -> top-k for the given rows."""
    wl = inp.wl
    kb, pos = inp.key_base_pos(rows)
    qs = inp.q_idx_scale[rows] if inp.q_idx_scale is not None else None
    u, s = oracle.fold(inp.q_idx[rows], qs, inp.W)
    sc = oracle.scores(u, s, inp.k_idx, inp.k_idx_scale, kb, pos + 1, int(pos.max()) + 1)
    return oracle.topk(sc, pos + 1, wl.k), pos


def _consistency(prob, rows_begin, rows_count):
    """Fused selection == dsa_topk(dsa_index_scores) on a contiguous row range."""
    wl = prob.wl
    ld = prob.seqs.max_seqlen_k
    sc = torch.empty((rows_count, ld), dtype=torch.float32, device="cuda")
    ws = dsa.workspace(dsa.dsa_workspace_size(dsa.DSA_OP_INDEX_SCORES, prob.seqs, 0, prob.ia))
    dsa.dsa_index_scores(prob.seqs, prob.ia, rows_begin, rows_count, sc, ws)
    idx2 = torch.empty((rows_count, wl.k), dtype=torch.int32, device="cuda")
    dsa.dsa_topk(prob.seqs, sc, rows_begin, rows_count, wl.k, idx2, ws)
    dsa.check_device_status(ws, "scores+topk")
    a = prob.idx[rows_begin: rows_begin + rows_count].cpu().numpy()
    b = idx2.cpu().numpy()
    assert np.array_equal(a, b), f"fused selection differs from topk(scores) in {np.any(a != b, axis=1).sum()} rows"


def _boundary_rows(wl):
    """Rows at the positions where the selection changes character: pos = k-1
    (the last row that keeps its whole prefix), k, k+1."""
    T, k = wl.total_q, wl.k
    return np.array([p for p in (k - 1, k, k + 1) if 0 <= p < T], dtype=np.int64)


def _run(name, n_sel_rows, n_attn_rows, consistency_ranges):
    wl = W.WORKLOADS[name] if isinstance(name, str) else name
    inp, prob = make(wl)
    prob.out.fill_(float("nan"))
    prob.forward()
    prob.check("forward")
    T = wl.total_q
    for rb, rc in consistency_ranges:
        _consistency(prob, rb, min(rc, T - rb))
    g_idx_all = prob.idx
    rows = stratified_rows(T, n_sel_rows, seed=1)
    o_idx, pos = _oracle_select(inp, rows)
    g_idx = g_idx_all[torch.from_numpy(rows).cuda()].cpu().numpy()
    mean_ov, min_ov = overlap(g_idx, o_idx, pos + 1, wl.k)
    assert mean_ov >= OVERLAP_MIN, (mean_ov, min_ov)
    for r in range(len(rows)):
        K = min(wl.k, int(pos[r]) + 1)
        assert np.all(g_idx[r, K:] == -1) and np.all(np.diff(g_idx[r, :K]) > 0)
        assert g_idx[r, :K].min() >= 0 and g_idx[r, :K].max() <= pos[r]
    arows = np.unique(np.concatenate([stratified_rows(T, n_attn_rows, seed=2), _boundary_rows(wl)])) \
        if wl.batch == 1 else stratified_rows(T, n_attn_rows, seed=2)
    g_idx_a = g_idx_all[torch.from_numpy(arows).cuda()].cpu().numpy()
    o, olse = oracle_attention_rows(inp, arows, g_idx_a)
    g, glse = gpu_out_rows(prob, arows)
    err = np.abs(g - o).max()
    assert err <= ATOL[wl.attn_dtype], err
    assert np.abs(glse - olse).max() <= (1e-5 if wl.attn_dtype == "f32" else 2e-2)
    return mean_ov


def test_forward_tiny_l512():
    inp, prob = make("tiny_l512")
    prob.forward()
    prob.check("forward")
    rows = np.arange(512)
    o_idx, pos = _oracle_select(inp, rows)
    g_idx = prob.idx.cpu().numpy()
    assert overlap(g_idx, o_idx, pos + 1, 64)[0] >= OVERLAP_MIN
    # every query with pos+1 <= k keeps its whole causal prefix
    for p in range(64):
        assert list(g_idx[p, : p + 1]) == list(range(p + 1))
    o, olse = oracle_attention_rows(inp, rows, g_idx)
    g, glse = gpu_out_rows(prob, rows)
    assert np.abs(g - o).max() <= ATOL["f32"]
    assert np.abs(glse - olse).max() <= 1e-5


def test_forward_small_prefill_selection_heavy():
    """k much smaller than L: every row's k-th score is deep in its tail."""
    wl = W.custom("prefill_l3000_k256", (3000,), (3000,), base="prefill_l8192", k=256)
    _run(wl, 3000, 48, [(0, 3000)])


def test_forward_batched_prefill():
    wl = W.custom("prefill_b3", (700, 1500, 129), (700, 1500, 129), base="prefill_l8192", k=300)
    _run(wl, 2329, 32, [(0, 2329)])


def test_forward_prefill_l8192():
    _run("prefill_l8192", 1024, 64, [(0, 8192)])


def test_forward_decode_b64():
    _run("decode_b64", 64, 64, [(0, 64)])


def test_forward_prefill_l32768():
    _run("prefill_l32768", 256, 128, [(0, 128), (16384, 256), (32768 - 128, 128)])


def test_forward_prefill_l131072():
    _run("prefill_l131072", 256, 128, [(131072 - 128, 128), (65536, 128)])


def test_fused_selection_matches_oracle_topk_l32768():
    """The fused selection at L=32768 against the oracle's top-k of the GPU's
    own scores (dsa_index_scores), row by row: identical index sets on 256
    rows spread over every position band plus the rows at pos = k-1, k, k+1
    (the comparison does not go through dsa_topk)."""
    wl = W.WORKLOADS["prefill_l32768"]
    inp, prob = make(wl)
    dsa.dsa_select(prob.seqs, prob.ia, wl.k, prob.idx, prob.ws)
    prob.check("select")
    rows = np.unique(np.concatenate([stratified_rows(wl.total_q, 256, seed=3), _boundary_rows(wl)]))
    ld = prob.seqs.max_seqlen_k
    sc = torch.empty((1, ld), dtype=torch.float32, device="cuda")
    ws = dsa.workspace(dsa.dsa_workspace_size(dsa.DSA_OP_INDEX_SCORES, prob.seqs, 0, prob.ia))
    g_sc = np.empty((len(rows), ld), dtype=np.float32)
    for i, r in enumerate(rows):
        dsa.dsa_index_scores(prob.seqs, prob.ia, int(r), 1, sc, ws)
        g_sc[i] = sc[0].cpu().numpy()
    dsa.check_device_status(ws, "index_scores")
    _, pos = inp.key_base_pos(rows)
    o_idx = oracle.topk(g_sc, pos + 1, wl.k)
    g_idx = prob.idx[torch.from_numpy(rows).cuda()].cpu().numpy()
    sets_equal(g_idx, o_idx, pos + 1, wl.k)


@pytest.mark.parametrize("name", ["prefill_l8192", "batched"])
def test_forward_host_matches_forward(name):
    """dsa_forward_host (query and output in pinned host memory, chunked and
    pipelined over three streams) returns exactly dsa_forward's output, lse and
    indices: 8 chunks at L=8192, 3 chunks for a ragged batch of 2329 rows."""
    wl = W.WORKLOADS[name] if name != "batched" else \
        W.custom("prefill_b3h", (700, 1500, 129), (700, 1500, 129), base="prefill_l8192", k=300)
    inp, prob = make(wl)
    prob.forward()
    prob.check("forward")
    ref_out, ref_lse, ref_idx = prob.out.clone(), prob.lse.clone(), prob.idx.clone()
    q_host = torch.empty(prob.q.shape, dtype=prob.q.dtype, pin_memory=True)
    q_host.copy_(prob.q)
    out_host = torch.full(prob.out.shape, float("nan"), dtype=prob.out.dtype, pin_memory=True)
    lse = torch.full_like(prob.lse, float("nan"))
    idx = torch.full_like(prob.idx, -7)
    aa = dsa.attn_args(q_host, prob.K, prob.V, wl.scale, out_host, lse)
    ws = dsa.workspace(dsa.dsa_workspace_size(dsa.DSA_OP_FORWARD_HOST, prob.seqs, wl.k, prob.ia, aa))
    h2d, d2h = torch.cuda.Stream(), torch.cuda.Stream()
    dsa.dsa_forward_host(prob.seqs, prob.ia, aa, wl.k, idx, ws, h2d, d2h)
    dsa.check_device_status(ws, "forward_host")
    torch.cuda.current_stream().synchronize()
    assert torch.equal(idx, ref_idx)
    assert torch.equal(lse, ref_lse)
    assert torch.equal(out_host, ref_out.cpu())
