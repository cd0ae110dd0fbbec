"""Dynamic k: a per-query k ("DeepSeek-V3.2与稀疏注意力技术革新", §6 names a
dynamic k as a future direction), through the C ABI.

Query t keeps K_t = min(clamp(k_t, 0, k), pos_t + 1) keys.  Checked on the
three selection paths, with per-query k drawn uniformly in [0, k] plus the
edge values 0, 1, k and past k:
  * prefill_l32768: the fused tensor-core indexer / top-k;
  * prefill_l8192: 64 row blocks over 8192 keys, which selects in two
    launches (split tensor-core score sweep, then the histogram top-k);
  * decode_b64: the scan + the histogram top-k.
Each is checked as follows:
  * the fused selection equals, bit for bit, the exact top-K_t of the GPU's
    own scores (dsa_index_scores ranked by the oracle's top-k), in ascending
    order, -1 after;
  * its overlap with the oracle's own selection (oracle scores) is >= 0.999;
  * the attention output on those indices matches the oracle's (bf16 2e-2).
"""
import numpy as np
import pytest
import torch

import oracle
from sparse_attention_11_b200 import dsa, workloads as W

from gpu_util import ATOL, OVERLAP_MIN, gpu_out_rows, gpu_scores, make, oracle_attention_rows, stratified_rows

pytestmark = pytest.mark.gpu


def _k_rows(T, k, seed):
    rng = np.random.default_rng(seed)
    kr = rng.integers(0, k + 1, size=T).astype(np.int32)
    kr[::97] = 0
    kr[1::89] = 1
    kr[2::83] = k
    kr[3::79] = k + 500  # clamped to k
    return kr


@pytest.mark.parametrize("name", ["prefill_l32768", "prefill_l8192", "decode_b64"])
def test_dynamic_k(name):
    wl = W.WORKLOADS[name]
    inp, prob = make(wl)
    T = wl.total_q
    kr = _k_rows(T, wl.k, 5)
    ia = dsa.indexer_args(prob.q_idx, prob.q_idx_scale, prob.W, prob.k_idx, prob.k_idx_scale,
                          k_per_row=torch.from_numpy(kr).cuda())
    idx = torch.full((T, wl.k), -7, dtype=torch.int32, device="cuda")
    prob.out.fill_(float("nan"))
    ws = dsa.workspace(dsa.dsa_workspace_size(dsa.DSA_OP_FORWARD, prob.seqs, wl.k, ia))
    dsa.dsa_forward(prob.seqs, ia, prob.aa, wl.k, idx, ws)
    dsa.check_device_status(ws, "dynamic-k forward")
    g_all = idx.cpu().numpy()
    _, pos_all = inp.key_base_pos(np.arange(T))
    kt = np.minimum(np.clip(kr, 0, wl.k), pos_all + 1)

    # 1) bit-exact against the exact top-K_t of the GPU's own scores
    ranges = [(0, min(64, T))] if T <= 256 else [(0, 64), (T // 2 - 32, 64), (T - 64, 64)]
    for rb, rc in ranges:
        sc = gpu_scores(prob, rb, rc).cpu().numpy()
        rows = np.arange(rb, rb + rc)
        exp = oracle.topk_dyn(sc, pos_all[rows] + 1, kr[rows], wl.k)
        for i, r in enumerate(rows):
            K = int(kt[r])
            g = g_all[r]
            assert np.all(g[K:] == -1), f"row {r}: padding"
            assert np.all(np.diff(g[:K]) > 0), f"row {r}: not ascending"
            assert np.array_equal(g[:K], np.sort(exp[i, :K])), f"row {r}: selection differs"

    # 2) against the oracle's own selection
    rows = stratified_rows(T, 128, seed=4)
    kb, pos = inp.key_base_pos(rows)
    qs = inp.q_idx_scale[rows] if inp.q_idx_scale is not None else None
    u, s = oracle.fold(inp.q_idx[rows], qs, inp.W)
    osc = oracle.scores(u, s, inp.k_idx, inp.k_idx_scale, kb, pos + 1, int(pos.max()) + 1)
    o_idx = oracle.topk_dyn(osc, pos + 1, kr[rows], wl.k)
    fr = []
    for i, r in enumerate(rows):
        K = int(kt[r])
        if K:
            fr.append(len(np.intersect1d(g_all[r, :K], o_idx[i, :K])) / K)
    assert np.mean(fr) >= OVERLAP_MIN, (np.mean(fr), np.min(fr))

    # 3) attention on the GPU's indices against the oracle
    arows = stratified_rows(T, 48, seed=6)
    o, olse = oracle_attention_rows(inp, arows, g_all[arows])
    g, glse = gpu_out_rows(prob, arows)
    assert np.abs(g - o).max() <= ATOL["bf16"]
    empty = kt[arows] == 0
    assert np.all(g[empty] == 0) and np.all(np.isneginf(glse[empty]))
