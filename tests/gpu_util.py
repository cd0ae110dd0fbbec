"""Helpers shared by the GPU parity tests: upload, oracle calls on the same
seeded inputs, and the comparison rules.

Comparison rules (written here once, used by every GPU test):
* indexer scores: |gpu - oracle| <= 1e-2 |oracle| + 1e-5 * max|oracle| of the
  row (the floor covers fp32 accumulation on rows whose dot products cancel);
* top-k from identical scores: identical index sets (bit-exact);
* end-to-end selection: mean over rows of |gpu set & oracle set| / K_t >= 0.999;
* attention against the oracle run on the GPU's own indices: 2e-2 absolute
  for bf16, 1e-5 absolute for fp32.
"""
import numpy as np
import torch

import oracle
from sparse_attention_11_b200 import dsa, workloads as W
from sparse_attention_11_b200.problem import DeviceProblem

SCORE_REL, SCORE_FLOOR = 1e-2, 1e-5
OVERLAP_MIN = 0.999
ATOL = {"bf16": 2e-2, "f32": 1e-5}


def bf16_np(t):
    return t.detach().cpu().view(torch.int16).numpy().view(np.uint16)


def bf16_to_f64(bits):
    return W.bf16_bits_to_f32(bits).astype(np.float64)


def stratified_rows(T, n, seed=0):
    """n query rows spread over every position band, always incl. first/last."""
    if n >= T:
        return np.arange(T)
    rng = np.random.default_rng(seed)
    edges = np.linspace(0, T, n + 1).astype(np.int64)
    rows = np.array([rng.integers(a, max(a + 1, b)) for a, b in zip(edges[:-1], edges[1:])], dtype=np.int64)
    rows[0], rows[-1] = 0, T - 1
    return np.unique(rows)


def assert_scores_close(g, o, ncand):
    for r in range(g.shape[0]):
        n = int(ncand[r])
        gg, oo = g[r, :n].astype(np.float64), o[r, :n].astype(np.float64)
        tol = SCORE_REL * np.abs(oo) + SCORE_FLOOR * (np.abs(oo).max() if n else 0.0)
        bad = np.abs(gg - oo) > tol
        assert not bad.any(), f"row {r}: {bad.sum()} scores off, e.g. s={np.argmax(bad)} gpu={gg[bad][0]} oracle={oo[bad][0]}"
        assert np.all(np.isneginf(g[r, n:])), f"row {r}: entries past the causal limit are not -inf"
        assert np.all(gg >= 0) and not np.any(np.signbit(g[r, :n])), f"row {r}: negative or -0.0 score"


def sets_equal(g_idx, o_idx, ncand, k):
    for r in range(g_idx.shape[0]):
        K = min(k, int(ncand[r]))
        gs = g_idx[r, :K]
        assert np.all(g_idx[r, K:] == -1), f"row {r}: padding"
        assert np.array_equal(np.sort(gs), np.sort(o_idx[r, :K])), f"row {r}: selection differs"
        assert np.all(np.diff(gs) > 0), f"row {r}: not in ascending order"


def overlap(g_idx, o_idx, ncand, k):
    fr = []
    for r in range(g_idx.shape[0]):
        K = min(k, int(ncand[r]))
        fr.append(len(np.intersect1d(g_idx[r, :K], o_idx[r, :K])) / K)
    return float(np.mean(fr)), float(np.min(fr))


def oracle_attention_rows(inp, rows, idx_rows):
    """Oracle attention for the given rows on the given (GPU) indices."""
    wl = inp.wl
    kb, _ = inp.key_base_pos(rows)
    q = inp.q_rows(rows)
    K = inp.K
    if inp.V is None:
        V, vs = K, wl.dk
    else:
        V, vs = inp.V, wl.dv
    return oracle.attention(q, K.ravel(), wl.dk, V.ravel(), vs, kb, idx_rows, wl.scale, wl.dv)


def gpu_out_rows(prob, rows):
    r = torch.from_numpy(np.asarray(rows)).to(prob.out.device)
    o = prob.out[r]
    o = o.float() if o.dtype == torch.bfloat16 else o
    lse = prob.lse[r].cpu().numpy().astype(np.float64) if prob.lse is not None else None
    return o.cpu().numpy().astype(np.float64), lse


def gpu_fold(prob):
    wl = prob.wl
    T = wl.total_q
    u = torch.empty((T, 128), dtype=torch.float32 if wl.idx_dtype == "f32" else torch.uint8, device=prob.out.device)
    s = torch.empty(T, dtype=torch.float32, device=prob.out.device)
    ws = dsa.workspace(dsa.dsa_workspace_size(dsa.DSA_OP_FOLD, prob.seqs), prob.out.device)
    dsa.dsa_fold(prob.seqs, prob.ia, u, s, ws)
    dsa.check_device_status(ws, "fold")
    return u.cpu().numpy(), s.cpu().numpy()


def gpu_scores(prob, row_begin, row_count):
    ld = prob.seqs.max_seqlen_k
    sc = torch.empty((row_count, ld), dtype=torch.float32, device=prob.out.device)
    ws = dsa.workspace(dsa.dsa_workspace_size(dsa.DSA_OP_INDEX_SCORES, prob.seqs, 0, prob.ia), prob.out.device)
    dsa.dsa_index_scores(prob.seqs, prob.ia, row_begin, row_count, sc, ws)
    dsa.check_device_status(ws, "index_scores")
    return sc


def make(name_or_wl, **kw):
    wl = W.WORKLOADS[name_or_wl] if isinstance(name_or_wl, str) else name_or_wl
    inp = W.generate(wl, device="cuda")
    return inp, DeviceProblem(inp, **kw)
