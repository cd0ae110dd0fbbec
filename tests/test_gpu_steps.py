"""GPU parity of each step of the path, through the C ABI, against the CPU
oracle on the same seeded inputs (fold, indexer scores, top-k, attention).
Sizes span several tiles with a ragged tail; the comparison rules are in
gpu_util."""
import numpy as np
import pytest
import torch

import oracle
from sparse_attention_11_b200 import dsa, workloads as W

from gpu_util import (ATOL, assert_scores_close, gpu_fold, gpu_out_rows, gpu_scores, make,
                      oracle_attention_rows, sets_equal)

pytestmark = pytest.mark.gpu


def _fp8_prefill(L, k=2048, name=None, **kw):
    return W.custom(name or f"prefill_l{L}_k{k}", (L,), (L,), base="prefill_l8192", k=k, **kw)


def _fp8_decode(ctx, name="decode_small"):
    return W.custom(name, (1,) * len(ctx), tuple(ctx), base="decode_b64")


# ---------------------------------------------------------------- a1 fold
@pytest.mark.parametrize("wl", ["tiny_l512", "fp8_1000", "fp8_3000", "fp8_20000"])
def test_fold(wl):
    # 1000 rows: a column of W per thread; 3000: 2 rows per warp; 20000: 8 rows
    # per warp on persistent CTAs, ragged last group
    wl = W.WORKLOADS["tiny_l512"] if wl == "tiny_l512" else _fp8_prefill(int(wl[4:]))
    inp, prob = make(wl)
    u, s = gpu_fold(prob)
    uo, so = oracle.fold(inp.q_idx, inp.q_idx_scale, inp.W)
    if wl.idx_dtype == "f32":
        assert np.allclose(u, uo, rtol=1e-5, atol=1e-6)
        assert np.all(s == 1)
        return
    # codes equal except, rarely, one e4m3 step where the fp32 fold sits on a
    # rounding midpoint; scales within 1e-6
    assert np.allclose(s, so, rtol=1e-6, atol=0)
    diff = u != uo
    assert diff.mean() <= 1e-3, diff.mean()
    if diff.any():
        gd = torch.from_numpy(u[diff]).view(torch.float8_e4m3fn).float().numpy()
        od = torch.from_numpy(uo[diff]).view(torch.float8_e4m3fn).float().numpy()
        step = np.maximum(np.abs(od), 2.0 ** -6) / 8
        assert np.all(np.abs(gd - od) <= step * 1.001)


# ---------------------------------------------------------------- a2 scores
@pytest.mark.parametrize("case", ["tiny", "fp8_tc", "fp8_scan"])
def test_index_scores(case):
    if case == "tiny":
        wl = W.WORKLOADS["tiny_l512"]
    elif case == "fp8_tc":
        wl = _fp8_prefill(1300, k=256)           # 11 row blocks, 6 key tiles, ragged
    else:
        wl = _fp8_decode([700, 3000, 1])
    inp, prob = make(wl)
    T = wl.total_q
    rb, rc = (0, T) if T < 64 or case != "fp8_tc" else (100, T - 150)
    g = gpu_scores(prob, rb, rc).cpu().numpy()
    u, s = gpu_fold(prob)
    rows = np.arange(rb, rb + rc)
    kb, pos = inp.key_base_pos(rows)
    o = oracle.scores(u[rows], s[rows], inp.k_idx, inp.k_idx_scale, kb, pos + 1, g.shape[1])
    assert_scores_close(g, o, pos + 1)


# ---------------------------------------------------------------- a3 top-k
def _adversarial_scores(rng, n_rows, n_cols):
    kind = rng.integers(0, 6, size=n_rows)
    out = np.empty((n_rows, n_cols), np.float32)
    for r in range(n_rows):
        if kind[r] == 0:
            out[r] = rng.standard_normal(n_cols)
        elif kind[r] == 1:     # few levels: heavy ties at the threshold
            out[r] = rng.integers(0, 4, n_cols).astype(np.float32)
        elif kind[r] == 2:     # ReLU-like: half zeros, +0/-0 mix
            x = np.maximum(rng.standard_normal(n_cols), 0).astype(np.float32)
            x[rng.random(n_cols) < 0.3] = -0.0
            out[r] = x
        elif kind[r] == 3:     # all equal
            out[r] = 1.5
        elif kind[r] == 4:     # denormals, infinities, NaN
            x = (rng.standard_normal(n_cols) * 1e-39).astype(np.float32)
            x[rng.random(n_cols) < 0.05] = np.inf
            x[rng.random(n_cols) < 0.05] = -np.inf
            x[rng.random(n_cols) < 0.05] = np.nan
            out[r] = x
        else:                  # values differing in the last mantissa bits
            base = np.float32(3.0)
            out[r] = (base + rng.integers(0, 8, n_cols) * np.spacing(base)).astype(np.float32)
    return out


@pytest.mark.parametrize("L,k", [(300, 64), (5000, 2048), (3000, 100)])
def test_topk_bitexact(L, k):
    rng = np.random.default_rng(L + k)
    wl = W.custom(f"topk_{L}", (L,), (L,), base="prefill_l8192", k=k)
    seqs = dsa.Seqs([0, L], [0, L])
    sc = _adversarial_scores(rng, L, L)
    idx = torch.full((L, k), -7, dtype=torch.int32, device="cuda")
    ws = dsa.workspace(dsa.dsa_workspace_size(dsa.DSA_OP_TOPK, seqs))
    dsa.dsa_topk(seqs, torch.from_numpy(sc).cuda(), 0, L, k, idx, ws)
    dsa.check_device_status(ws, "topk")
    g = idx.cpu().numpy()
    ncand = np.arange(L) + 1
    rows = np.unique(np.concatenate([np.arange(0, L, 7), np.arange(L - 40, L), [k - 1, k, k + 1]]))
    rows = rows[(rows >= 0) & (rows < L)]
    o = oracle.topk(sc[rows], ncand[rows], k)
    sets_equal(g[rows], o, ncand[rows], k)


def test_topk_batched_decode_rows():
    rng = np.random.default_rng(5)
    ctx = [3000, 2049, 2048, 10, 5000]
    seqs = dsa.Seqs(np.arange(6), np.concatenate([[0], np.cumsum(ctx)]))
    ld = max(ctx)
    sc = _adversarial_scores(rng, 5, ld)
    k = 2048
    idx = torch.empty((5, k), dtype=torch.int32, device="cuda")
    ws = dsa.workspace(256)
    dsa.dsa_topk(seqs, torch.from_numpy(sc).cuda(), 0, 5, k, idx, ws)
    dsa.check_device_status(ws, "topk")
    ncand = np.array(ctx)
    sets_equal(idx.cpu().numpy(), oracle.topk(sc, ncand, k), ncand, k)


# ---------------------------------------------------------------- a4 attention
def _random_idx(rng, inp, rows, k_sel, pad_frac=0.0):
    kb, pos = inp.key_base_pos(rows)
    idx = np.full((len(rows), k_sel), -1, np.int32)
    for i, p in enumerate(pos):
        n = min(k_sel, p + 1)
        sel = rng.choice(p + 1, size=n, replace=False).astype(np.int32)
        if pad_frac:
            sel[rng.random(n) < pad_frac] = -1
        idx[i, :n] = sel
    return idx


@pytest.mark.parametrize("case", ["aliased", "separate", "padded", "short"])
def test_sparse_attn_bf16(case):
    rng = np.random.default_rng(11)
    ctx = [5000, 3000, 70, 2500]
    wl = _fp8_decode(ctx, name="attn_" + case)
    inp, prob = make(wl, v_separate=(case == "separate"))
    rows = np.arange(wl.total_q)
    k_sel = {"short": 100}.get(case, 2048)
    idx = _random_idx(rng, inp, rows, k_sel, pad_frac=0.3 if case == "padded" else 0.0)
    idx_t = torch.from_numpy(idx).cuda()
    prob.out.fill_(float("nan"))
    dsa.dsa_sparse_attn(prob.seqs, prob.aa, idx_t, k_sel, prob.ws)
    prob.check("sparse_attn")
    g, glse = gpu_out_rows(prob, rows)
    o, olse = oracle_attention_rows(inp, rows, idx)
    err = np.abs(g - o).max()
    assert err <= ATOL["bf16"], err
    assert np.allclose(glse, olse, atol=2e-2), np.abs(glse - olse).max()


def test_sparse_attn_single_key_is_v_row():
    rng = np.random.default_rng(12)
    wl = _fp8_decode([900, 1200], name="attn_single")
    inp, prob = make(wl)
    idx = np.full((2, 128), -1, np.int32)
    idx[0, 77] = 13
    idx[1, 0] = 1199
    dsa.dsa_sparse_attn(prob.seqs, prob.aa, torch.from_numpy(idx).cuda(), 128, prob.ws)
    prob.check("sparse_attn")
    g, _ = gpu_out_rows(prob, [0, 1])
    K = inp.K
    v0 = W.bf16_bits_to_f32(K[13, :512])
    v1 = W.bf16_bits_to_f32(K[900 + 1199, :512])
    assert np.array_equal(g[0], np.broadcast_to(v0, (128, 512)))
    assert np.array_equal(g[1], np.broadcast_to(v1, (128, 512)))


def test_sparse_attn_empty_rows():
    wl = _fp8_decode([300, 400], name="attn_empty")
    inp, prob = make(wl)
    idx = np.full((2, 64), -1, np.int32)
    dsa.dsa_sparse_attn(prob.seqs, prob.aa, torch.from_numpy(idx).cuda(), 64, prob.ws)
    prob.check("sparse_attn")
    g, lse = gpu_out_rows(prob, [0, 1])
    assert np.all(g == 0) and np.all(np.isneginf(lse))


def test_sparse_attn_f32_tiny():
    rng = np.random.default_rng(13)
    inp, prob = make("tiny_l512")
    rows = np.arange(512)
    idx = _random_idx(rng, inp, rows, 64, pad_frac=0.1)
    dsa.dsa_sparse_attn(prob.seqs, prob.aa, torch.from_numpy(idx).cuda(), 64, prob.ws)
    prob.check("sparse_attn")
    g, glse = gpu_out_rows(prob, rows)
    o, olse = oracle_attention_rows(inp, rows, idx)
    assert np.abs(g - o).max() <= ATOL["f32"]
    assert np.abs(glse - olse).max() <= 1e-5


def test_out_of_range_index_is_reported():
    wl = _fp8_decode([300], name="attn_oob")
    inp, prob = make(wl)
    idx = np.full((1, 64), -1, np.int32)
    idx[0, :3] = [5, 300, 7]       # 300 is past seqlen_k
    dsa.dsa_sparse_attn(prob.seqs, prob.aa, torch.from_numpy(idx).cuda(), 64, prob.ws)
    code, _ = dsa.dsa_sync_status(prob.ws)
    assert code == dsa.DSA_ERR_INDEX
    assert dsa.dsa_sync_status(prob.ws)[0] == dsa.DSA_OK   # cleared


def test_wait_timeout_selftest():
    ws = dsa.workspace(256)
    dsa.dsa_selftest_wait_timeout(ws, 2_000_000)
    code, detail = dsa.dsa_sync_status(ws)
    assert code == dsa.DSA_ERR_TIMEOUT and detail == 0x5E1F
    # the context is still usable afterwards
    x = torch.ones(4, device="cuda")
    assert float(x.sum()) == 4.0
