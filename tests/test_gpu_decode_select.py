"""Decode-shaped selection (FP8 scan, then the top-k from the score histogram)
on inputs built to reach each of its paths:

- random keys: the k-th score's histogram bin is listed and ranked on chip;
- keys from three vectors: three score values with thousands of ties, so
  the bin is refined by radix passes down to one value;
- all keys equal, and a zero query: every score equal (all zero);
- keys differing only in one code: scores a few ulps apart, many of them in
  the k-th score's bin;
- dynamic k.

Contexts run from 1 key to 70000, across the k = 2048 boundary.  For every
row the selection equals the oracle's top-k of the scores of
dsa_index_scores (highest first, ties to the lower index) and, with one k for
all rows, dsa_topk on those scores (bit for bit)."""
import math

import numpy as np
import pytest
import torch

import oracle
from sparse_attention_11_b200 import dsa, workloads as W

from gpu_util import sets_equal

pytestmark = pytest.mark.gpu

CTX = [3000, 2049, 2048, 1, 10, 40000, 70000, 2100]


def _inputs(case, rng):
    n = len(CTX)
    tk = int(sum(CTX))
    q = rng.standard_normal((n, 128), dtype=np.float32)
    if case == "random":
        k = rng.standard_normal((tk, 128), dtype=np.float32)
    elif case == "levels":
        base = rng.standard_normal((3, 128), dtype=np.float32)
        k = base[rng.integers(0, 3, tk)]
    elif case in ("equal", "zero_query"):
        k = np.broadcast_to(rng.standard_normal(128, dtype=np.float32), (tk, 128)).copy()
        if case == "zero_query":
            k = rng.standard_normal((tk, 128), dtype=np.float32)
            q[:] = 0
    elif case == "near":
        k = np.broadcast_to(rng.standard_normal(128, dtype=np.float32), (tk, 128)).copy()
        k[:, 5] += rng.integers(0, 40, tk).astype(np.float32) * np.float32(1e-3)
    else:
        raise ValueError(case)
    q_idx, q_sc = W.quantize_e4m3_rows(q)
    k_idx, k_sc = W.quantize_e4m3_rows(k)
    Wf = rng.standard_normal((128, 128), dtype=np.float32) / np.float32(math.sqrt(128.0))
    Wb = torch.from_numpy(W.to_bf16_bits(Wf).view(np.int16)).view(torch.bfloat16).cuda()
    return q_idx, q_sc, Wb, k_idx, k_sc


@pytest.mark.parametrize("case", ["random", "levels", "equal", "zero_query", "near", "random_dynk"])
def test_decode_selection_paths(case):
    rng = np.random.default_rng(["random", "levels", "equal", "zero_query", "near", "random_dynk"].index(case) + 17)
    k = 2048
    n = len(CTX)
    cu_q = np.arange(n + 1, dtype=np.int64)
    cu_k = np.concatenate([[0], np.cumsum(CTX)]).astype(np.int64)
    seqs = dsa.Seqs(cu_q, cu_k, device=torch.device("cuda"))
    q_idx, q_sc, Wb, k_idx, k_sc = _inputs("random" if case == "random_dynk" else case, rng)
    k_rows = None
    if case == "random_dynk":
        k_rows = torch.from_numpy(rng.integers(0, 3000, n).astype(np.int32)).cuda()
    ia = dsa.indexer_args(torch.from_numpy(q_idx).cuda(), torch.from_numpy(q_sc).cuda(), Wb,
                          torch.from_numpy(k_idx).cuda(), torch.from_numpy(k_sc).cuda(), k_per_row=k_rows)
    ws = dsa.workspace(dsa.dsa_workspace_size(dsa.DSA_OP_FORWARD, seqs, k, ia))
    idx = torch.full((n, k), -7, dtype=torch.int32, device="cuda")
    dsa.dsa_select(seqs, ia, k, idx, ws)
    dsa.check_device_status(ws, "decode select")
    g = idx.cpu().numpy()

    ld = max(CTX)
    sc = torch.empty((n, ld), dtype=torch.float32, device="cuda")
    ws2 = dsa.workspace(dsa.dsa_workspace_size(dsa.DSA_OP_INDEX_SCORES, seqs, 0, ia))
    dsa.dsa_index_scores(seqs, ia, 0, n, sc, ws2)
    if k_rows is None:  # (dsa_topk takes one k for all rows)
        idx2 = torch.empty((n, k), dtype=torch.int32, device="cuda")
        dsa.dsa_topk(seqs, sc, 0, n, k, idx2, ws2)
        dsa.check_device_status(ws2, "scores+topk")
        assert np.array_equal(g, idx2.cpu().numpy())

    scn = sc.cpu().numpy()
    kk = k_rows.cpu().numpy() if k_rows is not None else np.full(n, k)
    ncand = np.array(CTX)
    for r in range(n):
        kr = min(int(kk[r]), k)  # the library clamps k_t to [0, k]
        o = oracle.topk(scn[r:r + 1], ncand[r:r + 1], max(kr, 1))
        if kr == 0:
            assert np.all(g[r] == -1)
            continue
        sets_equal(g[r:r + 1, :kr], o, ncand[r:r + 1], kr)
        assert np.all(g[r, min(kr, ncand[r]):] == -1)
    if case in ("equal", "zero_query"):
        for r in range(n):
            K = min(k, CTX[r])
            assert np.array_equal(g[r, :K], np.arange(K))   # all scores equal: the lowest indices
