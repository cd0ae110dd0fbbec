"""Backward of the sparse attention through the C ABI, against the oracle.

"DeepSeek-V3.2与稀疏注意力技术革新" §2.3 / §3.1 (the attention over the
selected rows, V the latent part of the KV row), §4.1 (the sparse training
stage runs this attention, so it needs gradients).

For each case the forward runs first (dsa_forward), and the backward then
takes the forward's own selection, output and lse, with a seeded d_out.
The oracle (oracle/backward.py, float64) is given the same selection and
the same stored output, which is where D = d_out . out comes from.  Every
element of d_q, d_K and d_V is compared within a tolerance relative to the
tensor's largest magnitude: 1e-4 for fp32 inputs, 1e-3 for bf16 inputs (the
kernel computes in fp32; the 2e-2 forward tolerance does not enter, since
both sides use the same stored output).
  * tiny_l512: fp32, 4 heads, dk = dv = 64, V its own tensor, k = 64
    (rows with fewer than k keys carry -1 slots);
  * a 640-token bf16 MLA prefill, 128 heads, dk 576, dv 512, k = 128, with
    V = K[:, :512] and d_V passed as d_K's first 512 columns.  d_K then
    holds the tied gradient of the KV row.
An index past its sequence is reported as DSA_ERR_INDEX.
"""
import numpy as np
import pytest
import torch

from oracle import backward as B
from sparse_attention_11_b200 import dsa, workloads as W

from gpu_util import bf16_np, bf16_to_f64, make

pytestmark = pytest.mark.gpu


def _global_idx(inp, idx):
    kb, _ = inp.key_base_pos(np.arange(idx.shape[0]))
    return np.where(idx >= 0, idx.astype(np.int64) + kb[:, None], -1)


def _close(g, o, rel):
    tol = rel * np.abs(o).max() + 1e-6
    err = np.abs(g - o).max()
    assert err <= tol, (err, tol)


def test_backward_tiny_fp32():
    wl = W.WORKLOADS["tiny_l512"]
    inp, prob = make(wl)
    prob.forward()
    prob.check("forward")
    T, H = wl.total_q, wl.heads
    gen = torch.Generator().manual_seed(21)
    d_out = torch.randn((T, H, wl.dv), generator=gen).cuda()
    d_q = torch.full((T, H, wl.dk), float("nan"), device="cuda")
    d_k = torch.zeros((wl.total_k, wl.dk), device="cuda")
    d_v = torch.zeros((wl.total_k, wl.dv), device="cuda")
    ws = dsa.workspace(256)
    dsa.dsa_sparse_attn_bwd(prob.seqs, prob.aa, prob.idx, wl.k, d_out, d_q, d_k, d_v, ws)
    dsa.check_device_status(ws, "backward")
    idx = _global_idx(inp, prob.idx.cpu().numpy())
    dq, dK, dV = B.sparse_attn_bwd(inp.q_host, inp.K, inp.V, idx, wl.scale, d_out.cpu().numpy(),
                                   O=prob.out.cpu().numpy())
    _close(d_q.cpu().numpy(), dq, 1e-4)
    _close(d_k.cpu().numpy(), dK, 1e-4)
    _close(d_v.cpu().numpy(), dV, 1e-4)


def test_backward_bf16_mla_tied():
    wl = W.custom("prefill_l640_k128", (640,), (640,), base="prefill_l8192", k=128)
    inp, prob = make(wl)
    prob.forward()
    prob.check("forward")
    T, H = wl.total_q, wl.heads
    gen = torch.Generator().manual_seed(22)
    d_out = torch.randn((T, H, wl.dv), generator=gen).to(torch.bfloat16).cuda()
    d_q = torch.full((T, H, wl.dk), float("nan"), device="cuda")
    d_kv = torch.zeros((wl.total_k, wl.dk), device="cuda")
    ws = dsa.workspace(256)
    dsa.dsa_sparse_attn_bwd(prob.seqs, prob.aa, prob.idx, wl.k, d_out, d_q, d_kv, d_kv[:, : wl.dv], ws)
    dsa.check_device_status(ws, "backward")
    idx = _global_idx(inp, prob.idx.cpu().numpy())
    q = bf16_to_f64(inp.q_rows(np.arange(T)))
    K = bf16_to_f64(inp.K)
    dq, dK, dV = B.sparse_attn_bwd(q, K, K[:, : wl.dv], idx, wl.scale, bf16_to_f64(bf16_np(d_out)),
                                   O=bf16_to_f64(bf16_np(prob.out)))
    _close(d_q.cpu().numpy(), dq, 1e-3)
    _close(d_kv.cpu().numpy(), B.mla_tied_grad(dK, dV), 1e-3)


def test_backward_reports_bad_index():
    wl = W.WORKLOADS["tiny_l512"]
    inp, prob = make(wl)
    prob.forward()
    prob.check("forward")
    idx = prob.idx.clone()
    idx[5, 0] = 100000  # past the sequence
    T, H = wl.total_q, wl.heads
    d_out = torch.zeros((T, H, wl.dv), device="cuda")
    d_q = torch.empty((T, H, wl.dk), device="cuda")
    d_k = torch.zeros((wl.total_k, wl.dk), device="cuda")
    d_v = torch.zeros((wl.total_k, wl.dv), device="cuda")
    ws = dsa.workspace(256)
    dsa.dsa_sparse_attn_bwd(prob.seqs, prob.aa, idx, wl.k, d_out, d_q, d_k, d_v, ws)
    code, detail = dsa.dsa_sync_status(ws)
    assert code == dsa.DSA_ERR_INDEX and detail == 5
