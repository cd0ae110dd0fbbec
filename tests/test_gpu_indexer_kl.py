"""The indexer's KL distillation (sparse stage) through the C ABI, against
the oracle.

"DeepSeek-V3.2与稀疏注意力技术革新" §4.1 (the indexer imitates the main
attention's distribution through a KL loss, in the sparse stage over the
selected keys), §2.2 (I = ReLU(q W_index k)).

* dsa_attn_target: the head-averaged attention probabilities of the selected
  keys.  It uses the forward's own selection and lse, and is compared with
  the oracle's attention_target over the same selected set (1e-5 absolute
  for fp32 inputs, 1e-4 for bf16): tiny_l512 and a 640-token bf16 MLA
  prefill.
* dsa_indexer_kl: per-query loss and the gradients in the indexer query, W
  and the indexer keys, against the oracle's kl_loss / kl_grads with the same
  target (each tensor within 1e-4 of its largest magnitude):
  - tiny_l512 (fp32 indexer inputs);
  - the 640-token prefill, whose e4m3 indexer codes times their scales are
    the real-valued inputs.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import backward as B
from sparse_attention_11_b200 import dsa, workloads as W

from gpu_util import bf16_to_f64, make

pytestmark = pytest.mark.gpu


def _global_idx(inp, idx):
    kb, _ = inp.key_base_pos(np.arange(idx.shape[0]))
    return np.where(idx >= 0, idx.astype(np.int64) + kb[:, None], -1)


def _dense(p_slots, idx_g, nk):
    d = np.zeros((p_slots.shape[0], nk))
    for t in range(p_slots.shape[0]):
        v = idx_g[t] >= 0
        d[t, idx_g[t][v]] = p_slots[t][v]
    return d


def _close(g, o, rel, floor=1e-7):
    tol = rel * np.abs(o).max() + floor
    err = np.abs(g - o).max()
    assert err <= tol, (err, tol)


def _indexer_f32(inp):
    if inp.wl.idx_dtype == "f32":
        return inp.q_idx.astype(np.float32), inp.W.astype(np.float32), inp.k_idx.astype(np.float32)
    lut = np.array([oracle.e4m3_decode(c) for c in range(256)])
    q = (lut[inp.q_idx] * inp.q_idx_scale[:, None]).astype(np.float32)
    k = (lut[inp.k_idx] * inp.k_idx_scale[:, None]).astype(np.float32)
    Wf = W.bf16_bits_to_f32(inp.W).astype(np.float32)
    return q, Wf, k


@pytest.mark.parametrize("case", ["tiny", "mla640"])
def test_indexer_kl(case):
    wl = W.WORKLOADS["tiny_l512"] if case == "tiny" else \
        W.custom("prefill_l640_k128", (640,), (640,), base="prefill_l8192", k=128)
    inp, prob = make(wl)
    prob.forward()
    prob.check("forward")
    T, nk = wl.total_q, wl.total_k
    ws = dsa.workspace(256)
    p = torch.full((T, wl.k), float("nan"), device="cuda")
    dsa.dsa_attn_target(prob.seqs, prob.aa, prob.idx, wl.k, p, ws)
    dsa.check_device_status(ws, "attn target")
    idx_g = _global_idx(inp, prob.idx.cpu().numpy())
    cand = B.selected_candidates(idx_g, nk)
    if case == "tiny":
        q, K = inp.q_host, inp.K
    else:
        q, K = bf16_to_f64(inp.q_rows(np.arange(T))), bf16_to_f64(inp.K)
    p_or = B.attention_target(q, K, wl.scale, cand)
    p_gpu = p.cpu().numpy()
    assert np.all(p_gpu[prob.idx.cpu().numpy() < 0] == 0)
    _close(_dense(p_gpu, idx_g, nk), p_or, 0, 1e-5 if case == "tiny" else 1e-4)

    qf, Wf, kf = _indexer_f32(inp)
    qd, Wd, kd = torch.from_numpy(qf).cuda(), torch.from_numpy(Wf).cuda(), torch.from_numpy(kf).cuda()
    loss = torch.full((T,), float("nan"), device="cuda")
    d_q = torch.full((T, 128), float("nan"), device="cuda")
    d_W = torch.zeros((128, 128), device="cuda")
    d_k = torch.zeros((nk, 128), device="cuda")
    dsa.dsa_indexer_kl(prob.seqs, qd, Wd, kd, prob.idx, wl.k, p, loss, d_q, d_W, d_k, ws)
    dsa.check_device_status(ws, "indexer kl")
    p_d = _dense(p_gpu.astype(np.float64), idx_g, nk)
    per_row = np.array([B.kl_loss(p_d[t:t + 1], B.indexer_logits(qf[t:t + 1], Wf, kf)[1], cand[t:t + 1])[0]
                        for t in range(T)])
    _close(loss.cpu().numpy(), per_row, 1e-4, 1e-6)
    _, dW, dq, dk = B.kl_grads(qf, Wf, kf, p_d, cand)
    _close(d_q.cpu().numpy(), dq, 1e-4)
    _close(d_W.cpu().numpy(), dW, 1e-4)
    _close(d_k.cpu().numpy(), dk, 1e-4)
