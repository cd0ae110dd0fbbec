"""Pins of the training-side oracle (oracle/backward.py) against what the
mathematics fixes, independent of the formulas it implements.

"DeepSeek-V3.2与稀疏注意力技术革新" §2.3 / §3.1 (sparse MQA attention, V the
latent part of the KV row), §4.1 (indexer KL distillation in the dense
warm-up and the sparse stage).

* Attention backward: central finite differences of the forward for every
  coordinate of q, K and V, on rows with padding slots and an empty row;
  closed forms (one selected key: dq = dK = 0, dV = sum of dO over heads;
  equal selected keys: dq = 0); invariance of the output under a common
  shift of every key row, which forces sum_j dK_j = 0; the MLA-tied
  gradient against finite differences of the tied forward.  The numpy
  forward is pinned to the C oracle's attention.
* KL: finite differences of the loss in W, q_idx and k_idx; zero loss and
  zero gradient when the target equals the indexer's distribution;
  KL >= 0; the sparse stage's candidate set equals the causal prefix when
  k covers it.
"""
import numpy as np
import pytest

import oracle
from oracle import backward as B


def _attn_case(seed=0, n=4, H=3, dk=6, dv=4, nk=9, k=5):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((n, H, dk))
    K = rng.standard_normal((nk, dk))
    V = rng.standard_normal((nk, dv))
    idx = np.full((n, k), -1, dtype=np.int64)
    for t in range(n - 1):  # the last row stays empty
        m = int(rng.integers(1, k + 1))
        idx[t, :m] = rng.choice(nk, size=m, replace=False)
    rng.shuffle(idx[0])  # padding slots anywhere in the row
    dO = rng.standard_normal((n, H, dv))
    return q, K, V, idx, dO, 0.7


def _fd(f, x, h=1e-6):
    g = np.zeros_like(x)
    it = np.nditer(x, flags=["multi_index"])
    for _ in it:
        i = it.multi_index
        old = x[i]
        x[i] = old + h
        fp = f()
        x[i] = old - h
        fm = f()
        x[i] = old
        g[i] = (fp - fm) / (2 * h)
    return g


def test_attention_backward_finite_differences():
    q, K, V, idx, dO, sc = _attn_case()
    loss = lambda: float((B.sparse_attn_fwd(q, K, V, idx, sc)[0] * dO).sum())
    dq, dK, dV = B.sparse_attn_bwd(q, K, V, idx, sc, dO)
    for name, x, g in (("q", q, dq), ("K", K, dK), ("V", V, dV)):
        num = _fd(loss, x)
        assert np.allclose(g, num, rtol=1e-6, atol=1e-8), (name, np.abs(g - num).max())
    assert np.all(dq[-1] == 0)  # the empty row
    used = np.unique(idx[idx >= 0])
    unused = np.setdiff1d(np.arange(K.shape[0]), used)
    assert np.all(dK[unused] == 0) and np.all(dV[unused] == 0)


def test_attention_backward_stored_output():
    """D from the stored output equals D = sum_j P_j dP_j when the output is
    exact; a perturbed output moves only D."""
    q, K, V, idx, dO, sc = _attn_case(seed=10)
    O, _ = B.sparse_attn_fwd(q, K, V, idx, sc)
    a = B.sparse_attn_bwd(q, K, V, idx, sc, dO)
    b = B.sparse_attn_bwd(q, K, V, idx, sc, dO, O=O)
    for x, y in zip(a, b):
        assert np.allclose(x, y, rtol=0, atol=1e-13)
    c = B.sparse_attn_bwd(q, K, V, idx, sc, dO, O=O * 1.01)
    assert np.array_equal(c[2], a[2])           # dV does not involve D
    assert not np.allclose(c[0], a[0])          # dq does


def test_attention_backward_single_key():
    q, K, V, idx, dO, sc = _attn_case(seed=1)
    idx[:, 1:] = -1
    idx[:-1, 0] = [2, 5, 2]
    dq, dK, dV = B.sparse_attn_bwd(q, K, V, idx, sc, dO)
    assert np.allclose(dq, 0, atol=1e-14) and np.allclose(dK, 0, atol=1e-14)
    exp = np.zeros_like(V)
    for t, j in enumerate(idx[:-1, 0]):
        exp[j] += dO[t].sum(axis=0)
    assert np.allclose(dV, exp, atol=1e-14)


def test_attention_backward_equal_keys():
    q, K, V, idx, dO, sc = _attn_case(seed=2, n=2)
    idx[0] = [0, 1, 2, 3, -1]
    K[[0, 1, 2, 3]] = K[0]
    dq, dK, dV = B.sparse_attn_bwd(q, K, V, idx, sc, dO)
    assert np.allclose(dq[0], 0, atol=1e-13)


def test_attention_backward_shift_invariance():
    """Shifting every key row by one vector shifts each query's scores by a
    constant, which the softmax ignores, so the loss is flat along it."""
    q, K, V, idx, dO, sc = _attn_case(seed=3)
    c = np.random.default_rng(9).standard_normal(K.shape[1])
    O0 = B.sparse_attn_fwd(q, K, V, idx, sc)[0]
    O1 = B.sparse_attn_fwd(q, K + c, V, idx, sc)[0]
    assert np.allclose(O0, O1, atol=1e-12)
    _, dK, _ = B.sparse_attn_bwd(q, K, V, idx, sc, dO)
    assert np.allclose(dK.sum(axis=0), 0, atol=1e-12)


def test_attention_backward_mla_tied():
    rng = np.random.default_rng(4)
    n, H, dk, dv, nk = 3, 2, 8, 5, 7
    q = rng.standard_normal((n, H, dk))
    KV = rng.standard_normal((nk, dk))
    idx = np.array([[0, 3, 6, -1], [1, 2, 4, 5], [6, -1, -1, -1]])
    dO = rng.standard_normal((n, H, dv))
    loss = lambda: float((B.sparse_attn_fwd(q, KV, KV[:, :dv], idx, 0.3)[0] * dO).sum())
    _, dK, dV = B.sparse_attn_bwd(q, KV, KV[:, :dv], idx, 0.3, dO)
    g = B.mla_tied_grad(dK, dV)
    assert np.allclose(g, _fd(loss, KV), rtol=1e-6, atol=1e-8)


def test_attention_forward_matches_c_oracle():
    rng = np.random.default_rng(5)
    n, H, dk, dv, nk = 5, 4, 64, 64, 40
    q = rng.standard_normal((n, H, dk)).astype(np.float32)
    K = rng.standard_normal((nk, dk)).astype(np.float32)
    V = rng.standard_normal((nk, dv)).astype(np.float32)
    idx = np.stack([rng.choice(nk, size=8, replace=False) for _ in range(n)]).astype(np.int32)
    idx[1, 5:] = -1
    O, lse = B.sparse_attn_fwd(q, K, V, idx, 0.125)
    Oc, lc = oracle.attention(q, K, dk, V, dv, np.zeros(n, dtype=np.int64), idx, 0.125, dv)
    assert np.allclose(O, Oc, rtol=0, atol=1e-12) and np.allclose(lse, lc, rtol=0, atol=1e-12)


def _kl_case(seed=6, n=5, nk=12, d=16):
    rng = np.random.default_rng(seed)
    qi = rng.standard_normal((n, d))
    W = rng.standard_normal((d, d)) / np.sqrt(d)
    ki = rng.standard_normal((nk, d))
    pos = np.array([3, 6, 8, 11, 11])
    cand = B.causal_candidates(n, pos, nk)
    q = rng.standard_normal((n, 2, 6))
    K = rng.standard_normal((nk, 6))
    p = B.attention_target(q, K, 0.5, cand)
    return qi, W, ki, p, cand


def test_kl_finite_differences():
    qi, W, ki, p, cand = _kl_case()
    x, _ = B.indexer_logits(qi, W, ki)
    assert np.abs(x).min() > 1e-4  # no ReLU kink inside the difference step
    f = lambda: B.kl_loss(p, B.indexer_logits(qi, W, ki)[1], cand)[0]
    loss, dW, dq, dk = B.kl_grads(qi, W, ki, p, cand)
    assert np.isclose(loss, f())
    for name, x_, g in (("W", W, dW), ("q_idx", qi, dq), ("k_idx", ki, dk)):
        num = _fd(f, x_, h=1e-7)
        assert np.allclose(g, num, rtol=1e-5, atol=1e-7), (name, np.abs(g - num).max())


def test_kl_zero_at_match_and_nonnegative():
    qi, W, ki, p, cand = _kl_case(seed=7)
    _, I = B.indexer_logits(qi, W, ki)
    loss, r = B.kl_loss(p, I, cand)
    assert loss > 0
    for t in range(p.shape[0]):
        assert np.isclose(r[t].sum(), 1.0) and np.isclose(p[t].sum(), 1.0)
    # the target equal to the indexer's own distribution: zero loss, zero gradient
    loss0, dW, dq, dk = B.kl_grads(qi, W, ki, r, cand)
    assert abs(loss0) < 1e-12
    assert np.allclose(dW, 0, atol=1e-12) and np.allclose(dq, 0, atol=1e-12) and np.allclose(dk, 0, atol=1e-12)
    # KL >= 0 on random targets over the candidates
    rng = np.random.default_rng(8)
    for _ in range(20):
        pr = rng.random(p.shape) * cand
        pr /= pr.sum(axis=1, keepdims=True)
        assert B.kl_loss(pr, I, cand)[0] >= 0


def test_candidate_sets():
    n, nk, k = 6, 10, 16
    pos = np.array([0, 2, 4, 6, 8, 9])
    idx = np.full((n, k), -1)
    for t in range(n):
        idx[t, : pos[t] + 1] = np.arange(pos[t] + 1)[::-1]
    assert np.array_equal(B.selected_candidates(idx, nk), B.causal_candidates(n, pos, nk))
    # sparse stage: the target over the selected set is the sparse attention's own
    rng = np.random.default_rng(9)
    q = rng.standard_normal((n, 3, 5))
    K = rng.standard_normal((nk, 5))
    sel = np.array([[0, -1], [1, 2], [0, 4], [5, 6], [8, 2], [9, 3]])
    p = B.attention_target(q, K, 0.4, B.selected_candidates(sel, nk))
    for t in range(n):
        s = sel[t][sel[t] >= 0]
        z = 0.4 * q[t] @ K[s].T
        e = np.exp(z - z.max(axis=1, keepdims=True))
        assert np.allclose(p[t, s], (e / e.sum(axis=1, keepdims=True)).mean(axis=0))
        assert np.isclose(p[t].sum(), 1.0)
