"""Pins for the oracle's selection and sparse attention.

Selection ("DeepSeek-V3.2与稀疏注意力技术革新", §2.3): each query keeps the
k highest-scoring keys of its causal prefix; ties go to the lower index.
Pinned by brute force on tiny rows, by the pairwise definition of a top-k
set, and by the consequences the pages fix (pos+1 <= k keeps every causal
key; order-preserving rescaling keeps the set).

Attention (§2.3, §3.1): standard softmax attention restricted to the
selected rows, every head sharing one K/V.  Pinned by dense causal attention
computed with numpy matrices when k >= L, and by closed-form special cases.
"""
import itertools

import numpy as np
import pytest
from scipy.special import logsumexp

import oracle


def _before(a, b, sa, sb):
    """Does candidate a rank before b (strict order used by the definition)?"""
    if np.isnan(sa) or np.isnan(sb):
        if np.isnan(sa) and np.isnan(sb):
            return a < b
        return np.isnan(sb)
    if sa != sb:
        return sa > sb
    return a < b


def _check_topk_set(scores, ncand, k, sel):
    K = min(k, ncand)
    chosen = [int(x) for x in sel[:K]]
    assert len(set(chosen)) == K and all(0 <= c < ncand for c in chosen)
    assert np.all(sel[K:] == -1)
    rest = set(range(ncand)) - set(chosen)
    for a in chosen:
        for b in rest:
            assert _before(a, b, scores[a], scores[b]), (a, b)


@pytest.mark.parametrize("seed", range(6))
def test_topk_brute_force_ties(seed):
    rng = np.random.default_rng(seed)
    n, ld = 30, 40
    levels = np.array([0.0, -0.0, 1.0, 2.5, 2.5, 1e-40, np.nan, 7.0], dtype=np.float32)
    sc = levels[rng.integers(0, len(levels), size=(n, ld))].astype(np.float32)
    ncand = rng.integers(1, ld + 1, size=n)
    for k in (1, 3, 8, 40):
        idx = oracle.topk(sc, ncand, k)
        for r in range(n):
            _check_topk_set(sc[r], int(ncand[r]), k, idx[r])
            # brute force: Python's sort on an explicit key
            order = sorted(range(int(ncand[r])),
                           key=lambda s: (1, 0.0, s) if np.isnan(sc[r, s]) else (0, -float(sc[r, s]), s))
            K = min(k, int(ncand[r]))
            assert list(idx[r, :K]) == order[:K]


@pytest.mark.parametrize("seed", range(4))
def test_topk_dynamic_k_brute_force(seed):
    """Dynamic k (a per-query k, [V32] §6): row r keeps
    min(clamp(k_r, 0, k), ncand_r) keys by the same order as top-k, then -1
    up to the row width k.  Brute force with Python's sort, on tie-heavy rows,
    with k_r of 0, 1, beyond the row, above k and negative."""
    rng = np.random.default_rng(100 + seed)
    n, ld, k = 40, 60, 24
    levels = np.array([0.0, -0.0, 1.0, 2.5, 2.5, 1e-40, np.nan, 7.0, 3.0], dtype=np.float32)
    sc = levels[rng.integers(0, len(levels), size=(n, ld))].astype(np.float32)
    ncand = rng.integers(1, ld + 1, size=n)
    k_rows = rng.integers(-3, k + 10, size=n).astype(np.int32)
    k_rows[:4] = [0, 1, k, 1000]
    idx = oracle.topk_dyn(sc, ncand, k_rows, k)
    assert idx.shape == (n, k)
    for r in range(n):
        kr = min(max(int(k_rows[r]), 0), k)
        order = sorted(range(int(ncand[r])),
                       key=lambda s: (1, 0.0, s) if np.isnan(sc[r, s]) else (0, -float(sc[r, s]), s))
        K = min(kr, int(ncand[r]))
        assert list(idx[r, :K]) == order[:K]
        assert np.all(idx[r, K:] == -1)
    # k_r >= k everywhere is plain top-k
    assert np.array_equal(oracle.topk_dyn(sc, ncand, np.full(n, k, np.int32), k), oracle.topk(sc, ncand, k))


def test_topk_all_causal_when_prefix_fits():
    rng = np.random.default_rng(7)
    sc = rng.standard_normal((20, 64)).astype(np.float32)
    ncand = np.arange(1, 21)
    idx = oracle.topk(sc, ncand, 20)
    for r in range(20):
        assert sorted(idx[r, : r + 1]) == list(range(r + 1))


def test_topk_equal_rows_take_lowest_indices():
    for val in (0.0, 3.0):
        sc = np.full((3, 50), val, dtype=np.float32)
        idx = oracle.topk(sc, np.array([50, 30, 10]), 16)
        assert list(idx[0]) == list(range(16))
        assert list(idx[1]) == list(range(16))
        assert list(idx[2, :10]) == list(range(10)) and np.all(idx[2, 10:] == -1)


def test_topk_invariant_under_power_of_two_scaling():
    rng = np.random.default_rng(8)
    sc = np.abs(rng.standard_normal((10, 100))).astype(np.float32)
    sc[:, ::7] = 0
    nc = np.full(10, 100)
    a = oracle.topk(sc, nc, 17)
    for m in (-20, 5):
        assert np.array_equal(a, oracle.topk(sc * np.float32(2.0 ** m), nc, 17))


def _dense_causal(q, K, V, scale):
    """softmax(scale q K^T + causal mask) V with numpy matrices, per head."""
    L, H, dk = q.shape
    out = np.zeros((L, H, V.shape[1]))
    lse = np.zeros((L, H))
    mask = np.triu(np.ones((L, L), bool), 1)
    for h in range(H):
        z = scale * (q[:, h, :].astype(np.float64) @ K.astype(np.float64).T)
        z[mask] = -np.inf
        lse[:, h] = logsumexp(z, axis=1)
        p = np.exp(z - lse[:, h: h + 1])
        out[:, h, :] = p @ V.astype(np.float64)
    return out, lse


def test_attention_full_selection_equals_dense_causal():
    rng = np.random.default_rng(9)
    L, H, dk, dv = 48, 3, 16, 8
    q = rng.standard_normal((L, H, dk)).astype(np.float32)
    K = rng.standard_normal((L, dk)).astype(np.float32)
    V = rng.standard_normal((L, dv)).astype(np.float32)
    idx = np.full((L, L), -1, np.int32)
    for t in range(L):
        idx[t, : t + 1] = rng.permutation(t + 1)   # any order: set semantics
    out, lse = oracle.attention(q, K.ravel(), dk, V.ravel(), dv, np.zeros(L), idx, 0.3, dv)
    ref, rlse = _dense_causal(q, K, V, 0.3)
    assert np.allclose(out, ref, atol=1e-12, rtol=1e-10)
    assert np.allclose(lse, rlse, atol=1e-12, rtol=1e-12)


def test_attention_special_cases():
    rng = np.random.default_rng(10)
    H, dk, dv, T = 4, 8, 6, 10
    q = rng.standard_normal((2, H, dk)).astype(np.float32)
    K = rng.standard_normal((T, dk)).astype(np.float32)
    V = rng.standard_normal((T, dv)).astype(np.float32)
    # a single selected row: the output is that V row, lse its logit
    idx = np.array([[6, -1, -1], [-1, 2, -1]], np.int32)
    out, lse = oracle.attention(q, K.ravel(), dk, V.ravel(), dv, np.zeros(2), idx, 0.5, dv)
    for r, j in ((0, 6), (1, 2)):
        assert np.allclose(out[r], np.broadcast_to(V[j], (H, dv)), atol=0, rtol=0)
        assert np.allclose(lse[r], 0.5 * (q[r].astype(np.float64) @ K[j].astype(np.float64)), rtol=1e-14)
    # identical V rows: output equals that row whatever the weights
    V2 = np.tile(V[:1], (T, 1))
    idx2 = np.array([[0, 3, 5, 9], [1, 2, 4, 8]], np.int32)
    out2, _ = oracle.attention(q, K.ravel(), dk, V2.ravel(), dv, np.zeros(2), idx2, 0.5, dv)
    assert np.allclose(out2, V2[0], atol=1e-14)
    # nothing selected: zeros and lse = -inf
    out3, lse3 = oracle.attention(q, K.ravel(), dk, V.ravel(), dv, np.zeros(2), np.full((2, 3), -1, np.int32), 0.5, dv)
    assert np.all(out3 == 0) and np.all(np.isneginf(lse3))


def test_attention_strided_v_inside_k():
    """V read as the first dv columns of the K rows (MLA latent layout)."""
    rng = np.random.default_rng(11)
    T, H, dk, dv = 12, 2, 10, 7
    q = rng.standard_normal((3, H, dk)).astype(np.float32)
    K = rng.standard_normal((T, dk)).astype(np.float32)
    idx = np.array([[0, 1, 2, 3], [4, 11, -1, 5], [7, 7, 8, 9]], np.int32)
    out, _ = oracle.attention(q, K.ravel(), dk, K.ravel(), dk, np.zeros(3), idx, 0.2, dv)
    ref, _ = oracle.attention(q, K.ravel(), dk, np.ascontiguousarray(K[:, :dv]).ravel(), dv, np.zeros(3), idx, 0.2, dv)
    assert np.array_equal(out, ref)
