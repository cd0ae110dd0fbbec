"""Pins for the oracle's lightning indexer (fold + scores).

Definition pinned: I[t,s] = ReLU(q_t . W_index . k_s) ("DeepSeek-V3.2与稀疏注意力
技术革新", §2.2), W_index folded into the query first.  Checked against
numpy's float64 matmul (an independent library), exact rational arithmetic on
tiny FP8 cases, and the invariants the formula fixes (scores >= 0, W = I
reduces to a plain dot product, q = 0 gives 0).
"""
from fractions import Fraction

import numpy as np
import torch

import oracle
from sparse_attention_11_b200 import workloads as W


def _rng(s):
    return np.random.default_rng(s)


def test_fold_f32_is_row_vector_times_matrix():
    rng = _rng(0)
    q = rng.standard_normal((7, 128)).astype(np.float32)
    Wm = rng.standard_normal((128, 128)).astype(np.float32)   # not symmetric
    u, s_row = oracle.fold(q, None, Wm)
    ref = (q.astype(np.float64) @ Wm.astype(np.float64)).astype(np.float32)
    assert np.array_equal(u, ref)
    assert np.all(s_row == 1.0)
    wrong = (q.astype(np.float64) @ Wm.T.astype(np.float64)).astype(np.float32)
    assert not np.allclose(u, wrong, rtol=1e-2)


def test_scores_f32_match_bilinear_form():
    rng = _rng(1)
    n = 40
    q = rng.standard_normal((n, 128)).astype(np.float32)
    k = rng.standard_normal((n, 128)).astype(np.float32)
    Wm = (rng.standard_normal((128, 128)) / np.sqrt(128)).astype(np.float32)
    u, s_row = oracle.fold(q, None, Wm)
    ncand = np.arange(n) + 1
    sc = oracle.scores(u, s_row, k, None, np.zeros(n), ncand, n)
    ref = np.einsum("ti,ij,sj->ts", q.astype(np.float64), Wm.astype(np.float64), k.astype(np.float64))
    for t in range(n):
        r = np.maximum(ref[t, : t + 1], 0.0)
        # fp32 rounding of the folded query only: relative error ~ 2^-24 * sqrt(128) * |terms|
        bound = 1e-5 * (np.abs(q[t].astype(np.float64) @ np.abs(Wm.astype(np.float64))) @ np.abs(k[: t + 1].T) + 1e-30)
        assert np.all(np.abs(sc[t, : t + 1] - r) <= bound + 1e-6)
        assert np.all(sc[t, : t + 1] >= 0)
        assert np.all(np.isneginf(sc[t, t + 1:]))
    # zeros are +0.0, never -0.0
    z = sc[np.isfinite(sc)]
    assert not np.any(np.signbit(z))


def test_scores_identity_W_reduces_to_dot():
    rng = _rng(2)
    n = 16
    q = rng.standard_normal((n, 128)).astype(np.float32)
    k = rng.standard_normal((n, 128)).astype(np.float32)
    u, s_row = oracle.fold(q, None, np.eye(128, dtype=np.float32))
    assert np.array_equal(u, q)
    sc = oracle.scores(u, s_row, k, None, np.zeros(n), np.full(n, n), n)
    ref = np.maximum(q.astype(np.float64) @ k.astype(np.float64).T, 0.0).astype(np.float32)
    assert np.array_equal(sc, ref)


def _torch_e4m3(codes):
    return torch.from_numpy(np.ascontiguousarray(codes)).view(torch.float8_e4m3fn).to(torch.float64).numpy()


def test_fold_e4m3_requantisation_properties():
    rng = _rng(3)
    x = W.bf16_bits_to_f32(W.to_bf16_bits(rng.standard_normal((64, 128)).astype(np.float32)))
    codes, s_q = W.quantize_e4m3_rows(x)
    codes[5] = 0   # an all-zero query row
    Wb = W.to_bf16_bits((rng.standard_normal((128, 128)) / np.sqrt(128)).astype(np.float32))
    u8, s_row = oracle.fold(codes, s_q, Wb)
    Wf = W.bf16_bits_to_f32(Wb).astype(np.float64)
    ref = (_torch_e4m3(codes) @ Wf).astype(np.float32)       # q8 . W, fp32
    deq = _torch_e4m3(u8)
    for r in range(64):
        amax = np.abs(ref[r]).max()
        if amax == 0:
            assert np.all(u8[r] == 0) and s_row[r] == s_q[r]
            continue
        s_u = np.float32(amax / 448.0)
        assert s_row[r] == np.float32(np.float64(s_q[r]) * np.float64(s_u))
        assert np.abs(deq[r]).max() == 448.0
        # each element is the nearest e4m3 value: within half an e4m3 step
        y = ref[r].astype(np.float64) / np.float64(s_u)
        step = np.where(np.abs(y) >= 2.0 ** -6, 2.0 ** (np.floor(np.log2(np.maximum(np.abs(y), 1e-300))) - 3), 2.0 ** -9)
        assert np.all(np.abs(deq[r] - y) <= 0.5 * step * (1 + 1e-6))


def test_scores_e4m3_exact_rational():
    rng = _rng(4)
    n = 12
    xq = rng.standard_normal((n, 128)).astype(np.float32)
    xk = rng.standard_normal((n, 128)).astype(np.float32)
    xk[3] = 0.0
    qc, qs = W.quantize_e4m3_rows(xq)
    kc, ks = W.quantize_e4m3_rows(xk)
    # use the codes directly as the folded query (fold is pinned separately)
    sc = oracle.scores(qc, qs, kc, ks, np.zeros(n), np.full(n, n), n)
    qd, kd = _torch_e4m3(qc), _torch_e4m3(kc)
    for t in range(n):
        for s in range(n):
            dot = sum(Fraction(float(a)) * Fraction(float(b)) for a, b in zip(qd[t], kd[s]))
            x = Fraction(float(qs[t])) * Fraction(float(ks[s])) * dot
            want = np.float32(float(x)) if x > 0 else np.float32(0.0)
            got = sc[t, s]
            assert abs(float(got) - float(want)) <= abs(float(want)) * 2.0 ** -23, (t, s)
    assert np.all(sc[:, 3] == 0)


def test_zero_query_gives_zero_scores():
    n = 8
    rng = _rng(5)
    k = rng.standard_normal((n, 128)).astype(np.float32)
    u, s_row = oracle.fold(np.zeros((n, 128), np.float32), None, np.eye(128, dtype=np.float32))
    sc = oracle.scores(u, s_row, k, None, np.zeros(n), np.full(n, n), n)
    assert np.all(sc == 0) and not np.any(np.signbit(sc))
