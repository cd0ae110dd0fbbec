"""CPU oracle for the training-side steps of DSA: the sparse attention's
backward over the selected set, and the lightning indexer's KL distillation
loss with its gradients.

TEST INFRASTRUCTURE: only the tests may import this module; no product path
does.  Plain numpy in float64, one definition per function, no blocking or
fusion.

Sources ("DeepSeek-V3.2与稀疏注意力技术革新"):
  §2.3  attention runs as standard attention over the k selected keys;
  §3.1  MLA in MQA form: every head attends to the same KV row of
        512 latent + 64 rope columns, and V is the latent part;
  §2.2  the indexer score I[t,s] = ReLU(q_t · W_index · k_s);
  §4.1  training has two stages.  In the dense warm-up the main model is
        frozen and only the indexer learns, through a KL-divergence loss
        that makes it imitate the dense model's attention distribution.  In
        the sparse stage the indexer keeps that KL loss (the main model
        trains on the language-modelling loss).

The pages give no formula for the KL term.  Readings (the plainest ones
the text supports):
  * target p_t: the main attention's probabilities of query t, averaged
    over the heads, over the candidate keys C_t.  C_t is the causal prefix
    s <= pos_t in the dense warm-up, and the selected set in the sparse
    stage, where p is renormalised over it;
  * indexer distribution r_t = softmax over C_t of the scores I[t, .];
  * loss = sum over queries of KL(p_t || r_t);
  * the training arithmetic is real-valued (float64 here).  The e4m3
    storage of the pages concerns the inference key cache.
"""
import numpy as np


def _f64(x):
    return np.asarray(x, dtype=np.float64)


# ----------------------------------------------------------------------------- attention over the selected set
def sparse_attn_fwd(q, K, V, idx, scale):
    """Forward of the sparse MQA attention (§2.3, §3.1).

    q [n,H,dk], K [Nk,dk], V [Nk,dv], idx [n,k] int (row indices into K/V;
    -1 = empty slot).  For query t and head h, over the valid slots j:
      z_j = scale * q[t,h] . K[idx_j],  O = sum_j softmax(z)_j V[idx_j],
      lse = log sum_j exp(z_j).
    A query with no valid slot gives O = 0 and lse = -inf."""
    q, K, V = _f64(q), _f64(K), _f64(V)
    n, H, _ = q.shape
    dv = V.shape[1]
    O = np.zeros((n, H, dv))
    lse = np.full((n, H), -np.inf)
    for t in range(n):
        sel = idx[t][idx[t] >= 0]
        if sel.size == 0:
            continue
        z = scale * (q[t] @ K[sel].T)            # [H, |sel|]
        m = z.max(axis=1, keepdims=True)
        e = np.exp(z - m)
        ssum = e.sum(axis=1, keepdims=True)
        O[t] = (e / ssum) @ V[sel]
        lse[t] = (m + np.log(ssum))[:, 0]
    return O, lse


def sparse_attn_bwd(q, K, V, idx, scale, dO, O=None):
    """Gradients of sum(dO * O) for sparse_attn_fwd.

    Returns dq [n,H,dk], dK [Nk,dk], dV [Nk,dv].  Every selected key
    collects its contributions from every query and head that selected it.
    The softmax backward, per (t, h):
      P_j  = softmax(z)_j
      dP_j = dO . V[idx_j]
      D    = sum_j P_j dP_j        (= dO . O)
      dz_j = P_j (dP_j - D)
      dq   = scale * sum_j dz_j K[idx_j]
      dK[idx_j] += scale * dz_j q
      dV[idx_j] += P_j dO
    Indices in a row must be distinct (a selection is a set).

    O: optional forward output [n,H,dv].  When given, D = dO . O is taken
    from it, as a training kernel does with the output it stored.  With the
    exact output this is the same D."""
    q, K, V, dO = _f64(q), _f64(K), _f64(V), _f64(dO)
    n, H, dk = q.shape
    dq = np.zeros_like(q)
    dK = np.zeros_like(K)
    dV = np.zeros_like(V)
    for t in range(n):
        sel = idx[t][idx[t] >= 0]
        if sel.size == 0:
            continue
        if np.unique(sel).size != sel.size:
            raise ValueError(f"row {t}: repeated index")
        z = scale * (q[t] @ K[sel].T)
        P = np.exp(z - z.max(axis=1, keepdims=True))
        P /= P.sum(axis=1, keepdims=True)        # [H, m]
        dP = dO[t] @ V[sel].T                    # [H, m]
        if O is None:
            D = (P * dP).sum(axis=1, keepdims=True)
        else:
            D = (dO[t] * _f64(O[t])).sum(axis=1, keepdims=True)
        dz = P * (dP - D)
        dq[t] = scale * (dz @ K[sel])
        np.add.at(dK, sel, scale * (dz.T @ q[t]))
        np.add.at(dV, sel, P.T @ dO[t])
    return dq, dK, dV


def mla_tied_grad(dK, dV):
    """Gradient of the one stored KV row when V is its first dv columns
    (§3.1): the K-side gradient plus the V-side one on the latent part."""
    g = np.array(dK, dtype=np.float64, copy=True)
    g[:, : dV.shape[1]] += dV
    return g


# ----------------------------------------------------------------------------- indexer KL distillation
def indexer_logits(q_idx, W, k_idx):
    """x[t,s] = (q_t W) . k_s and I = ReLU(x) (§2.2), real-valued."""
    x = (_f64(q_idx) @ _f64(W)) @ _f64(k_idx).T
    return x, np.maximum(x, 0.0)


def attention_target(q, K, scale, cand):
    """p[t,s]: the attention probabilities of query t over its candidates
    cand[t] (a boolean row), averaged over the heads.  Each head's softmax
    runs over the candidates only; zero off the candidates."""
    q, K = _f64(q), _f64(K)
    n, H, _ = q.shape
    p = np.zeros((n, K.shape[0]))
    for t in range(n):
        c = np.nonzero(cand[t])[0]
        if c.size == 0:
            continue
        z = scale * (q[t] @ K[c].T)
        e = np.exp(z - z.max(axis=1, keepdims=True))
        p[t, c] = (e / e.sum(axis=1, keepdims=True)).mean(axis=0)
    return p


def kl_loss(p, I, cand):
    """sum over t of KL(p_t || softmax over cand[t] of I[t, .]).
    Returns (loss, r) with r the indexer distribution (zero off the
    candidates).  Terms with p = 0 contribute 0."""
    p, I = _f64(p), _f64(I)
    r = np.zeros_like(I)
    loss = 0.0
    for t in range(I.shape[0]):
        c = np.nonzero(cand[t])[0]
        if c.size == 0:
            continue
        z = I[t, c]
        lr = z - z.max() - np.log(np.exp(z - z.max()).sum())   # log softmax
        r[t, c] = np.exp(lr)
        pc = p[t, c]
        nz = pc > 0
        loss += float((pc[nz] * (np.log(pc[nz]) - lr[nz])).sum())
    return loss, r


def kl_grads(q_idx, W, k_idx, p, cand):
    """The loss of kl_loss on I = ReLU(q_idx W k_idx^T), and its gradients
    with respect to W, q_idx and k_idx.

    With r = softmax(I) over the candidates, dL/dI[t,s] = r - p on the
    candidates (p sums to 1 there); ReLU passes it where x > 0, and the
    bilinear form x = (q W) k^T gives
      dW = q_idx^T G k_idx,  dq_idx = G k_idx W^T,  dk_idx = G^T q_idx W,
    with G = (r - p) * [x > 0] on the candidates, 0 elsewhere."""
    x, I = indexer_logits(q_idx, W, k_idx)
    loss, r = kl_loss(p, I, cand)
    G = np.where(cand, r - _f64(p), 0.0) * (x > 0)
    qf, Wf, kf = _f64(q_idx), _f64(W), _f64(k_idx)
    dW = qf.T @ G @ kf
    dq = G @ kf @ Wf.T
    dk = G.T @ (qf @ Wf)
    return loss, dW, dq, dk


def causal_candidates(n, pos, nk):
    """cand[t, s] = s <= pos[t] (the dense warm-up's candidate set)."""
    return np.arange(nk)[None, :] <= np.asarray(pos)[:, None]


def selected_candidates(idx, nk):
    """cand[t, s] = s is in the selection idx[t] (the sparse stage's set)."""
    cand = np.zeros((idx.shape[0], nk), dtype=bool)
    for t in range(idx.shape[0]):
        sel = idx[t][idx[t] >= 0]
        cand[t, sel] = True
    return cand
