"""Context-parallel prefill on the GPU, ranks emulated one after another.

One process and one GPU run every rank's chunks in turn.  Each rank's
chunks run against the whole key side, which is what the all-gather leaves
in every rank's memory.  The ranks' kernels never wait on one another, so
running them in sequence is the same computation as running them on G
GPUs.  The collective itself is covered by the gloo tests
(test_context_parallel.py).

Checked on prefill_l8192 ("DeepSeek-V3.2与稀疏注意力技术革新", §2.2-§3.1)
under the zigzag, balanced and contiguous plans:
  * each rank's idx, out and lse rows equal, bit for bit, the rows of one
    dsa_forward over the whole sequence;
  * context_parallel.forward at world size 1 (the gather's local path and
    both zigzag chunks) equals it as well;
  * a short chunk at the end of the sequence (42 queries over 8192 keys),
    which takes the scan + histogram top-k selection path, agrees in its
    selection (overlap >= 0.999).  Where its index rows are identical, the
    attention output is identical.
"""
import numpy as np
import pytest
import torch

from sparse_attention_11_b200 import context_parallel as cp, workloads as W

from gpu_util import OVERLAP_MIN, make

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def full():
    wl = W.WORKLOADS["prefill_l8192"]
    inp, prob = make(wl)
    prob.forward()
    prob.check("full forward")
    torch.cuda.synchronize()
    return wl, prob


def _rank_run(wl, prob, chunks):
    rows = torch.cat([torch.arange(a, b) for a, b in chunks]).cuda()
    n = rows.numel()
    q_idx, q_sc, q = prob.q_idx[rows], prob.q_idx_scale[rows], prob.q[rows]
    out = torch.full((n, wl.heads, wl.dv), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((n, wl.heads), float("nan"), dtype=torch.float32, device="cuda")
    idx = torch.full((n, wl.k), -7, dtype=torch.int32, device="cuda")
    run = cp.LocalForward(chunks, wl.k, q_idx, q_sc, prob.W, prob.k_idx, prob.k_idx_scale, q, prob.K, prob.V,
                          wl.scale, out, lse, idx)
    run()
    run.check()
    return rows, idx, out, lse


@pytest.mark.parametrize("world,scheme", [(2, "zigzag"), (3, "balanced"), (4, "contiguous")])
def test_ranks_match_single_forward(full, world, scheme):
    wl, prob = full
    seen = torch.zeros(wl.total_q, dtype=torch.int64, device="cuda")
    for r, chunks in enumerate(cp.plan(wl.total_q, world, scheme, k=wl.k)):
        rows, idx, out, lse = _rank_run(wl, prob, chunks)
        assert torch.equal(idx, prob.idx[rows]), f"rank {r}: selection differs"
        assert torch.equal(out.view(torch.int16), prob.out[rows].view(torch.int16)), f"rank {r}: output differs"
        assert torch.equal(lse, prob.lse[rows]), f"rank {r}: lse differs"
        seen[rows] += 1
    assert bool((seen == 1).all())


def test_forward_world1(full):
    wl, prob = full
    p = cp.plan(wl.total_q, 1, "zigzag")
    assert len(p[0]) == 2
    rows = torch.cat([torch.arange(a, b) for a, b in p[0]]).cuda()
    out = torch.empty((rows.numel(), wl.heads, wl.dv), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((rows.numel(), wl.heads), dtype=torch.float32, device="cuda")
    idx = torch.empty((rows.numel(), wl.k), dtype=torch.int32, device="cuda")
    kv_shard = prob.K[rows]
    k_idx, k_sc, K, V = cp.forward(p, 0, wl.k, prob.q_idx[rows], prob.q_idx_scale[rows], prob.W, prob.k_idx[rows],
                                   prob.k_idx_scale[rows], prob.q[rows], kv_shard, wl.dv, wl.scale, out, lse, idx)
    assert torch.equal(k_idx, prob.k_idx) and torch.equal(K.view(torch.int16), prob.K.view(torch.int16))
    assert torch.equal(idx, prob.idx[rows])
    assert torch.equal(out.view(torch.int16), prob.out[rows].view(torch.int16))
    assert torch.equal(lse, prob.lse[rows])


def test_short_tail_chunk(full):
    wl, prob = full
    L = wl.total_q
    rows, idx, out, lse = _rank_run(wl, prob, [(L - 42, L)])
    g, f = idx.cpu().numpy(), prob.idx[rows].cpu().numpy()
    fr = [len(np.intersect1d(g[i], f[i])) / wl.k for i in range(len(g))]
    assert np.all(g >= 0) and np.mean(fr) >= OVERLAP_MIN, np.mean(fr)
    same = np.where((g == f).all(axis=1))[0]
    assert len(same) > 0
    s = torch.from_numpy(same).cuda()
    assert torch.equal(out[s].view(torch.int16), prob.out[rows][s].view(torch.int16))
