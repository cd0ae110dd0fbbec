"""dsa_select_noalloc: the selection entry point for callers that cannot
allocate device memory (a host framework owning all GPU memory through its own
pool, or a latency-critical path that must not allocate).  It keeps its
scratch in a static array inside the library instead of a caller workspace.

Checked through the C ABI against dsa_select (the workspace form) on the same
inputs, twice in a row (the second call reuses the shared static scratch
left by the first); indices must match exactly, the rule every selection
test here uses.  This file is collected last on purpose."""
import numpy as np
import pytest
import torch

from sparse_attention_11_b200 import dsa, workloads as W
from sparse_attention_11_b200.problem import DeviceProblem

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("L,k", [(3000, 256), (8192, 2048)])
def test_select_noalloc_matches_select(L, k):
    wl = W.custom(f"noalloc_l{L}_k{k}", (L,), (L,), base="prefill_l8192", k=k)
    inp = W.generate(wl, device="cuda")
    prob = DeviceProblem(inp)
    ref = torch.empty((L, k), dtype=torch.int32, device="cuda")
    dsa.dsa_select(prob.seqs, prob.ia, k, ref, prob.ws)
    dsa.check_device_status(prob.ws, "dsa_select")
    ref = ref.cpu().numpy()
    for _ in range(2):
        out = torch.full((L, k), -7, dtype=torch.int32, device="cuda")
        dsa.dsa_select_noalloc(prob.seqs, prob.ia, k, out)
        assert np.array_equal(out.cpu().numpy(), ref)


def test_select_noalloc_ragged_batch_dynamic_k():
    """A ragged batch of three prefill sequences with a per-query k (k_t
    uniform in [0, k] plus 0 and past k), against dsa_select."""
    k = 512
    wl = W.custom("noalloc_batch", (1500, 700, 2300), (1500, 900, 2300), base="prefill_l8192", k=k)
    inp = W.generate(wl, device="cuda")
    prob = DeviceProblem(inp)
    rng = np.random.default_rng(3)
    kr = rng.integers(0, k + 1, size=wl.total_q).astype(np.int32)
    kr[:5] = 0
    kr[-5:] = k + 100
    ia = dsa.indexer_args(prob.q_idx, prob.q_idx_scale, prob.W, prob.k_idx, prob.k_idx_scale,
                          k_per_row=torch.from_numpy(kr).cuda())
    ref = torch.empty((wl.total_q, k), dtype=torch.int32, device="cuda")
    dsa.dsa_select(prob.seqs, ia, k, ref, prob.ws)
    dsa.check_device_status(prob.ws, "dsa_select")
    out = torch.full((wl.total_q, k), -7, dtype=torch.int32, device="cuda")
    dsa.dsa_select_noalloc(prob.seqs, ia, k, out)
    assert np.array_equal(out.cpu().numpy(), ref.cpu().numpy())


def test_select_noalloc_rejects_oversize_and_unsupported():
    # more query rows than the static scratch holds: rejected before launch
    L = 32769
    seqs = dsa.Seqs([0, L], [0, L])
    q = torch.zeros((L, 128), dtype=torch.uint8, device="cuda")
    sc = torch.ones(L, dtype=torch.float32, device="cuda")
    Wm = torch.zeros((128, 128), dtype=torch.bfloat16, device="cuda")
    ia = dsa.indexer_args(q, sc, Wm, q, sc)
    idx = torch.empty((L, 8), dtype=torch.int32, device="cuda")
    with pytest.raises(dsa.DsaError) as e:
        dsa.dsa_select_noalloc(seqs, ia, 8, idx)
    assert e.value.code == dsa.DSA_ERR_WORKSPACE
    # decode-shaped inputs need a score buffer: not served without a workspace
    seqs = dsa.Seqs([0, 1, 2], [0, 600, 1200])
    with pytest.raises(dsa.DsaError) as e:
        dsa.dsa_select_noalloc(seqs, ia, 8, idx[:2])
    assert e.value.code == dsa.DSA_ERR_UNSUPPORTED
