"""Context-parallel prefill, host side (CPU, gloo).

The split of one sequence over G ranks ("DeepSeek-V3.2与稀疏注意力技术革新",
§3.2 cost model; §6 million-token direction) is checked without a GPU:
  * the row plans partition [0, L) and balance the indexer's O(pos) cost
    (zigzag) and the attention's min(k, pos+1) cost;
  * a chunk's sequence description puts its queries at positions a..b-1;
  * the all-gather of the key side, at world sizes 2 and 3 with ragged
    chunks, reassembles every key-side tensor bit for bit (e4m3 codes,
    fp32 scales, bf16 KV rows);
  * each rank's rows, computed by the oracle from its own query rows and
    the gathered keys at the chunk positions, equal the oracle's
    single-process forward (so the gather and the position mapping lose
    nothing).
"""
import os
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from sparse_attention_11_b200 import context_parallel as cp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("scheme", ["zigzag", "balanced", "contiguous"])
@pytest.mark.parametrize("L", [0, 1, 7, 512, 1001, 32768])
@pytest.mark.parametrize("world", [1, 2, 3, 8])
def test_plan_partitions(scheme, L, world):
    p = cp.plan(L, world, scheme)
    assert len(p) == world
    assert len({len(c) for c in p}) == 1  # the same chunk slots on every rank
    cover = np.zeros(L, dtype=np.int64)
    for chunks in p:
        for a, b in chunks:
            assert 0 <= a <= b <= L
            cover[a:b] += 1
    assert np.all(cover == 1)
    sizes = [cp.local_rows(c) for c in p]
    assert sum(sizes) == L
    if scheme != "balanced":
        assert max(sizes) - min(sizes) <= (2 if scheme == "zigzag" else 1)


def _costs(p, k):
    ix = [sum((b * (b + 1) - a * (a + 1)) // 2 for a, b in c) for c in p]  # sum of (pos+1)
    at = [sum(sum(min(k, t + 1) for t in range(a, b)) for a, b in c) for c in p]
    return np.array(ix, dtype=np.float64), np.array(at, dtype=np.float64)


@pytest.mark.parametrize("world", [2, 4, 8])
def test_plans_balance_cost(world):
    L, k = 32768, 2048
    ix, at = _costs(cp.plan(L, world, "zigzag"), k)
    assert ix.max() / ix.min() < 1.001  # the indexer's O(pos) cost, exactly even
    ixc, _ = _costs(cp.plan(L, world, "contiguous"), k)
    assert ixc.max() / ixc.min() > 2.0  # what zigzag removes
    # the modelled total (attention keys + per-row overhead + indexer pairs)
    # is even under "balanced" only
    a, o = cp.INDEXER_PAIR_COST, cp.ROW_OVERHEAD
    rows = lambda p: np.array([cp.local_rows(c) for c in p], dtype=np.float64)
    tot = lambda p: (lambda i, t: t + a * i)(*_costs(p, k)) + o * rows(p)
    tb = tot(cp.plan(L, world, "balanced"))
    assert tb.max() / tb.min() < 1.005
    tz = tot(cp.plan(L, world, "zigzag"))
    assert tz.max() / tz.min() > 1.03
    assert np.isclose(tb.sum(), tz.sum())
    # row_cost is that model, row by row
    p = cp.plan(L, world, "balanced")
    direct = np.array([sum(cp.row_cost(np.arange(s, e), k).sum() for s, e in c) for c in p])
    assert np.allclose(direct, tb)


def test_chunk_positions():
    s = cp.chunk_seqs((300, 420), "cpu")
    cq, ck = s.cu_q.numpy(), s.cu_k.numpy()
    assert list(cq) == [0, 120] and list(ck) == [0, 420]
    sq, sk = cq[1] - cq[0], ck[1] - ck[0]
    pos = (sk - sq) + np.arange(sq)  # the library's rule for query i of a sequence
    assert np.array_equal(pos, np.arange(300, 420))


def _worker(rank, world, port, scheme, q):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import oracle
    from sparse_attention_11_b200 import context_parallel as cpm, workloads as W

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        inp = W.generate(W.WORKLOADS["tiny_l512"], q_on_device=False)
        wl = inp.wl
        L = wl.total_q
        p = cpm.plan(L, world, scheme)
        mine = p[rank]
        rows = np.concatenate([np.arange(a, b) for a, b in mine]).astype(np.int64)
        # key side of this rank, gathered
        g_kidx = cpm.all_gather_rows(torch.from_numpy(inp.k_idx[rows]), p, rank).numpy()
        g_K = cpm.all_gather_rows(torch.from_numpy(inp.K[rows]), p, rank).numpy()
        g_V = cpm.all_gather_rows(torch.from_numpy(inp.V[rows]), p, rank).numpy()
        # the storage types of the FP8 / BF16 configuration
        rng = np.random.default_rng(3)
        codes = rng.integers(0, 256, size=(L, 128), dtype=np.uint8)
        scales = rng.random(L, dtype=np.float32)
        kv = torch.from_numpy(rng.standard_normal((L, 576), dtype=np.float32)).to(torch.bfloat16)
        ok_types = (np.array_equal(cpm.all_gather_rows(torch.from_numpy(codes[rows]), p, rank).numpy(), codes) and
                    np.array_equal(cpm.all_gather_rows(torch.from_numpy(scales[rows]), p, rank).numpy(), scales) and
                    torch.equal(cpm.all_gather_rows(kv[torch.from_numpy(rows)], p, rank), kv))
        # into a preallocated buffer (the per-step form), twice over the same buffer
        buf = torch.full_like(kv, float("nan"))
        for _ in range(2):
            got = cpm.all_gather_rows(kv[torch.from_numpy(rows)], p, rank, out=buf)
            ok_types = ok_types and got is buf and torch.equal(buf, kv)
        # this rank's rows at the chunk positions, against the gathered keys
        pos = np.concatenate([np.arange(a, b) for a, b in mine]).astype(np.int64)
        kb = np.zeros_like(pos)
        idx, out, lse = oracle.forward_rows(inp.q_idx[rows], None, inp.W, g_kidx, None, kb, pos, wl.k,
                                            inp.q_host[rows], g_K, g_K.shape[1], g_V, g_V.shape[1], wl.scale, wl.dv)
        same = (np.array_equal(g_kidx, inp.k_idx) and np.array_equal(g_K, inp.K) and np.array_equal(g_V, inp.V))
        q.put((rank, rows, idx, out, lse, same, ok_types))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,scheme", [(2, "zigzag"), (3, "balanced"), (3, "contiguous")])
def test_context_parallel_gloo(world, scheme):
    import oracle
    from sparse_attention_11_b200 import workloads as W

    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29600 + (os.getpid() + 7 * world + len(scheme)) % 1000
    procs = [ctx.Process(target=_worker, args=(r, world, port, scheme, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=240) for _ in range(world)]
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    inp = W.generate(W.WORKLOADS["tiny_l512"], q_on_device=False)
    wl = inp.wl
    L = wl.total_q
    kb, pos = inp.key_base_pos(np.arange(L))
    idx, out, lse = oracle.forward_rows(inp.q_idx, None, inp.W, inp.k_idx, None, kb, pos, wl.k, inp.q_host, inp.K,
                                        inp.K.shape[1], inp.V, inp.V.shape[1], wl.scale, wl.dv)
    seen = np.zeros(L, dtype=np.int64)
    for rank, rows, ridx, rout, rlse, same, ok_types in res:
        assert same, f"rank {rank}: gathered keys differ"
        assert ok_types, f"rank {rank}: gathered e4m3 / fp32 / bf16 rows differ"
        seen[rows] += 1
        assert np.array_equal(ridx, idx[rows])
        assert np.array_equal(rout, out[rows]) and np.array_equal(rlse, lse[rows])
    assert np.all(seen == 1)
