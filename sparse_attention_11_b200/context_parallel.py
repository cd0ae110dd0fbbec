"""Context-parallel prefill: one long sequence split over the ranks of a
process group by query rows, with the key side all-gathered once.

Method: "DeepSeek-V3.2与稀疏注意力技术革新".  §2.2-§2.3 give the per-query
indexer and top-k.  §3.1 gives the attention over the k selected rows.
§3.2 gives the cost, O(L²) in the indexer plus O(Lk) in the attention.
Every query row depends only on its own query and on the keys 0..pos.
So the rows split freely across GPUs once each GPU holds the whole key
side.  The pages name million-token contexts as the direction (§6); this is
the split that scales one sequence over several GPUs.

Plan.  The sequence's L rows are cut into chunks:
  * "zigzag": 2·G chunks of near-equal length; rank r takes chunks r and
    2G-1-r.  The indexer's work on a row grows with its position, so
    pairing an early chunk with a late one evens the ranks' indexer cost.
    The attention's work is k rows per query once pos >= k, so it is even
    under either plan.
  * "balanced": the zigzag pairing with boundaries placed on the modelled
    row cost, so the cheap first k rows of the attention are evened too.
  * "contiguous": one chunk per rank.
Each rank starts with the rows of its own chunks, for both the query side
(q_idx + scales, q) and the key side (k_idx + scales, the KV rows).

Exchange.  One all-gather per key-side tensor assembles the full sequence
in every rank's memory, in sequence order: 16 + 4 + 1152 bytes per token in
the FP8-indexer / BF16 MLA configuration.  That is 38 MB at L = 32K, small
against the compute.  Outputs stay sharded; nothing is reduced.

Compute.  A chunk [a, b) is, for the library, a sequence whose b keys are
rows 0..b-1 of the gathered buffers and whose b-a queries are its last
positions.  That is the library's rule pos = seqlen_k - seqlen_q + i, so
each chunk is one dsa_forward call on this rank's rows.  Every step runs
in libdsa's kernels.  This module only plans, gathers and marshals.
"""
import numpy as np
import torch

from . import dsa


# Modelled cost of a rank's rows, in units of the attention's cost of one
# selected key.  The three terms are fitted by least squares to 24 measured
# rank times (3 plans x 8 ranks, L = 32K, ranks emulated on a B200; RMS
# residual 0.1 ms of about 4.4 ms):
#   0.395 ns per selected key (attention);
#   54.6 ns per query row, 138 keys' worth (the per-query work of the
#     attention and the selection);
#   7.45e-12 s per causal (query, key) pair, 0.0189 keys' worth (the
#     key-split selection that a rank's chunks take).
INDEXER_PAIR_COST = 0.0189
ROW_OVERHEAD = 138.0


def row_cost(pos, k, alpha=INDEXER_PAIR_COST, overhead=ROW_OVERHEAD):
    """Modelled cost of query rows at positions `pos`: min(k, pos+1)
    selected keys, a per-row overhead, and alpha per causal indexer pair."""
    pos = np.asarray(pos, dtype=np.float64)
    return np.minimum(float(k), pos + 1.0) + overhead + alpha * (pos + 1.0)


def plan(L, world, scheme="zigzag", k=2048, alpha=INDEXER_PAIR_COST, overhead=ROW_OVERHEAD):
    """Chunks of query rows per rank: a list (rank) of lists of (begin, end),
    in the order the rank stores its rows.

    zigzag: 2G chunks of near-equal length, rank r takes chunks r and
    2G-1-r (evens the indexer's O(pos) cost exactly).  balanced: the same
    pairing, with boundaries placed on the cumulative row_cost so that the
    G chunks of each half carry equal cost, which also evens the cheap
    first k rows of the attention.  contiguous: one chunk per rank."""
    if L < 0 or world < 1:
        raise ValueError("need L >= 0 and world >= 1")
    n = 2 * world
    if scheme == "zigzag":
        b = [(i * L) // n for i in range(n + 1)]
    elif scheme == "balanced":
        c = np.concatenate([[0.0], np.cumsum(row_cost(np.arange(L), k, alpha, overhead))])
        half = L // 2
        first = [c[half] * j / world for j in range(world + 1)]
        second = [c[half] + (c[L] - c[half]) * j / world for j in range(1, world + 1)]
        b = [int(np.searchsorted(c, x, side="left")) for x in first + second]
        b[0], b[world], b[n] = 0, half, L
        for i in range(1, n + 1):
            b[i] = max(b[i], b[i - 1])
    elif scheme == "contiguous":
        b = [(i * L) // world for i in range(world + 1)]
        return [[(b[r], b[r + 1])] for r in range(world)]
    else:
        raise ValueError(f"unknown scheme {scheme!r}")
    return [[(b[r], b[r + 1]), (b[n - 1 - r], b[n - r])] for r in range(world)]


def local_rows(chunks):
    """Number of rows a rank holds."""
    return sum(e - s for s, e in chunks)


def shard(x, chunks):
    """The rows of `chunks` of a full [L, ...] tensor, concatenated in chunk
    order (a rank's starting layout)."""
    return torch.cat([x[s:e] for s, e in chunks]) if chunks else x[:0]


def chunk_seqs(chunk, device):
    """The library's sequence description of one chunk [a, b): b keys, the
    last b-a of them are the queries."""
    a, b = chunk
    return dsa.Seqs([0, b - a], [0, b], device=device)


def all_gather_rows(x, plans, rank, group=None, out=None):
    """Assemble the full [L, ...] tensor from every rank's shard `x` (the rows
    of plans[rank], in chunk order), into `out` when given (rows in sequence
    order; it must be [L, ...] of x's dtype), else into a new tensor.

    One all-gather per chunk slot (the j-th chunk of every rank).  Each
    rank's piece is padded to the slot's longest chunk, because the
    collective moves equal-sized pieces.  Every rank makes the same calls in
    the same order.
    """
    import torch.distributed as dist

    world = len(plans)
    L = max(e for p in plans for _, e in p) if any(plans) else 0
    if out is not None:
        if tuple(out.shape) != (L,) + tuple(x.shape[1:]) or out.dtype != x.dtype:
            raise ValueError("out must be [L, ...] with the shard's dtype")
        full = out
    else:
        full = torch.empty((L,) + tuple(x.shape[1:]), dtype=x.dtype, device=x.device)
    if world == 1:
        off = 0
        for s, e in plans[0]:
            full[s:e].copy_(x[off:off + e - s])
            off += e - s
        return full
    nslot = len(plans[0])
    if any(len(p) != nslot for p in plans):
        raise ValueError("every rank needs the same number of chunks")
    off = 0
    for j in range(nslot):
        lens = [p[j][1] - p[j][0] for p in plans]
        m = max(lens)
        mine = x[off:off + lens[rank]]
        off += lens[rank]
        if m == 0:
            continue
        send = mine if lens[rank] == m else torch.cat(
            [mine, torch.zeros((m - lens[rank],) + tuple(x.shape[1:]), dtype=x.dtype, device=x.device)])
        recv = [torch.empty_like(send) for _ in range(world)]
        dist.all_gather(recv, send.contiguous(), group=group)
        for r in range(world):
            s, e = plans[r][j]
            full[s:e].copy_(recv[r][:e - s])
    return full


class LocalForward:
    """This rank's forward over the full (gathered) key side: one dsa_forward
    per chunk, on the rank's rows of the query-side inputs and outputs.

    q_idx [n, 128] (uint8 e4m3 or fp32), q_scale [n] or None, q [n, H, dk]:
    the rank's rows in chunk order.  W_index as in indexer_args.  k_idx
    [L, 128], k_scale [L] or None, K [L, >=dk], V [L, >=dv] (may be a view
    of K's first columns): the gathered key side.  out [n, H, dv], lse [n, H]
    or None, idx [n, k]: this rank's rows of the results, in chunk order.
    """

    def __init__(self, chunks, k, q_idx, q_scale, W, k_idx, k_scale, q, K, V, scale, out, lse, idx):
        dev = q.device
        self.k = int(k)
        self.calls = []
        off = 0
        for ch in chunks:
            n = ch[1] - ch[0]
            if n == 0:
                continue
            sl = slice(off, off + n)
            off += n
            seqs = chunk_seqs(ch, dev)
            ia = dsa.indexer_args(q_idx[sl], q_scale[sl] if q_scale is not None else None, W, k_idx[:ch[1]],
                                  k_scale[:ch[1]] if k_scale is not None else None)
            aa = dsa.attn_args(q[sl], K[:ch[1]], V[:ch[1]], scale, out[sl], lse[sl] if lse is not None else None)
            self.calls.append((seqs, ia, aa, idx[sl]))
        need = max((dsa.dsa_workspace_size(dsa.DSA_OP_FORWARD, s, self.k, ia, aa) for s, ia, aa, _ in self.calls),
                   default=256)
        self.ws = dsa.workspace(need, dev)

    def __call__(self):
        for seqs, ia, aa, ix in self.calls:
            dsa.dsa_forward(seqs, ia, aa, self.k, ix, self.ws)

    def check(self, where="context-parallel forward"):
        dsa.check_device_status(self.ws, where)


class ContextParallelForward:
    """One rank's context-parallel forward, with every buffer allocated once:
    the gathered key side (index codes, their scales, the KV rows) and the
    per-chunk calls of LocalForward over them.  Each step all-gathers the
    ranks' key-side shards into those buffers and runs the rank's chunks.

    q_idx, q_scale, q, out, lse, idx: this rank's rows in chunk order, as in
    LocalForward.  The shards passed to step() are this rank's key-side rows
    in chunk order: k_idx [n, 128], k_scale [n] or None, kv [n, dk].  V is
    the first dv columns of the gathered KV rows (MLA)."""

    def __init__(self, plans, rank, k, q_idx, q_scale, W, q, dk, dv, scale, out, lse, idx, k_idx_dtype,
                 kv_dtype, group=None):
        self.plans, self.rank, self.group = plans, rank, group
        L = max(e for p in plans for _, e in p)
        dev = q.device
        self.k_idx = torch.empty((L, 128), dtype=k_idx_dtype, device=dev)
        self.k_scale = torch.empty((L,), dtype=torch.float32, device=dev) if q_scale is not None else None
        self.kv = torch.empty((L, dk), dtype=kv_dtype, device=dev)
        self.local = LocalForward(plans[rank], k, q_idx, q_scale, W, self.k_idx, self.k_scale, q, self.kv,
                                  self.kv[:, :dv], scale, out, lse, idx)

    def step(self, k_idx_shard, k_scale_shard, kv_shard):
        all_gather_rows(k_idx_shard, self.plans, self.rank, self.group, out=self.k_idx)
        if self.k_scale is not None:
            all_gather_rows(k_scale_shard, self.plans, self.rank, self.group, out=self.k_scale)
        all_gather_rows(kv_shard, self.plans, self.rank, self.group, out=self.kv)
        self.local()

    def check(self, where="context-parallel forward"):
        self.local.check(where)


def forward(plans, rank, k, q_idx, q_scale, W, k_idx_shard, k_scale_shard, q, kv_shard, dv, scale, out, lse, idx,
            v_shard=None, group=None):
    """Context-parallel forward on this rank in one call: all-gather the key
    side (indexer codes, their scales, the KV rows), then run the rank's
    chunks.  V is the first dv columns of the KV rows (the MLA latent part)
    unless v_shard gives V's rows separately.  Returns the gathered
    (k_idx, k_scale, K, V).  Repeated steps should use
    ContextParallelForward, which allocates once."""
    k_idx = all_gather_rows(k_idx_shard, plans, rank, group)
    k_scale = all_gather_rows(k_scale_shard, plans, rank, group) if k_scale_shard is not None else None
    K = all_gather_rows(kv_shard, plans, rank, group)
    V = all_gather_rows(v_shard, plans, rank, group) if v_shard is not None else K[:, :dv]
    run = LocalForward(plans[rank], k, q_idx, q_scale, W, k_idx, k_scale, q, K, V, scale, out, lse, idx)
    run()
    run.check()
    return k_idx, k_scale, K, V
