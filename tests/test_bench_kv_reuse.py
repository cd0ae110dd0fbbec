"""The index rows of the cross-query KV-tile reuse prototype (bench.py,
pair_union_rows), checked on CPU against a set-based construction: for each
adjacent pair, the ascending union of both selections, each query's own keys
kept and its partner's masked (-1), then -1 padding."""
import os
import sys

import numpy as np
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def test_pair_union_rows_brute_force():
    import bench
    rng = np.random.default_rng(4)
    T, k1, L = 9, 8, 30
    own = np.full((T, k1), -1, np.int32)
    for t in range(T):
        n = int(rng.integers(0, k1 + 1))            # rows with padding, and an empty row
        own[t, :n] = np.sort(rng.choice(L, size=n, replace=False))
    own[2] = own[3]                                 # a pair with identical selections
    rows, usize = bench.pair_union_rows(torch.from_numpy(own))
    rows = rows.numpy()
    assert rows.shape == (T, 2 * k1)
    for i in range(T // 2):
        A = set(own[2 * i][own[2 * i] >= 0].tolist())
        B = set(own[2 * i + 1][own[2 * i + 1] >= 0].tolist())
        U = sorted(A | B)
        assert int(usize[i]) == len(U)
        for r, S in ((2 * i, A), (2 * i + 1, B)):
            assert rows[r, :len(U)].tolist() == [x if x in S else -1 for x in U]
            assert np.all(rows[r, len(U):] == -1)
    assert rows[T - 1, :k1].tolist() == own[T - 1].tolist() and np.all(rows[T - 1, k1:] == -1)
