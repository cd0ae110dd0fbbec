"""The bench's launch count per prefill step (bench.step_launches: fold +
fused indexer/top-k + attention, or fold + score sweep + top-k + attention)
follows the library's own path choice, read here from dsa_workspace_size:
the two-launch path is the one whose workspace holds a score buffer of
total_q x max_seqlen_k floats next to the index buffer.  CPU only (no kernel runs)."""
import ctypes
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


@pytest.fixture(scope="module")
def lib():
    from sparse_attention_11_b200 import build
    build.build()
    from sparse_attention_11_b200 import dsa
    return dsa


@pytest.mark.parametrize("L,k", [(3000, 256), (8192, 2048), (10112, 2048), (10240, 2048), (12288, 2048),
                                 (32768, 2048), (2048, 2048)])
def test_step_launches_follow_the_library(lib, L, k):
    import bench
    from sparse_attention_11_b200 import workloads as W
    wl = W.custom(f"l{L}", (L,), (L,), base="prefill_l8192", k=k)
    ia = lib.dsa_indexer_args(lib.DSA_E4M3, 0x100000, 0x110000, lib.DSA_BF16, 0x200000, 0x300000, 0x310000)
    S = lib.dsa_seqs(1, L, L, L, L, 0x1000, 0x2000)
    n = ctypes.c_size_t(0)
    assert lib.raw_call("dsa_workspace_size", lib.DSA_OP_FORWARD, ctypes.byref(S), k, ctypes.byref(ia), None,
                        ctypes.byref(n)) == 0
    two_launch = n.value >= L * L * 4 + L * k * 4   # the score buffer on top of the index buffer
    assert bench.step_launches(wl) == (4 if two_launch else 3), (L, n.value)
