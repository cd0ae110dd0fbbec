"""Multi-rank host logic of bench.py on CPU (gloo, world size 2): the
max-over-ranks timing reduction, the barrier, and the reference arm's
rank-0-only output.  The data path has no collective (independent replicas),
so this is the whole N>1 logic."""
import json
import os
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _worker(rank, world, port, q):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bench.barrier(world)
        m = bench.max_over_ranks(10.0 + 5.0 * rank, world)
        tokens = world * 32768 * 4 / (m / 1e3)
        q.put((rank, m, tokens))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + os.getpid() % 1000
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    assert [r[1] for r in res] == [15.0, 15.0]      # both ranks see the max
    assert res[0][2] == res[1][2] == 2 * 32768 * 4 / 0.015


def test_reference_arm_prints_only_on_rank0():
    env = dict(os.environ, WORLD_SIZE="2", RANK="1", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload",
                        "tiny_l512", "--steps", "1", "--warmup", "0"], env=env, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == ""
    env.update(RANK="0", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload",
                        "tiny_l512", "--steps", "1", "--warmup", "0"], env=env, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["e2e"]["h2d_bytes_per_step"] == 0


def test_indexer_roofline_arithmetic():
    """The selection stage's roofline: one sweep's 2·128·Σ(pos+1) FLOP per
    event time, against the FP8 GEMM peak measured in the same run."""
    sys.path.insert(0, ROOT)
    import bench
    from sparse_attention_11_b200 import workloads as W
    wl = W.custom("probe", (1000,), (1000,), base="prefill_l8192", k=100)
    info = bench.workload_info(wl)
    assert info["pairs"] == 1000 * 1001 // 2 and info["sum_sel"] == 100 * 101 // 2 + 900 * 100
    fp8 = {"fp8_tflops": 10.0, "how": "test"}
    r = bench.indexer_roofline(info, 2.0, fp8)
    assert r["peak"] == 10.0
    assert abs(r["achieved"] - 2 * 128 * 500500 / 2e-3 / 1e12) < 1e-12
    assert abs(r["frac"] - r["achieved"] / 10.0) < 1e-15
    assert r["index_out_bytes"] == 4 * info["sum_sel"]
