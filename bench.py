#!/usr/bin/env python
"""Benchmark of the DSA forward hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl native|reference]
                    [--workload prefill_l32768]

One step = one pass of the whole path over one batch: fold W_index into the
indexer queries, fused FP8 indexer + exact top-2048 (scores stay on chip),
sparse MQA attention over the selected rows.  The headline workload is the
L=32768 prefill (tokens/s); the same line carries the decode measurement
(batch 64, contexts 16K-64K; tokens/s = 64 / step time).  Inputs are
synthetic and seeded (sparse_attention_11_b200.workloads) and larger than
L2, so no flush is needed between steps.

Under torchrun (N > 1) every rank runs an independent replica of the
workload (the path shards by independent sequences; no collective on the
data path); value = all ranks' tokens / max-over-ranks device time.
With --cp the ranks instead split ONE sequence by query rows (context
parallel): the key side is all-gathered over NCCL each step and value = L
tokens / max-over-ranks time ("scaling": "strong").  At N = 1 the default
line carries "context_parallel": the same split at 8 ranks, emulated rank
by rank on one GPU (compute only).

--impl reference times the CPU oracle (oracle/), as it stands, on the host
cores on a bounded stratified sample of the same workload.
"""
import argparse
import datetime
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "DSA prefill tokens/s at L=32K (indexer+top-2048+sparse attn); decode tok/s"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--workload", default="prefill_l32768")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-dynk", action="store_true", help="skip the dynamic-k line")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-cp", action="store_true", help="skip the emulated context-parallel line")
    ap.add_argument("--cp", action="store_true",
                    help="under torchrun: split one sequence over the ranks (context parallel) instead of replicas")
    ap.add_argument("--cp-scheme", choices=["balanced", "zigzag", "contiguous"], default="balanced")
    ap.add_argument("--kv-reuse", action="store_true",
                    help="also measure the cross-query KV-tile reuse prototype (adjacent query pairs, k = 1024)")
    ap.add_argument("--bwd", action="store_true",
                    help="also time the sparse attention's backward (dsa_sparse_attn_bwd) on the workload")
    ap.add_argument("--cpu-seconds", type=float, default=15.0, help="target CPU seconds of the oracle sample")
    ap.add_argument("--probe-fp8-peak", action="store_true",
                    help="only measure the dense FP8 (e4m3) GEMM peak of this GPU (burst and sustained) and print it")
    ap.add_argument("--profile-case", choices=["select", "decode-small", "decode"],
                    help="run a lean case for a profiler (no timing line): 'select' = dsa_select on --workload with "
                         "the indexer inputs only; 'decode-small' = decode select + attention, 64 sequences with "
                         "contexts 16K-24K; 'decode' = the same on decode_b64 (contexts 16K-64K)")
    ap.add_argument("--reps", type=int, default=3, help="calls of the --profile-case")
    return ap.parse_args()


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def fp8_peak(burst_reps=10, sustained_s=0.0, n=8192):
    """Dense FP8 tensor peak of this GPU, measured: torch._scaled_mm on e4m3
    operands, n^3 (2 n^3 FLOP per call), bf16 out, per-tensor fp32 scales.
    Burst = best of `burst_reps` calls timed with CUDA events; sustained =
    back-to-back calls for `sustained_s` seconds.  No clock or power setting is
    touched."""
    import torch
    g = torch.Generator(device="cuda")
    g.manual_seed(1234)
    a = torch.randn((n, n), generator=g, device="cuda").to(torch.float8_e4m3fn)
    bt = torch.randn((n, n), generator=g, device="cuda").to(torch.float8_e4m3fn)
    sa = torch.ones((), device="cuda")
    sb = torch.ones((), device="cuda")
    st = torch.cuda.current_stream()

    def mm():
        return torch._scaled_mm(a, bt.t(), sa, sb, out_dtype=torch.bfloat16)

    for _ in range(3):
        mm()
    torch.cuda.synchronize()
    best = float("inf")
    for _ in range(burst_reps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(st)
        mm()
        e1.record(st)
        torch.cuda.synchronize()
        best = min(best, e0.elapsed_time(e1))
    flop = 2.0 * n ** 3
    res = {"fp8_tflops": flop / (best / 1e3) / 1e12, "n": n, "how": f"torch._scaled_mm e4m3 {n}^3, best of {burst_reps}"}
    if sustained_s > 0:
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        calls = max(1, int(sustained_s / (best / 1e3)))
        e0.record(st)
        for _ in range(calls):
            mm()
        e1.record(st)
        torch.cuda.synchronize()
        res["fp8_tflops_sustained"] = flop * calls / (e0.elapsed_time(e1) / 1e3) / 1e12
        res["sustained_calls"] = calls
    del a, bt
    torch.cuda.empty_cache()
    return res


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi samples of this GPU's clocks and throttle reasons."""
    FIELDS = ["clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.active",
              "clocks_event_reasons.hw_slowdown", "clocks_event_reasons.hw_thermal_slowdown",
              "clocks_event_reasons.sw_thermal_slowdown", "clocks_event_reasons.sw_power_cap"]

    def __init__(self, device_index):
        import torch
        self.ident = None
        try:
            props = torch.cuda.get_device_properties(device_index)
            u = str(getattr(props, "uuid", ""))
            if u:
                self.ident = u if u.startswith("GPU-") else "GPU-" + u
        except Exception:
            self.ident = None
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        cmd = ["nvidia-smi", "--query-gpu=" + ",".join(self.FIELDS), "--format=csv,noheader,nounits", "-lms", "100"]
        if self.ident:
            cmd += ["-i", self.ident]
        try:
            self.proc = subprocess.Popen(cmd, stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.15)
        self.proc.terminate()
        self.proc.wait(timeout=10)
        sm, mx, pw, reasons = [], [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < len(self.FIELDS):
                    continue
                try:
                    sm.append(float(parts[0]))
                    mx.append(float(parts[1]))
                    pw.append(float(parts[2]))
                except ValueError:
                    continue
                for n, v in zip(names, parts[4:8]):
                    if v.lower().startswith("active"):
                        reasons.add(n)
        os.unlink(self.path)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        # samples under load: power above half of the run's maximum
        pmax = max(pw) if pw else 0
        loaded = [s for s, p in zip(sm, pw) if p >= 0.5 * pmax] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm), "power_w_max": pmax}


# ----------------------------------------------------------------------------- distributed
def dist_setup(args):
    import torch
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    return ws, rank, local


def barrier(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x, ws, device=None):
    if ws == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ----------------------------------------------------------------------------- workloads
def workload_info(wl):
    import numpy as np
    pos = []
    for sq, sk in zip(wl.seqlens_q, wl.seqlens_k):
        pos.append(np.arange(sk - sq, sk, dtype=np.int64))
    pos = np.concatenate(pos)
    sel = np.minimum(pos + 1, wl.k)
    return {"tokens": int(wl.total_q), "sum_sel": int(sel.sum()), "pairs": int((pos + 1).sum())}


def indexer_roofline(info, sel_ms, fp8):
    """The selection stage (fold + indexer/top-k) against the FP8 tensor
    peak.  The work is one score sweep's algorithmic FLOP, 2·128·Σ(pos+1),
    divided by the stage's event time; the index rows it writes are reported
    beside it.  The peak is this GPU's dense e4m3 GEMM burst, measured in the
    same run (fp8_peak)."""
    flops = 2.0 * 128 * info["pairs"]
    peak = fp8["fp8_tflops"]
    achieved = flops / (sel_ms / 1e3) / 1e12
    out_bytes = 4 * info["sum_sel"]
    return {"stage": "select (fold + indexer/top-k)", "bound": "tensor", "achieved": achieved, "peak": peak,
            "unit": "TFLOP/s", "frac": achieved / peak,
            "peak_kind": "fp8 burst, measured in this run (" + fp8["how"] + ")", "flops_per_call": flops,
            "index_out_bytes": out_bytes, "index_out_gbs": out_bytes / (sel_ms / 1e3) / 1e9}


def attn_flops(wl, info):
    return 2.0 * wl.heads * (wl.dk + wl.dv) * info["sum_sel"]


def attn_bytes(wl, info):
    """Algorithmic HBM bytes of one attention launch: gathered KV rows (V is the
    latent part of K, so a row is dk bf16), q, out, lse, idx."""
    row = wl.dk * 2 if wl.v_in_k else (wl.dk + wl.dv) * 2
    return info["sum_sel"] * row + wl.total_q * wl.heads * (wl.dk + wl.dv) * 2 + wl.total_q * wl.heads * 4 + \
        wl.total_q * wl.k * 4


def captured_traffic(workload, kernel):
    """DRAM bytes per launch from the committed ncu capture, or None when the
    kernel's sources changed since the counters were taken."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        tr = json.load(f)
    h = hashlib.sha256()
    for rel in tr.get("kernel_sources", []):
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    if h.hexdigest() != tr.get("kernel_sources_sha256"):
        return None
    return tr.get(workload, {}).get(kernel)


def step_launches(wl):
    """Kernel launches of one prefill step (dsa_select + dsa_sparse_attn),
    by the library's selection rule (include/dsa.h, dsa_select).  The fused
    path is fold, indexer/top-k.  Fewer than 80 128-row blocks over more
    than 2048 keys add one launch: fold, score sweep, histogram top-k."""
    blocks = wl.batch * ((max(wl.seqlens_q) + 127) // 128)
    split = max(wl.seqlens_q) >= 64 and blocks < 80 and max(wl.seqlens_k) > 2048
    return (4 if split else 3)


def run_native_workload(wl, steps, warmup, ws_n, rank, sampler=None, v_separate=None, inp=None):
    """Device-timed steps of select + attention on one workload (v_separate:
    V in a tensor of its own instead of the latent part of K)."""
    import torch
    from sparse_attention_11_b200 import dsa, workloads as W
    from sparse_attention_11_b200.problem import DeviceProblem
    if inp is None:
        inp = W.generate(wl, device="cuda")
    prob = DeviceProblem(inp, v_separate=v_separate)
    st = torch.cuda.current_stream()

    def step(evs=None):
        if evs:
            evs[0].record(st)
        dsa.dsa_select(prob.seqs, prob.ia, wl.k, prob.idx, prob.ws)
        if evs:
            evs[1].record(st)
        dsa.dsa_sparse_attn(prob.seqs, prob.aa, prob.idx, wl.k, prob.ws)
        if evs:
            evs[2].record(st)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    prob.check("warmup")
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(ws_n)
    torch.cuda.synchronize()
    if sampler:
        sampler.start()
    t0.record(st)
    for i in range(steps):
        step(evs[i])
    t1.record(st)
    torch.cuda.synchronize()
    clocks = sampler.stop() if sampler else None
    barrier(ws_n)
    prob.check("timed steps")
    ms = t0.elapsed_time(t1)
    sel_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    att_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
    return inp, prob, ms, sel_ms, att_ms, clocks


def dynamic_k_native(inp, prob, steps, warmup, lo=256, seed=11):
    """Dynamic k (a per-query k): the same prefill step with k_t drawn
    uniformly in [lo, k] per query (seeded), device-timed like the main line."""
    import numpy as np
    import torch
    from sparse_attention_11_b200 import dsa
    wl = prob.wl
    rng = np.random.default_rng(seed)
    kr = rng.integers(lo, wl.k + 1, size=wl.total_q).astype(np.int32)
    ia = dsa.indexer_args(prob.q_idx, prob.q_idx_scale, prob.W, prob.k_idx, prob.k_idx_scale,
                          k_per_row=torch.from_numpy(kr).cuda())
    st = torch.cuda.current_stream()

    def step(evs=None):
        if evs:
            evs[0].record(st)
        dsa.dsa_select(prob.seqs, ia, wl.k, prob.idx, prob.ws)
        if evs:
            evs[1].record(st)
        dsa.dsa_sparse_attn(prob.seqs, prob.aa, prob.idx, wl.k, prob.ws)
        if evs:
            evs[2].record(st)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    for i in range(steps):
        step(evs[i])
    torch.cuda.synchronize()
    dsa.check_device_status(prob.ws, "dynamic k")
    ms = statistics.mean(e[0].elapsed_time(e[2]) for e in evs)
    sel_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    att_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
    pos = np.concatenate([np.arange(sk - sq, sk) for sq, sk in zip(wl.seqlens_q, wl.seqlens_k)])
    sum_sel = int(np.minimum(kr, pos + 1).sum())
    flops = 2.0 * wl.heads * (wl.dk + wl.dv) * sum_sel
    return {"k_per_query": f"uniform [{lo}, {wl.k}] (seed {seed}); K_t = min(k_t, pos+1)",
            "value": wl.total_q / (ms / 1e3), "unit": "tokens/s", "ms_per_step": ms, "steps": steps,
            "stages_ms": {"select": sel_ms, "attention": att_ms}, "sum_selected": sum_sel,
            "attention_tflops": flops / (att_ms / 1e3) / 1e12}


def pair_union_rows(own):
    """Index rows for adjacent query pairs (2i, 2i+1) sharing their key
    tiles: row 2i (2i+1) holds the ascending union of both queries'
    selections, with the keys only the partner selected set to -1 (masked),
    then -1 padding, width 2 * own.shape[1].  A trailing unpaired row keeps
    its own selection.  Returns the rows and the union size of each pair."""
    import torch
    T, k1 = own.shape
    npair = T // 2
    big = torch.iinfo(torch.int64).max
    a = own[0:2 * npair:2].to(torch.int64)
    b = own[1:2 * npair:2].to(torch.int64)
    cat = torch.cat([a, b], dim=1)
    cat = torch.where(cat < 0, torch.full_like(cat, big), cat)
    srt, _ = torch.sort(cat, dim=1)
    dup = torch.zeros_like(srt, dtype=torch.bool)
    dup[:, 1:] = srt[:, 1:] == srt[:, :-1]
    uni, _ = torch.sort(torch.where(dup, torch.full_like(srt, big), srt), dim=1)
    usize = (uni != big).sum(dim=1)

    def masked(rows):
        o, _ = torch.sort(torch.where(rows < 0, torch.full_like(rows, big), rows), dim=1)
        j = torch.searchsorted(o, uni).clamp(max=o.shape[1] - 1)
        hit = (torch.gather(o, 1, j) == uni) & (uni != big)
        return torch.where(hit, uni, torch.full_like(uni, -1)).to(torch.int32)

    out = torch.full((T, 2 * k1), -1, dtype=torch.int32, device=own.device)
    out[0:2 * npair:2] = masked(a)
    out[1:2 * npair:2] = masked(b)
    if T % 2:
        out[T - 1, :k1] = own[T - 1]
    return out, usize


def kv_reuse_prototype(prob, steps, warmup, k1=1024):
    """Cross-query KV-tile reuse (adjacent query pairs), a measured prototype
    on the shipped attention kernel.  Each query of a pair (2i, 2i+1) gets
    the pair's union of top-k1 selections as its index row (at most 2*k1
    slots, ascending), with the slots only its partner selected masked (-1):
    the kernel then runs S, the softmax and PV over the union's tiles with a
    per-query mask, which is the per-query compute of a kernel that gathers
    each union tile once for both queries.  A masked slot gathers row 0 (an
    L2 hit) instead of the partner's key and the tiles after the query's last
    own slot are skipped, so the time is a lower bound for such a kernel.
    The baseline is each query over its own k1 keys; outputs must agree
    (masked slots carry zero weight).  Union sizes give the gather saving."""
    import numpy as np
    import torch
    from sparse_attention_11_b200 import dsa
    wl = prob.wl
    T = wl.total_q
    st = torch.cuda.current_stream()
    ws = dsa.workspace(dsa.dsa_workspace_size(dsa.DSA_OP_FORWARD, prob.seqs, 2 * k1, prob.ia, prob.aa))
    own = torch.full((T, k1), -1, dtype=torch.int32, device="cuda")
    dsa.dsa_select(prob.seqs, prob.ia, k1, own, ws)
    dsa.check_device_status(ws, "kv reuse: select")
    npair = T // 2
    idx_u, usize = pair_union_rows(own)

    def timed(idx, ksel):
        for _ in range(warmup):
            dsa.dsa_sparse_attn(prob.seqs, prob.aa, idx, ksel, ws)
        torch.cuda.synchronize()
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(steps)]
        for e in evs:
            e[0].record(st)
            dsa.dsa_sparse_attn(prob.seqs, prob.aa, idx, ksel, ws)
            e[1].record(st)
        torch.cuda.synchronize()
        dsa.check_device_status(ws, "kv reuse: attention")
        return statistics.mean(e[0].elapsed_time(e[1]) for e in evs)

    base_ms = timed(own, k1)
    out_base = prob.out.clone()
    lse_base = prob.lse.clone() if prob.lse is not None else None
    union_ms = timed(idx_u, 2 * k1)
    diff = float((prob.out.float() - out_base.float()).abs().max())
    ldiff = float((prob.lse - lse_base).abs().max()) if lse_base is not None else None
    del out_base, lse_base
    us = usize.float().cpu().numpy()
    n_own = int((own >= 0).sum())
    return {"k_per_query": k1, "pairs": npair, "union_keys_mean": float(us.mean()),
            "union_keys_p5_p95": [float(np.percentile(us, 5)), float(np.percentile(us, 95))],
            "attention_ms_own": base_ms, "attention_ms_union_masked": union_ms, "time_ratio": union_ms / base_ms,
            "gathered_rows_own": n_own, "gathered_rows_shared_tiles": int(usize.sum()) + (k1 if T % 2 else 0),
            "gather_saving": 1.0 - (int(usize.sum()) + (k1 if T % 2 else 0)) / n_own,
            "max_abs_diff_out": diff, "max_abs_diff_lse": ldiff,
            "note": "union tiles with a per-query mask on the shipped kernel: a lower bound of a shared-tile kernel's time"}


def context_parallel_emulated(prob, world, schemes, steps, warmup):
    """Context-parallel prefill with its ranks emulated in turn on this GPU.
    Each rank's chunks run against the whole key side, which is what the
    all-gather leaves in every rank's memory, and are timed with CUDA
    events.  The ranks never wait on one another, so max(rank time) is the
    compute time of a G-GPU run.  The all-gather is not timed here; its
    bytes are reported."""
    import torch
    from sparse_attention_11_b200 import context_parallel as cp
    wl = prob.wl
    L = wl.total_q
    st = torch.cuda.current_stream()
    res = {"emulated_world": world, "note": "ranks run one after another on one GPU; all-gather not timed"}
    for scheme in schemes:
        plans = cp.plan(L, world, scheme, k=wl.k)
        rank_ms = []
        for chunks in plans:
            rows = torch.cat([torch.arange(a, b) for a, b in chunks]).cuda()
            n = rows.numel()
            out = torch.empty((n, wl.heads, wl.dv), dtype=torch.bfloat16, device="cuda")
            lse = torch.empty((n, wl.heads), dtype=torch.float32, device="cuda")
            idx = torch.empty((n, wl.k), dtype=torch.int32, device="cuda")
            run = cp.LocalForward(chunks, wl.k, prob.q_idx[rows], prob.q_idx_scale[rows], prob.W, prob.k_idx,
                                  prob.k_idx_scale, prob.q[rows], prob.K, prob.V, wl.scale, out, lse, idx)
            for _ in range(warmup):
                run()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            torch.cuda.synchronize()
            e0.record(st)
            for _ in range(steps):
                run()
            e1.record(st)
            torch.cuda.synchronize()
            run.check("context-parallel (emulated)")
            rank_ms.append(e0.elapsed_time(e1) / steps)
            del run, out, lse, idx
        mx = max(rank_ms)
        res[scheme] = {"rank_ms": [round(x, 3) for x in rank_ms], "max_rank_ms": mx,
                       "imbalance": mx / statistics.mean(rank_ms), "tokens_per_s_at_max_rank": L / (mx / 1e3)}
    res["allgather_bytes_per_rank"] = int((L - L // world) * (128 + 4 + wl.dk * 2))
    return res


def context_parallel_native(args, ws_n, rank, dev, sampler):
    """Context-parallel prefill on ws_n GPUs: one sequence, query rows split
    by the plan, the key side all-gathered over NCCL every step, each rank's
    chunks through dsa_forward.  Strong scaling: value = L tokens per step /
    max-over-ranks device time."""
    import torch
    from sparse_attention_11_b200 import context_parallel as cp, workloads as W
    from sparse_attention_11_b200.problem import DeviceProblem
    wl = W.WORKLOADS[args.workload]
    L = wl.total_q
    if wl.batch != 1 or wl.idx_dtype != "e4m3" or not wl.v_in_k:
        raise SystemExit("--cp needs a single-sequence FP8 / MLA prefill workload")
    inp = W.generate(wl, device="cuda")
    full = DeviceProblem(inp, with_lse=False)
    plans = cp.plan(L, ws_n, args.cp_scheme, k=wl.k)
    mine = plans[rank]
    rows = torch.cat([torch.arange(a, b) for a, b in mine]).cuda()
    n = rows.numel()
    q_idx, q_sc, q = full.q_idx[rows], full.q_idx_scale[rows], full.q[rows]
    k_idx_sh, k_sc_sh, kv_sh = full.k_idx[rows], full.k_idx_scale[rows], full.K[rows]
    W_index = full.W
    del full, inp
    torch.cuda.empty_cache()
    out = torch.empty((n, wl.heads, wl.dv), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((n, wl.heads), dtype=torch.float32, device=dev)
    idx = torch.empty((n, wl.k), dtype=torch.int32, device=dev)
    st = torch.cuda.current_stream()
    run = cp.ContextParallelForward(plans, rank, wl.k, q_idx, q_sc, W_index, q, wl.dk, wl.dv, wl.scale, out, lse,
                                    idx, k_idx_sh.dtype, kv_sh.dtype)

    def step():
        run.step(k_idx_sh, k_sc_sh, kv_sh)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    run.check("context-parallel warm-up")
    barrier(ws_n)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    sampler.start()
    t0.record(st)
    for _ in range(args.steps):
        step()
    t1.record(st)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    barrier(ws_n)
    run.check("context-parallel timed steps")
    ms_max = max_over_ranks(t0.elapsed_time(t1), ws_n, dev)
    return {
        "metric": METRIC, "value": L * args.steps / (ms_max / 1e3), "unit": "tokens/s", "n_gpus": ws_n,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_max / args.steps, "higher_is_better": True,
        "scaling": "strong", "vs_baseline": None, "dtype": "bf16",
        "dtypes": {"indexer": "e4m3", "attention": "bf16", "accumulate": "f32"}, "data": "synthetic",
        "config": {"workload": wl.name, "batch": 1, "seq_len": L, "top_k": wl.k, "heads": wl.heads, "dk": wl.dk,
                   "dv": wl.dv, "v": "latent part of K", "l2": "inputs larger than L2 (no flush)",
                   "parallelism": f"context-parallel x{ws_n} ({args.cp_scheme})"},
        "allgather_bytes_per_rank": int((L - n) * (128 + 4 + wl.dk * 2)),
        "gpu_launches": 3 * len([c for c in mine if c[1] > c[0]]) * args.steps, "clocks": clocks,
    }


def backward_native(prob, steps, warmup, seed=23):
    """The sparse attention's backward over the forward's own selection,
    output and lse, with a seeded bf16 d_out; the MLA-tied gradient (d_V is
    d_K's first dv columns).  Device-timed per call; d_K is zeroed between
    calls outside the timed region."""
    import torch
    from sparse_attention_11_b200 import dsa
    wl = prob.wl
    T, H = wl.total_q, wl.heads
    gen = torch.Generator(device="cuda")
    gen.manual_seed(seed)
    d_out = torch.randn((T, H, wl.dv), generator=gen, device="cuda").to(torch.bfloat16)
    d_q = torch.empty((T, H, wl.dk), device="cuda")
    d_kv = torch.zeros((wl.total_k, wl.dk), device="cuda")
    ws = dsa.workspace(256)
    run = lambda: dsa.dsa_sparse_attn_bwd(prob.seqs, prob.aa, prob.idx, wl.k, d_out, d_q, d_kv, d_kv[:, :wl.dv], ws)
    for _ in range(warmup):
        d_kv.zero_()
        run()
    st = torch.cuda.current_stream()
    ts = []
    for _ in range(steps):
        d_kv.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(st)
        run()
        e1.record(st)
        torch.cuda.synchronize()
        ts.append(e0.elapsed_time(e1))
    dsa.check_device_status(ws, "backward")
    pos = np.concatenate([np.arange(sk - sq, sk) for sq, sk in zip(wl.seqlens_q, wl.seqlens_k)])
    flops = 2.0 * H * (3 * wl.dk + 2 * wl.dv) * float(np.minimum(wl.k, pos + 1).sum())
    ms = statistics.mean(ts)
    return {"kernel": "attn_bwd_kernel (CUDA cores, fp32)", "ms": ms, "steps": steps,
            "tflops": flops / (ms / 1e3) / 1e12, "flops_per_call": flops,
            "tokens_per_s": T / (ms / 1e3)}


def e2e_native(inp, prob, steps):
    """The same metric through the host-memory API, dsa_forward_host: every
    step copies its inputs from pinned host memory (the key-side tensors on the
    compute stream; the queries chunk by chunk inside the call, overlapped with
    the attention and with the output copies) and reads the attention output
    back into pinned host memory."""
    import torch
    from sparse_attention_11_b200 import dsa
    small = [prob.K, prob.q_idx, prob.k_idx, prob.W] + \
        [t for t in (prob.q_idx_scale, prob.k_idx_scale) if t is not None]
    if prob.V.data_ptr() != prob.K.data_ptr():
        small.append(prob.V)
    small_host = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in small]
    for h, d in zip(small_host, small):
        h.copy_(d)
    q_host = torch.empty(prob.q.shape, dtype=prob.q.dtype, pin_memory=True)
    q_host.copy_(prob.q)
    out_host = torch.empty(prob.out.shape, dtype=prob.out.dtype, pin_memory=True)
    h2d = sum(t.numel() * t.element_size() for t in small_host) + q_host.numel() * q_host.element_size()
    d2h = out_host.numel() * out_host.element_size()
    aa = dsa.attn_args(q_host, prob.K, prob.V, prob.wl.scale, out_host, prob.lse)
    ws = dsa.workspace(dsa.dsa_workspace_size(dsa.DSA_OP_FORWARD_HOST, prob.seqs, prob.wl.k, prob.ia, aa))
    h2d_stream, d2h_stream = torch.cuda.Stream(), torch.cuda.Stream()
    st = torch.cuda.current_stream()

    def step():
        for h, d in zip(small_host, small):
            d.copy_(h, non_blocking=True)
        dsa.dsa_forward_host(prob.seqs, prob.ia, aa, prob.wl.k, prob.idx, ws, h2d_stream, d2h_stream)

    step()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(st)
    for _ in range(steps):
        step()
    t1.record(st)
    torch.cuda.synchronize()
    dsa.check_device_status(ws, "e2e")
    if not torch.equal(out_host[:: max(1, out_host.shape[0] // 64)], prob.out[:: max(1, out_host.shape[0] // 64)].cpu()):
        raise RuntimeError("e2e: host output differs from the device-resident run")
    return t0.elapsed_time(t1) / steps, h2d, d2h


def cpu_baseline(inp, target_s, max_rows=4096):
    """The oracle, as it stands, on a stratified sample of query rows."""
    import oracle
    wl = inp.wl
    T = wl.total_q
    thr = oracle.num_threads()

    def rows_for(n):
        n = max(1, min(n, T))
        return np.unique(np.linspace(0, T - 1, n).round().astype(np.int64))

    def run(rows):
        kb, pos = inp.key_base_pos(rows)
        q = inp.q_rows(rows)
        qs = inp.q_idx_scale[rows] if inp.q_idx_scale is not None else None
        V = inp.K if inp.V is None else inp.V
        vs = wl.dk if inp.V is None else wl.dv
        t = time.perf_counter()
        oracle.forward_rows(inp.q_idx[rows], qs, inp.W, inp.k_idx, inp.k_idx_scale, kb, pos, wl.k, q,
                            inp.K.ravel(), wl.dk, V.ravel(), vs, wl.scale, wl.dv)
        return time.perf_counter() - t

    cal = rows_for(thr)
    t_cal = run(cal)
    n = int(min(max_rows, max(len(cal), len(cal) * target_s / max(t_cal, 1e-3))))
    rows = rows_for(n)
    t = run(rows)
    return {"value": len(rows) / t, "unit": "tokens/s", "cores": thr, "kind": "oracle",
            "sample": f"{len(rows)} query rows of {wl.name} evenly spaced over all positions "
                      f"(fold, scores, top-{wl.k}, attention per row), {t:.1f} s; tokens/s = rows/s",
            "seconds": t}


# ----------------------------------------------------------------------------- native arm
def native(args):
    import torch
    from sparse_attention_11_b200 import workloads as W
    ws_n, rank, local = dist_setup(args)
    dev = torch.device("cuda", torch.cuda.current_device())
    peaks = load_peaks()
    wl = W.WORKLOADS[args.workload]
    info = workload_info(wl)
    sampler = ClockSampler(torch.cuda.current_device())
    if args.cp:
        res = context_parallel_native(args, ws_n, rank, dev, sampler)
        if rank == 0:
            print(json.dumps(res), flush=True)
        if ws_n > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return
    inp, prob, ms, sel_ms, att_ms, clocks = run_native_workload(wl, args.steps, args.warmup, ws_n, rank, sampler)
    ms_max = max_over_ranks(ms, ws_n, dev)
    tokens_per_step = info["tokens"]
    value = ws_n * tokens_per_step * args.steps / (ms_max / 1e3)
    att_max = max_over_ranks(att_ms, ws_n, dev)
    flops = attn_flops(wl, info)
    achieved_tf = flops / (att_max / 1e3) / 1e12
    # the burst peak is the denominator: the bf16 matmul's sustained figure was
    # taken under the power cap at a lower clock than a bench run holds
    peak = peaks["bf16_tflops"]
    res = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": ws_n, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_max / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16",
        "dtypes": {"indexer": "e4m3", "attention": "bf16", "accumulate": "f32"},
        "data": "synthetic",
        "config": {"workload": wl.name, "batch": wl.batch, "seq_len": int(max(wl.seqlens_k)), "top_k": wl.k,
                   "heads": wl.heads, "dk": wl.dk, "dv": wl.dv, "v": "latent part of K" if wl.v_in_k else "own tensor",
                   "l2": "inputs larger than L2 (no flush)", "parallelism": f"replicas x{ws_n}"},
        "stages_ms": {"select": sel_ms, "attention": att_ms},
        "roofline": {"kernel": "attn_tc_kernel", "bound": "tensor", "achieved": achieved_tf,
                     "peak": peak, "unit": "TFLOP/s", "frac": achieved_tf / peak,
                     "peak_kind": f"bf16 {peaks['source']} burst", "flops_per_launch": flops,
                     "frac_of_sustained": achieved_tf / peaks["bf16_tflops_sustained"], "traffic": None},
        "gpu_launches": step_launches(wl) * args.steps,
        "clocks": clocks,
    }
    if wl.idx_dtype == "e4m3":
        fp8 = fp8_peak()
        res["stage_rooflines"] = {"indexer_topk": indexer_roofline(info, max_over_ranks(sel_ms, ws_n, dev), fp8)}
    tr = captured_traffic(wl.name, "attn_tc_kernel")
    if tr:
        res["roofline"]["traffic"] = tr["bytes_per_launch"]
        res["roofline"]["traffic_source"] = tr["source"]
    if not args.no_e2e:
        e2e_ms, h2d, d2h = e2e_native(inp, prob, max(1, min(args.steps, 5)))
        e2e_max = max_over_ranks(e2e_ms, ws_n, dev)
        res["e2e"] = {"value": ws_n * tokens_per_step / (e2e_max / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                      "d2h_bytes_per_step": d2h, "ms_per_step": e2e_max, "api": "dsa_forward_host"}
    # the backward runs on the fixed-k forward's selection, output and lse
    if args.bwd and wl.attn_dtype == "bf16":
        res["backward"] = backward_native(prob, max(1, min(args.steps, 3)), 1)
    # dynamic k last: it writes the problem's indices and output with another selection
    if not args.no_dynk and wl.name != "decode_b64":
        res["dynamic_k"] = dynamic_k_native(inp, prob, max(3, min(args.steps, 10)), args.warmup)
    if args.kv_reuse and wl.batch == 1 and wl.attn_dtype == "bf16":
        res["kv_reuse_prototype"] = kv_reuse_prototype(prob, max(3, min(args.steps, 10)), args.warmup)
    if not args.no_cp and ws_n == 1 and wl.batch == 1 and wl.idx_dtype == "e4m3":
        res["context_parallel"] = context_parallel_emulated(prob, 8, ("balanced", "zigzag", "contiguous"), 5, 2)
    if not args.no_decode and wl.name != "decode_b64":
        del prob
        torch.cuda.empty_cache()
        dwl = W.WORKLOADS["decode_b64"]
        dinfo = workload_info(dwl)
        dsteps = max(args.steps, 20)
        dinp, dprob, dms, dsel, datt, _ = run_native_workload(dwl, dsteps, args.warmup, ws_n, rank, None)
        dms_max = max_over_ranks(dms, ws_n, dev)
        datt_max = max_over_ranks(datt, ws_n, dev)
        byts = attn_bytes(dwl, dinfo)
        scan_bytes = dinfo["pairs"] * 132
        res["decode"] = {
            "workload": dwl.name, "value": ws_n * dinfo["tokens"] * dsteps / (dms_max / 1e3), "unit": "tokens/s",
            "ms_per_step": dms_max / dsteps, "steps": dsteps, "stages_ms": {"select": dsel, "attention": datt},
            "roofline": {"kernel": "attn_tc_kernel", "bound": "hbm", "achieved": byts / (datt_max / 1e3) / 1e9,
                         "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": byts / (datt_max / 1e3) / 1e9 / peaks["hbm_gbs"], "bytes_per_launch": byts},
            "select_hbm": {"bytes_scan": scan_bytes, "achieved_gbs": scan_bytes / (dsel / 1e3) / 1e9},
            "gpu_launches": 4 * dsteps,  # fold, scan, top-k, attention
        }
        if not args.no_e2e:
            e2e_ms, h2d, d2h = e2e_native(dinp, dprob, 5)
            res["decode"]["e2e"] = {"value": ws_n * dinfo["tokens"] / (max_over_ranks(e2e_ms, ws_n, dev) / 1e3),
                                    "unit": "tokens/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}
        del dprob
        torch.cuda.empty_cache()
        # the same decode step with V in a tensor of its own: every selected row gathers
        # K (576) and V (512) columns, 2176 bytes
        _, vprob, vms, vsel, vatt, _ = run_native_workload(dwl, dsteps, args.warmup, ws_n, rank, None,
                                                           v_separate=True, inp=dinp)
        vatt_max = max_over_ranks(vatt, ws_n, dev)
        vbytes = dinfo["sum_sel"] * (dwl.dk + dwl.dv) * 2 + dwl.total_q * dwl.heads * (dwl.dk + dwl.dv) * 2 + \
            dwl.total_q * dwl.heads * 4 + dwl.total_q * dwl.k * 4
        res["decode_v_separate"] = {
            "workload": dwl.name + " (V a separate tensor)", "ms_per_step": max_over_ranks(vms, ws_n, dev) / dsteps,
            "stages_ms": {"select": vsel, "attention": vatt},
            "roofline": {"kernel": "attn_tc_kernel", "bound": "hbm", "achieved": vbytes / (vatt_max / 1e3) / 1e9,
                         "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": vbytes / (vatt_max / 1e3) / 1e9 / peaks["hbm_gbs"], "bytes_per_launch": vbytes}}
        del vprob
    if rank == 0 and ws_n == 1 and not args.no_cpu_baseline:
        res["cpu_baseline"] = cpu_baseline(inp, args.cpu_seconds)
    if rank == 0:
        print(json.dumps(res), flush=True)
    if ws_n > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


# ----------------------------------------------------------------------------- reference arm
def reference(args):
    ws_n = int(os.environ.get("WORLD_SIZE", "1"))
    if int(os.environ.get("RANK", "0")) != 0:
        return
    from sparse_attention_11_b200 import workloads as W
    wl = W.WORKLOADS[args.workload]
    inp = W.generate(wl, device="cpu", q_on_device=False) if wl.attn_dtype == "f32" else None
    if inp is None:
        # the attention queries are drawn on the GPU; without one, draw them on the CPU generator
        import torch
        dev = "cuda" if torch.cuda.is_available() else "cpu"
        inp = W.generate(wl, device=dev)
    per_step_s = max(2.0, 60.0 / max(1, args.steps + args.warmup))
    for _ in range(args.warmup):
        cpu_baseline(inp, per_step_s / 4)
    vals, secs = [], []
    for _ in range(args.steps):
        r = cpu_baseline(inp, per_step_s)
        vals.append(r["value"])
        secs.append(r["seconds"])
    v = statistics.median(vals)
    res = {"impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": ws_n, "steps": args.steps,
           "warmup": args.warmup, "ms_per_step": 1e3 * statistics.mean(secs), "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
           "config": {"workload": wl.name, "batch": wl.batch, "seq_len": int(max(wl.seqlens_k)), "top_k": wl.k,
                      "heads": wl.heads, "dk": wl.dk, "dv": wl.dv},
           "cpu_baseline": {"kind": "oracle", "cores": r["cores"], "sample": r["sample"], "value": v},
           "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(res), flush=True)


def profile_case(args):
    """Lean cases for profiler captures: the device holds only what the
    captured kernels read and write (a few GB at most)."""
    import torch
    from sparse_attention_11_b200 import dsa, workloads as W
    from sparse_attention_11_b200.problem import DeviceProblem
    if args.profile_case == "select":
        wl = W.WORKLOADS[args.workload]
        s = wl.seed
        cu_q = np.concatenate([[0], np.cumsum(wl.seqlens_q)]).astype(np.int64)
        cu_k = np.concatenate([[0], np.cumsum(wl.seqlens_k)]).astype(np.int64)
        qf = W.bf16_bits_to_f32(W.to_bf16_bits(W._sub_rng(s, "q_idx").standard_normal((wl.total_q, 128),
                                                                                        dtype=np.float32)))
        kf = W.bf16_bits_to_f32(W.to_bf16_bits(W._indexer_keys(W._sub_rng(s, "k_idx"), wl.total_k)))
        q_idx, q_sc = W.quantize_e4m3_rows(qf)
        k_idx, k_sc = W.quantize_e4m3_rows(kf)
        Wf = W._sub_rng(s, "W_index").standard_normal((128, 128), dtype=np.float32) / np.float32(math.sqrt(128.0))
        Wb = torch.from_numpy(W.to_bf16_bits(Wf).view(np.int16)).view(torch.bfloat16).cuda()
        seqs = dsa.Seqs(cu_q, cu_k, device=torch.device("cuda"))
        ia = dsa.indexer_args(torch.from_numpy(q_idx).cuda(), torch.from_numpy(q_sc).cuda(), Wb,
                              torch.from_numpy(k_idx).cuda(), torch.from_numpy(k_sc).cuda())
        ws = dsa.workspace(dsa.dsa_workspace_size(dsa.DSA_OP_FORWARD, seqs, wl.k, ia))
        idx = torch.empty((wl.total_q, wl.k), dtype=torch.int32, device="cuda")
        for _ in range(args.reps):
            dsa.dsa_select(seqs, ia, wl.k, idx, ws)
        torch.cuda.synchronize()
        dsa.check_device_status(ws, "profile case select")
    else:
        if args.profile_case == "decode":
            wl = W.WORKLOADS["decode_b64"]
        else:
            rng = np.random.default_rng(0)
            ctx = tuple(int(x) for x in rng.integers(16384, 24577, size=64))
            wl = W.custom("decode_b64_ctx16k_24k", (1,) * 64, ctx, base="decode_b64")
        prob = DeviceProblem(W.generate(wl, device="cuda"))
        for _ in range(args.reps):
            dsa.dsa_select(prob.seqs, prob.ia, wl.k, prob.idx, prob.ws)
            dsa.dsa_sparse_attn(prob.seqs, prob.aa, prob.idx, wl.k, prob.ws)
        torch.cuda.synchronize()
        prob.check("profile case decode-small")
    print("profile case done:", args.profile_case, wl.name, flush=True)


def main():
    args = parse()
    if args.profile_case:
        profile_case(args)
        return
    if args.probe_fp8_peak:
        print(json.dumps(fp8_peak(burst_reps=10, sustained_s=4.0)), flush=True)
        return
    if args.impl == "reference":
        reference(args)
    else:
        native(args)


if __name__ == "__main__":
    main()
