"""Seeded synthetic workloads for the DSA forward path.

This module only draws inputs.  It holds none of the method's arithmetic (no
fold, score, selection or attention); both the CUDA path and the CPU oracle
consume exactly the bytes produced here.

Recipe (shapes follow the workloads the DSA pages discuss; the values are
synthetic stand-ins for model activations, since no weights or datasets are
involved):

* tiny_l512: batch 1, L=512.  Indexer q, k fp32 N(0,1) [512,128];
  W_index fp32 N(0,1/128); k=64; attention q fp32 N(0,1) [512,4,64],
  K and V separate fp32 N(0,1) [512,64]; scale 1/8.
* prefill_l{8192,32768,131072}: batch 1.  Indexer q: bf16 N(0,1) [L,128].
  Indexer k: bf16 of z + c_m for planted keys (probability 1/16, cluster
  m ~ U{0..15}, centres c_j = 3 g_j, g_j ~ N(0,I_128)), z ~ N(0,I_128)
  otherwise.  Both are stored as OCP e4m3 codes with a per-token fp32 scale
  amax/448.  W_index bf16 N(0,1/128).  MLA latent KV cache bf16 N(0,1)
  [L,576] (512 latent + 64 rope); V is the latent part, K[:, :512].
  Attention q bf16 N(0,1) [L,128,576] drawn on the GPU (torch Philox).
  k=2048, scale 1/sqrt(576).
* decode_b64: 64 sequences, context lengths U{16384..65536}, one query per
  sequence at the last position; key-side tensors as in prefill, packed by
  cu_seqlens_k.

Every tensor has its own sub-seed derived from (seed, tensor name).
"""
import math
import zlib
from dataclasses import dataclass, field

import numpy as np
import torch


@dataclass(frozen=True)
class Workload:
    name: str
    seqlens_q: tuple
    seqlens_k: tuple
    idx_dtype: str      # "f32" | "e4m3"
    w_dtype: str        # "f32" | "bf16"
    k: int
    heads: int
    dk: int
    dv: int
    attn_dtype: str     # "f32" | "bf16"
    scale: float
    seed: int = 0
    v_in_k: bool = True  # V = K[:, :dv] (MLA latent) instead of its own tensor

    @property
    def batch(self):
        return len(self.seqlens_q)

    @property
    def total_q(self):
        return int(sum(self.seqlens_q))

    @property
    def total_k(self):
        return int(sum(self.seqlens_k))


def _sub_rng(seed, name):
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, zlib.crc32(name.encode())])))


def _sub_seed(seed, name):
    return int(np.random.SeedSequence([seed, zlib.crc32(name.encode())]).generate_state(1)[0])


def _decode_lengths(seed, b=64, lo=16384, hi=65536):
    return tuple(int(x) for x in _sub_rng(seed, "ctx_lengths").integers(lo, hi + 1, size=b))


def _prefill(name, L, k=2048, seed=0):
    return Workload(name, (L,), (L,), "e4m3", "bf16", k, 128, 576, 512, "bf16", 1.0 / math.sqrt(576), seed, True)


WORKLOADS = {
    "tiny_l512": Workload("tiny_l512", (512,), (512,), "f32", "f32", 64, 4, 64, 64, "f32", 1.0 / 8.0, 0, False),
    "prefill_l8192": _prefill("prefill_l8192", 8192),
    "prefill_l32768": _prefill("prefill_l32768", 32768),
    "decode_b64": Workload("decode_b64", (1,) * 64, _decode_lengths(0), "e4m3", "bf16", 2048, 128, 576, 512,
                           "bf16", 1.0 / math.sqrt(576), 0, True),
    "prefill_l131072": _prefill("prefill_l131072", 131072),
}


def custom(name, seqlens_q, seqlens_k, base="prefill_l8192", **kw):
    """A workload with the dtypes/dims of `base` and other sequence lengths."""
    b = WORKLOADS[base]
    d = dict(b.__dict__)
    d.update(name=name, seqlens_q=tuple(seqlens_q), seqlens_k=tuple(seqlens_k))
    d.update(kw)
    return Workload(**d)


def to_bf16_bits(x):
    """float array -> uint16 bf16 bit patterns (round to nearest even, via torch)."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def bf16_bits_to_f32(b):
    return (b.astype(np.uint32) << 16).view(np.float32)


def quantize_e4m3_rows(x):
    """Per-row absmax/448 fp32 scale and e4m3 codes (uint8), via torch's
    float8_e4m3fn cast after clamping to the finite range."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    amax = np.abs(x).max(axis=1)
    scale = np.where(amax > 0, amax / np.float32(448.0), np.float32(1.0)).astype(np.float32)
    y = torch.from_numpy(x / scale[:, None]).clamp_(-448.0, 448.0)
    codes = y.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    return codes, scale


@dataclass
class Inputs:
    wl: Workload
    cu_q: np.ndarray
    cu_k: np.ndarray
    q_idx: np.ndarray            # f32 [Tq,128] or uint8 e4m3 codes
    q_idx_scale: np.ndarray      # f32 [Tq] or None
    W: np.ndarray                # f32 or uint16 bf16 bits [128,128]
    k_idx: np.ndarray            # f32 [Tk,128] or uint8
    k_idx_scale: np.ndarray      # f32 [Tk] or None
    K: np.ndarray                # f32 [Tk,dk] or uint16 [Tk,dk]
    V: np.ndarray                # None when V is K[:, :dv]
    q_host: np.ndarray = None    # [Tq,H,dk] when drawn on the host
    q_dev: "torch.Tensor" = None  # when drawn on the GPU
    extra: dict = field(default_factory=dict)

    def key_base_pos(self, rows):
        """Packed row of each query's first key, and each query's position:
        queries are the last seqlen_q positions of their sequence."""
        rows = np.asarray(rows, dtype=np.int64)
        b = np.searchsorted(self.cu_q, rows, side="right") - 1
        sq = self.cu_q[b + 1] - self.cu_q[b]
        sk = self.cu_k[b + 1] - self.cu_k[b]
        pos = (sk - sq) + (rows - self.cu_q[b])
        return self.cu_k[b], pos

    def q_rows(self, rows):
        rows = np.asarray(rows, dtype=np.int64)
        if self.q_host is not None:
            return self.q_host[rows]
        t = self.q_dev[torch.from_numpy(rows).to(self.q_dev.device)].cpu()
        if t.dtype == torch.bfloat16:
            return t.view(torch.int16).numpy().view(np.uint16)
        return t.numpy()


def _indexer_keys(rng, n):
    z = rng.standard_normal((n, 128), dtype=np.float32)
    centres = np.float32(3.0) * rng.standard_normal((16, 128), dtype=np.float32)
    planted = rng.random(n) < 1.0 / 16.0
    member = rng.integers(0, 16, size=n)
    z[planted] += centres[member[planted]]
    return z


def generate(wl, device=None, q_on_device=None):
    """Draw every input of `wl`.  Large attention queries are drawn on
    `device` (default: on the GPU when the workload is not tiny)."""
    s = wl.seed
    cu_q = np.concatenate([[0], np.cumsum(wl.seqlens_q)]).astype(np.int64)
    cu_k = np.concatenate([[0], np.cumsum(wl.seqlens_k)]).astype(np.int64)
    Tq, Tk = wl.total_q, wl.total_k
    if wl.idx_dtype == "f32":
        q_idx = _sub_rng(s, "q_idx").standard_normal((Tq, 128), dtype=np.float32)
        k_idx = _sub_rng(s, "k_idx").standard_normal((Tk, 128), dtype=np.float32)
        q_sc = k_sc = None
    else:
        qf = bf16_bits_to_f32(to_bf16_bits(_sub_rng(s, "q_idx").standard_normal((Tq, 128), dtype=np.float32)))
        kf = bf16_bits_to_f32(to_bf16_bits(_indexer_keys(_sub_rng(s, "k_idx"), Tk)))
        q_idx, q_sc = quantize_e4m3_rows(qf)
        k_idx, k_sc = quantize_e4m3_rows(kf)
    Wf = _sub_rng(s, "W_index").standard_normal((128, 128), dtype=np.float32) / np.float32(math.sqrt(128.0))
    W = Wf if wl.w_dtype == "f32" else to_bf16_bits(Wf)
    rk = _sub_rng(s, "kv")
    if wl.attn_dtype == "f32":
        K = rk.standard_normal((Tk, wl.dk), dtype=np.float32)
        V = None if wl.v_in_k else _sub_rng(s, "v").standard_normal((Tk, wl.dv), dtype=np.float32)
    else:
        K = to_bf16_bits(rk.standard_normal((Tk, wl.dk), dtype=np.float32))
        V = None if wl.v_in_k else to_bf16_bits(_sub_rng(s, "v").standard_normal((Tk, wl.dv), dtype=np.float32))
    inp = Inputs(wl, cu_q, cu_k, q_idx, q_sc, W, k_idx, k_sc, K, V)
    if q_on_device is None:
        q_on_device = wl.attn_dtype == "bf16"
    if q_on_device:
        dev = torch.device(device if device is not None else "cuda")
        g = torch.Generator(device=dev)
        g.manual_seed(_sub_seed(s, "q"))
        dt = torch.bfloat16 if wl.attn_dtype == "bf16" else torch.float32
        inp.q_dev = torch.randn((Tq, wl.heads, wl.dk), generator=g, device=dev, dtype=dt)
    else:
        if wl.attn_dtype == "f32":
            inp.q_host = _sub_rng(s, "q").standard_normal((Tq, wl.heads, wl.dk), dtype=np.float32)
        else:
            inp.q_host = to_bf16_bits(_sub_rng(s, "q").standard_normal((Tq, wl.heads, wl.dk), dtype=np.float32))
    return inp
