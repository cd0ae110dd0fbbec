"""Device-side placement of a generated workload for the C entry points.

Uploads the tensors drawn by `workloads.generate` and builds the argument
structs of include/dsa.h.  Marshalling only: no step of the path runs here.
"""
import numpy as np
import torch

from . import dsa


def _bf16(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)


class DeviceProblem:
    def __init__(self, inp, device="cuda", with_lse=True, v_separate=None):
        wl = inp.wl
        self.inp, self.wl = inp, wl
        dev = torch.device(device)
        self.seqs = dsa.Seqs(inp.cu_q, inp.cu_k, device=dev)
        if wl.idx_dtype == "f32":
            self.q_idx = torch.from_numpy(inp.q_idx).to(dev)
            self.k_idx = torch.from_numpy(inp.k_idx).to(dev)
            self.q_idx_scale = self.k_idx_scale = None
            self.W = torch.from_numpy(inp.W).to(dev)
        else:
            self.q_idx = torch.from_numpy(inp.q_idx).to(dev)
            self.k_idx = torch.from_numpy(inp.k_idx).to(dev)
            self.q_idx_scale = torch.from_numpy(inp.q_idx_scale).to(dev)
            self.k_idx_scale = torch.from_numpy(inp.k_idx_scale).to(dev)
            self.W = _bf16(inp.W).to(dev)
        if wl.attn_dtype == "f32":
            self.K = torch.from_numpy(inp.K).to(dev)
            self.V = self.K[:, : wl.dv] if inp.V is None else torch.from_numpy(inp.V).to(dev)
            dt = torch.float32
        else:
            self.K = _bf16(inp.K).to(dev)
            self.V = self.K[:, : wl.dv] if inp.V is None else _bf16(inp.V).to(dev)
            dt = torch.bfloat16
        if v_separate and inp.V is None:  # same values, own tensor
            self.V = self.V.contiguous()
        if inp.q_dev is not None:
            self.q = inp.q_dev
        else:
            self.q = torch.from_numpy(inp.q_host.view(np.int16)).view(torch.bfloat16).to(dev) \
                if wl.attn_dtype == "bf16" else torch.from_numpy(inp.q_host).to(dev)
        T = wl.total_q
        self.out = torch.empty((T, wl.heads, wl.dv), dtype=dt, device=dev)
        self.lse = torch.empty((T, wl.heads), dtype=torch.float32, device=dev) if with_lse else None
        self.idx = torch.empty((T, wl.k), dtype=torch.int32, device=dev)
        self.ia = dsa.indexer_args(self.q_idx, self.q_idx_scale, self.W, self.k_idx, self.k_idx_scale)
        self.aa = dsa.attn_args(self.q, self.K, self.V, wl.scale, self.out, self.lse)
        self.ws = dsa.workspace(dsa.dsa_workspace_size(dsa.DSA_OP_FORWARD, self.seqs, wl.k, self.ia, self.aa), dev)

    def forward(self, idx_out=True):
        dsa.dsa_forward(self.seqs, self.ia, self.aa, self.wl.k, self.idx if idx_out else None, self.ws)

    def check(self, where="dsa"):
        dsa.check_device_status(self.ws, where)
