"""Device-side set-up of the synthetic workloads (no method arithmetic).

Moves synth arrays (bf16 bit patterns) to the GPU as torch.bfloat16 tensors
and prepares decode caches, calling only the library for any computation.
"""
from __future__ import annotations

import numpy as np
import torch

from . import infv2, synth


def to_dev(a: np.ndarray, device="cuda") -> torch.Tensor:
    """uint16 bf16 bit patterns -> torch.bfloat16 tensor on the device."""
    t = torch.from_numpy(np.ascontiguousarray(a).view(np.int16))
    return t.to(device).view(torch.bfloat16)


def to_host_bits(t: torch.Tensor) -> np.ndarray:
    """torch.bfloat16 tensor -> uint16 numpy bit patterns."""
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def fill_kc1_cache(p, k_cache: torch.Tensor, kc1_cache: torch.Tensor, lens, stream=None):
    """Compress each (sequence, kv head) cache row range [0, L) into kc1_cache
    with the library's stage-1 kernel ([L, 1, d] views, one head at a time)."""
    p1 = infv2.params(1, 1, k=max(p.n_init + p.n_local, 1), n_init=p.n_init, n_local=p.n_local)
    batch, h_kv = k_cache.shape[0], k_cache.shape[1]
    for s in range(batch):
        L = int(lens[s])
        for g in range(h_kv):
            if L >= p.l_c1:
                src = k_cache[s, g, :L].unsqueeze(1)
                dst = kc1_cache[s, g, :infv2.num_kernels(p, L)].unsqueeze(1)
                infv2.infv2_compress_k(p1, src, dst, stream=stream)


class DecodeState:
    """KV caches, K^C1 cache, lengths and workspace of one batched decode."""

    def __init__(self, shape: synth.Shape, data: dict, device="cuda"):
        self.p = infv2.params_of(shape)
        self.cap = data["cap"]
        self.k_cache = to_dev(data["k_cache"], device)
        self.v_cache = to_dev(data["v_cache"], device)
        batch, h_kv = self.k_cache.shape[:2]
        self.batch = batch
        cap_c1 = infv2.num_kernels(self.p, self.cap)
        self.kc1_cache = torch.zeros((batch, h_kv, max(cap_c1, 1), shape.d), dtype=torch.bfloat16,
                                     device=device)
        self.lens0 = data["lens"].copy()
        fill_kc1_cache(self.p, self.k_cache, self.kc1_cache, self.lens0)
        self.seqlens = torch.from_numpy(self.lens0.astype(np.int32)).to(device)
        ws = infv2.infv2_decode_workspace_size(self.p, batch, self.cap)
        self.workspace = torch.empty(max(ws, 256), dtype=torch.uint8, device=device)
        self.q = to_dev(data["q"], device)          # [steps, batch, h_q, d]
        self.k_new = to_dev(data["k_new"], device)  # [steps, batch, h_kv, d]
        self.v_new = to_dev(data["v_new"], device)

    def step(self, t: int, o=None, lse=None, idx_out=None, stream=None):
        return infv2.infv2_decode(self.p, self.q[t], self.k_new[t], self.v_new[t], self.k_cache,
                                  self.v_cache, self.kc1_cache, self.seqlens, self.workspace,
                                  idx_out=idx_out, o=o, lse=lse, stream=stream)
