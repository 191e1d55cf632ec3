"""Upload synthetic workloads to device memory as torch tensors.

Plumbing only: it copies the generator's bf16 bit patterns into device
tensors and allocates output buffers.  It imports neither the CUDA library nor
the oracle.
"""
from __future__ import annotations

import numpy as np
import torch

from . import DecodeWorkload, PrefillWorkload


def bf16_tensor(u16: np.ndarray, device="cuda") -> torch.Tensor:
    """uint16 bf16 bit patterns -> torch.bfloat16 tensor (bit-exact)."""
    a = np.ascontiguousarray(u16).view(np.int16)
    return torch.from_numpy(a).to(device).view(torch.bfloat16)


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """torch.bfloat16 tensor -> uint16 bit patterns on the host."""
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


class DecodeBuffers:
    """Device tensors of one decode workload plus output buffers.

    `layers` > 1 makes independent copies of the K/V/stats pools (distinct
    addresses, same contents) so that consecutive steps can rotate through
    more bytes than the L2 cache holds.
    """

    def __init__(self, w: DecodeWorkload, device="cuda", pad: int = 0, layers: int = 1):
        self.w = w
        self.device = device
        kh, vh = w.make_pools(pad)
        k0 = bf16_tensor(kh, device)
        v0 = bf16_tensor(vh, device)
        del kh, vh
        self.k_pools = [k0] + [k0.clone() for _ in range(layers - 1)]
        self.v_pools = [v0] + [v0.clone() for _ in range(layers - 1)]
        self.q = bf16_tensor(w.q, device)
        self.block_table = torch.from_numpy(np.ascontiguousarray(w.block_table)).to(device)
        self.ctx_lens = torch.from_numpy(np.ascontiguousarray(w.ctx_lens, dtype=np.int32)).to(device)
        self.head_kind = torch.from_numpy(np.ascontiguousarray(w.head_kind)).to(device)
        g = w.N_P // w.N_L
        self.stats = [torch.zeros((w.num_pool_pages, w.H_kv, g, 2, w.D), dtype=torch.bfloat16,
                                  device=device) for _ in range(layers)]
        self.sel = [torch.full((w.B, w.H_kv, w.top_k), -7, dtype=torch.int32, device=device)
                    for _ in range(layers)]
        self.sel_count = [torch.full((w.B, w.H_kv), -7, dtype=torch.int32, device=device)
                          for _ in range(layers)]
        self.scores = torch.full((w.B, w.H_kv, w.max_pages), float("nan"), dtype=torch.float32,
                                 device=device)
        self.out = torch.empty((w.B, w.H_q, w.D), dtype=torch.bfloat16, device=device)
        self.lse = torch.empty((w.B, w.H_q), dtype=torch.float32, device=device)

    @property
    def k_pool(self):
        return self.k_pools[0]

    @property
    def v_pool(self):
        return self.v_pools[0]


class PrefillBuffers:
    def __init__(self, w: PrefillWorkload, device="cuda"):
        self.w = w
        self.q = bf16_tensor(w.q(), device)
        self.k = bf16_tensor(w.k(), device)
        self.v = bf16_tensor(w.v(), device)
        self.out = torch.empty((w.T, w.H_q, w.D), dtype=torch.bfloat16, device=device)
        self.lse = torch.empty((w.H_q, w.T), dtype=torch.float32, device=device)
