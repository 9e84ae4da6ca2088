"""Device-memory holder for one attention layer's paged cache (PyTorch plumbing).

Allocates the buffers include/resa.h describes as torch CUDA tensors and
builds the C structs; all computation goes through block_sparse_long_resa_b200.resa.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch

from . import resa


@dataclass
class LayerCache:
    k: torch.Tensor            # [num_pages][Hkv][b][d] bf16
    v: torch.Tensor
    desc: torch.Tensor         # [num_pages][Hkv][2][d] bf16
    page_table: torch.Tensor   # [B][max_pages] int32
    seq_len: torch.Tensor      # [B] int32 (tokens incl. the decode token)

    @classmethod
    def from_problem(cls, p, device) -> "LayerCache":
        dev = torch.device(device)
        k = p.k_cache.to(dev)
        return cls(k=k, v=p.v_cache.to(dev),
                   desc=torch.zeros(p.num_pages, p.num_kv_heads, 2, p.head_dim,
                                    dtype=torch.bfloat16, device=dev),
                   page_table=p.page_table.to(dev), seq_len=p.ctx_len.to(dev).clone())

    def struct(self, seq_len=None, rows=None) -> resa.resa_cache_t:
        """The C struct; ``rows`` (int32 device tensor) restricts a call to
        those rows of the page table, in that order."""
        return resa.make_cache(self.k, self.v, self.desc, self.page_table,
                               self.seq_len if seq_len is None else seq_len, rows)

    @property
    def batch(self) -> int:
        return int(self.page_table.shape[0])

    @property
    def max_pages(self) -> int:
        return int(self.page_table.shape[1])


def workspace(cfg: resa.resa_config_t, batch: int, max_pages: int, max_chunk: int, device,
              stream=None) -> torch.Tensor:
    """Allocate and zero a workspace tensor for the given sizes."""
    n = resa.resa_workspace_size(cfg, batch, max_pages, max_chunk)
    ws = torch.empty(n, dtype=torch.uint8, device=device)
    resa.resa_workspace_init(ws, stream)
    return ws
