"""The paged KV cache as the library's entry points take it: four device
tensors in the layout of the C ABI (``sa_kv_cache``).

  * k, v       : bf16 ``[num_pages][Hkv][P][d]`` -- one (page, kv head) tile is
    contiguous (``P*d*2`` bytes);
  * page_table : int32 ``[B][max_pages_per_seq]`` (logical page -> physical page);
  * seq_lens   : int32 ``[B]``.
"""
from __future__ import annotations

import dataclasses

import torch


@dataclasses.dataclass
class PagedCache:
    k: torch.Tensor            # bf16 [num_pages][Hkv][P][d]
    v: torch.Tensor            # bf16 [num_pages][Hkv][P][d]
    page_table: torch.Tensor   # int32 [B][max_pages]
    seq_lens: torch.Tensor     # int32 [B]

    @property
    def batch(self) -> int:
        return int(self.page_table.shape[0])

    @property
    def num_kv_heads(self) -> int:
        return int(self.k.shape[1])

    @property
    def page_size(self) -> int:
        return int(self.k.shape[2])

    @property
    def head_dim(self) -> int:
        return int(self.k.shape[3])

    @property
    def max_pages(self) -> int:
        return int(self.page_table.shape[1])

    @property
    def num_pages(self) -> int:
        return int(self.k.shape[0])

    def with_v(self, v: torch.Tensor) -> "PagedCache":
        return PagedCache(self.k, v, self.page_table, self.seq_lens)

    def to(self, device) -> "PagedCache":
        return PagedCache(self.k.to(device), self.v.to(device),
                          self.page_table.to(device), self.seq_lens.to(device))
