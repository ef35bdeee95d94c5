"""Paged KV-cache storage for the decode megakernel (torch device memory).

Layout per layer (bf16): ``[num_pages, n_kv_heads, page_size, head_dim]``, so
one KV head's page is one contiguous block that a single bulk copy moves.
Sequence b's position p lives in physical page ``block_table[b, p // page]``
at slot ``p % page``.  Pages are handed to sequences in a caller-chosen order
(a seeded permutation by default, so paging is exercised).
"""

from __future__ import annotations

from typing import List, Optional, Sequence

import torch

from .mk import KVCacheView


class PagedKVCache:
    def __init__(self, cfg: dict, max_batch: int, max_tokens: Sequence[int], page: int = 16,
                 device="cuda", page_order: Optional[torch.Tensor] = None):
        """``max_tokens[b]``: positions sequence b may ever use (its pages are
        mapped up front)."""
        self.cfg, self.page, self.device = cfg, page, device
        L, Hkv, d = cfg["n_layers"], cfg["n_kv_heads"], cfg["head_dim"]
        need = [(int(n) + page - 1) // page for n in max_tokens]
        self.max_pages_per_seq = max(1, max(need))
        self.num_pages = max(1, sum(need))
        order = (torch.arange(self.num_pages) if page_order is None
                 else page_order[: self.num_pages])
        bt = torch.full((max_batch, self.max_pages_per_seq), -1, dtype=torch.int32)
        k = 0
        for b, n in enumerate(need):
            bt[b, :n] = order[k:k + n].to(torch.int32)
            k += n
        self.block_table_cpu = bt
        self.block_table = bt.to(device)
        shape = (self.num_pages, Hkv, page, d)
        self.k = [torch.zeros(shape, dtype=torch.bfloat16, device=device) for _ in range(L)]
        self.v = [torch.zeros(shape, dtype=torch.bfloat16, device=device) for _ in range(L)]
        self.view = KVCacheView(self.k, self.v, self.block_table)

    def load_history(self, hist: List[dict], lengths: Sequence[int]):
        """Scatter a contiguous history (synth.make_kv_history) into the pages."""
        P = self.page
        for l, hl in enumerate(hist):
            for b, n in enumerate(lengths):
                if n == 0:
                    continue
                pos = torch.arange(n)
                phys = self.block_table_cpu[b, pos // P].long().to(self.device)
                slot = (pos % P).to(self.device)
                kb = hl["k"][b, :, :n].to(self.device).permute(1, 0, 2)   # [n, Hkv, d]
                vb = hl["v"][b, :, :n].to(self.device).permute(1, 0, 2)
                self.k[l][phys, :, slot] = kb
                self.v[l][phys, :, slot] = vb

    def token(self, l: int, b: int, p: int):
        """K and V [Hkv, d] stored for sequence b at position p."""
        ph = int(self.block_table_cpu[b, p // self.page])
        s = p % self.page
        return self.k[l][ph, :, s], self.v[l][ph, :, s]
