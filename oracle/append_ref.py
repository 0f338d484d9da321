"""CPU oracle of the KV append that precedes a decode step -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg
may import this module.  It shares nothing with the CUDA path.

What is computed ("FlashMLA: 高性能GPU注意力机制计算库", section 项目主要功能: the
latent KV cache is paged, 64 tokens per block, addressed through a block
table; "FlashAttention终极指南": ``cache_seqlens`` holds the number of cached
tokens of each request):

* request b's cache_seqlens entry L counts the s_q tokens being appended, so
  they are its last s_q cache positions: new token s (0-based) is position
  j = L - s_q + s;
* position j lives in page ``block_table[b, j // 64]`` at slot ``j % 64``;
* the token's whole 576-wide latent row is stored there unchanged (the row is
  the key; its first 512 values are the value), nothing else in the cache
  changes.

Reading taken where the pages are silent: a request with L < s_q has no
position for its first s_q - L new tokens; those rows are dropped (the CUDA
path also flags them in its error word).

The copy is exact (no arithmetic), so the result keeps the cache's dtype.
"""

from __future__ import annotations

from typing import Tuple

import torch

from oracle.mla_ref import mla_decode_ref

PAGE = 64


def append_kv_ref(kcache: torch.Tensor, block_table: torch.Tensor, cache_seqlens: torch.Tensor,
                  kv_new: torch.Tensor) -> torch.Tensor:
    """A copy of ``kcache`` [pages, 64, 1, 576] with ``kv_new`` [b, s_q, 576] written in.

    One row per (request, new token), in plain loops.
    """
    out = kcache.clone()
    b, s_q, _ = kv_new.shape
    for r in range(b):
        L = int(cache_seqlens[r])
        for s in range(s_q):
            j = L - s_q + s  # cache position of new token s
            if j < 0:
                continue
            page = int(block_table[r, j // PAGE])
            slot = j % PAGE
            out[page, slot, 0, :] = kv_new[r, s, :]
    return out


def decode_with_append_ref(q: torch.Tensor, kv_new: torch.Tensor, kcache: torch.Tensor,
                           block_table: torch.Tensor, cache_seqlens: torch.Tensor, softmax_scale: float,
                           causal: bool) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """Append, then the plain fp64 decode of ``mla_ref``: (appended cache, out, lse)."""
    appended = append_kv_ref(kcache, block_table, cache_seqlens, kv_new)
    out, lse = mla_decode_ref(q, appended, block_table, cache_seqlens, softmax_scale, causal)
    return appended, out, lse
