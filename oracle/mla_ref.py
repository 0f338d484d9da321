"""fp64 CPU oracle of paged MLA decode attention -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg
may import this module.  It shares nothing with the CUDA path.

What is computed (the plain definition, which the split-KV / online-softmax
kernel reaches up to rounding order):

* "FlashMLA 在 Hopper GPU 上的 MHA 内核调度优化解析", section
  计算边界特性与优化方向抉择: one latent KV head; every cached token is a row of
  d_k = 576 values that serves as the key, and its first d_v = 512 values serve
  as the value (the FLOP count 2*h_q*s_q*s_k*(d_k+d_v) and byte count 2*s_k*d_k
  both say the 576-wide row is read once and used for both products).
* "FlashMLA: 高性能GPU注意力机制计算库" (hanhandi.cn doc-0479), section
  项目主要功能: the cache is paged in blocks of 64 tokens, BF16 or FP16.
* same page, section 4. Softmax数值稳定性优化: the maximum is subtracted before
  exponentiating (here: an explicit first pass for the row max, a second pass
  for the exponentials and their sum -- not an online softmax).
* "FlashMLA 在 Hopper GPU 上的 MHA 内核调度优化解析", section 跷跷板调度的数学重构:
  any rescaled/online accumulation order must be mathematically identical to
  the standard softmax accumulation -- which is why the oracle is the plain
  definition.
* "DeepSeek开源FlashMLA全解析", section 2.1 item 4 (结果融合) and the same
  hotdry page's section 辅助优化：可编程依赖启动与瓦片调度 (splitkv_mla +
  combine kernels): chunk outputs are merged with weights derived from their
  log-sum-exp -- ``mla_partial_ref`` / ``merge_partials_ref``.
* "FlashAttention终极指南" (cnnetsun.cn): ``cache_seqlens`` holds the number of
  cached tokens per request, ``causal`` masks future tokens, and the
  log-sum-exp of the scaled scores is returned beside the output.

Readings taken where the pages are silent:

* lse is the natural log of sum_j exp(scale * q.k_j) (scaled-score units).
* causal with s_q > 1 is aligned bottom-right: query position s (0-based) of
  s_q sees keys j <= L - s_q + s.
* a row that sees no key has out = 0 and lse = -inf.
* slots of the last page at or beyond L are never read.
* ``softmax_scale`` multiplies q.k (the workloads use 576**-0.5).

Layouts (all row-major, as the C-ABI):
  q            [b, s_q, h_q, 576]
  kcache       [num_pages, 64, 1, 576]
  block_table  [b, >= ceil(L_b/64)] int
  cache_seqlens[b] int
  out          [b, s_q, h_q, 512]
  lse          [b, h_q, s_q]       (note: heads before query positions)
"""

from __future__ import annotations

import math
from typing import Iterable, List, Optional, Sequence, Tuple

import torch

D_K = 576
D_V = 512
PAGE = 64

_F64 = torch.float64


def visible_key_count(seqlen: int, s_q: int, s: int, causal: bool) -> int:
    """Number of keys that query position ``s`` (0-based, of ``s_q``) attends to.

    Non-causal: all ``seqlen`` cached keys.  Causal: bottom-right alignment,
    keys 0 .. seqlen - s_q + s inclusive, never negative.
    """
    if not causal:
        return int(seqlen)
    return max(0, int(seqlen) - (s_q - 1 - s))


def gather_keys(kcache: torch.Tensor, block_table_row: torch.Tensor, seqlen: int) -> torch.Tensor:
    """Token rows 0..seqlen-1 of one request, as fp64 [seqlen, 576].

    Token j lives in page ``block_table_row[j // 64]`` at slot ``j % 64``.
    Written as the per-token definition (one index pair per token), so a reader
    can check it by eye; the fancy index gathers exactly those rows.
    """
    seqlen = int(seqlen)
    if seqlen == 0:
        return torch.zeros(0, D_K, dtype=_F64)
    tok = torch.arange(seqlen)
    page_of_tok = block_table_row.to(torch.int64)[tok // PAGE]
    slot_of_tok = tok % PAGE
    rows = kcache[page_of_tok, slot_of_tok, 0, :]
    return rows.to(_F64)


def _softmax_rows(z: torch.Tensor, v: torch.Tensor) -> Tuple[torch.Tensor, torch.Tensor]:
    """Two-pass softmax of score rows z [n_rows, n_keys] applied to v [n_keys, 512].

    Pass 1: m = row max.  Pass 2: w = exp(z - m), Z = sum w.
    Returns (out = w @ v / Z, lse = m + ln Z).  n_keys must be > 0.
    """
    m = z.max(dim=1).values
    w = torch.exp(z - m[:, None])
    zsum = w.sum(dim=1)
    out = (w @ v) / zsum[:, None]
    lse = m + torch.log(zsum)
    return out, lse


def mla_decode_ref(
    q: torch.Tensor,
    kcache: torch.Tensor,
    block_table: torch.Tensor,
    cache_seqlens: torch.Tensor,
    softmax_scale: float,
    causal: bool,
    requests: Optional[Sequence[int]] = None,
) -> Tuple[torch.Tensor, torch.Tensor]:
    """fp64 reference of paged MLA decode.

    Returns ``(out, lse)`` with ``out`` [n, s_q, h_q, 512] and ``lse``
    [n, h_q, s_q] in fp64, where n = len(requests) (default: all b requests,
    in order).  Inputs may be bf16/fp16/fp32/fp64 CPU tensors; every value is
    converted exactly to fp64 before any arithmetic.
    """
    b, s_q, h_q, dk = q.shape
    if dk != D_K:
        raise ValueError(f"q last dim must be {D_K}, got {dk}")
    if tuple(kcache.shape[1:]) != (PAGE, 1, D_K):
        raise ValueError(f"kcache must be [pages, {PAGE}, 1, {D_K}], got {tuple(kcache.shape)}")
    reqs = list(range(b)) if requests is None else [int(r) for r in requests]
    out = torch.zeros(len(reqs), s_q, h_q, D_V, dtype=_F64)
    lse = torch.full((len(reqs), h_q, s_q), -math.inf, dtype=_F64)
    scale = float(softmax_scale)
    for i, r in enumerate(reqs):
        seqlen = int(cache_seqlens[r])
        keys = gather_keys(kcache, block_table[r], seqlen)  # [L, 576]
        vals = keys[:, :D_V]  # V is the first 512 columns of the same rows
        qr = q[r].to(_F64)  # [s_q, h_q, 576]
        for s in range(s_q):
            n_vis = visible_key_count(seqlen, s_q, s, causal)
            if n_vis == 0:
                continue  # out stays 0, lse stays -inf
            z = scale * (qr[s] @ keys[:n_vis].T)  # [h_q, n_vis]
            o, l = _softmax_rows(z, vals[:n_vis])
            out[i, s] = o
            lse[i, :, s] = l
    return out, lse


def mla_partial_ref(
    q: torch.Tensor,
    kcache: torch.Tensor,
    block_table: torch.Tensor,
    cache_seqlens: torch.Tensor,
    softmax_scale: float,
    causal: bool,
    request: int,
    key_begin: int,
    key_end: int,
) -> Tuple[torch.Tensor, torch.Tensor]:
    """Chunk result of one request over keys [key_begin, key_end) only.

    This is one split of the split-KV rewrite: the normalised output of the
    chunk o_c [s_q, h_q, 512] and its log-sum-exp lse_c [h_q, s_q], with the
    same visibility rule as ``mla_decode_ref``.  A row with no visible key in
    the chunk has o_c = 0 and lse_c = -inf (weight zero in the merge).
    """
    b, s_q, h_q, _ = q.shape
    seqlen = int(cache_seqlens[request])
    keys = gather_keys(kcache, block_table[request], seqlen)
    vals = keys[:, :D_V]
    qr = q[request].to(_F64)
    o = torch.zeros(s_q, h_q, D_V, dtype=_F64)
    lse = torch.full((h_q, s_q), -math.inf, dtype=_F64)
    for s in range(s_q):
        hi = min(int(key_end), visible_key_count(seqlen, s_q, s, causal))
        lo = int(key_begin)
        if hi <= lo:
            continue
        z = float(softmax_scale) * (qr[s] @ keys[lo:hi].T)
        oc, lc = _softmax_rows(z, vals[lo:hi])
        o[s] = oc
        lse[:, s] = lc
    return o, lse


def merge_partials_ref(
    partials: Iterable[Tuple[torch.Tensor, torch.Tensor]]
) -> Tuple[torch.Tensor, torch.Tensor]:
    """Merge chunk results (o_c, lse_c) of one request into (out, lse).

    lse = ln sum_c exp(lse_c)   (computed around the max for stability)
    out = sum_c exp(lse_c - lse) * o_c
    Rows where every chunk has lse_c = -inf get out = 0, lse = -inf.
    o_c: [s_q, h_q, 512], lse_c: [h_q, s_q].
    """
    parts: List[Tuple[torch.Tensor, torch.Tensor]] = list(partials)
    if not parts:
        raise ValueError("merge of zero chunks")
    lses = torch.stack([p[1].to(_F64) for p in parts])  # [C, h_q, s_q]
    outs = torch.stack([p[0].to(_F64) for p in parts])  # [C, s_q, h_q, 512]
    m = lses.max(dim=0).values  # [h_q, s_q]
    finite = torch.isfinite(m)
    m_safe = torch.where(finite, m, torch.zeros_like(m))
    wsum = torch.exp(lses - m_safe[None]).sum(dim=0)
    lse = torch.where(finite, m_safe + torch.log(wsum), torch.full_like(m, -math.inf))
    lse_safe = torch.where(finite, lse, torch.zeros_like(lse))
    weights = torch.exp(lses - lse_safe[None])  # [C, h_q, s_q]; -inf rows -> 0
    weights = torch.where(finite[None], weights, torch.zeros_like(weights))
    out = (weights.permute(0, 2, 1)[..., None] * outs).sum(dim=0)  # [s_q, h_q, 512]
    return out, lse
