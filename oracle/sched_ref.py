"""CPU re-derivation of the tile scheduler -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg
may import this module.  It is written from the pages, independently of the
device scheduler, in plain Python integers, one 64-token block at a time.

Sources:
* "FlashMLA: 高性能GPU注意力机制计算库" (hanhandi.cn doc-0479), section
  6. SM资源调度优化: each of num_sm_parts partitions gets
  ceil_div(total_num_blocks, num_sm_parts) blocks plus fixed_overhead_num_blocks
  to compensate the fixed cost of a piece of work; a sequence may be cut
  between partitions; the goal is equal work per SM for variable lengths.
* "FlashMLA 在 Hopper GPU 上的 MHA 内核调度优化解析", section
  辅助优化：可编程依赖启动与瓦片调度: the tile scheduler hands requests and
  blocks to the SMs so variable-length batches stay balanced.
* same walk-through, section 项目主要功能: a block is one 64-token page.

Reading taken here (the pages give the share formula, not the assignment):
* n_r = ceil(L_r / 64) blocks per request; F = 3 units of fixed overhead per
  request that has blocks.  The pages name fixed_overhead_num_blocks without a
  value; F is a tuning constant of the scheduler (every F gives a valid
  schedule with the bounds below), set to the value the device library uses.  Requests are laid end to end on a line of units:
  request r occupies F overhead units followed by its n_r block units, so its
  block k sits at unit x = cum_r + F + k, where cum_r is the sum of (F + n_t)
  over the non-empty requests t < r.  total = sum over non-empty requests of
  (F + n_r).
* share S = ceil(total / P); partition p owns the units [p*S, (p+1)*S), so
  block (r, k) belongs to partition (cum_r + F + k) // S.
* A partition's chunks are its maximal runs of blocks of one request.  Its real
  work is its blocks plus F per chunk; at most its first chunk has its overhead
  units outside the partition, so the work is at most S + F = the pages'
  ceil_div(total, P) + fixed_overhead, and (for all but the last partition) at
  least S - F.
* Output, per partition, 8 int32: begin_req, begin_blk, end_req, end_blk,
  begin_split, 0, 0, 0.  The partition owns every block (r, k), k < n_r, with
  (begin_req, begin_blk) <= (r, k) < (end_req, end_blk) lexicographically;
  (end_req, end_blk) is the next partition's begin, and the last partition ends
  at (b, 0).  A partition boundary at unit x lies at (r, max(0, x - cum_r - F))
  for the last request r with cum_r <= x, or at (b, 0) when x >= total.
  begin_split is the index, among the chunks of begin_req, of the partition's
  first chunk when it continues a request (begin_blk > 0), else 0.
  num_splits[0] = 0 and num_splits[r + 1] = num_splits[r] + (chunks of r).
"""

from __future__ import annotations

from typing import Dict, List, Sequence, Tuple

PAGE_BLOCK = 64
FIXED_OVERHEAD_BLOCKS = 3
META_INTS = 8


def _ceil_div(a: int, b: int) -> int:
    return -(-a // b)


def block_owners(seqlens: Sequence[int], num_parts: int, fixed_overhead: int = FIXED_OVERHEAD_BLOCKS):
    """Partition of every block, by walking the unit line block by block.

    Returns (owner, n_blk, share) with owner[(r, k)] = partition of block k of request r.
    """
    if num_parts < 1:
        raise ValueError("num_parts must be >= 1")
    if any(int(L) < 0 for L in seqlens):
        raise ValueError("negative sequence length")
    F = int(fixed_overhead)
    n_blk = [_ceil_div(int(L), PAGE_BLOCK) for L in seqlens]
    total = sum(F + n for n in n_blk if n > 0)
    share = _ceil_div(total, num_parts) if total > 0 else 0
    owner: Dict[Tuple[int, int], int] = {}
    x = 0  # next unit on the line
    for r, n in enumerate(n_blk):
        if n == 0:
            continue
        x += F  # the request's overhead units
        for k in range(n):
            owner[(r, k)] = x // share
            x += 1
    return owner, n_blk, share


def tile_schedule_ref(
    seqlens: Sequence[int], num_parts: int, fixed_overhead: int = FIXED_OVERHEAD_BLOCKS
) -> Tuple[List[List[int]], List[int]]:
    """Return (meta [num_parts][8], num_splits [b + 1]) for the given lengths."""
    owner, n_blk, _ = block_owners(seqlens, num_parts, fixed_overhead)
    b = len(seqlens)
    # chunks: maximal runs of (request, partition), in order
    chunks: List[Tuple[int, int, int, int, int]] = []  # (part, req, lo, hi, split index)
    per_req: Dict[int, int] = {}
    for r in range(b):
        k = 0
        while k < n_blk[r]:
            part = owner[(r, k)]
            lo = k
            while k < n_blk[r] and owner[(r, k)] == part:
                k += 1
            chunks.append((part, r, lo, k, per_req.get(r, 0)))
            per_req[r] = per_req.get(r, 0) + 1
    num_splits = [0] * (b + 1)
    for r in range(b):
        num_splits[r + 1] = num_splits[r] + per_req.get(r, 0)
    # each partition begins where the blocks before it end: at its first block, or, when it has
    # none, at the first block of a later partition (or (b, 0))
    first_of_part: Dict[int, Tuple[int, int, int]] = {}
    for part, r, lo, hi, si in chunks:
        if part not in first_of_part:
            first_of_part[part] = (r, lo, si if lo > 0 else 0)
    begins: List[Tuple[int, int, int]] = [(b, 0, 0)] * (num_parts + 1)
    nxt = (b, 0, 0)
    for p in range(num_parts - 1, -1, -1):
        if p in first_of_part:
            nxt = first_of_part[p]
        begins[p] = nxt
    meta = []
    for p in range(num_parts):
        br, bk, bs = begins[p]
        er, ek, _ = begins[p + 1]
        meta.append([br, bk, er, ek, bs, 0, 0, 0])
    return meta, num_splits


def chunks_of_part(meta_row: Sequence[int], seqlens: Sequence[int]) -> List[Tuple[int, int, int, int]]:
    """Expand one partition's range into chunks (request, blk_begin, blk_end, split_idx)."""
    br, bk, er, ek, bs = (int(x) for x in meta_row[:5])
    out = []
    r = br
    while r < len(seqlens) and (r < er or (r == er and ek > 0)):
        n = _ceil_div(int(seqlens[r]), PAGE_BLOCK)
        lo = bk if r == br else 0
        hi = ek if r == er else n
        if hi > lo:
            out.append((r, lo, hi, bs if r == br else 0))
        r += 1
    return out
