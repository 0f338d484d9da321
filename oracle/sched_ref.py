"""CPU re-derivation of the tile scheduler -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg
may import this module.  It is written from the pages, independently of the
device scheduler, in plain Python integers.

Sources:
* "FlashMLA: 高性能GPU注意力机制计算库" (hanhandi.cn doc-0479), section
  6. SM资源调度优化: the per-partition share is
  ceil_div(total_num_blocks, num_sm_parts) + fixed_overhead_num_blocks; the
  partitions split the work of all sequences roughly equally, which may cut a
  sequence into several pieces; each piece costs a fixed overhead.
* "FlashMLA 在 Hopper GPU 上的 MHA 内核调度优化解析", section
  辅助优化：可编程依赖启动与瓦片调度: the tile scheduler hands requests and
  blocks to the SMs so variable-length batches stay balanced.
* same walk-through, section 项目主要功能: a block is one 64-token page.

Readings (the pages give the formula, not the walk; listed in the design doc):
* n_r = ceil(L_r / 64) blocks per request; a request with n_r = 0 has no chunk.
* total = sum over requests with n_r > 0 of (n_r + F); F = 5.
* quota = ceil(total / P) + F for P partitions (total = 0: every part empty).
* The walk visits requests in order.  Partition p starts with budget = quota.
  At request r with k blocks already assigned, need = (n_r - k) + F.
  If need <= budget, or p is the last partition, the rest of r joins p
  (budget -= need) and the walk moves to r + 1.  Otherwise p takes
  t = budget - F blocks of r when t > 0 (a split) and closes; when t <= 0 it
  closes without taking anything.  (The "last partition takes the rest" clause
  is a safety net: with the +F in the quota no input tried has needed it.)
* Output, per partition, 8 int32: begin_req, begin_blk, end_req, end_blk,
  begin_split, 0, 0, 0.  The part owns every block (r, k), k < n_r, with
  (begin_req, begin_blk) <= (r, k) < (end_req, end_blk) in lexicographic order;
  begin_split is the chunk index, within request begin_req, of the part's first
  chunk.  num_splits[0] = 0 and num_splits[r + 1] = num_splits[r] + (number of
  chunks of request r).
"""

from __future__ import annotations

from typing import List, Sequence, Tuple

PAGE_BLOCK = 64
FIXED_OVERHEAD_BLOCKS = 5
META_INTS = 8


def _ceil_div(a: int, b: int) -> int:
    return -(-a // b)


def tile_schedule_ref(
    seqlens: Sequence[int], num_parts: int, fixed_overhead: int = FIXED_OVERHEAD_BLOCKS
) -> Tuple[List[List[int]], List[int]]:
    """Return (meta [num_parts][8], num_splits [b + 1]) for the given lengths."""
    if num_parts < 1:
        raise ValueError("num_parts must be >= 1")
    b = len(seqlens)
    n_blk = [_ceil_div(int(L), PAGE_BLOCK) for L in seqlens]
    if any(int(L) < 0 for L in seqlens):
        raise ValueError("negative sequence length")
    F = int(fixed_overhead)
    total = sum(n + F for n in n_blk if n > 0)
    quota = _ceil_div(total, num_parts) + F if total > 0 else 0

    meta: List[List[int]] = []
    num_splits = [0] * (b + 1)
    chunks_so_far = 0
    r, k, split = 0, 0, 0
    for p in range(num_parts):
        begin = (r, k, split)
        budget = quota
        last = p == num_parts - 1
        while r < b:
            if n_blk[r] == 0:
                num_splits[r + 1] = chunks_so_far
                r += 1
                continue
            need = (n_blk[r] - k) + F
            if need <= budget or last:
                budget -= need
                chunks_so_far += split + 1
                num_splits[r + 1] = chunks_so_far
                r, k, split = r + 1, 0, 0
            else:
                t = budget - F
                if t > 0:
                    k += t
                    split += 1
                break
        meta.append([begin[0], begin[1], r, k, begin[2], 0, 0, 0])
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
