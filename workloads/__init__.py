"""Seeded synthetic inputs for paged MLA decode (shared by tests and bench).

This module only draws random numbers and lays them out; it holds none of the
attention arithmetic, so both the CPU oracle and the CUDA path can be fed from
it without sharing any of the method's code.

Every tensor is generated on the CPU with ``torch.Generator`` (seed fixed per
workload) so the oracle and the GPU see the same bytes.  The five named
workloads follow the shapes of the pages' use case (DeepSeek decode: one latent
KV head, 576-wide cache rows, 64-token pages, h_q up to 128, BF16/FP16):

=============== ===== ==== ==== ======================== ======= ========== ======
name            batch s_q  h_q  cached tokens L          dtype   value std  causal
=============== ===== ==== ==== ======================== ======= ========== ======
tiny              1    1    16  256                      bf16    1.0        no
memory-bound     64    1    16  4096 each                bf16    1.0        no
compute-bound   128    1   128  4096 each                bf16    1.0        no
varlen-mtp      132    2   128  uniform int in [1,16384] bf16    1.0        yes
long-fp16        16    2    64  32768 + uniform [-2048,2048] fp16 0.5       yes
=============== ===== ==== ==== ======================== ======= ========== ======

``memory-bound-fp8`` / ``compute-bound-fp8`` are ``memory-bound`` / ``compute-bound`` with an
e5m2 cache (one byte per value).  An e5m2
cache is drawn as raw codes (no rounding of any number happens here): sign and 2-bit mantissa
uniform, exponent field uniform in [10, 16] (magnitudes 2^-5 .. 3.5, a spread like the 16-bit
caches' N(0, 1)); its poison is code 0x71 (10240).

Page pools: ``tiny`` has its 4 pages plus 4 unreferenced pages filled with 1e4;
``memory-bound`` uses exactly 4096 pages with ``randperm(4096)`` as its table;
``compute-bound`` 8192 pages in random order; the two variable-length workloads
use a shared pool of sum(ceil(L/64)) pages in random order, table slots past a
request's last page are -1, and the slots past L in a request's last page are
filled with 1e4 (they must never be read).  softmax_scale = 576 ** -0.5.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Dict, List, Optional, Sequence

import torch

D_K = 576
PAGE = 64
POISON = 1.0e4


@dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    s_q: int
    h_q: int
    dtype: torch.dtype
    std: float
    causal: bool
    seed: int
    seqlen_kind: str  # "fixed", "uniform", "around"
    seqlen_a: int
    seqlen_b: int = 0
    pool_kind: str = "exact"  # "exact" | "shared"
    extra_poison_pages: int = 0
    description: str = ""
    kv_fp8: bool = False  # cache of e5m2 codes (uint8) instead of ``dtype``

    @property
    def rows(self) -> int:
        return self.s_q * self.h_q


WORKLOADS: Dict[str, Workload] = {
    w.name: w
    for w in [
        Workload("tiny", 1, 1, 16, torch.bfloat16, 1.0, False, 1000, "fixed", 256,
                 extra_poison_pages=4,
                 description="batch 1, s_q 1, h_q 16, seqlen 256, bf16"),
        Workload("memory-bound", 64, 1, 16, torch.bfloat16, 1.0, False, 1001, "fixed", 4096,
                 description="batch 64, s_q 1, h_q 16, seqlen 4096, bf16"),
        Workload("memory-bound-fp8", 64, 1, 16, torch.bfloat16, 1.0, False, 1005, "fixed", 4096,
                 description="batch 64, s_q 1, h_q 16, seqlen 4096, bf16 q, e5m2 cache", kv_fp8=True),
        Workload("compute-bound-fp8", 128, 1, 128, torch.bfloat16, 1.0, False, 1006, "fixed", 4096,
                 description="batch 128, s_q 1, h_q 128, seqlen 4096, bf16 q, e5m2 cache", kv_fp8=True),
        Workload("compute-bound", 128, 1, 128, torch.bfloat16, 1.0, False, 1002, "fixed", 4096,
                 description="batch 128, s_q 1, h_q 128, seqlen 4096, bf16"),
        Workload("varlen-mtp", 132, 2, 128, torch.bfloat16, 1.0, True, 1003, "uniform", 1, 16384,
                 pool_kind="shared",
                 description="batch 132, s_q 2 causal, h_q 128, seqlen U[1,16384], bf16"),
        Workload("long-fp16", 16, 2, 64, torch.float16, 0.5, True, 1004, "around", 32768, 2048,
                 pool_kind="shared",
                 description="batch 16, s_q 2 causal, h_q 64, seqlen 32768+U[-2048,2048], fp16"),
    ]
}


@dataclass
class Inputs:
    q: torch.Tensor  # [b, s_q, h_q, 576]
    kcache: torch.Tensor  # [pages, 64, 1, 576]
    block_table: torch.Tensor  # [b, width] int32
    cache_seqlens: torch.Tensor  # [b] int32
    softmax_scale: float
    causal: bool
    meta: dict = field(default_factory=dict)

    @property
    def batch(self) -> int:
        return self.q.shape[0]

    @property
    def s_q(self) -> int:
        return self.q.shape[1]

    @property
    def h_q(self) -> int:
        return self.q.shape[2]


def _randn(g: torch.Generator, shape: Sequence[int], std: float, dtype: torch.dtype) -> torch.Tensor:
    """N(0, std^2) values drawn in fp32 then rounded to ``dtype``, in slabs to bound memory."""
    shape = tuple(int(s) for s in shape)
    out = torch.empty(shape, dtype=dtype)
    flat = out.view(shape[0], -1)
    step = max(1, (1 << 24) // max(1, flat.shape[1]))
    for i in range(0, shape[0], step):
        j = min(shape[0], i + step)
        slab = torch.randn((j - i, flat.shape[1]), generator=g, dtype=torch.float32)
        if std != 1.0:
            slab.mul_(std)
        flat[i:j] = slab.to(dtype)
    return out


E5M2_POISON_CODE = 0x71  # 1.25 * 2^13 = 10240


def _rand_e5m2_codes(g: torch.Generator, shape: Sequence[int]) -> torch.Tensor:
    """uint8 e5m2 codes: random sign and mantissa, exponent field in [10, 16], drawn in slabs."""
    shape = tuple(int(s) for s in shape)
    out = torch.empty(shape, dtype=torch.uint8)
    flat = out.view(shape[0], -1)
    step = max(1, (1 << 24) // max(1, flat.shape[1]))
    for i in range(0, shape[0], step):
        j = min(shape[0], i + step)
        n = (j - i, flat.shape[1])
        sign = torch.randint(0, 2, n, generator=g, dtype=torch.int32)
        expo = torch.randint(10, 17, n, generator=g, dtype=torch.int32)
        mant = torch.randint(0, 4, n, generator=g, dtype=torch.int32)
        flat[i:j] = ((sign << 7) | (expo << 2) | mant).to(torch.uint8)
    return out


def make_case(
    batch: int,
    s_q: int,
    h_q: int,
    seqlens: Sequence[int],
    *,
    dtype: torch.dtype = torch.bfloat16,
    std: float = 1.0,
    causal: bool = False,
    seed: int = 0,
    extra_poison_pages: int = 0,
    table_pad: int = 0,
    poison_tail: bool = True,
    softmax_scale: Optional[float] = None,
    kv_fp8: bool = False,
) -> Inputs:
    """Build one seeded paged-cache case with the given per-request lengths.

    Pages are drawn for every request (ceil(L/64) each), the pool is shuffled
    with ``randperm`` and ``extra_poison_pages`` unreferenced pages filled with
    1e4 are mixed in.  ``table_pad`` extra -1 columns are appended to the table.
    ``kv_fp8``: the cache is uint8 e5m2 codes (poison code 0x71 = 10240).
    """
    g = torch.Generator().manual_seed(int(seed))
    seqlens = [int(x) for x in seqlens]
    assert len(seqlens) == batch
    n_pages = [-(-L // PAGE) for L in seqlens]
    used = sum(n_pages)
    pool = used + int(extra_poison_pages)
    width = max([1] + n_pages) + int(table_pad)
    q = _randn(g, (batch, s_q, h_q, D_K), std, dtype)
    if kv_fp8:
        kcache = _rand_e5m2_codes(g, (max(pool, 1), PAGE, 1, D_K))
        poison = torch.tensor(E5M2_POISON_CODE, dtype=torch.uint8)
    else:
        kcache = _randn(g, (max(pool, 1), PAGE, 1, D_K), std, dtype)
        poison = torch.tensor(POISON, dtype=dtype)
    perm = torch.randperm(max(pool, 1), generator=g)
    table = torch.full((batch, width), -1, dtype=torch.int32)
    pos = 0
    for r, n in enumerate(n_pages):
        table[r, :n] = perm[pos:pos + n].to(torch.int32)
        pos += n
    # unreferenced pages of the pool are poison
    if pool > used:
        kcache[perm[used:pool]] = poison
    # slots past L in a request's last page are poison too
    if poison_tail:
        for r, L in enumerate(seqlens):
            if L % PAGE:
                kcache[int(table[r, n_pages[r] - 1]), L % PAGE:] = poison
    scale = D_K ** -0.5 if softmax_scale is None else float(softmax_scale)
    return Inputs(q, kcache, table, torch.tensor(seqlens, dtype=torch.int32), scale, causal,
                  meta={"seed": seed, "pool_pages": pool, "used_pages": used})


def draw_seqlens(w: Workload, g: torch.Generator) -> List[int]:
    if w.seqlen_kind == "fixed":
        return [w.seqlen_a] * w.batch
    if w.seqlen_kind == "uniform":
        return torch.randint(w.seqlen_a, w.seqlen_b + 1, (w.batch,), generator=g).tolist()
    if w.seqlen_kind == "around":
        d = torch.randint(-w.seqlen_b, w.seqlen_b + 1, (w.batch,), generator=g)
        return (w.seqlen_a + d).tolist()
    raise ValueError(w.seqlen_kind)


def make_workload(name: str) -> Inputs:
    """Inputs of one named workload (deterministic for its seed)."""
    w = WORKLOADS[name]
    g = torch.Generator().manual_seed(w.seed)
    seqlens = draw_seqlens(w, g)
    if name in ("memory-bound", "memory-bound-fp8"):
        # exactly the 4096-page pool, table = randperm(4096) viewed as [64, 64]
        q = _randn(g, (w.batch, w.s_q, w.h_q, D_K), w.std, w.dtype)
        if w.kv_fp8:
            kcache = _rand_e5m2_codes(g, (4096, PAGE, 1, D_K))
        else:
            kcache = _randn(g, (4096, PAGE, 1, D_K), w.std, w.dtype)
        table = torch.randperm(4096, generator=g).to(torch.int32).view(64, 64).contiguous()
        return Inputs(q, kcache, table, torch.tensor(seqlens, dtype=torch.int32), D_K ** -0.5, w.causal,
                      meta={"seed": w.seed, "pool_pages": 4096, "used_pages": 4096})
    return make_case(w.batch, w.s_q, w.h_q, seqlens, dtype=w.dtype, std=w.std, causal=w.causal,
                     seed=w.seed + 7919, extra_poison_pages=w.extra_poison_pages, kv_fp8=w.kv_fp8)


def algorithmic_cost(seqlens: Sequence[int], s_q: int, h_q: int, elem_bytes: int = 2,
                     kv_elem_bytes: Optional[int] = None) -> Dict[str, float]:
    """FLOPs and bytes of one decode call by the pages' cost model.

    FLOPs = 2 * h_q * s_q * (576 + 512) * sum(L); bytes = 576 * kv_elem * sum(L)
    (each cached row read once, V being part of it) + q + out + lse (elem bytes each;
    kv_elem defaults to elem, 1 for an e5m2 cache).
    """
    kv_elem = elem_bytes if kv_elem_bytes is None else kv_elem_bytes
    tot = float(sum(int(x) for x in seqlens))
    b = len(seqlens)
    rows = s_q * h_q
    flops = 2.0 * rows * (576 + 512) * tot
    kv_bytes = 576.0 * kv_elem * tot
    io_bytes = b * rows * (576 * elem_bytes + 512 * elem_bytes + 4)
    return {"flops": flops, "kv_bytes": kv_bytes, "bytes": kv_bytes + io_bytes, "tokens": tot}


def seqlens_of(name: str) -> List[int]:
    w = WORKLOADS[name]
    g = torch.Generator().manual_seed(w.seed)
    return draw_seqlens(w, g)


__all__ = ["WORKLOADS", "Workload", "Inputs", "make_case", "make_workload", "algorithmic_cost",
           "seqlens_of", "POISON", "E5M2_POISON_CODE", "PAGE", "D_K"]
