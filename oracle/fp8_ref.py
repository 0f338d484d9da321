"""CPU oracle of the FP8 (e5m2) latent-cache variant -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg
may import this module.  It shares nothing with the CUDA path.

What is computed:

* "云上AI推理新突破：FlashMLA赋能DeepSeek-V2-Lite提速16%", section 3. 动态精度缩放:
  the query and the keys are cast to float8_e5m2 and Q.K^T is formed from those
  8-bit operands; the softmax and the value-weighted sum are done back at FP16
  precision, with V cast to fp16.
* "DeepSeek开源FlashMLA全解析", section 1.2 计算模式创新: the same mixed
  pipeline (quantise q and k to fp8, multiply, then softmax and P.V).
* Everything else -- the paged 576-wide latent row that is both the key and
  (first 512 values) the value, the block table, lengths, causal rule, lse --
  is the 16-bit decode of ``oracle.mla_ref``, which this module calls on the
  dequantised operands.

Readings taken where the pages are silent or loose:

* The cache itself holds e5m2 bytes (one byte per value): storing the keys in
  the format they are multiplied in halves the bytes a decode step reads, and
  the same bytes serve as V (widened to fp16, which is exact: every finite
  e5m2 value is an fp16 value).
* e5m2 is the 8-bit binary format with 1 sign bit, 5 exponent bits (bias 15)
  and 2 mantissa bits, with subnormals (exponent field 0: m/4 * 2^-14); the
  exponent field 31 holds +-inf (mantissa 0) and NaN.
* Casting to e5m2 rounds to the nearest value, ties to the even mantissa;
  finite values beyond the largest finite e5m2 value, 57344, become +-57344
  (saturating); NaN stays NaN.  The pages name no overflow rule; the
  workloads never come near it.
* The query is quantised from its bf16/fp16 values; the scores are
  scale * (Qq . Kq^T) and are not rounded again: the page's cast of the
  scores to fp16 before the softmax is read as "the softmax runs at no less
  than fp16 precision" (the CUDA path keeps them in fp32; this oracle in
  fp64).
* P.V: the exact e5m2 values of V, weights in fp64 here (the CUDA path rounds
  P to fp16, the precision the page names).

Parity status: pinned by ``tests/fp8_pins.py`` (the 256 codes against a
hand-worked table and torch's own float8_e5m2 type, rounding against torch's
cast, ties to even, saturation, idempotence, the error bound, a hand-worked
two-key decode, and the reduction to ``mla_decode_ref`` when the query is
already on the e5m2 grid) and by planted mistakes in
``tests/test_oracle_mutants.py``.
"""

from __future__ import annotations

import math
from typing import Optional, Sequence, Tuple

import torch

from oracle.append_ref import append_kv_ref
from oracle.mla_ref import mla_decode_ref

_F64 = torch.float64

E5M2_BIAS = 15
E5M2_MANT_BITS = 2
E5M2_MAX = 57344.0  # (1 + 3/4) * 2^15, code 0x7B
E5M2_MIN_NORMAL_EXP = 1 - E5M2_BIAS  # -14
E5M2_SUBNORMAL_STEP = 2.0 ** (E5M2_MIN_NORMAL_EXP - E5M2_MANT_BITS)  # 2^-16


def e5m2_value(code: int) -> float:
    """Value of one e5m2 code (0..255), from the field definition."""
    code = int(code) & 0xFF
    sign = -1.0 if code >> 7 else 1.0
    e = (code >> 2) & 0x1F
    m = code & 0x3
    if e == 0x1F:
        return sign * math.inf if m == 0 else math.nan
    if e == 0:
        return sign * (m / 4.0) * 2.0 ** E5M2_MIN_NORMAL_EXP
    return sign * (1.0 + m / 4.0) * 2.0 ** (e - E5M2_BIAS)


# value of every code, indexed by the code
E5M2_TABLE = torch.tensor([e5m2_value(c) for c in range(256)], dtype=_F64)


def e5m2_decode(codes: torch.Tensor) -> torch.Tensor:
    """fp64 values of a uint8 tensor of e5m2 codes (table look-up, any shape)."""
    return E5M2_TABLE[codes.to(torch.int64)]


def e5m2_quantize(x: torch.Tensor) -> torch.Tensor:
    """x rounded to the e5m2 grid (nearest, ties to even; saturating), as fp64.

    For a finite nonzero |x| with binade exponent E = floor(log2 |x|), the
    e5m2 values in [2^E, 2^(E+1)) are spaced 2^(E-2); below the smallest
    normal binade (E < -14) the subnormals are spaced 2^-16.  |x| / spacing
    is then rounded to the nearest integer, ties to even (torch.round), which
    is the same as rounding the 2-bit mantissa to nearest-even: an odd
    multiple of the spacing is an odd mantissa.  A result that rounds up to
    2^(E+1) is the next binade's first value, still on the grid.
    """
    x = x.to(_F64)
    a = x.abs()
    finite_nz = torch.isfinite(a) & (a > 0)
    safe = torch.where(finite_nz, a, torch.ones_like(a))
    _, k = torch.frexp(safe)  # safe = f * 2^k, f in [0.5, 1): E = k - 1
    e = (k.to(torch.int64) - 1).clamp(min=E5M2_MIN_NORMAL_EXP)
    spacing = torch.pow(torch.full_like(safe, 2.0), (e - E5M2_MANT_BITS).to(_F64))
    q = torch.round(safe / spacing) * spacing
    q = torch.clamp(q, max=E5M2_MAX)
    out = torch.where(finite_nz, torch.copysign(q, x), x)
    # +-inf saturate like every other out-of-range value; NaN and +-0 pass through
    out = torch.where(torch.isinf(x), torch.copysign(torch.full_like(x, E5M2_MAX), x), out)
    return out


def e5m2_encode(x: torch.Tensor) -> torch.Tensor:
    """uint8 codes of x after ``e5m2_quantize`` (NaN -> 0x7F).

    The code of a grid value is found by search in the code table (the
    inverse of ``e5m2_value`` over the finite codes, with the sign of zero
    kept), so it needs no bit arithmetic of its own.
    """
    q = e5m2_quantize(x).reshape(-1)
    finite_codes = [c for c in range(256) if math.isfinite(e5m2_value(c))]
    table = {}
    for c in finite_codes:
        v = e5m2_value(c)
        key = (v, math.copysign(1.0, v))
        table.setdefault(key, c)
    out = torch.empty(q.numel(), dtype=torch.uint8)
    for i, v in enumerate(q.tolist()):
        if math.isnan(v):
            out[i] = 0x7F
        else:
            out[i] = table[(v, math.copysign(1.0, v))]
    return out.view(x.shape)


def mla_decode_fp8_ref(
    q: torch.Tensor,
    kcache_codes: torch.Tensor,
    block_table: torch.Tensor,
    cache_seqlens: torch.Tensor,
    softmax_scale: float,
    causal: bool,
    requests: Optional[Sequence[int]] = None,
) -> Tuple[torch.Tensor, torch.Tensor]:
    """Paged MLA decode over an e5m2 cache: ``(out, lse)`` in fp64.

    q: [b, s_q, h_q, 576] bf16/fp16 (any dtype exact in fp64); kcache_codes:
    [pages, 64, 1, 576] uint8 e5m2 codes.  The query is cast to e5m2 (the
    page's q.to(float8_e5m2)), the bytes of each request's pages are read as
    their e5m2 values, and the plain fp64 decode of ``mla_decode_ref`` runs on
    those values, request by request.
    """
    if kcache_codes.dtype != torch.uint8:
        raise ValueError("kcache_codes must hold uint8 e5m2 codes")
    b, s_q, h_q, _ = q.shape
    reqs = list(range(b)) if requests is None else [int(r) for r in requests]
    out = torch.zeros(len(reqs), s_q, h_q, 512, dtype=_F64)
    lse = torch.full((len(reqs), h_q, s_q), -math.inf, dtype=_F64)
    for i, r in enumerate(reqs):
        # only this request's pages are read as e5m2 values; they become pages 0 .. n-1 of its own table
        seqlen = int(cache_seqlens[r])
        n = -(-seqlen // 64)
        pages = block_table[r, :n].to(torch.int64)
        k8 = e5m2_decode(kcache_codes[pages])
        table = torch.arange(max(n, 1), dtype=torch.int32)[None]
        q8 = e5m2_quantize(q[r:r + 1].to(_F64))  # this request's query rows cast to e5m2
        o, l = mla_decode_ref(q8, k8.reshape(n, 64, 1, 576), table, cache_seqlens[r:r + 1],
                              softmax_scale, causal)
        out[i] = o[0]
        lse[i] = l[0]
    return out, lse


def append_kv_fp8_ref(kcache_codes: torch.Tensor, block_table: torch.Tensor, cache_seqlens: torch.Tensor,
                      kv_new: torch.Tensor) -> torch.Tensor:
    """A copy of the e5m2 cache with the new rows cast to e5m2 and written to their slots.

    kv_new: [b, s_q, 576] bf16/fp16.  Positions and slots are those of
    ``append_kv_ref``; each written byte is ``e5m2_encode`` of the new value.
    """
    return append_kv_ref(kcache_codes, block_table, cache_seqlens, e5m2_encode(kv_new.to(_F64)))
