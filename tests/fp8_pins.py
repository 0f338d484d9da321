"""Pins for the FP8 (e5m2) cache oracle (``oracle.fp8_ref``).

Each ``pin_*`` takes the module and raises AssertionError if it disagrees.  What fixes the
answers, independently of the oracle's own arithmetic:

* the e5m2 format's field definition, worked by hand for a table of codes;
* torch's own ``float8_e5m2`` dtype (a library implementation of the same format and of the
  round-to-nearest-even cast the page names, ``q.to(torch.float8_e5m2)``, in
  "云上AI推理新突破：FlashMLA赋能DeepSeek-V2-Lite提速16%", section 3. 动态精度缩放);
* closed forms: ties go to the even mantissa, out-of-range values saturate, rounding moves a
  value by at most half a grid step, a hand-worked two-key decode;
* the reduction to the pinned 16-bit decode when the query already lies on the e5m2 grid.
"""

from __future__ import annotations

import math

import torch

import oracle.mla_ref as attn

F64 = torch.float64


def _codes_to_f64_by_torch(codes: torch.Tensor) -> torch.Tensor:
    return codes.to(torch.uint8).view(torch.float8_e5m2).to(F64)


def pin_code_table_hand_values(mod):
    """Codes worked by hand from the fields (sign | 5-bit exponent, bias 15 | 2-bit mantissa)."""
    want = {
        0x00: 0.0, 0x01: 2.0 ** -16, 0x02: 2.0 ** -15, 0x03: 3 * 2.0 ** -16, 0x04: 2.0 ** -14,
        0x38: 0.5, 0x3C: 1.0, 0x3D: 1.25, 0x3E: 1.5, 0x3F: 1.75, 0x40: 2.0, 0x42: 3.0, 0x43: 3.5,
        0x7B: 57344.0, 0x7C: math.inf, 0xBC: -1.0, 0xFB: -57344.0, 0xFC: -math.inf,
    }
    got = mod.e5m2_decode(torch.tensor(list(want), dtype=torch.uint8))
    for (c, v), g in zip(want.items(), got.tolist()):
        assert g == v, f"code {c:#04x}: {g} != {v}"
    neg0 = float(mod.e5m2_decode(torch.tensor([0x80], dtype=torch.uint8))[0])
    assert neg0 == 0.0 and math.copysign(1.0, neg0) < 0
    for c in (0x7D, 0x7E, 0x7F, 0xFD):
        assert math.isnan(float(mod.e5m2_decode(torch.tensor([c], dtype=torch.uint8))[0]))


def pin_decode_matches_torch_float8(mod):
    """All 256 codes against torch's float8_e5m2 type."""
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    mine = mod.e5m2_decode(codes)
    lib = _codes_to_f64_by_torch(codes)
    same = (mine == lib) | (torch.isnan(mine) & torch.isnan(lib))
    assert bool(same.all()), f"codes differ: {codes[~same].tolist()}"


def pin_quantize_matches_torch_cast(mod):
    """Round to nearest even on random values over every binade, subnormals included."""
    g = torch.Generator().manual_seed(77)
    n = 100000
    x = torch.randn(n, generator=g, dtype=F64) * torch.pow(2.0, torch.randint(-22, 16, (n,), generator=g).to(F64))
    x = x[x.abs() < 57344.0]
    mine = mod.e5m2_quantize(x)
    lib = x.to(torch.float8_e5m2).to(F64)
    assert torch.equal(mine, lib), f"{int((mine != lib).sum())} values differ"
    # bf16 / fp16 inputs (what the query arrives as) go through the same rounding
    for dt in (torch.bfloat16, torch.float16):
        xs = x[x.abs() < 60000.0].to(dt)
        assert torch.equal(mod.e5m2_quantize(xs.to(F64)), xs.to(torch.float8_e5m2).to(F64))


def pin_ties_to_even(mod):
    """Midpoints between neighbours go to the even mantissa (hand-worked and exhaustively)."""
    cases = {1.125: 1.0, 1.375: 1.5, 1.625: 1.5, 1.875: 2.0, -1.125: -1.0, 3.25: 3.0, 3.75: 4.0,
             0.5 * 2.0 ** -16: 0.0, 1.5 * 2.0 ** -16: 2.0 ** -15, 2.5 * 2.0 ** -16: 2.0 ** -15,
             3.5 * 2.0 ** -16: 2.0 ** -14}
    got = mod.e5m2_quantize(torch.tensor(list(cases), dtype=F64)).tolist()
    for (x, v), g in zip(cases.items(), got):
        assert g == v, f"{x}: {g} != {v}"
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    vals = _codes_to_f64_by_torch(codes)
    grid = torch.unique(vals[torch.isfinite(vals) & (vals >= 0)])
    mid = (grid[:-1] + grid[1:]) / 2
    q = mod.e5m2_quantize(mid)
    # of the two neighbours, the one whose code has an even mantissa (last bit 0)
    even = {float(v): int(c) & 1 == 0 for v, c in zip(vals.tolist(), codes.tolist()) if math.isfinite(v) and v >= 0}
    for lo, hi, r in zip(grid[:-1].tolist(), grid[1:].tolist(), q.tolist()):
        assert r == (lo if even[lo] else hi), f"tie {lo}/{hi} -> {r}"


def pin_saturation(mod):
    """Beyond the largest finite value (57344 = 1.75 * 2^15) results clamp; NaN stays NaN."""
    x = torch.tensor([57344.0, 60000.0, 61440.0, 1e6, -1e9, math.inf, -math.inf], dtype=F64)
    got = mod.e5m2_quantize(x).tolist()
    assert got == [57344.0, 57344.0, 57344.0, 57344.0, -57344.0, 57344.0, -57344.0], got
    assert math.isnan(float(mod.e5m2_quantize(torch.tensor([math.nan], dtype=F64))[0]))


def pin_grid_is_fixed_and_codes_round_trip(mod):
    """Every finite e5m2 value quantises to itself and encodes back to its own code."""
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    vals = _codes_to_f64_by_torch(codes)
    fin = torch.isfinite(vals)
    assert torch.equal(mod.e5m2_quantize(vals[fin]), vals[fin])
    assert torch.equal(mod.e5m2_encode(vals[fin]), codes[fin])


def pin_rounding_error_bound(mod):
    """|q(x) - x| <= 2^-3 |x| on the normal range and <= 2^-17 below it; q is monotone."""
    g = torch.Generator().manual_seed(5)
    x = torch.sort(torch.randn(50000, generator=g, dtype=F64) * 300.0).values
    q = mod.e5m2_quantize(x)
    normal = x.abs() >= 2.0 ** -14
    assert bool(((q - x).abs()[normal] <= x.abs()[normal] * 2.0 ** -3).all())
    small = torch.linspace(-2.0 ** -14, 2.0 ** -14, 4001, dtype=F64)
    assert bool(((mod.e5m2_quantize(small) - small).abs() <= 2.0 ** -17).all())
    assert bool((q[1:] >= q[:-1]).all())


def _one_page_case(q_row: dict, keys: list, seqlen: int):
    """One request, one page; q_row maps column -> value; keys[j] maps column -> e5m2 code."""
    q = torch.zeros(1, 1, 1, 576, dtype=torch.bfloat16)
    for c, v in q_row.items():
        q[0, 0, 0, c] = v
    kc = torch.zeros(1, 64, 1, 576, dtype=torch.uint8)
    for j, row in enumerate(keys):
        for c, code in row.items():
            kc[0, j, 0, c] = code
    return q, kc, torch.zeros(1, 1, dtype=torch.int32), torch.tensor([seqlen], dtype=torch.int32)


def pin_golden_two_keys(mod):
    """Hand-worked: q = (1.125, 3.3) quantises to (1.0, 3.5); k0 = e0 (code 0x3C = 1.0),
    k1 = 0.5 e1 (code 0x38).  Scores (scale 1): z0 = 1.0, z1 = 3.5 * 0.5 = 1.75, so
    out = (w0 * 1.0, w1 * 0.5, 0, ...) with w1 = e^0.75 / (1 + e^0.75), and
    lse = ln(e^1 + e^1.75)."""
    q, kc, bt, sl = _one_page_case({0: 1.125, 1: 3.3}, [{0: 0x3C}, {1: 0x38}], 2)
    out, lse = mod.mla_decode_fp8_ref(q, kc, bt, sl, 1.0, False)
    w1 = math.exp(0.75) / (1.0 + math.exp(0.75))
    w0 = 1.0 - w1
    want = torch.zeros(512, dtype=F64)
    want[0] = w0 * 1.0
    want[1] = w1 * 0.5
    assert torch.allclose(out[0, 0, 0], want, rtol=0, atol=1e-15), out[0, 0, 0, :2]
    assert abs(float(lse[0, 0, 0]) - math.log(math.exp(1.0) + math.exp(1.75))) < 1e-14


def _random_codes(g, shape, lo_exp=10, hi_exp=17):
    """e5m2 codes with exponent fields in [lo_exp, hi_exp) (values ~2^-5 .. 2^2), random sign and mantissa."""
    e = torch.randint(lo_exp, hi_exp, shape, generator=g)
    m = torch.randint(0, 4, shape, generator=g)
    s = torch.randint(0, 2, shape, generator=g)
    return ((s << 7) | (e << 2) | m).to(torch.uint8)


def _paged_case(seed, lens, s_q, h_q):
    g = torch.Generator().manual_seed(seed)
    pages = sum(-(-L // 64) for L in lens) + 2
    kc = _random_codes(g, (pages, 64, 1, 576))
    perm = torch.randperm(pages, generator=g)
    width = max(-(-L // 64) for L in lens)
    bt = torch.zeros(len(lens), width, dtype=torch.int32)
    pos = 0
    for r, L in enumerate(lens):
        n = -(-L // 64)
        bt[r, :n] = perm[pos:pos + n].to(torch.int32)
        pos += n
    q = torch.randn(len(lens), s_q, h_q, 576, generator=g).to(torch.bfloat16)
    return q, kc, bt, torch.tensor(lens, dtype=torch.int32)


def pin_grid_query_reduces_to_plain_decode(mod):
    """A query already on the e5m2 grid: the FP8 decode is the 16-bit decode of the cache's values."""
    q, kc, bt, sl = _paged_case(11, [70, 130, 5], 2, 3)
    qg = _codes_to_f64_by_torch(_random_codes(torch.Generator().manual_seed(12), tuple(q.shape)))
    out8, lse8 = mod.mla_decode_fp8_ref(qg.to(torch.bfloat16), kc, bt, sl, 0.07, True)
    out, lse = attn.mla_decode_ref(qg, _codes_to_f64_by_torch(kc), bt, sl, 0.07, True)
    assert torch.equal(out8, out) and torch.equal(lse8, lse)


def pin_query_is_cast_like_torch(mod):
    """An off-grid query: the FP8 decode equals the 16-bit decode of torch's e5m2 cast of q."""
    q, kc, bt, sl = _paged_case(13, [64, 100], 1, 4)
    out8, lse8 = mod.mla_decode_fp8_ref(q, kc, bt, sl, 0.05, False)
    qc = q.to(torch.float8_e5m2).to(F64)
    out, lse = attn.mla_decode_ref(qc, _codes_to_f64_by_torch(kc), bt, sl, 0.05, False)
    assert torch.equal(out8, out) and torch.equal(lse8, lse)
    out16, _ = attn.mla_decode_ref(q, _codes_to_f64_by_torch(kc), bt, sl, 0.05, False)
    assert not torch.equal(out8, out16)  # the cast of q does change the result


def pin_append_writes_cast_bytes(mod):
    """The appended bytes are torch's e5m2 cast of the new rows, at the positions the 16-bit append uses."""
    q, kc, bt, sl = _paged_case(17, [65, 3], 2, 1)
    g = torch.Generator().manual_seed(18)
    kv = (torch.randn(2, 2, 576, generator=g) * 2.0).to(torch.bfloat16)
    out = mod.append_kv_fp8_ref(kc, bt, sl, kv)
    want = kc.clone()
    for r, L in enumerate(sl.tolist()):
        for s in range(2):
            j = L - 2 + s
            want[int(bt[r, j // 64]), j % 64, 0] = kv[r, s].to(torch.float8_e5m2).view(torch.uint8)
    assert torch.equal(out, want)
    assert torch.equal(kc, _paged_case(17, [65, 3], 2, 1)[1])  # the input is untouched


ALL_FP8_PINS = [pin_code_table_hand_values, pin_decode_matches_torch_float8, pin_quantize_matches_torch_cast,
                pin_ties_to_even, pin_saturation, pin_grid_is_fixed_and_codes_round_trip, pin_rounding_error_bound,
                pin_golden_two_keys, pin_grid_query_reduces_to_plain_decode, pin_query_is_cast_like_torch,
                pin_append_writes_cast_bytes]
