"""FP8 (e5m2) cache path through the C ABI against the CPU oracle (needs a B200).

The decode over an e5m2 cache must match ``oracle.mla_decode_fp8_ref`` (the query cast to e5m2,
the cache bytes read as e5m2 values, the plain fp64 decode) within the parity tolerances of the
16-bit path: both sides multiply the same e5m2 values, so what remains is the fp32 accumulation,
P rounded to fp16 (the page's FP16 weighting) and the output's rounding.  The append that casts
new rows to e5m2 must match ``oracle.append_kv_fp8_ref`` byte for byte.
"""

import pytest
import torch

import oracle
from gpu_util import compare, run_gpu
from workloads import E5M2_POISON_CODE, make_case, make_workload

pytestmark = pytest.mark.gpu

CASES = [
    # batch, s_q, h_q, seqlens, q dtype, causal, parts, seed
    (3, 1, 16, [1, 63, 200], torch.bfloat16, False, None, 1),         # 16 rows: one tile, NP = 16
    (2, 1, 32, [64, 300], torch.float16, False, None, 2),             # 32 rows: one full tile
    (2, 2, 16, [129, 2], torch.bfloat16, True, None, 3),              # causal, s_q = 2
    (2, 1, 64, [70, 1000], torch.bfloat16, False, None, 4),           # 64 rows: one half-empty tile
    (2, 2, 128, [70, 1], torch.bfloat16, True, None, 5),              # 2 row tiles; a row with no visible key
    (2, 1, 33, [300, 64], torch.float16, False, None, 6),             # 33 rows: the 128-row kernel
    (4, 1, 16, [0, 5, 0, 640], torch.bfloat16, False, 3, 7),          # empty requests, splits
    (1, 1, 16, [1000], torch.bfloat16, False, 7, 8),                  # one request cut in many chunks
    (1, 2, 8, [513], torch.float16, True, 1, 9),                      # single partition
    (5, 1, 1, [17, 64, 65, 128, 129], torch.bfloat16, False, 2, 10),  # one query row
    (600, 1, 16, [(37 * i) % 211 for i in range(600)], torch.bfloat16, False, None, 11),  # many short requests
    (1, 8, 128, [700], torch.bfloat16, True, None, 12),               # 1024 rows: 8 row tiles
    (4, 1, 64, [0, 5, 0, 640], torch.float16, False, 3, 13),          # 128-row kernel with splits
    (3, 1, 128, [4096, 70, 1], torch.bfloat16, False, None, 14),      # one full 128-row tile, long request
    (2, 2, 100, [300, 77], torch.float16, True, None, 15),            # 200 rows: a ragged second tile
]


def _ref(inp):
    return oracle.mla_decode_fp8_ref(inp.q, inp.kcache, inp.block_table, inp.cache_seqlens, inp.softmax_scale,
                                     inp.causal)


@pytest.mark.parametrize("case", CASES, ids=[f"b{c[0]}_sq{c[1]}_h{c[2]}_{c[7]}" for c in CASES])
def test_fp8_cache_small_cases(case):
    b, s_q, h_q, lens, dtype, causal, parts, seed = case
    inp = make_case(b, s_q, h_q, lens, dtype=dtype, causal=causal, seed=700 + seed, extra_poison_pages=3,
                    table_pad=2, kv_fp8=True)
    out, lse, _, _, flags = run_gpu(inp, parts)
    assert flags[0] == 0, flags
    assert out.dtype == dtype
    ref_out, ref_lse = _ref(inp)
    compare(out, lse, ref_out, ref_lse, what=f"fp8 {case[:4]}")


def test_fp8_cache_poison_is_never_read():
    """Pages outside the table and slots past L hold 10240 (code 0x71); reading any of them would
    dominate the softmax."""
    inp = make_case(3, 1, 16, [65, 130, 7], seed=720, extra_poison_pages=4, kv_fp8=True)
    assert int((inp.kcache == E5M2_POISON_CODE).sum()) > 4 * 64 * 576
    out, lse, _, _, flags = run_gpu(inp)
    assert flags[0] == 0
    ref_out, ref_lse = _ref(inp)
    compare(out, lse, ref_out, ref_lse, "fp8 poison")
    assert float(out.abs().max()) < 100.0


def test_fp8_cache_repeated_runs_identical():
    inp = make_case(8, 1, 16, [3000] * 8, seed=721, kv_fp8=True)
    first = run_gpu(inp, 37)
    for _ in range(3):
        again = run_gpu(inp, 37)
        assert torch.equal(first[0], again[0]) and torch.equal(first[1], again[1])


def test_fp8_cache_memory_bound_workload_every_request():
    """The full-size e5m2 workload (64 requests x 4096 tokens, 16 rows), every request checked."""
    inp = make_workload("memory-bound-fp8")
    out, lse, _, _, flags = run_gpu(inp)
    assert flags[0] == 0
    ref_out, ref_lse = _ref(inp)
    compare(out, lse, ref_out, ref_lse, "memory-bound-fp8")


APPEND = [
    # batch, s_q, h_q, lengths (counting the new tokens), dtype, causal, seed
    (4, 1, 16, [65, 1, 64, 300], torch.bfloat16, False, 1),
    (3, 2, 64, [129, 2, 700], torch.float16, True, 2),
    (2, 2, 128, [2, 1000], torch.bfloat16, True, 3),
]


def _append_inputs(case, extremes=False):
    b, s_q, h_q, lens, dtype, causal, seed = case
    inp = make_case(b, s_q, h_q, lens, dtype=dtype, causal=causal, seed=740 + seed, extra_poison_pages=2,
                    kv_fp8=True)
    g = torch.Generator().manual_seed(760 + seed)
    kv_new = (torch.randn(b, s_q, 576, generator=g) * 2.0).to(dtype)
    if extremes:
        # ties to even and saturation.  Only for the byte-exact append check: a saturated key (57344)
        # gives scores of ~2400, whose lse fp32 cannot hold to the decode's absolute 1e-3
        kv_new[0, 0, :4] = torch.tensor([1.125, 1.375, -3.25, 1.0e5])
    return inp, kv_new


@pytest.mark.parametrize("case", APPEND, ids=[f"b{c[0]}_sq{c[1]}_h{c[2]}" for c in APPEND])
def test_fp8_append_is_bit_exact(case):
    import mla_decode_attention_16_b200 as mla

    inp, kv_new = _append_inputs(case, extremes=True)
    kc = inp.kcache.cuda()
    ws = mla.alloc_workspace(inp.batch, inp.s_q * inp.h_q, 1)
    mla.mla_append_kv(kv_new.cuda(), kc, inp.block_table.cuda(), inp.cache_seqlens.cuda(), ws)
    torch.cuda.synchronize()
    assert mla.mla_read_device_status(ws) == (0, 0)
    want = oracle.append_kv_fp8_ref(inp.kcache, inp.block_table, inp.cache_seqlens, kv_new)
    got = kc.cpu()
    assert torch.equal(got, want), f"{int((got != want).sum())} cache bytes differ from the oracle"


@pytest.mark.parametrize("case", APPEND, ids=[f"b{c[0]}_sq{c[1]}_h{c[2]}" for c in APPEND])
def test_fp8_decode_fused_with_append_matches_oracle(case):
    import mla_decode_attention_16_b200 as mla

    inp, kv_new = _append_inputs(case)
    q, kc = inp.q.cuda(), inp.kcache.cuda()
    bt, sl = inp.block_table.cuda(), inp.cache_seqlens.cuda()
    rows = inp.s_q * inp.h_q
    parts = mla.mla_get_num_sm_parts(rows, kv_fp8=True)
    meta, ns = mla.mla_get_metadata(sl, rows, parts)
    ws = mla.alloc_workspace(inp.batch, rows, parts)
    out, lse = mla.mla_decode_fwd_append(q, kv_new.cuda(), kc, bt, sl, inp.softmax_scale, inp.causal, meta, ns, ws)
    torch.cuda.synchronize()
    assert mla.mla_read_device_status(ws) == (0, 0)
    cache = oracle.append_kv_fp8_ref(inp.kcache, inp.block_table, inp.cache_seqlens, kv_new)
    assert torch.equal(kc.cpu(), cache)
    ref_out, ref_lse = oracle.mla_decode_fp8_ref(inp.q, cache, inp.block_table, inp.cache_seqlens,
                                                 inp.softmax_scale, inp.causal)
    compare(out.cpu(), lse.cpu(), ref_out, ref_lse, f"fp8 append+decode {case[:3]}")


def test_fp8_partition_count():
    import mla_decode_attention_16_b200 as mla

    sms = torch.cuda.get_device_properties(0).multi_processor_count
    assert mla.mla_get_num_sm_parts(16, kv_fp8=True) == sms
    assert mla.mla_get_num_sm_parts(32, kv_fp8=True) == sms
    assert mla.mla_get_num_sm_parts(33, kv_fp8=True) == sms // 2   # one 128-row tile, two CTAs
    assert mla.mla_get_num_sm_parts(128, kv_fp8=True) == sms // 2
    assert mla.mla_get_num_sm_parts(1024, kv_fp8=True) == sms // 16


def test_fp8_cache_compute_bound_workload_every_request():
    """The full-size e5m2 workload with 128 query rows (128 requests x 4096 tokens), every request
    checked: the 128-row-tile kernel."""
    inp = make_workload("compute-bound-fp8")
    out, lse, _, _, flags = run_gpu(inp)
    assert flags[0] == 0
    ref_out, ref_lse = _ref(inp)
    compare(out, lse, ref_out, ref_lse, "compute-bound-fp8")
