"""CUDA path vs the fp64 CPU oracle, through the C ABI (needs a B200)."""

import math
import random

import pytest
import torch

import oracle
from gpu_util import compare, run_gpu
from workloads import WORKLOADS, make_case, make_workload

pytestmark = pytest.mark.gpu

SMALL = [
    # batch, s_q, h_q, seqlens, dtype, causal, parts, seed
    (3, 1, 16, [1, 63, 200], torch.bfloat16, False, None, 1),
    (2, 1, 128, [64, 300], torch.bfloat16, False, None, 2),
    (2, 2, 64, [129, 2], torch.float16, True, None, 3),
    (2, 2, 128, [70, 1], torch.bfloat16, True, None, 4),          # 2 row tiles; a row with no visible key
    (4, 1, 16, [0, 5, 0, 640], torch.bfloat16, False, 3, 5),      # empty requests, splits
    (1, 1, 16, [1000], torch.bfloat16, False, 7, 6),              # one request cut in many chunks
    (1, 2, 8, [513], torch.float16, True, 1, 7),                  # single partition
    (5, 1, 1, [17, 64, 65, 128, 129], torch.bfloat16, False, 2, 8),  # one query row
    (2, 2, 100, [300, 77], torch.bfloat16, True, None, 9),        # ragged second row tile (200 rows)
    (3, 1, 32, [4096, 1, 2000], torch.float16, False, None, 10),
    (2, 1, 33, [300, 64], torch.bfloat16, False, None, 11),       # 33 rows: pair kernel, 2 quadrants idle
    (2, 2, 16, [100, 500], torch.bfloat16, True, None, 12),       # 32 rows, causal: narrow kernel at N = 32
    (1, 8, 128, [700], torch.bfloat16, True, None, 13),           # 1024 rows (the maximum): 8 row tiles
    (600, 1, 16, [(37 * i) % 211 for i in range(600)], torch.bfloat16, False, None, 14),  # many short requests
    (300, 1, 128, [(53 * i) % 307 for i in range(300)], torch.float16, False, None, 15),
    (4, 1, 64, [0, 5, 0, 640], torch.bfloat16, False, 3, 16),      # pair kernel: empty requests, splits
]


@pytest.mark.parametrize("case", SMALL, ids=[f"b{c[0]}_sq{c[1]}_h{c[2]}_{c[7]}" for c in SMALL])
def test_small_cases(case):
    b, s_q, h_q, lens, dtype, causal, parts, seed = case
    inp = make_case(b, s_q, h_q, lens, dtype=dtype, causal=causal, seed=seed, extra_poison_pages=3, table_pad=2)
    out, lse, meta, ns, flags = run_gpu(inp, parts)
    assert flags[0] == 0, flags
    ref_out, ref_lse = oracle.mla_decode_ref(inp.q, inp.kcache, inp.block_table, inp.cache_seqlens,
                                             inp.softmax_scale, inp.causal)
    compare(out, lse, ref_out, ref_lse, what=str(case[:4]))


FEW_ROWS = [c for c in SMALL if c[1] * c[2] <= 32]


@pytest.mark.parametrize("variant", ["few-rows-one-cta", "few-rows-pair", "row-tile-pair"])
@pytest.mark.parametrize("case", FEW_ROWS, ids=[f"b{c[0]}_sq{c[1]}_h{c[2]}_{c[7]}" for c in FEW_ROWS])
def test_few_row_cases_every_kernel_variant(variant, case):
    """Every split-KV kernel that can take s_q * h_q <= 32 rows gives the oracle's result."""
    import mla_decode_attention_16_b200 as mla

    b, s_q, h_q, lens, dtype, causal, parts, seed = case
    inp = make_case(b, s_q, h_q, lens, dtype=dtype, causal=causal, seed=seed, extra_poison_pages=3, table_pad=2)
    mla.mla_set_kernel_variant(variant)
    try:
        assert mla.mla_get_kernel_variant(s_q * h_q) == variant
        out, lse, meta, ns, flags = run_gpu(inp, parts)
    finally:
        mla.mla_set_kernel_variant("auto")
    assert flags[0] == 0, flags
    ref_out, ref_lse = oracle.mla_decode_ref(inp.q, inp.kcache, inp.block_table, inp.cache_seqlens,
                                             inp.softmax_scale, inp.causal)
    compare(out, lse, ref_out, ref_lse, what=f"{variant} {case[:4]}")


def test_tiny_workload():
    inp = make_workload("tiny")
    out, lse, _, _, flags = run_gpu(inp)
    assert flags[0] == 0
    ref_out, ref_lse = oracle.mla_decode_ref(inp.q, inp.kcache, inp.block_table, inp.cache_seqlens,
                                             inp.softmax_scale, inp.causal)
    compare(out, lse, ref_out, ref_lse, "tiny")


def test_metadata_bit_exact():
    import mla_decode_attention_16_b200 as mla
    rng = random.Random(7)
    cases = [([192, 640, 1, 0, 130], 3), ([4096] * 64, 74), ([4096] * 128, 74), ([0, 0, 0], 5), ([1], 148),
             ([rng.randint(0, 3000) for _ in range(16384)], 148),   # the largest batch
             ([rng.randint(0, 3000) for _ in range(2000)], 1024)]   # the most partitions
    for _ in range(20):
        b = rng.choice([1, 3, 16, 132, 500])
        cases.append(([rng.choice([0, 1, 64, 65, rng.randint(1, 40000)]) for _ in range(b)],
                      rng.choice([1, 2, 37, 74, 148])))
    for lens, P in cases:
        sl = torch.tensor(lens, dtype=torch.int32, device="cuda")
        meta, ns = mla.mla_get_metadata(sl, 16, P)
        ref_meta, ref_ns = oracle.tile_schedule_ref(lens, P)
        assert meta.cpu().tolist() == ref_meta, (lens[:8], P)
        assert ns.cpu().tolist() == ref_ns, (lens[:8], P)


def test_split_counts_agree():
    """The same request computed in one piece and in many pieces agrees within tolerance."""
    inp = make_case(2, 2, 64, [3000, 1500], dtype=torch.bfloat16, causal=True, seed=21)
    o1, l1, _, ns1, _ = run_gpu(inp, 1)
    o2, l2, _, ns2, _ = run_gpu(inp, 74)
    assert int(ns1[-1]) == 2 and int(ns2[-1]) > 2
    ref_out, ref_lse = oracle.mla_decode_ref(inp.q, inp.kcache, inp.block_table, inp.cache_seqlens,
                                             inp.softmax_scale, inp.causal)
    compare(o1, l1, ref_out, ref_lse, "unsplit")
    compare(o2, l2, ref_out, ref_lse, "split")


def test_deterministic_and_page_permutation_invariant():
    inp = make_case(3, 1, 128, [700, 64, 1300], seed=22, extra_poison_pages=5)
    o1, l1, *_ = run_gpu(inp)
    o2, l2, *_ = run_gpu(inp)
    assert torch.equal(o1, o2) and torch.equal(l1, l2), "not deterministic"
    pool = inp.kcache.shape[0]
    perm = torch.randperm(pool, generator=torch.Generator().manual_seed(3))
    inv = torch.empty_like(perm)
    inv[perm] = torch.arange(pool)
    inp.kcache = inp.kcache[perm].contiguous()
    inp.block_table = torch.where(inp.block_table >= 0, inv[inp.block_table.clamp(min=0).long()].to(torch.int32),
                                  inp.block_table)
    o3, l3, *_ = run_gpu(inp)
    assert torch.equal(o1, o3) and torch.equal(l1, l3), "page relabelling changed the result"


@pytest.mark.parametrize("case", [
    (1, 8, 128, [700], True, None, 13),          # pair kernel: 8 row tiles, partitions of one or two blocks
    (6, 1, 64, [300, 1, 64, 2000, 65, 129], False, 5, 23),  # pair kernel: chunks cut across few partitions
    (4, 2, 8, [513, 1, 700, 64], True, 7, 24),   # narrow kernel
], ids=["pair_8_tiles", "pair_few_parts", "narrow"])
def test_repeated_runs_identical(case):
    """The first launch matches the oracle and five more give the same bits (catches pipeline races
    that show only under some launch timings, e.g. the first launch after loading)."""
    b, s_q, h_q, lens, causal, parts, seed = case
    inp = make_case(b, s_q, h_q, lens, causal=causal, seed=seed, extra_poison_pages=3)
    o1, l1, _, _, flags = run_gpu(inp, parts)
    assert flags[0] == 0, flags
    ref_out, ref_lse = oracle.mla_decode_ref(inp.q, inp.kcache, inp.block_table, inp.cache_seqlens,
                                             inp.softmax_scale, inp.causal)
    compare(o1, l1, ref_out, ref_lse, str(case))
    for _ in range(5):
        o, l, *_ = run_gpu(inp, parts)
        assert torch.equal(o, o1) and torch.equal(l, l1), "a later launch gave different bits"


def test_combine_stage_against_oracle_merge():
    """Second stage alone: synthetic partials in the workspace, merged vs the oracle's merge."""
    import mla_decode_attention_16_b200 as mla
    g = torch.Generator().manual_seed(5)
    b, s_q, h_q, parts = 4, 2, 8, 3
    rows = s_q * h_q
    chunks = [3, 1, 0, 2]  # chunk counts per request (1 => written by the first stage, untouched here)
    ns = torch.tensor([0] + list(torch.tensor(chunks).cumsum(0)), dtype=torch.int32)
    ws = mla.alloc_workspace(b, rows, parts)
    nchunk = int(ns[-1])
    lse_acc = torch.randn(nchunk, rows, generator=g, dtype=torch.float64) * 3
    lse_acc[0, 3] = -math.inf  # an empty chunk
    o_acc = torch.randn(nchunk, rows, 512, generator=g, dtype=torch.float64)
    lse_off = 256
    o_off = (256 + (b + parts) * rows * 4 + 255) // 256 * 256
    ws.view(torch.uint8)[lse_off:lse_off + nchunk * rows * 4].view(torch.float32).copy_(
        lse_acc.flatten().float())
    ws[o_off:o_off + nchunk * rows * 512 * 4].view(torch.float32).copy_(o_acc.flatten().float())
    out = torch.full((b, s_q, h_q, 512), 7.0, dtype=torch.bfloat16, device="cuda")
    lse = torch.full((b, h_q, s_q), 7.0, dtype=torch.float32, device="cuda")
    sl = torch.tensor([100, 100, 0, 100], dtype=torch.int32, device="cuda")
    mla.mla_combine_fwd(sl, s_q, h_q, torch.bfloat16, ns.cuda(), parts, ws, out, lse)
    torch.cuda.synchronize()
    out, lse = out.cpu().double(), lse.cpu().double()
    for r in range(b):
        c0, c = int(ns[r]), chunks[r]
        if c == 1:
            assert bool((out[r] == 7.0).all()) and bool((lse[r] == 7.0).all()), "single-chunk request touched"
            continue
        if c == 0:
            assert bool((out[r] == 0).all()) and bool(torch.isneginf(lse[r]).all())
            continue
        parts_in = []
        for k in range(c):
            o = o_acc[c0 + k].view(s_q, h_q, 512).float().double()
            l_ = lse_acc[c0 + k].float().double().view(s_q, h_q).T.contiguous()
            parts_in.append((o, l_))
        ref_o, ref_l = oracle.merge_partials_ref(parts_in)
        err = (out[r] - ref_o).abs()
        assert float((err - (1e-2 + 1e-2 * ref_o.abs())).max()) <= 0
        assert float((lse[r] - ref_l).abs().max()) <= 1e-4


def test_bad_page_index_is_flagged_not_faulted():
    """A block-table entry outside the pool is caught by the kernel's bounds check."""
    inp = make_case(2, 1, 16, [100, 100], seed=23)
    inp.block_table[1, 1] = inp.kcache.shape[0] + 5
    out, lse, _, _, flags = run_gpu(inp)
    assert flags[0] & 2, flags
    assert flags[1] == inp.kcache.shape[0] + 5
    ref_out, ref_lse = oracle.mla_decode_ref(inp.q, inp.kcache, inp.block_table, inp.cache_seqlens,
                                             inp.softmax_scale, inp.causal, requests=[0])
    compare(out[:1], lse[:1], ref_out, ref_lse, "unaffected request")


FULL = ["memory-bound", "compute-bound", "varlen-mtp", "long-fp16"]


@pytest.mark.parametrize("name", FULL)
def test_full_size_workload_every_request(name):
    """Full-size workload in the bench's launch configuration; every request of it is checked element
    by element against the fp64 oracle (out and lse), and the error is reported against the tolerance."""
    inp = make_workload(name)
    out, lse, meta, ns, flags = run_gpu(inp)
    assert flags[0] == 0, flags
    ref_out, ref_lse = oracle.mla_decode_ref(inp.q, inp.kcache, inp.block_table, inp.cache_seqlens,
                                             inp.softmax_scale, inp.causal)
    assert ref_out.shape[0] == inp.q.shape[0]
    compare(out, lse, ref_out, ref_lse, name)
    err = (out.double() - ref_out).abs()
    ratio = float((err / (1e-2 + 1e-2 * ref_out.abs())).max())
    fin = torch.isfinite(ref_lse)
    lerr = float((lse.double()[fin] - ref_lse[fin]).abs().max())
    print(f"\n{name}: {inp.q.shape[0]} requests, max |out-ref|/tol {ratio:.3f}, max |lse-ref| {lerr:.2e}")
