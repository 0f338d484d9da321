"""KV append and the decode step fused with it, through the C ABI, against the CPU oracle (needs a B200).

mla_append_kv writes each request's s_q new latent rows to cache positions L - s_q + s; the cache
after the call must equal oracle.append_kv_ref bit for bit (a plain copy).  mla_decode_fwd_append
does the append and then the decode on the same stream; its output must match the oracle's
"append, then decode" within the parity tolerances, including a new token that opens a fresh page
(slot 0) and requests whose only cached tokens are the new ones.
"""

import pytest
import torch

import oracle
from gpu_util import compare
from workloads import make_case

pytestmark = pytest.mark.gpu

CASES = [
    # batch, s_q, h_q, lengths (counting the new tokens), dtype, causal, seed
    (4, 1, 16, [65, 1, 64, 300], torch.bfloat16, False, 1),     # 65: the new token opens page 1 at slot 0
    (3, 2, 64, [129, 2, 700], torch.float16, True, 2),           # 129: positions 127 | 128 (fresh page)
    (2, 2, 128, [2, 1000], torch.bfloat16, True, 3),             # a request made only of new tokens
    (5, 1, 1, [1, 2, 63, 64, 65], torch.bfloat16, False, 4),
]


def _inputs(case):
    b, s_q, h_q, lens, dtype, causal, seed = case
    inp = make_case(b, s_q, h_q, lens, dtype=dtype, causal=causal, seed=500 + seed, extra_poison_pages=2)
    g = torch.Generator().manual_seed(600 + seed)
    kv_new = (torch.randn(b, s_q, 576, generator=g) * 2.0).to(dtype)
    return inp, kv_new


@pytest.mark.parametrize("case", CASES, ids=[f"b{c[0]}_sq{c[1]}_h{c[2]}" for c in CASES])
def test_append_is_bit_exact(case):
    import mla_decode_attention_16_b200 as mla

    inp, kv_new = _inputs(case)
    kc = inp.kcache.cuda()
    ws = mla.alloc_workspace(inp.batch, inp.s_q * inp.h_q, 1)
    mla.mla_append_kv(kv_new.cuda(), kc, inp.block_table.cuda(), inp.cache_seqlens.cuda(), ws)
    torch.cuda.synchronize()
    assert mla.mla_read_device_status(ws) == (0, 0)
    want = oracle.append_kv_ref(inp.kcache, inp.block_table, inp.cache_seqlens, kv_new)
    assert torch.equal(kc.cpu(), want), "cache after the append differs from the oracle"


@pytest.mark.parametrize("case", CASES, ids=[f"b{c[0]}_sq{c[1]}_h{c[2]}" for c in CASES])
def test_decode_fused_with_append_matches_oracle(case):
    import mla_decode_attention_16_b200 as mla

    inp, kv_new = _inputs(case)
    q, kc = inp.q.cuda(), inp.kcache.cuda()
    bt, sl = inp.block_table.cuda(), inp.cache_seqlens.cuda()
    rows = inp.s_q * inp.h_q
    parts = mla.mla_get_num_sm_parts(rows)
    meta, ns = mla.mla_get_metadata(sl, rows, parts)
    ws = mla.alloc_workspace(inp.batch, rows, parts)
    out, lse = mla.mla_decode_fwd_append(q, kv_new.cuda(), kc, bt, sl, inp.softmax_scale, inp.causal, meta, ns,
                                         ws)
    torch.cuda.synchronize()
    assert mla.mla_read_device_status(ws) == (0, 0)
    appended, ref_out, ref_lse = oracle.decode_with_append_ref(inp.q, kv_new, inp.kcache, inp.block_table,
                                                               inp.cache_seqlens, inp.softmax_scale, inp.causal)
    assert torch.equal(kc.cpu(), appended)
    compare(out.cpu(), lse.cpu(), ref_out, ref_lse, f"append+decode {case[:4]}")


def test_append_flags_rows_without_a_slot():
    """L < s_q (no position for the first new token) and a page outside the pool are flagged, and
    those rows are skipped; every other row is still written."""
    import mla_decode_attention_16_b200 as mla

    inp, kv_new = _inputs((3, 2, 16, [1, 100, 100], torch.bfloat16, False, 9))
    bt = inp.block_table.clone()
    bt[2, 1] = inp.kcache.shape[0] + 3  # request 2's new tokens (positions 98, 99) sit in page slot 1
    kc = inp.kcache.cuda()
    ws = mla.alloc_workspace(3, 32, 1)
    mla.mla_append_kv(kv_new.cuda(), kc, bt.cuda(), inp.cache_seqlens.cuda(), ws)
    torch.cuda.synchronize()
    bits, page = mla.mla_read_device_status(ws)
    assert bits == 2 | 4 and page == inp.kcache.shape[0] + 3, (bits, page)
    keep = inp.block_table.clone()
    keep[2] = -1  # the oracle skips nothing, so drop request 2 there: its rows were not written
    want = oracle.append_kv_ref(inp.kcache, keep, torch.tensor([1, 100, 0], dtype=torch.int32), kv_new)
    assert torch.equal(kc.cpu(), want)
