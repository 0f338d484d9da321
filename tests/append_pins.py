"""Pins for the KV-append oracle (``oracle.append_ref``): facts fixed by the pages' paged-cache
layout and by the attention it feeds.

Each ``pin_*`` takes the append module and raises AssertionError if it disagrees.  None re-types
the oracle's position arithmetic: a hand-worked golden case (``golden/append_fresh_page.json``,
including a token that opens a fresh page at slot 0), a read-back through the attention oracle's
independently pinned gather, closed forms of the decode that follows (a lone new token is the
output), the causal reading (a query does not see the token after it) and a short request.
"""

from __future__ import annotations

import json
import os

import torch

import oracle.mla_ref as attn

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
F64 = torch.float64


def _changed_rows(a: torch.Tensor, b: torch.Tensor):
    diff = (a != b).any(dim=-1).any(dim=-1)  # [pages, 64]
    return [(int(p), int(s)) for p, s in diff.nonzero().tolist()]


def pin_golden_fresh_page(mod):
    g = json.load(open(os.path.join(GOLDEN, "append_fresh_page.json")))
    s_q = g["s_q"]
    table = torch.tensor(g["block_table"], dtype=torch.int32)
    lens = torch.tensor(g["cache_seqlens"], dtype=torch.int32)
    kc = torch.zeros(g["pool_pages"], 64, 1, 576, dtype=F64)
    b = table.shape[0]
    kv = torch.arange(1, b * s_q * 576 + 1, dtype=F64).view(b, s_q, 576)  # every row distinct, non-zero
    out = mod.append_kv_ref(kc, table, lens, kv)
    want = sorted((w["page"], w["slot"]) for w in g["expected_writes"])
    assert sorted(_changed_rows(out, kc)) == want
    for w in g["expected_writes"]:
        assert torch.equal(out[w["page"], w["slot"], 0], kv[w["request"], w["token"]])
    assert bool((kc == 0).all()), "the input cache must not be modified"


def _case(seed, lens, s_q, pool_extra=2):
    g = torch.Generator().manual_seed(seed)
    n_pages = [-(-L // 64) for L in lens]
    pool = sum(n_pages) + pool_extra
    kc = torch.randn(pool, 64, 1, 576, generator=g, dtype=F64)
    perm = torch.randperm(pool, generator=g)
    table = torch.full((len(lens), max(n_pages) + 1), -1, dtype=torch.int32)
    pos = 0
    for r, n in enumerate(n_pages):
        table[r, :n] = perm[pos:pos + n].to(torch.int32)
        pos += n
    kv = torch.randn(len(lens), s_q, 576, generator=g, dtype=F64)
    return kc, table, torch.tensor(lens, dtype=torch.int32), kv


def pin_read_back_through_gather(mod):
    """Gathering each request's tokens (the attention oracle's reader) after the append gives the
    old tokens followed by the new rows; exactly one cache row per new token changed."""
    for s_q, lens in ((1, [1, 64, 65, 130]), (2, [2, 64, 65, 129]), (3, [3, 66, 191, 200])):
        kc, table, sl, kv = _case(7 + s_q, lens, s_q)
        out = mod.append_kv_ref(kc, table, sl, kv)
        for r, L in enumerate(lens):
            before = attn.gather_keys(kc, table[r], L)
            after = attn.gather_keys(out, table[r], L)
            assert torch.equal(after[:L - s_q], before[:L - s_q])
            assert torch.equal(after[L - s_q:], kv[r])
        assert len(_changed_rows(out, kc)) == sum(1 for _ in lens) * s_q


def pin_lone_new_token_is_the_output(mod):
    """A request whose only cached token is the new one: the decode returns that token's value
    exactly and lse = scale * q.k (single-key closed form)."""
    kc, table, _, kv = _case(11, [1, 1], 1)
    kc[:] = 1.0e4  # whatever was in the slot before must not matter
    sl = torch.tensor([1, 1], dtype=torch.int32)
    g = torch.Generator().manual_seed(12)
    q = torch.randn(2, 1, 4, 576, generator=g, dtype=F64)
    appended, out, lse = mod.decode_with_append_ref(q, kv, kc, table, sl, 0.05, False)
    for r in range(2):
        assert torch.allclose(out[r, 0], kv[r, 0, :512].expand(4, 512), rtol=0, atol=1e-12)
        assert torch.allclose(lse[r, :, 0], 0.05 * (q[r, 0] @ kv[r, 0]), rtol=0, atol=1e-12)


def pin_causal_query_does_not_see_the_next_new_token(mod):
    kc, table, sl, kv = _case(13, [70, 3], 2)
    g = torch.Generator().manual_seed(14)
    q = torch.randn(2, 2, 3, 576, generator=g, dtype=F64)
    _, out1, lse1 = mod.decode_with_append_ref(q, kv, kc, table, sl, 0.04, True)
    kv2 = kv.clone()
    kv2[:, 1] += 3.0  # change only the second new token
    _, out2, lse2 = mod.decode_with_append_ref(q, kv2, kc, table, sl, 0.04, True)
    assert torch.equal(out1[:, 0], out2[:, 0]) and torch.equal(lse1[:, :, 0], lse2[:, :, 0])
    assert not torch.allclose(out1[:, 1], out2[:, 1])


def pin_short_request_keeps_only_positioned_tokens(mod):
    """L = 1 with s_q = 2: only the second new token has a position (0); the first is dropped."""
    kc, table, _, kv = _case(15, [1], 2)
    sl = torch.tensor([1], dtype=torch.int32)
    out = mod.append_kv_ref(kc, table, sl, kv)
    assert len(_changed_rows(out, kc)) == 1
    assert torch.equal(attn.gather_keys(out, table[0], 1)[0], kv[0, 1])


ALL_APPEND_PINS = [pin_golden_fresh_page, pin_read_back_through_gather, pin_lone_new_token_is_the_output,
                   pin_causal_query_does_not_see_the_next_new_token, pin_short_request_keeps_only_positioned_tokens]
