"""Pins for the CPU oracle: facts fixed by the pages and by mathematics.

Each ``pin_*`` takes the oracle's attention module (normally ``oracle.mla_ref``)
and raises AssertionError if it disagrees.  ``tests/test_oracle_pins.py`` runs
them on the real oracle; ``tests/test_oracle_mutants.py`` runs them on copies
of the oracle with planted mistakes and requires every mistake to be caught.

None of these re-types the oracle's formula: they use closed forms (single key,
equal scores, a hand-worked three-key example), invariances (page permutation,
logit shift), a reduction (causal row == shorter non-causal call), an exact
rewrite (split + merge == direct) and two independent computations (pure-Python
scalar loops; torch's fused scaled-dot-product attention).
"""

from __future__ import annotations

import json
import math
import os

import torch

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
F64 = torch.float64


def _case(batch, s_q, h_q, seqlens, seed, dtype=torch.float64, pool_extra=3, std=1.0):
    """Small random case built here (fp64 values, shuffled pool)."""
    g = torch.Generator().manual_seed(seed)
    n_pages = [-(-L // 64) for L in seqlens]
    pool = sum(n_pages) + pool_extra
    q = (torch.randn(batch, s_q, h_q, 576, generator=g, dtype=F64) * std).to(dtype)
    kc = (torch.randn(pool, 64, 1, 576, generator=g, dtype=F64) * std).to(dtype)
    perm = torch.randperm(pool, generator=g)
    table = torch.full((batch, max(n_pages + [1]) + 1), -1, dtype=torch.int32)
    pos = 0
    for r, n in enumerate(n_pages):
        table[r, :n] = perm[pos:pos + n].to(torch.int32)
        pos += n
    return q, kc, table, torch.tensor(seqlens, dtype=torch.int32)


def _close(a, b, atol=1e-12, rtol=1e-12, what=""):
    a = torch.as_tensor(a, dtype=F64)
    b = torch.as_tensor(b, dtype=F64)
    fin_a, fin_b = torch.isfinite(a), torch.isfinite(b)
    assert torch.equal(fin_a, fin_b), f"{what}: finite pattern differs"
    assert torch.equal(a[~fin_a], b[~fin_b]), f"{what}: infinities differ"
    if fin_a.any():
        err = (a[fin_a] - b[fin_b]).abs()
        tol = atol + rtol * b[fin_b].abs()
        assert bool((err <= tol).all()), f"{what}: max err {float(err.max()):.3e}"


# --------------------------------------------------------------------------- closed forms

def pin_single_key(ref):
    """L = 1: softmax over one key is 1, so out = V_0 = K_0[:512] and lse = scale*q.K_0."""
    q, kc, table, lens = _case(2, 1, 3, [1, 1], seed=11)
    scale = 0.37
    out, lse = ref.mla_decode_ref(q, kc, table, lens, scale, False)
    for r in range(2):
        k0 = kc[int(table[r, 0]), 0, 0].to(F64)
        for h in range(3):
            _close(out[r, 0, h], k0[:512], what="single-key out")
            _close(lse[r, h, 0], scale * float(q[r, 0, h].to(F64) @ k0), what="single-key lse")


def pin_equal_scores(ref):
    """All scores equal -> uniform weights: out = mean of V rows, lse = z + ln L.

    q is zero on dims 0..511 and every key shares dims 512..575 (the part only
    K uses), while dims 0..511 (V) are distinct; with q == 0 entirely,
    lse = ln L exactly.
    """
    L = 150
    q, kc, table, lens = _case(1, 1, 2, [L], seed=12)
    rope = torch.randn(64, dtype=F64, generator=torch.Generator().manual_seed(5))
    kc[:, :, 0, 512:] = rope
    q[:, :, :, :512] = 0.0
    q[0, 0, 1] = 0.0  # head 1: q == 0 entirely
    scale = 0.1
    out, lse = ref.mla_decode_ref(q, kc, table, lens, scale, False)
    tok = torch.arange(L)
    rows = kc[table[0].long()[tok // 64], tok % 64, 0].to(F64)
    mean_v = rows[:, :512].mean(dim=0)
    _close(out[0, 0, 0], mean_v, atol=1e-12, what="equal-score mean")
    _close(out[0, 0, 1], mean_v, atol=1e-12, what="zero-q mean")
    z = scale * float(q[0, 0, 0, 512:].to(F64) @ rope)
    _close(lse[0, 0, 0], z + math.log(L), what="equal-score lse")
    _close(lse[0, 1, 0], math.log(L), what="zero-q lse = ln L")


def pin_golden_three_keys(ref):
    """Hand-worked example stored in tests/golden/three_keys.json (closed form)."""
    with open(os.path.join(GOLDEN, "three_keys.json")) as f:
        gold = json.load(f)
    q = torch.zeros(1, 1, 1, 576, dtype=F64)
    kc = torch.zeros(2, 64, 1, 576, dtype=F64)
    for idx, val in gold["q_nonzero"]:
        q[0, 0, 0, idx] = val
    for page, slot, idx, val in gold["k_nonzero"]:
        kc[page, slot, 0, idx] = val
    table = torch.tensor([gold["block_table"]], dtype=torch.int32)
    lens = torch.tensor([gold["seqlen"]], dtype=torch.int32)
    out, lse = ref.mla_decode_ref(q, kc, table, lens, gold["softmax_scale"], False)
    exp_out = torch.zeros(512, dtype=F64)
    for idx, val in gold["expected_out_nonzero"]:
        exp_out[idx] = val
    _close(out[0, 0, 0], exp_out, atol=1e-12, what="three-key out")
    _close(lse[0, 0, 0], gold["expected_lse"], what="three-key lse")


# --------------------------------------------------------------------------- invariances

def pin_page_permutation(ref):
    """Relabelling the pool pages (and the table with them) changes nothing, bit for bit."""
    q, kc, table, lens = _case(3, 2, 2, [70, 128, 5], seed=13, pool_extra=4)
    out, lse = ref.mla_decode_ref(q, kc, table, lens, 0.05, True)
    pool = kc.shape[0]
    perm = torch.randperm(pool, generator=torch.Generator().manual_seed(99))
    inv = torch.empty_like(perm)
    inv[perm] = torch.arange(pool)
    kc2 = kc[perm]  # new page i holds old page perm[i]
    table2 = torch.where(table >= 0, inv[table.clamp(min=0).long()].to(torch.int32), table)
    out2, lse2 = ref.mla_decode_ref(q, kc2, table2, lens, 0.05, True)
    assert torch.equal(out, out2) and torch.equal(lse, lse2), "page permutation changed the result"


def pin_logit_shift(ref):
    """Adding c to every score leaves out unchanged and adds c to lse (large c: stability).

    A key dimension that every key shares (dim 575 = 1) and a q value there
    shifts all scores of a row by the same amount.
    """
    q, kc, table, lens = _case(1, 1, 2, [90], seed=14)
    kc[:, :, 0, 575] = 1.0
    q[:, :, :, 575] = 0.0
    scale = 0.05
    out0, lse0 = ref.mla_decode_ref(q, kc, table, lens, scale, False)
    shift = 2000.0
    q[:, :, :, 575] = shift / scale
    out1, lse1 = ref.mla_decode_ref(q, kc, table, lens, scale, False)
    _close(out1, out0, atol=1e-9, rtol=1e-9, what="shifted out")
    _close(lse1, lse0 + shift, atol=1e-9, rtol=1e-12, what="shifted lse")


def pin_causal_reduction(ref):
    """Causal row s of an s_q-query call == non-causal 1-query call over the first L-s_q+s+1 keys."""
    s_q, L = 3, 70
    q, kc, table, lens = _case(1, s_q, 2, [L], seed=15)
    out, lse = ref.mla_decode_ref(q, kc, table, lens, 0.06, True)
    for s in range(s_q):
        q1 = q[:, s:s + 1].clone()
        l1 = torch.tensor([L - s_q + s + 1], dtype=torch.int32)
        o1, e1 = ref.mla_decode_ref(q1, kc, table, l1, 0.06, False)
        _close(out[0, s], o1[0, 0], what=f"causal row {s} out")
        _close(lse[0, :, s], e1[0, :, 0], what=f"causal row {s} lse")


def pin_empty_rows(ref):
    """A row that sees no key: out = 0, lse = -inf (L = 0, and causal L = 1 with s_q = 2)."""
    q, kc, table, lens = _case(2, 2, 2, [0, 1], seed=16)
    out, lse = ref.mla_decode_ref(q, kc, table, lens, 0.1, True)
    assert torch.equal(out[0], torch.zeros_like(out[0]))
    assert bool(torch.isneginf(lse[0]).all())
    assert torch.equal(out[1, 0], torch.zeros_like(out[1, 0]))
    assert bool(torch.isneginf(lse[1, :, 0]).all())
    k0 = kc[int(table[1, 0]), 0, 0].to(F64)
    _close(out[1, 1, 0], k0[:512], what="row with one visible key")


# --------------------------------------------------------------------------- split rewrite

def pin_split_merge(ref):
    """Split-KV rewrite: merging chunk results over any cut points equals the direct result."""
    s_q, L = 2, 300
    q, kc, table, lens = _case(1, s_q, 3, [L], seed=17)
    out, lse = ref.mla_decode_ref(q, kc, table, lens, 0.05, True)
    for cuts in ([0, 64, 128, 300], [0, 1, 299, 300], [0, 299, 300], [0, 300]):
        parts = [ref.mla_partial_ref(q, kc, table, lens, 0.05, True, 0, a, b)
                 for a, b in zip(cuts[:-1], cuts[1:])]
        mo, ml = ref.merge_partials_ref(parts)
        _close(mo, out[0], atol=1e-12, rtol=1e-10, what=f"merge {cuts} out")
        _close(ml, lse[0], atol=1e-12, rtol=1e-12, what=f"merge {cuts} lse")


def pin_merge_closed_form(ref):
    """Two chunks with lse a, b and outputs x, y merge to ln(e^a+e^b) and (e^a x + e^b y)/(e^a+e^b)."""
    a, b = 1.25, -0.5
    x = torch.full((1, 1, 512), 2.0, dtype=F64)
    y = torch.full((1, 1, 512), -4.0, dtype=F64)
    la = torch.tensor([[a]], dtype=F64)
    lb = torch.tensor([[b]], dtype=F64)
    mo, ml = ref.merge_partials_ref([(x, la), (y, lb)])
    ea, eb = math.exp(a), math.exp(b)
    _close(ml[0, 0], math.log(ea + eb), what="merge lse")
    _close(mo[0, 0], torch.full((512,), (2.0 * ea - 4.0 * eb) / (ea + eb), dtype=F64), what="merge out")
    # an empty chunk (lse -inf) has weight 0
    z = torch.zeros_like(x)
    ninf = torch.tensor([[-math.inf]], dtype=F64)
    mo2, ml2 = ref.merge_partials_ref([(x, la), (z, ninf)])
    _close(ml2, la, what="merge with empty chunk lse")
    _close(mo2, x, what="merge with empty chunk out")
    mo3, ml3 = ref.merge_partials_ref([(z, ninf), (z, ninf)])
    assert bool(torch.isneginf(ml3).all()) and torch.equal(mo3, z)


# --------------------------------------------------------------------------- independent computations

def pin_bruteforce_scalar(ref):
    """Pure-Python scalar loops (math.exp, explicit sums) on a tiny mixed case.

    Covers the block-table gather, the V slice, causal alignment, and the
    [b, s_q, h_q, 512] / [b, h_q, s_q] output layouts element by element.
    """
    s_q, h_q = 2, 3
    seqlens = [67, 3]
    q, kc, table, lens = _case(2, s_q, h_q, seqlens, seed=18, pool_extra=2)
    scale = 0.045
    out, lse = ref.mla_decode_ref(q, kc, table, lens, scale, True)
    ql = q.tolist()
    for r, L in enumerate(seqlens):
        keys = []
        for j in range(L):
            page = int(table[r, j // 64])
            keys.append(kc[page, j % 64, 0].tolist())
        for s in range(s_q):
            n_vis = L - (s_q - 1 - s)
            for h in range(h_q):
                zs = [scale * sum(a * b for a, b in zip(ql[r][s][h], keys[j])) for j in range(n_vis)]
                m = max(zs)
                ws = [math.exp(z - m) for z in zs]
                tot = sum(ws)
                for c in (0, 1, 255, 511):
                    val = sum(ws[j] * keys[j][c] for j in range(n_vis)) / tot
                    _close(out[r, s, h, c], val, atol=1e-12, rtol=1e-10, what=f"bf out r{r}s{s}h{h}c{c}")
                _close(lse[r, h, s], m + math.log(tot), atol=1e-12, what=f"bf lse r{r}h{h}s{s}")


def pin_sdpa_library(ref):
    """torch's scaled_dot_product_attention (fp64, CPU) on the gathered contiguous keys."""
    seqlens = [200, 64]
    q, kc, table, lens = _case(2, 1, 4, seqlens, seed=19)
    scale = 576 ** -0.5
    out, _ = ref.mla_decode_ref(q, kc, table, lens, scale, False)
    for r, L in enumerate(seqlens):
        pages = table[r, : -(-L // 64)].long()
        k = kc[pages].reshape(-1, 576)[:L].to(F64)  # contiguous gather, written differently
        v = k[:, :512]
        qq = q[r, 0].to(F64)  # [h, 576]
        o = torch.nn.functional.scaled_dot_product_attention(
            qq[None, :, None, :], k[None, None].expand(1, 4, L, 576), v[None, None].expand(1, 4, L, 512),
            scale=scale)
        _close(out[r, 0], o[0, :, 0], atol=1e-12, rtol=1e-10, what="sdpa")


ALL_PINS = [
    pin_single_key,
    pin_equal_scores,
    pin_golden_three_keys,
    pin_page_permutation,
    pin_logit_shift,
    pin_causal_reduction,
    pin_empty_rows,
    pin_split_merge,
    pin_merge_closed_form,
    pin_bruteforce_scalar,
    pin_sdpa_library,
]
