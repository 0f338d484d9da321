"""Planted mistakes in copies of the oracle must each fail at least one pin (no GPU).

A mutant is the oracle module's source with one plausible mistake substituted
(a dropped term, a wrong sign or index, a transposed layout ...), loaded as a
fresh module on the CPU.  The real oracle is never modified.
"""

import importlib.util
import inspect
import sys
import types

import pytest

import oracle.append_ref as app
import oracle.fp8_ref as fp8
import oracle.mla_ref as ref
import oracle.sched_ref as sched
from append_pins import ALL_APPEND_PINS
from fp8_pins import ALL_FP8_PINS
from oracle_pins import ALL_PINS
from sched_pins import ALL_SCHED_PINS

ATTN_MUTANTS = {
    "V is the last 512 columns": ("vals = keys[:, :D_V]", "vals = keys[:, D_K - D_V:]"),
    "V slice in partials": ("    vals = keys[:, :D_V]\n    qr = q[request]", "    vals = keys[:, 64:]\n    qr = q[request]"),
    "scale dropped": ("z = scale * (qr[s] @ keys[:n_vis].T)", "z = (qr[s] @ keys[:n_vis].T)"),
    "lse in log2": ("lse = m + torch.log(zsum)", "lse = (m + torch.log(zsum)) / 0.6931471805599453"),
    "lse without max": ("lse = m + torch.log(zsum)", "lse = torch.log(zsum)"),
    "no max subtraction": ("w = torch.exp(z - m[:, None])", "w = torch.exp(z)"),
    "causal off by one": ("return max(0, int(seqlen) - (s_q - 1 - s))", "return max(0, int(seqlen) - (s_q - s))"),
    "causal top-left": ("return max(0, int(seqlen) - (s_q - 1 - s))", "return min(int(seqlen), s + 1)"),
    "page index by modulo": ("page_of_tok = block_table_row.to(torch.int64)[tok // PAGE]",
                             "page_of_tok = block_table_row.to(torch.int64)[tok % PAGE]"),
    "slot ignores page offset": ("slot_of_tok = tok % PAGE", "slot_of_tok = tok // PAGE"),
    "reads the whole last page": [("    if not causal:\n        return int(seqlen)",
                                   "    if not causal:\n        return -(-int(seqlen) // PAGE) * PAGE"),
                                  ("tok = torch.arange(seqlen)", "tok = torch.arange(-(-seqlen // PAGE) * PAGE)")],
    "lse stored [s, h]": ("lse[i, :, s] = l", "lse[i, s % lse.shape[1], :] = l[: lse.shape[2]].sum()"),
    "empty row lse zero": ("lse = torch.full((len(reqs), h_q, s_q), -math.inf, dtype=_F64)",
                           "lse = torch.zeros((len(reqs), h_q, s_q), dtype=_F64)"),
    "merge weights not normalised": ("weights = torch.exp(lses - lse_safe[None])", "weights = torch.exp(lses - m_safe[None])"),
    "merge lse is max": ("lse = torch.where(finite, m_safe + torch.log(wsum), torch.full_like(m, -math.inf))",
                         "lse = torch.where(finite, m_safe, torch.full_like(m, -math.inf))"),
    "partial chunk ignores begin": ("        lo = int(key_begin)\n", "        lo = 0\n"),
}

SCHED_MUTANTS = {
    "share rounded down": ("share = _ceil_div(total, num_parts) if total > 0 else 0",
                           "share = max(1, total // num_parts) if total > 0 else 0"),
    "share without per-request overhead": ("total = sum(F + n for n in n_blk if n > 0)", "total = sum(n_blk)"),
    "no overhead units on the line": ("        x += F  # the request's overhead units\n", ""),
    "overhead after the blocks": [("        x += F  # the request's overhead units\n", ""),
                                  ("            x += 1\n", "            x += 1\n        x += F\n")],
    "block size 128": ("PAGE_BLOCK = 64", "PAGE_BLOCK = 128"),
    "split index not recorded": ("chunks.append((part, r, lo, k, per_req.get(r, 0)))", "chunks.append((part, r, lo, k, 0))"),
    "begin split dropped": ("first_of_part[part] = (r, lo, si if lo > 0 else 0)", "first_of_part[part] = (r, lo, 0)"),
    "chunk count off by one": ("num_splits[r + 1] = num_splits[r] + per_req.get(r, 0)",
                               "num_splits[r + 1] = num_splits[r] + per_req.get(r, 0) + (r == 0)"),
    "empty partitions end at (b, 0)": ("            nxt = first_of_part[p]\n        begins[p] = nxt",
                                       "            nxt = first_of_part[p]\n        begins[p] = nxt if p in first_of_part else (b, 0, 0)"),
}

APPEND_MUTANTS = {
    "position off by one": ("j = L - s_q + s  #", "j = L - s_q + s + 1  #"),
    "lengths exclude the new tokens": ("j = L - s_q + s  #", "j = L + s  #"),
    "new tokens in reverse order": ("out[page, slot, 0, :] = kv_new[r, s, :]",
                                    "out[page, slot, 0, :] = kv_new[r, s_q - 1 - s, :]"),
    "page by modulo": ("page = int(block_table[r, j // PAGE])", "page = int(block_table[r, j % PAGE])"),
    "slot by division": ("slot = j % PAGE", "slot = j // PAGE"),
    "first request's table": ("page = int(block_table[r, j // PAGE])", "page = int(block_table[0, j // PAGE])"),
    "writes into the input": ("out = kcache.clone()", "out = kcache"),
    "short request wraps around": ("            if j < 0:\n                continue\n", ""),
}

FP8_MUTANTS = {
    "ties round up": ("q = torch.round(safe / spacing) * spacing", "q = torch.floor(safe / spacing + 0.5) * spacing"),
    "truncation": ("q = torch.round(safe / spacing) * spacing", "q = torch.floor(safe / spacing) * spacing"),
    "exponent bias 16": ("E5M2_BIAS = 15", "E5M2_BIAS = 16"),
    "three mantissa bits": ("E5M2_MANT_BITS = 2", "E5M2_MANT_BITS = 3"),
    "no subnormal floor": ("e = (k.to(torch.int64) - 1).clamp(min=E5M2_MIN_NORMAL_EXP)", "e = k.to(torch.int64) - 1"),
    "binade off by one": ("e = (k.to(torch.int64) - 1).clamp(min=E5M2_MIN_NORMAL_EXP)",
                          "e = k.to(torch.int64).clamp(min=E5M2_MIN_NORMAL_EXP)"),
    "overflow not saturated": ("q = torch.clamp(q, max=E5M2_MAX)", "q = q"),
    "subnormals one binade low": ("return sign * (m / 4.0) * 2.0 ** E5M2_MIN_NORMAL_EXP",
                                  "return sign * (m / 4.0) * 2.0 ** (E5M2_MIN_NORMAL_EXP - 1)"),
    "mantissa bits swapped": ("m = code & 0x3", "m = ((code & 1) << 1) | ((code >> 1) & 1)"),
    "query not cast": ("q8 = e5m2_quantize(q[r:r + 1].to(_F64))", "q8 = q[r:r + 1].to(_F64)"),
    "append stores truncated bytes": ("e5m2_encode(kv_new.to(_F64)))", "kv_new.to(torch.uint8))"),
    "sign dropped": ("out = torch.where(finite_nz, torch.copysign(q, x), x)", "out = torch.where(finite_nz, q, x)"),
}


def _mutant(module: types.ModuleType, edits) -> types.ModuleType:
    """Copy of ``module`` with each (old, new) text substitution applied."""
    if isinstance(edits, tuple):
        edits = [edits]
    mutated = inspect.getsource(module)
    for old, new in edits:
        assert mutated.count(old) >= 1, f"mutation anchor not found: {old!r}"
        mutated = mutated.replace(old, new)
    name = module.__name__ + "_mutant"
    spec = importlib.util.spec_from_loader(name, loader=None)
    mod = importlib.util.module_from_spec(spec)
    mod.__dict__["__name__"] = name
    sys.modules[name] = mod  # dataclasses / inspect need it registered
    try:
        exec(compile(mutated, f"<{name}>", "exec"), mod.__dict__)
    finally:
        sys.modules.pop(name, None)
    return mod


def _caught(pins, mod) -> list:
    failed = []
    for pin in pins:
        try:
            pin(mod)
        except Exception as e:  # noqa: BLE001 - any failure counts as caught
            failed.append(f"{pin.__name__}: {type(e).__name__}")
    return failed


@pytest.mark.parametrize("name", sorted(ATTN_MUTANTS))
def test_attention_mutant_is_caught(name):
    mod = _mutant(ref, ATTN_MUTANTS[name])
    assert _caught(ALL_PINS, mod), f"mutant '{name}' passed every pin"


@pytest.mark.parametrize("name", sorted(APPEND_MUTANTS))
def test_append_mutant_is_caught(name):
    mod = _mutant(app, APPEND_MUTANTS[name])
    assert _caught(ALL_APPEND_PINS, mod), f"mutant '{name}' passed every pin"


@pytest.mark.parametrize("name", sorted(SCHED_MUTANTS))
def test_sched_mutant_is_caught(name):
    mod = _mutant(sched, SCHED_MUTANTS[name])
    assert _caught(ALL_SCHED_PINS, mod), f"mutant '{name}' passed every pin"


@pytest.mark.parametrize("name", sorted(FP8_MUTANTS))
def test_fp8_mutant_is_caught(name):
    mod = _mutant(fp8, FP8_MUTANTS[name])
    assert _caught(ALL_FP8_PINS, mod), f"mutant '{name}' passed every pin"
