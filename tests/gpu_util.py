"""Helpers of the GPU parity tests: run the CUDA path through the C ABI, compare with the oracle."""

from __future__ import annotations

import math

import torch

OUT_ATOL = 1e-2
OUT_RTOL = 1e-2
LSE_ATOL = 1e-3


def run_gpu(inp, num_sm_parts=None, device="cuda"):
    import mla_decode_attention_16_b200 as mla

    q = inp.q.to(device)
    kc = inp.kcache.to(device)
    bt = inp.block_table.to(device)
    sl = inp.cache_seqlens.to(device)
    b, s_q, h_q, _ = q.shape
    rows = s_q * h_q
    parts = num_sm_parts or mla.mla_get_num_sm_parts(rows, kv_fp8=inp.kcache.dtype == torch.uint8)
    meta, ns = mla.mla_get_metadata(sl, rows, parts)
    ws = mla.alloc_workspace(b, rows, parts, device)
    out, lse = mla.mla_decode_fwd(q, kc, bt, sl, inp.softmax_scale, inp.causal, meta, ns, ws)
    torch.cuda.synchronize()
    flags = mla.mla_read_device_status(ws)
    return out.cpu(), lse.cpu(), meta.cpu(), ns.cpu(), flags


def compare(out, lse, ref_out, ref_lse, what=""):
    """Element-wise check against the oracle with the stated tolerances; returns max errors."""
    o = out.to(torch.float64)
    assert o.shape == ref_out.shape, (o.shape, ref_out.shape)
    assert torch.isfinite(o).all(), f"{what}: non-finite output"
    err = (o - ref_out).abs()
    tol = OUT_ATOL + OUT_RTOL * ref_out.abs()
    bad = err > tol
    if bad.any():
        idx = tuple(int(i) for i in bad.nonzero()[0])
        raise AssertionError(f"{what}: {int(bad.sum())} outputs out of tolerance; first {idx}: "
                             f"gpu {float(o[idx]):.6g} ref {float(ref_out[idx]):.6g}; max err {float(err.max()):.3g}")
    l = lse.to(torch.float64)
    fin_ref = torch.isfinite(ref_lse)
    assert torch.equal(torch.isfinite(l), fin_ref), f"{what}: lse finite pattern differs"
    assert bool(torch.isneginf(l[~fin_ref]).all()), f"{what}: lse of empty rows must be -inf"
    lerr = (l[fin_ref] - ref_lse[fin_ref]).abs()
    if lerr.numel():
        assert float(lerr.max()) <= LSE_ATOL, f"{what}: lse max err {float(lerr.max()):.3g}"
    return float(err.max()) if err.numel() else 0.0, float(lerr.max()) if lerr.numel() else 0.0
