"""mla_decode_fwd_static_ws: the decode forward for callers that cannot allocate.

Callers such as a serving loop whose GPU memory is reserved up front by
another allocator, or code that must not call cudaMalloc (it can synchronise
the device), have no workspace buffer to hand over; this entry point keeps the
split-KV partials in a scratch array built into the library instead.  The test
calls it through the C ABI twice in a row (the scratch keeps the previous
call's contents) and checks both results against the fp64 CPU oracle and
against the regular entry point with the tolerances of the other parity tests,
and reads the scratch's device error word after each call.  It also checks
that a batch needing more scratch than the built-in 32 MiB, or a call with a
bad argument, is refused before anything is launched (the error word of the
previous call survives it).  This file is named so that pytest collects it
last.
"""

import ctypes

import pytest
import torch

import oracle
from gpu_util import LSE_ATOL, OUT_ATOL, OUT_RTOL, compare
from workloads import make_case

pytestmark = pytest.mark.gpu


def _bind(lib):
    vp, c_int, c_i64, c_f = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float
    fn = lib.mla_decode_fwd_static_ws
    fn.argtypes = [vp, vp, c_i64, vp, c_i64, vp, c_int, c_int, c_int, c_int, c_f, c_int, vp, vp, c_int, vp, vp, vp]
    fn.restype = c_int
    return fn


def _call(fn, inp, q, kc, bt, sl, meta, ns, parts, out, lse):
    b, s_q, h_q, _ = q.shape
    dtype = 0 if q.dtype == torch.bfloat16 else 1
    stream = torch.cuda.current_stream().cuda_stream
    return fn(q.data_ptr(), kc.data_ptr(), kc.shape[0], bt.data_ptr(), bt.stride(0), sl.data_ptr(), b, s_q, h_q,
              dtype, inp.softmax_scale, 1 if inp.causal else 0, meta.data_ptr(), ns.data_ptr(), parts,
              out.data_ptr(), lse.data_ptr(), stream)


def _status(lib):
    fn = lib.mla_static_ws_read_device_status
    fn.argtypes = [ctypes.c_void_p, ctypes.POINTER(ctypes.c_int32)]
    fn.restype = ctypes.c_int
    flags = (ctypes.c_int32 * 2)()
    rc = fn(torch.cuda.current_stream().cuda_stream, flags)
    assert rc == 0, lib.mla_status_string(rc)
    return int(flags[0]), int(flags[1])


def _close(a, b):
    a, b = a.double(), b.double()
    assert bool(((a - b).abs() <= OUT_ATOL + OUT_RTOL * b.abs()).all()), float((a - b).abs().max())


@pytest.mark.parametrize("case", [
    (6, 1, 16, [4096, 300, 1, 0, 2000, 64], torch.bfloat16, False, 1),
    (3, 2, 64, [900, 65, 2500], torch.float16, True, 2),
])
def test_static_scratch_matches_oracle_and_regular_entry_point(case):
    import mla_decode_attention_16_b200 as mla

    b, s_q, h_q, lens, dtype, causal, seed = case
    inp = make_case(b, s_q, h_q, lens, dtype=dtype, causal=causal, seed=100 + seed, extra_poison_pages=2)
    q, kc = inp.q.cuda(), inp.kcache.cuda()
    bt, sl = inp.block_table.cuda(), inp.cache_seqlens.cuda()
    rows = s_q * h_q
    parts = mla.mla_get_num_sm_parts(rows)
    meta, ns = mla.mla_get_metadata(sl, rows, parts)
    ref_out, ref_lse = mla.mla_decode_fwd(q, kc, bt, sl, inp.softmax_scale, causal, meta, ns)
    cpu_out, cpu_lse = oracle.mla_decode_ref(inp.q, inp.kcache, inp.block_table, inp.cache_seqlens,
                                             inp.softmax_scale, inp.causal)
    fn = _bind(mla.lib)
    for _ in range(2):  # second call runs on the scratch the first one left behind
        out = torch.full_like(ref_out, 3.0)
        lse = torch.full_like(ref_lse, 3.0)
        rc = _call(fn, inp, q, kc, bt, sl, meta, ns, parts, out, lse)
        assert rc == 0, mla.lib.mla_status_string(rc)
        torch.cuda.synchronize()
        assert _status(mla.lib) == (0, 0)
        compare(out.cpu(), lse.cpu(), cpu_out, cpu_lse, f"static scratch {case[:4]}")
        _close(out.cpu(), ref_out.cpu())
        fin = torch.isfinite(ref_lse)
        assert torch.equal(torch.isfinite(lse), fin)
        assert float((lse[fin] - ref_lse[fin]).abs().max()) <= LSE_ATOL


def test_static_scratch_rejects_oversize_batch():
    import mla_decode_attention_16_b200 as mla

    fn = _bind(mla.lib)
    b, s_q, h_q = 512, 1, 128  # (512 + parts) * 128 rows * 2 KB > 32 MiB
    dev = torch.zeros(16, dtype=torch.int32, device="cuda")
    p = dev.data_ptr()
    rc = fn(p, p, 1, p, 1, p, b, s_q, h_q, 0, 0.1, 0, p, p, 74, p, p, torch.cuda.current_stream().cuda_stream)
    assert rc == 3, mla.lib.mla_status_string(rc)


def test_static_scratch_rejected_call_enqueues_nothing():
    """A bad page index sets the scratch's error word; a later call that fails its host checks (here
    a misaligned output) returns before clearing it, so the word still reads the first call's error."""
    import mla_decode_attention_16_b200 as mla

    fn = _bind(mla.lib)
    inp = make_case(2, 1, 16, [100, 100], seed=123)
    inp.block_table[1, 1] = inp.kcache.shape[0] + 9
    q, kc = inp.q.cuda(), inp.kcache.cuda()
    bt, sl = inp.block_table.cuda(), inp.cache_seqlens.cuda()
    parts = mla.mla_get_num_sm_parts(16)
    meta, ns = mla.mla_get_metadata(sl, 16, parts)
    out = torch.empty(2, 1, 16, 512, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(2, 16, 1, dtype=torch.float32, device="cuda")
    assert _call(fn, inp, q, kc, bt, sl, meta, ns, parts, out, lse) == 0
    torch.cuda.synchronize()
    assert _status(mla.lib) == (2, inp.kcache.shape[0] + 9)
    flat = torch.empty(2 * 16 * 512 + 8, dtype=torch.bfloat16, device="cuda")
    bad_out = flat[1:1 + 2 * 16 * 512].view(2, 1, 16, 512)  # 2-byte offset: not 16-byte aligned
    assert _call(fn, inp, q, kc, bt, sl, meta, ns, parts, bad_out, lse) == 1
    torch.cuda.synchronize()
    assert _status(mla.lib) == (2, inp.kcache.shape[0] + 9)
    inp.block_table[1, 1] = 0  # a valid call clears the header again
    assert _call(fn, inp, q, kc, inp.block_table.cuda(), sl, meta, ns, parts, out, lse) == 0
    torch.cuda.synchronize()
    assert _status(mla.lib) == (0, 0)
