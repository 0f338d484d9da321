"""Bounded pipeline waits: a withheld arrival ends in a recorded timeout, not a hang (needs a B200).

The library's test hook (mla_test_withhold_q_ready) makes every split-KV launch leave out one
software arrival -- the "query rows are in tensor memory" signal of each partition's first chunk --
and shortens every pipeline wait to about 10 ms.  The stage waiting for that signal gives up,
records MLA_DEVERR_TIMEOUT in the workspace's error word and raises its CTA's abort flag; the TMA
producer waits for the page loads it already issued, the other roles return, and the launch
completes.  No TMA load or distributed shared memory store is left outstanding at the injection
point (the withheld signal comes before the first score exists, so nothing has been sent to a peer
CTA).  Afterwards the context is still usable: a normal launch matches the fp64 oracle.
"""

import ctypes
import time

import pytest
import torch

import oracle
from gpu_util import compare, run_gpu
from workloads import make_case

pytestmark = pytest.mark.gpu

WAIT_CYCLES = 20_000_000  # ~10 ms at the B200's clocks


def _hook(lib, enable, cycles):
    fn = lib.mla_test_withhold_q_ready
    fn.argtypes = [ctypes.c_int, ctypes.c_longlong]
    fn.restype = ctypes.c_int
    rc = fn(enable, cycles)
    assert rc == 0, lib.mla_status_string(rc)


@pytest.mark.parametrize("case", [
    (3, 1, 16, [700, 64, 2000], False, 1, "few-rows-one-cta"),
    (3, 1, 16, [700, 64, 2000], False, 1, "few-rows-pair"),
    (2, 2, 64, [900, 300], True, 2, "row-tile-pair"),
    (3, 1, 16, [700, 64, 2000], False, 3, "fp8-cache"),
    (2, 2, 64, [900, 300], True, 4, "fp8-cache-128-row-tiles"),
], ids=lambda c: c[-1])
def test_withheld_arrival_times_out_and_launch_returns(case):
    import mla_decode_attention_16_b200 as mla

    b, s_q, h_q, lens, causal, seed, variant = case
    kv_fp8 = variant.startswith("fp8-cache")  # the e5m2-cache kernels (kernel variants do not apply)
    inp = make_case(b, s_q, h_q, lens, causal=causal, seed=300 + seed, kv_fp8=kv_fp8)
    ref = oracle.mla_decode_fp8_ref if kv_fp8 else oracle.mla_decode_ref
    variant = "auto" if kv_fp8 else variant
    mla.mla_set_kernel_variant(variant)
    _hook(mla.lib, 1, WAIT_CYCLES)
    try:
        t0 = time.perf_counter()
        _, _, _, _, flags = run_gpu(inp)  # synchronises
        elapsed = time.perf_counter() - t0
    finally:
        _hook(mla.lib, 0, 0)
        mla.mla_set_kernel_variant("auto")
    assert flags[0] & 1, f"MLA_DEVERR_TIMEOUT not recorded: {flags}"
    assert elapsed < 30.0
    # the context is intact: the same inputs now run normally and match the oracle
    mla.mla_set_kernel_variant(variant)
    try:
        out, lse, _, _, flags = run_gpu(inp)
    finally:
        mla.mla_set_kernel_variant("auto")
    assert flags[0] == 0, flags
    ref_out, ref_lse = ref(inp.q, inp.kcache, inp.block_table, inp.cache_seqlens, inp.softmax_scale, inp.causal)
    compare(out, lse, ref_out, ref_lse, f"after timeout {case[:3]}")


def test_hook_rejects_bad_arguments():
    import mla_decode_attention_16_b200 as mla

    fn = mla.lib.mla_test_withhold_q_ready
    fn.argtypes = [ctypes.c_int, ctypes.c_longlong]
    fn.restype = ctypes.c_int
    assert fn(2, 0) == 1
    assert fn(1, -5) == 1
    assert fn(0, 0) == 0
