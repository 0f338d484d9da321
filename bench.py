"""Benchmark of paged MLA decode on B200 (one JSON line on stdout).

A step is one pass of the whole hot path over one batch: the tile scheduler
(mla_get_metadata) followed by the decode forward (split-KV kernel + combine
kernel), inputs resident in HBM.  The headline workload is the memory-bound
decode batch (64 requests x 4096 cached tokens, h_q 16, s_q 1, bf16); a
default run adds, under "per_workload", the same measurements for the three
workloads with h_q * s_q >= 128 (compute-bound, varlen-mtp, long-fp16) and for
the memory- and compute-bound batches over an e5m2 cache (memory-bound-fp8,
compute-bound-fp8), at most
--companion-steps timed steps each.  Pick one workload with --workload.
Throughput uses the pages' cost model: bytes = 576*e*sum(L) + q + out + lse
(e = 2 bytes per cached value, 1 for the e5m2 cache), FLOPs =
2*h_q*s_q*(576+512)*sum(L).

Timing: W warm-up steps, then exactly K steps between CUDA events on the
launching stream, with a barrier and a synchronize on both sides; two resident
copies of the cache (each larger than the 126 MB L2) alternate between steps so
no step finds its pages in L2.  Multi-GPU (torchrun): every rank runs its own
shard of requests (weak scaling, no collective on the data path); the elapsed
time is the max over ranks.

--impl reference times the CPU oracle (fp64, this host's cores) on a bounded
sample of the same workload instead.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

from workloads import WORKLOADS, algorithmic_cost, make_workload  # noqa: E402

METRIC = "MLA decode TFLOPS & HBM GB/s at 1 B200, % of roofline, vs CPU oracle"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
DEFAULT_WORKLOAD = "memory-bound"


# ----------------------------------------------------------------------------- helpers
def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def unit_of(name: str) -> str:
    w = WORKLOADS[name]
    return "GB/s" if w.rows < 128 else "TFLOPS"


def throughput(cost: dict, seconds: float, unit: str) -> float:
    if unit == "GB/s":
        return cost["bytes"] / seconds / 1e9
    return cost["flops"] / seconds / 1e12


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def reduce_max(value: float, device=None) -> float:
    """Max of a scalar over all ranks (identity without a process group)."""
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()):
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def shard_seed(base_seed: int, rank: int) -> int:
    """Seed of rank's shard of requests: rank 0 keeps the workload's own seed."""
    return base_seed + 7777 * rank


class ClockSampler:
    """Samples SM clock and clock-event reasons with NVML while running."""

    REASONS = {
        0x0000000000000004: "sw_power_cap",
        0x0000000000000008: "hw_slowdown",
        0x0000000000000020: "sw_thermal_slowdown",
        0x0000000000000040: "hw_thermal_slowdown",
        0x0000000000000080: "hw_power_brake_slowdown",
    }

    def __init__(self, index: int, period_s: float = 0.005):
        self.samples, self.reasons, self.ok = [], 0, False
        self.max_mhz = None
        self._stop = threading.Event()
        try:
            import pynvml

            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:  # noqa: BLE001 - NVML missing: report no clocks
            self.ok = False
        self.period = period_s
        self._t = None

    def _sample(self):
        try:
            self.samples.append(self._nv.nvmlDeviceGetClockInfo(self._h, self._nv.NVML_CLOCK_SM))
            fn = getattr(self._nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                self._nv.nvmlDeviceGetCurrentClocksThrottleReasons
            self.reasons |= int(fn(self._h))
        except Exception:  # noqa: BLE001
            pass

    def _run(self):
        while not self._stop.is_set():
            self._sample()
            time.sleep(self.period)

    def start(self):
        if self.ok:
            self._sample()
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()

    def stop(self):
        if self.ok:
            self._stop.set()
            self._t.join()
            self._sample()

    def summary(self):
        if not self.ok or not self.samples:
            return None
        names = [n for bit, n in self.REASONS.items() if self.reasons & bit]
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": names, "samples": len(self.samples)}


KERNELS = {  # variant -> (kernel name, source file)
    "few-rows-one-cta": ("splitkv_narrow_kernel", "splitkv_narrow.cu"),
    "few-rows-pair": ("splitkv_npair_kernel", "splitkv_npair.cu"),
    "row-tile-pair": ("splitkv_pair_kernel", "splitkv.cu"),
}


def variant_of(rows: int, variant: str = "auto") -> str:
    """The split-KV kernel variant the library runs for s_q * h_q = rows (its default choice for
    "auto": the one-CTA few-row kernel up to 32 rows, the row-tile pair kernel above)."""
    if variant != "auto":
        return variant
    return "few-rows-one-cta" if rows <= 32 else "row-tile-pair"


FP8_KERNELS = (("splitkv_fp8_kernel", "splitkv_fp8.cu"), ("splitkv_fp8_rt_kernel", "splitkv_fp8_rt.cu"))


def kernel_of(rows: int, variant: str = "auto", kv_fp8: bool = False):
    """(name, source file) of the split-KV kernel the library runs for s_q * h_q = rows (over an e5m2
    cache: the one-CTA kernel up to 32 rows, the 128-row-tile kernel above; variants do not apply)."""
    if kv_fp8:
        return FP8_KERNELS[0] if rows <= 32 else FP8_KERNELS[1]
    return KERNELS[variant_of(rows, variant)]


# Context denominators besides the measured ones: the ~8 TB/s HBM figure the target states, and
# the datasheet dense bf16 rate of one B200.
NOMINAL_HBM_GBS = 8000.0
NOMINAL_BF16_TFLOPS = 2250.0


def tensor_peak(peaks: dict, kv_fp8: bool, key: str = "bf16_tflops") -> float:
    """Tensor-core peak (TF/s) a decode's FLOPs are held to.  16-bit: the measured bf16 rate (fp16
    runs at the same dense rate).  e5m2 cache: Q.K^T (576 of the 1088 FLOPs per key and row) runs
    as an 8-bit MMA at twice that rate (the nominal fp8 : bf16 ratio), P.V at the 16-bit rate, so
    the peak is the FLOP-weighted harmonic blend of the two.  `key` picks the bf16 rate."""
    bf16 = float(peaks[key])
    if not kv_fp8:
        return bf16
    f_qk, f_pv = 576.0, 512.0
    return (f_qk + f_pv) / (f_qk / (2.0 * bf16) + f_pv / bf16)


def roofline_extras(unit: str, achieved: float, peaks: dict, kv_fp8: bool, read_gbs) -> dict:
    """The same achieved rate against the other denominators: for HBM-bound work the nominal
    8 TB/s and a read-only stream measured in the same run; for tensor-bound work the sustained
    (seconds-long, power-capped) bf16 rate and the datasheet rate, blended like the primary peak
    for an e5m2 cache."""
    if unit == "GB/s":
        return {"nominal_peak": NOMINAL_HBM_GBS, "frac_of_nominal": achieved / NOMINAL_HBM_GBS,
                "read_stream_gbs": read_gbs, "frac_of_read_stream": achieved / read_gbs if read_gbs else None}
    sustained = tensor_peak(peaks, kv_fp8, "bf16_tflops_sustained")
    nominal = tensor_peak({"bf16_tflops": NOMINAL_BF16_TFLOPS}, kv_fp8)
    return {"sustained_peak": sustained, "frac_of_sustained": achieved / sustained,
            "nominal_peak": nominal, "frac_of_nominal": achieved / nominal}


_READ_STREAM = {}


def read_stream_gbs(dev) -> float:
    """Read-only HBM stream of this GPU, measured once per process: a sum over 2 GiB of bf16
    (larger than L2), best of 5, CUDA events.  A denominator for context only (a library kernel,
    outside every timed region)."""
    if dev.index not in _READ_STREAM:
        x = torch.ones(1 << 30, dtype=torch.bfloat16, device=dev)
        best = float("inf")
        for _ in range(6):
            a, z = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            x.sum(dtype=torch.float32)
            z.record()
            torch.cuda.synchronize(dev)
            best = min(best, a.elapsed_time(z) / 1000.0)
        _READ_STREAM[dev.index] = x.numel() * x.element_size() / best / 1e9
        del x
        torch.cuda.empty_cache()
    return _READ_STREAM[dev.index]


def cost_of(inp, lens):
    """The pages' cost model for these requests of a workload (1 byte per value of an e5m2 cache)."""
    return algorithmic_cost(lens, inp.s_q, inp.h_q, kv_elem_bytes=inp.kcache.element_size())


def oracle_fn(inp):
    """The CPU oracle's decode for this workload's cache type."""
    import oracle

    return oracle.mla_decode_fp8_ref if inp.kcache.dtype == torch.uint8 else oracle.mla_decode_ref


def profile_traffic(name: str, kernel: str, source: str):
    """DRAM bytes per split-KV launch from the committed ncu summary, if it was taken from this source."""
    path = os.path.join(ROOT, "profiles", f"{kernel}_{name}.md")
    src = os.path.join(ROOT, "mla_decode_attention_16_b200", "csrc", source)
    try:
        text = open(path).read()
        digest = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    except OSError:
        return None
    m_sha = re.search(re.escape(source) + r" sha256\[:16\]:\s*([0-9a-f]{16})", text)
    m_tr = re.search(r"traffic_bytes_per_launch:\s*([0-9.eE+]+)", text)
    if not m_sha or not m_tr or m_sha.group(1) != digest:
        return None
    return float(m_tr.group(1))


# ----------------------------------------------------------------------------- CPU oracle legs
def oracle_sample(inp, budget_s: float, min_s: float = 3.0):
    """Time the fp64 oracle request by request; returns (seconds, requests timed, passes).

    Requests are taken in order and the workload is cycled until at least min(min_s, budget_s)
    seconds have passed (so a workload the oracle finishes quickly is still timed over a few
    seconds); it stops early once budget_s is reached.
    """
    decode = oracle_fn(inp)
    done, t0, passes = [], time.perf_counter(), 0
    floor = min(min_s, budget_s)
    while True:
        for r in range(inp.batch):
            decode(inp.q, inp.kcache, inp.block_table, inp.cache_seqlens, inp.softmax_scale, inp.causal,
                   requests=[r])
            done.append(r)
            if time.perf_counter() - t0 >= budget_s:
                return time.perf_counter() - t0, done, passes
        passes += 1
        if time.perf_counter() - t0 >= floor:
            return time.perf_counter() - t0, done, passes


def cpu_baseline(inp, name: str, unit: str, budget_s: float):
    secs, reqs, passes = oracle_sample(inp, budget_s)
    lens = [int(inp.cache_seqlens[r]) for r in reqs]
    cost = cost_of(inp, lens)
    what = (f"{passes} full pass(es) over the {inp.batch} requests" if len(reqs) == passes * inp.batch
            else f"{len(reqs)} request(s) in order")
    return {"value": throughput(cost, secs, unit), "unit": unit, "cores": torch.get_num_threads(),
            "kind": "oracle",
            "sample": f"{what} of the {name} workload, fp64 torch CPU, {secs:.1f} s"}


def run_reference(args, name: str):
    world, rank, _ = dist_env()
    if rank != 0:
        return 0
    unit = unit_of(name)
    inp = make_workload(name)
    per_step = max(0.05, min(10.0, 150.0 / max(1, args.steps + args.warmup)))  # whole run ~150 s of CPU
    for _ in range(args.warmup):
        oracle_sample(inp, per_step, per_step)
    vals, secs_tot = [], 0.0
    for _ in range(args.steps):
        secs, reqs, _ = oracle_sample(inp, per_step, per_step)
        lens = [int(inp.cache_seqlens[r]) for r in reqs]
        vals.append(throughput(cost_of(inp, lens), secs, unit))
        secs_tot += secs
    value = statistics.median(vals)
    w = WORKLOADS[name]
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": unit, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000.0 * secs_tot / max(1, args.steps),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": workload_config(name, world),
        "cpu_baseline": {"value": value, "unit": unit, "cores": torch.get_num_threads(), "kind": "oracle",
                         "sample": f"each step: requests of the {w.name} workload in order (cycling) until "
                                   f"{per_step:.1f} s of fp64 CPU work (median over steps)"},
        "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def workload_config(name: str, world: int):
    w = WORKLOADS[name]
    return {"workload": name, "description": w.description, "batch_per_gpu": w.batch, "global_batch": w.batch * world,
            "s_q": w.s_q, "h_q": w.h_q, "d_k": 576, "d_v": 512, "page": 64, "causal": w.causal,
            "l2": "inputs larger than L2; two resident cache copies alternate between steps",
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU"}


# ----------------------------------------------------------------------------- GPU leg
def init_dist():
    world, rank, local = dist_env()
    if world > 1:
        import datetime

        import torch.distributed as dist

        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return world, rank, torch.device("cuda", torch.cuda.current_device())


def measure_gpu(name: str, steps: int, warmup: int, world: int, rank: int, dev, cpu_seconds: float,
                variant: str = "auto"):
    """Device throughput, split-KV kernel time, end-to-end throughput (and, on rank 0 of a 1-GPU run
    with cpu_seconds > 0, the CPU oracle's) of one workload.  Every rank makes the same collective
    calls in the same order; rank 0 gets the result dict, the others None."""
    import mla_decode_attention_16_b200 as mla

    w = WORKLOADS[name]
    if w.kv_fp8:
        variant = "auto"  # the e5m2-cache kernel has no variants
    mla.mla_set_kernel_variant(variant)
    unit = unit_of(name)
    if rank == 0:
        inp = make_workload(name)
    else:
        import workloads as wl
        g = torch.Generator().manual_seed(shard_seed(w.seed, rank))  # same shapes and length law
        lens = wl.draw_seqlens(w, g)
        inp = wl.make_case(w.batch, w.s_q, w.h_q, lens, dtype=w.dtype, std=w.std, causal=w.causal,
                           seed=shard_seed(w.seed, rank) + 1, kv_fp8=w.kv_fp8)
    lens = [int(x) for x in inp.cache_seqlens.tolist()]
    cost = cost_of(inp, lens)

    b, s_q, h_q = inp.batch, inp.s_q, inp.h_q
    rows = s_q * h_q
    q = inp.q.to(dev)
    caches = [inp.kcache.to(dev), inp.kcache.to(dev)]
    bt = inp.block_table.to(dev)
    sl = inp.cache_seqlens.to(dev)
    parts = mla.mla_get_num_sm_parts(rows, dev.index, kv_fp8=w.kv_fp8)
    meta = torch.empty(parts, 8, dtype=torch.int32, device=dev)
    ns = torch.empty(b + 1, dtype=torch.int32, device=dev)
    ws = mla.alloc_workspace(b, rows, parts, dev)
    out = torch.empty(b, s_q, h_q, 512, dtype=q.dtype, device=dev)
    lse = torch.empty(b, h_q, s_q, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(i):
        mla.mla_get_metadata(sl, rows, parts, meta, ns, stream=stream)
        mla.mla_decode_fwd(q, caches[i & 1], bt, sl, inp.softmax_scale, inp.causal, meta, ns, ws, out, lse,
                           stream=stream)

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier()
        torch.cuda.synchronize(dev)

    # ---- warm-up
    for i in range(warmup):
        step(i)
    barrier()
    flags = mla.mla_read_device_status(ws, stream)
    if flags[0] != 0:
        raise RuntimeError(f"{name}: device error flags {flags}")

    # ---- timed region (device throughput, inputs resident)
    clocks = ClockSampler(dev.index)
    est_s = 2e-4 * steps
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    clocks.start()
    torch.cuda._sleep(int(min(est_s, 0.5) * 1.0e9))  # head start so the host enqueues ahead of the GPU
    ev0.record(stream)
    for i in range(steps):
        step(i)
    ev1.record(stream)
    barrier()
    clocks.stop()
    elapsed = ev0.elapsed_time(ev1) / 1000.0
    elapsed_max = reduce_max(elapsed, dev)
    value = throughput(cost, elapsed_max / steps, unit) * world

    # ---- split-KV kernel alone, CUDA events per launch on the launching stream (roofline)
    n_prof = max(3, min(steps, 200))
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n_prof)]
    mla.mla_get_metadata(sl, rows, parts, meta, ns, stream=stream)
    barrier()
    torch.cuda._sleep(int(min(2e-4 * n_prof, 0.5) * 1.0e9))
    for i, (a, z) in enumerate(evs):
        a.record(stream)
        mla.mla_splitkv_fwd(q, caches[i & 1], bt, sl, inp.softmax_scale, inp.causal, meta, ns, ws, out, lse,
                            stream=stream)
        z.record(stream)
    barrier()
    kern_s = reduce_max(statistics.mean(a.elapsed_time(z) for a, z in evs) / 1000.0, dev)

    # ---- end to end through the public API with pinned host buffers.  A serving loop pipelines
    # steps: step i's inputs go host -> device on one stream while step i-1 computes on another
    # and step i-2's result comes back on a third; device inputs and outputs are double-buffered
    # and events order every reuse.  Every step still copies its q, block table and lengths in
    # and its out and lse back.
    q_h = inp.q.pin_memory()
    bt_h = inp.block_table.pin_memory()
    sl_h = inp.cache_seqlens.pin_memory()
    out_h = [torch.empty(out.shape, dtype=out.dtype).pin_memory() for _ in range(2)]
    lse_h = [torch.empty(lse.shape, dtype=lse.dtype).pin_memory() for _ in range(2)]
    h2d = q_h.numel() * q_h.element_size() + bt_h.numel() * 4 + sl_h.numel() * 4
    d2h = out_h[0].numel() * out_h[0].element_size() + lse_h[0].numel() * 4
    n_e2e = max(3, min(steps, 200))
    q_d = [torch.empty_like(q) for _ in range(2)]
    bt_d = [torch.empty_like(bt) for _ in range(2)]
    sl_d = [torch.empty_like(sl) for _ in range(2)]
    out_d = [torch.empty_like(out) for _ in range(2)]
    lse_d = [torch.empty_like(lse) for _ in range(2)]
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_comp = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    used = [False, False]

    def e2e_step(i):
        k = i & 1
        with torch.cuda.stream(s_in):
            if used[k]:
                s_in.wait_event(ev_comp[k])  # step i-2 has finished reading q_d[k]
            q_d[k].copy_(q_h, non_blocking=True)
            bt_d[k].copy_(bt_h, non_blocking=True)
            sl_d[k].copy_(sl_h, non_blocking=True)
            ev_in[k].record(s_in)
        stream.wait_event(ev_in[k])
        if used[k]:
            stream.wait_event(ev_out[k])  # step i-2's result has left out_d[k]
        mla.mla_get_metadata(sl_d[k], rows, parts, meta, ns, stream=stream)
        mla.mla_decode_fwd(q_d[k], caches[i & 1], bt_d[k], sl_d[k], inp.softmax_scale, inp.causal, meta, ns, ws,
                           out_d[k], lse_d[k], stream=stream)
        ev_comp[k].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_comp[k])
            out_h[k].copy_(out_d[k], non_blocking=True)
            lse_h[k].copy_(lse_d[k], non_blocking=True)
            ev_out[k].record(s_out)
        used[k] = True

    for i in range(4):
        e2e_step(i)
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    # the same head start as the device-time loop: the host enqueues the steps while the input
    # stream sleeps, so the timed region measures the copies and kernels of a loop whose host keeps
    # ahead of the GPU (as a serving loop replaying CUDA graphs does), not Python's call overhead;
    # every step's copies in and out are still inside it
    with torch.cuda.stream(s_in):
        torch.cuda._sleep(int(min(4e-4 * n_e2e, 0.5) * 1.0e9))
    e0.record(s_in)
    for i in range(n_e2e):
        e2e_step(i)
    e1.record(s_out)  # after the last step's result is back on the host
    barrier()
    e2e_s = reduce_max(e0.elapsed_time(e1) / 1000.0 / n_e2e, dev)
    e2e_value = throughput(cost, e2e_s, unit) * world
    flags = mla.mla_read_device_status(ws, stream)
    if flags[0] != 0:
        raise RuntimeError(f"{name}: device error flags {flags}")
    del caches, q_d, out_d
    if rank != 0:
        return None

    peaks, peak_src = load_peaks()
    if unit == "GB/s":
        achieved = cost["bytes"] / kern_s / 1e9
        peak = float(peaks["hbm_gbs"])
        roof = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak}
    else:
        achieved = cost["flops"] / kern_s / 1e12
        peak = tensor_peak(peaks, w.kv_fp8)
        roof = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak}
    kname, ksrc = kernel_of(rows, variant, w.kv_fp8)
    roof["traffic"] = profile_traffic(name, kname, ksrc)
    roof.update(roofline_extras(unit, achieved, peaks, w.kv_fp8, read_stream_gbs(dev) if unit == "GB/s" else None))
    roof["peak_source"] = f"{peak_src} (MEASURED_PEAKS.json)" if peak_src == "measured" else "fallback"
    roof["kernel"] = kname
    roof["variant"] = "fp8-cache" if w.kv_fp8 else variant_of(rows, variant)
    roof["kernel_us"] = kern_s * 1e6
    roof["algorithmic_per_launch"] = cost["bytes"] if unit == "GB/s" else cost["flops"]
    res = {
        "value": value, "unit": unit, "steps": steps, "warmup": warmup,
        "ms_per_step": 1000.0 * elapsed_max / steps,
        "dtype": ("e5m2 q.k, fp16 p.v, " if w.kv_fp8 else "") + ("bf16" if q.dtype == torch.bfloat16 else "fp16"),
        "config": workload_config(name, world),
        "tflops": cost["flops"] / (elapsed_max / steps) / 1e12 * world,
        "gbps": cost["bytes"] / (elapsed_max / steps) / 1e9 * world,
        "roofline": roof,
        "e2e": {"value": e2e_value, "unit": unit, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": 3 * steps,
        "clocks": clocks.summary(),
    }
    if world == 1 and cpu_seconds > 0:
        res["cpu_baseline"] = cpu_baseline(inp, name, unit, cpu_seconds)
    return res


# ----------------------------------------------------------------------------- row-count study
SWEEP_H = (16, 32, 64, 128)
SWEEP_S = (1, 2, 4, 8)


def sweep_shapes():
    """(h_q, s_q) pairs of the row-count study: every combination, s_q * h_q up to 1024 rows."""
    return [(h, sq) for h in SWEEP_H for sq in SWEEP_S if h * sq <= 1024]


def variants_for(rows: int):
    """Kernel variants that can run s_q * h_q = rows query rows."""
    if rows <= 32:
        return ["few-rows-one-cta", "few-rows-pair", "row-tile-pair"]
    return ["row-tile-pair"]


def binding_roof(cost: dict, peaks: dict):
    """(seconds at the binding roofline, which roof) for one call: the larger of HBM time and
    tensor time at the measured peaks."""
    t_hbm = cost["bytes"] / (float(peaks["hbm_gbs"]) * 1e9)
    t_tc = cost["flops"] / (float(peaks["bf16_tflops"]) * 1e12)
    return (t_hbm, "hbm") if t_hbm >= t_tc else (t_tc, "tensor")


def run_sweep(args):
    """Split-KV kernel time of every kernel variant over h_q x s_q (batch 64, 4096 cached tokens per
    request, bf16, causal when s_q > 1): one JSON line per (shape, variant) with the fraction of the
    binding roofline, then one line naming the fastest variant per row count."""
    import mla_decode_attention_16_b200 as mla
    from workloads import make_case

    world, rank, dev = init_dist()
    peaks, _ = load_peaks()
    best = {}
    for h, sq in sweep_shapes():
        rows = h * sq
        inp = make_case(64, sq, h, [4096] * 64, causal=sq > 1, seed=5000 + rows + h)
        lens = [4096] * 64
        cost = algorithmic_cost(lens, sq, h)
        q = inp.q.to(dev)
        caches = [inp.kcache.to(dev), inp.kcache.to(dev)]
        bt, sl = inp.block_table.to(dev), inp.cache_seqlens.to(dev)
        out = torch.empty(64, sq, h, 512, dtype=q.dtype, device=dev)
        lse = torch.empty(64, h, sq, dtype=torch.float32, device=dev)
        stream = torch.cuda.current_stream(dev)
        for variant in variants_for(rows):
            mla.mla_set_kernel_variant(variant)
            parts = mla.mla_get_num_sm_parts(rows, dev.index)
            meta, ns = mla.mla_get_metadata(sl, rows, parts)
            ws = mla.alloc_workspace(64, rows, parts, dev)
            for i in range(max(3, args.warmup)):
                mla.mla_splitkv_fwd(q, caches[i & 1], bt, sl, inp.softmax_scale, inp.causal, meta, ns, ws, out, lse,
                                    stream=stream)
            torch.cuda.synchronize(dev)
            n = max(3, min(args.steps, 50))
            evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
            for i, (a, z) in enumerate(evs):
                a.record(stream)
                mla.mla_splitkv_fwd(q, caches[i & 1], bt, sl, inp.softmax_scale, inp.causal, meta, ns, ws, out, lse,
                                    stream=stream)
                z.record(stream)
            torch.cuda.synchronize(dev)
            flags = mla.mla_read_device_status(ws, stream)
            if flags[0] != 0:
                raise RuntimeError(f"sweep h_q {h} s_q {sq} {variant}: device error flags {flags}")
            secs = statistics.median(a.elapsed_time(z) for a, z in evs) / 1000.0
            roof_s, bound = binding_roof(cost, peaks)
            line = {"mode": "sweep", "h_q": h, "s_q": sq, "rows": rows, "variant": variant,
                    "kernel": KERNELS[variant][0], "kernel_us": secs * 1e6, "gbps": cost["bytes"] / secs / 1e9,
                    "tflops": cost["flops"] / secs / 1e12, "bound": bound, "frac": roof_s / secs,
                    "config": "batch 64, 4096 cached tokens per request, bf16, causal when s_q > 1"}
            if rank == 0:
                print(json.dumps(line), flush=True)
            if rows not in best or secs < best[rows][1]:
                best[rows] = (variant, secs)
            del ws
        del caches, q
        torch.cuda.empty_cache()
    mla.mla_set_kernel_variant("auto")
    if rank == 0:
        print(json.dumps({"mode": "sweep-best", "fastest": {str(r): v for r, (v, _) in sorted(best.items())}}),
              flush=True)
    return 0


# workloads whose numbers join the headline line of a default run: the pages' h_q * s_q >= 128
# configs, and the memory- and compute-bound batches over an e5m2 cache
COMPANIONS = ["compute-bound", "varlen-mtp", "long-fp16", "memory-bound-fp8", "compute-bound-fp8"]


def run_gpu(args, name: str, companions=()):
    world, rank, dev = init_dist()
    cpu_s = 0.0 if args.no_cpu_baseline else args.cpu_seconds
    head = measure_gpu(name, args.steps, args.warmup, world, rank, dev, cpu_s, args.variant)
    extra = {}
    for other in companions:
        torch.cuda.empty_cache()
        extra[other] = measure_gpu(other, min(args.steps, args.companion_steps), args.warmup, world, rank, dev,
                                   0.0 if args.no_cpu_baseline else args.companion_cpu_seconds, args.variant)
    if rank == 0:
        line = {"metric": METRIC, "value": head["value"], "unit": head["unit"], "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": head["ms_per_step"],
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": head["dtype"],
                "data": "synthetic"}
        for k in ("config", "tflops", "gbps", "roofline", "e2e", "gpu_launches", "clocks", "cpu_baseline"):
            if k in head:
                line[k] = head[k]
        if extra:
            line["per_workload"] = extra
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(WORKLOADS) + ["all", "sweep"])
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--companion-steps", type=int, default=200,
                    help="timed steps of each h_q*s_q >= 128 workload added to a default run's line")
    ap.add_argument("--companion-cpu-seconds", type=float, default=5.0)
    ap.add_argument("--variant", default="auto",
                    choices=["auto", "few-rows-one-cta", "few-rows-pair", "row-tile-pair"],
                    help="split-KV kernel variant (default: the library's choice by row count)")
    ap.add_argument("--headline-only", action="store_true",
                    help="a default run measures only the headline workload")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        names = [n for n in WORKLOADS if n != "tiny"] if args.workload == "all" else [args.workload]
        for name in names:
            rc = run_reference(args, name)
            if rc:
                return rc
        return 0
    if args.workload == "sweep":
        return run_sweep(args)
    if args.workload == "all":
        for name in [n for n in WORKLOADS if n != "tiny"]:
            rc = run_gpu(args, name)
            if rc:
                return rc
        return 0
    given = argv if argv is not None else sys.argv[1:]
    default_run = not any(a.startswith("--workload") for a in given)
    companions = COMPANIONS if default_run and not args.headline_only else ()
    return run_gpu(args, args.workload, companions)


if __name__ == "__main__":
    sys.exit(main())
