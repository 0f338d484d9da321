"""Host-side logic of bench.py (no GPU): kernel choice, cost model, units, seeds, profile lookup."""

import hashlib
import importlib
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

bench = importlib.import_module("bench")
from workloads import WORKLOADS, algorithmic_cost  # noqa: E402


def test_kernel_choice_by_rows():
    assert bench.kernel_of(1)[0] == "splitkv_narrow_kernel"
    assert bench.kernel_of(32) == ("splitkv_narrow_kernel", "splitkv_narrow.cu")
    assert bench.kernel_of(16, "few-rows-pair") == ("splitkv_npair_kernel", "splitkv_npair.cu")
    assert bench.kernel_of(33) == ("splitkv_pair_kernel", "splitkv.cu")
    assert bench.kernel_of(1024)[0] == "splitkv_pair_kernel"
    assert bench.kernel_of(16, "few-rows-one-cta") == ("splitkv_narrow_kernel", "splitkv_narrow.cu")
    assert bench.kernel_of(16, "row-tile-pair")[0] == "splitkv_pair_kernel"
    assert bench.variant_of(16) == "few-rows-one-cta" and bench.variant_of(128) == "row-tile-pair"


def test_cost_model_by_hand():
    # two requests of 64 and 100 cached tokens, s_q 2, h_q 8: 16 rows, 164 tokens
    c = algorithmic_cost([64, 100], 2, 8)
    assert c["tokens"] == 164
    assert c["flops"] == 2 * 16 * (576 + 512) * 164
    assert c["kv_bytes"] == 576 * 2 * 164
    assert c["bytes"] == 576 * 2 * 164 + 2 * 16 * (576 * 2 + 512 * 2 + 4)


def test_units_and_throughput():
    assert bench.unit_of("memory-bound") == "GB/s"
    for name in ("compute-bound", "varlen-mtp", "long-fp16"):
        assert bench.unit_of(name) == "TFLOPS", name
    cost = {"bytes": 3e9, "flops": 5e12}
    assert bench.throughput(cost, 0.5, "GB/s") == pytest.approx(6.0)
    assert bench.throughput(cost, 0.5, "TFLOPS") == pytest.approx(10.0)


def test_shard_seeds():
    seeds = [bench.shard_seed(1001, r) for r in range(8)]
    assert seeds[0] == 1001  # rank 0 runs the workload itself
    assert len(set(seeds)) == 8


def test_warmup_minimum_is_enforced():
    with pytest.raises(SystemExit):
        bench.main(["--warmup", "2", "--steps", "1"])


def test_profile_traffic_only_for_the_source_it_was_taken_from(tmp_path, monkeypatch):
    csrc = tmp_path / "mla_decode_attention_16_b200" / "csrc"
    csrc.mkdir(parents=True)
    (tmp_path / "profiles").mkdir()
    src = csrc / "splitkv.cu"
    src.write_bytes(b"// kernel source\n")
    digest = hashlib.sha256(src.read_bytes()).hexdigest()[:16]
    prof = tmp_path / "profiles" / "splitkv_pair_kernel_compute-bound.md"
    prof.write_text(f"splitkv.cu sha256[:16]: {digest}\ntraffic_bytes_per_launch: 628559360.0\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.profile_traffic("compute-bound", "splitkv_pair_kernel", "splitkv.cu") == 628559360.0
    src.write_bytes(b"// kernel source, changed\n")  # counters no longer describe this kernel
    assert bench.profile_traffic("compute-bound", "splitkv_pair_kernel", "splitkv.cu") is None
    assert bench.profile_traffic("memory-bound", "splitkv_narrow_kernel", "splitkv_narrow.cu") is None


def test_every_bench_workload_has_a_profile_summary():
    for name in WORKLOADS:
        if name == "tiny":
            continue
        kernel, _ = bench.kernel_of(WORKLOADS[name].rows, kv_fp8=WORKLOADS[name].kv_fp8)
        assert os.path.exists(os.path.join(ROOT, "profiles", f"{kernel}_{name}.md")), name


def test_sweep_shapes_and_variants():
    shapes = bench.sweep_shapes()
    assert (16, 1) in shapes and (128, 8) in shapes and len(shapes) == 16
    assert all(h * s <= 1024 for h, s in shapes)
    assert bench.variants_for(32) == ["few-rows-one-cta", "few-rows-pair", "row-tile-pair"]
    assert bench.variants_for(33) == ["row-tile-pair"]


def test_binding_roof_picks_the_slower_roof():
    peaks = {"hbm_gbs": 1000.0, "bf16_tflops": 100.0}
    t, b = bench.binding_roof({"bytes": 2e9, "flops": 1e12}, peaks)  # 2 ms of HBM vs 10 ms of tensor
    assert b == "tensor" and abs(t - 0.01) < 1e-12
    t, b = bench.binding_roof({"bytes": 2e10, "flops": 1e12}, peaks)
    assert b == "hbm" and abs(t - 0.02) < 1e-12


def test_fp8_workload_host_logic():
    """The e5m2-cache workload: its kernel, a cost model at one byte per cached value, and the FP8
    oracle for the CPU leg."""
    import torch

    import oracle
    from workloads import make_case

    assert bench.kernel_of(16, kv_fp8=True) == ("splitkv_fp8_kernel", "splitkv_fp8.cu")
    assert bench.kernel_of(32, kv_fp8=True)[0] == "splitkv_fp8_kernel"
    assert bench.kernel_of(33, kv_fp8=True) == ("splitkv_fp8_rt_kernel", "splitkv_fp8_rt.cu")
    assert bench.kernel_of(1024, "row-tile-pair", kv_fp8=True)[0] == "splitkv_fp8_rt_kernel"
    assert WORKLOADS["memory-bound-fp8"].kv_fp8 and not WORKLOADS["memory-bound"].kv_fp8
    assert "memory-bound-fp8" in bench.COMPANIONS
    inp8 = make_case(2, 1, 16, [100, 64], seed=3, kv_fp8=True)
    inp16 = make_case(2, 1, 16, [100, 64], seed=3)
    assert inp8.kcache.dtype == torch.uint8
    c8, c16 = bench.cost_of(inp8, [100, 64]), bench.cost_of(inp16, [100, 64])
    assert c8["kv_bytes"] == 576 * 164 and c16["kv_bytes"] == 2 * 576 * 164
    assert c8["flops"] == c16["flops"]
    assert bench.oracle_fn(inp8) is oracle.mla_decode_fp8_ref
    assert bench.oracle_fn(inp16) is oracle.mla_decode_ref


def test_tensor_peak_blends_fp8_and_fp16():
    """Over an e5m2 cache Q.K^T (576 of 1088 FLOPs per key) runs at twice the 16-bit rate."""
    peaks = {"bf16_tflops": 1000.0}
    assert bench.tensor_peak(peaks, False) == 1000.0
    blended = bench.tensor_peak(peaks, True)
    assert abs(blended - 1088.0 / (576.0 / 2000.0 + 512.0 / 1000.0)) < 1e-9
    assert 1000.0 < blended < 2000.0


def test_roofline_extras_denominators():
    """HBM-bound work is also held to the nominal 8 TB/s and to a read stream of the same run;
    tensor-bound work to the sustained and datasheet bf16 rates, blended for an e5m2 cache like
    the primary peak."""
    peaks = {"bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0}
    h = bench.roofline_extras("GB/s", 4000.0, peaks, False, 6400.0)
    assert h["frac_of_nominal"] == 0.5 and h["frac_of_read_stream"] == 0.625
    assert bench.roofline_extras("GB/s", 4000.0, peaks, False, None)["frac_of_read_stream"] is None
    t = bench.roofline_extras("TFLOPS", 700.0, peaks, False, None)
    assert t["sustained_peak"] == 1400.0 and t["frac_of_sustained"] == 0.5
    assert t["nominal_peak"] == 2250.0
    t8 = bench.roofline_extras("TFLOPS", 700.0, peaks, True, None)
    assert abs(t8["sustained_peak"] - bench.tensor_peak({"bf16_tflops": 1400.0}, True)) < 1e-9
    assert abs(t8["nominal_peak"] - bench.tensor_peak({"bf16_tflops": 2250.0}, True)) < 1e-9
