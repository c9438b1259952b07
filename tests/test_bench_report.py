"""bench.py's JSON line: every key the measurement contract names, and the
roofline arithmetic (achieved = gate/up FLOP / launch time, frac = achieved /
peak) for each kind of gate/up launch.  Pure host code: no GPU."""
import argparse
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from mixture_experts_layer_sqrt_b200 import synth  # noqa: E402

KEYS = ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
        "vs_baseline", "dtype", "data", "config", "roofline", "e2e", "gpu_launches", "clocks")


@pytest.mark.parametrize("name,kind,bound", [("mixtral_bf16", "tc_grouped_gemm", "tensor"),
                                             ("sqrt_fp4", "tc_fp4_gemm", "tensor"),
                                             ("tiny_f32", "grouped_gemm_simt", "alu")])
def test_report_keys_and_roofline(name, kind, bound):
    p = synth.PROBLEMS[name]
    args = argparse.Namespace(steps=10, warmup=3)
    rows = p.T * p.k
    gemm_ms, ms = 1.5, 2.5
    value = bench.whole_job_value(2, p.T, ms)
    e2e = {"value": 1.0, "unit": "tokens/s", "h2d_bytes_per_step": 1, "d2h_bytes_per_step": 1}
    res = bench.report(args, p, 2, rows, value, ms, [ms] * 10, gemm_ms, e2e, 80, None)
    for k in KEYS:
        assert k in res, k
    r = res["roofline"]
    assert r["kernel"].startswith(kind) and r["bound"] == bound and r["unit"] == "TFLOP/s"
    flops = 4.0 * rows * p.D * p.F
    assert r["achieved"] == pytest.approx(flops / (gemm_ms / 1e3) / 1e12)
    assert r["frac"] == pytest.approx(r["achieved"] / r["peak"])
    assert res["value"] == pytest.approx(2 * p.T / (ms / 1e3))
    assert res["n_gpus"] == 2 and res["scaling"] == "weak" and res["vs_baseline"] is None
    assert res["gpu_launches"] == 80 and res["gpu_launches_per_step"] == 8
    assert res["dtype"] == ("f32" if p.act == "f32" else "bf16")


def test_traffic_records_follow_their_kernel_sources(monkeypatch, tmp_path):
    # each recorded DRAM figure is keyed to a hash of its kernel's sources;
    # the record is void as soon as one of them differs
    rec = tmp_path / "traffic.txt"
    sha = bench.gemm_sources_sha(bench.TRAFFIC_SOURCES["gate_up_sqrt_fp4"])
    rec.write_text(f"# comment\ngate_up_sqrt_fp4 {sha} 123456\ngate_up_mixtral_bf16 0000000000000000 99\n")
    assert bench.profiled_traffic("gate_up_sqrt_fp4", str(rec)) == 123456.0
    assert bench.profiled_traffic("gate_up_mixtral_bf16", str(rec)) is None  # stale sources hash
    assert bench.profiled_traffic("gate_up_tiny_f32", str(rec)) is None
    changed = dict(bench.TRAFFIC_SOURCES, gate_up_sqrt_fp4=("gemm_fp4.cu", "api.cu"))
    monkeypatch.setattr(bench, "TRAFFIC_SOURCES", changed)
    assert bench.profiled_traffic("gate_up_sqrt_fp4", str(rec)) is None


def test_extrapolation_arithmetic():
    # ffn_s = 2 + 0.01 n exactly: the fit recovers both parts
    a, b = bench.extrapolate_ffn([(64, 2.64), (256, 4.56), (64, 2.64)])
    assert a == pytest.approx(2.0) and b == pytest.approx(0.01)
    # a decreasing fit falls back to the largest sample's rate through the origin
    a, b = bench.extrapolate_ffn([(64, 3.0), (256, 2.0)])
    assert a == 0.0 and b == pytest.approx(2.0 / 256)
    # one size only: linear through the origin
    a, b = bench.extrapolate_ffn([(32, 1.6)])
    assert a == 0.0 and b == pytest.approx(0.05)


def test_cpu_baseline_fields_small_workload():
    p = synth.PROBLEMS["mixtral_bf16"].with_(name="cb", T=96, D=128, F=64, E=4)
    cb = bench.cpu_baseline_leg(p, sizes=(8, 32))
    for k in ("value", "unit", "cores", "nproc", "threads", "kind", "extrapolated", "route_dispatch_s",
              "ffn_s_per_token", "ffn_fixed_s", "sample"):
        assert k in cb, k
    assert cb["kind"] == "oracle" and cb["extrapolated"] is True and cb["unit"] == "tokens/s"
    assert cb["nproc"] >= 1 and cb["threads"] >= 1 and cb["cores"] == cb["threads"]
    layer_s = cb["route_dispatch_s"] + cb["ffn_fixed_s"] + cb["ffn_s_per_token"] * p.T
    assert cb["value"] == pytest.approx(p.T / layer_s)


def test_reference_arm_line_small_workload():
    p = synth.PROBLEMS["capacity_bf16"].with_(name="ref", T=128, D=128, F=64, E=4)
    args = argparse.Namespace(steps=4, warmup=3)
    res = bench.run_reference(args, p)
    for k in KEYS:
        if k not in ("roofline", "gpu_launches", "clocks"):
            assert k in res, k
    assert res["impl"] == "reference" and res["dtype"] == "f64"
    assert res["cpu_baseline"]["value"] == res["value"]
    assert res["e2e"]["value"] == res["value"] and res["e2e"]["h2d_bytes_per_step"] == 0
    assert res["config"] == bench.workload_config(p, 1, res["config"]["rows_after_capacity"])
    assert 0 < res["config"]["rows_after_capacity"] <= p.T * p.k


def test_permute_combine_bandwidth():
    # Mixtral shape: gather 2 * 8192 rows * 4096 * 2 B, combine 8192 * 4096 * 4 + 4096 * 4096 * 4 B
    p = synth.PROBLEMS["mixtral_bf16"]
    stage_ms = {n: 0.0 for n in bench.STAGES}
    stage_ms.update(gather=0.02, combine=0.03)
    pc = bench.permute_combine(p, 8192, stage_ms, {"hbm": 6000.0, "src": "test"})
    assert pc["gather"]["bytes"] == 2 * 8192 * 4096 * 2
    assert pc["combine"]["bytes"] == 8192 * 4096 * 4 + 4096 * 4096 * 4
    assert pc["gather"]["gbs"] == pytest.approx(pc["gather"]["bytes"] / 0.02e-3 / 1e9)
    assert pc["combine"]["frac"] == pytest.approx(pc["combine"]["gbs"] / 6000.0)
    # the shared expert's fp32 row is read by combine too; NVFP4 rows carry a scale each
    q = synth.PROBLEMS["sqrt_fp4"]
    pq = bench.permute_combine(q, 49152, stage_ms, {"hbm": 6000.0, "src": "test"})
    assert pq["combine"]["bytes"] == 49152 * 4096 * 4 + 2 * 8192 * 4096 * 4
    assert pq["gather"]["bytes"] == 2 * 49152 * 4096 * 2 + 4 * 49152


def test_load_balance_diagnostic_hand_cases():
    # perfectly balanced: T k / E each -> 1; one expert takes everything -> E
    lb = bench.load_balance([4, 4, 4, 4], T=8, k=2)
    assert lb["loss"] == pytest.approx(1.0) and lb["kept"] == 16 and lb["drops"] == 0
    lb = bench.load_balance([16, 0, 0, 0], T=16, k=1)
    assert lb["loss"] == pytest.approx(4.0) and lb["max_count"] == 16 and lb["min_count"] == 0
    # 3 experts, T=3, k=2: counts 3,2,1 -> 3 * ((3/6)^2 + (2/6)^2 + (1/6)^2) = 3 * 14/36
    lb = bench.load_balance([3, 2, 1], T=3, k=2)
    assert lb["loss"] == pytest.approx(3 * 14 / 36)
    # capacity 2: kept min(count, 2) = 2 + 2 + 1, the rest dropped
    lb = bench.load_balance([3, 2, 1], T=3, k=2, capacity=2)
    assert lb["kept"] == 5 and lb["drops"] == 1
