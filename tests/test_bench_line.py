"""The benchmark's JSON line, assembled on CPU from synthetic measurements:
every key the line must carry is there, the throughput arithmetic is right,
and every extra measurement carries a roofline fraction of its own peak."""
import json
import types

import pytest

import bench
from ring_ulysses_sequence_b200.synth import BENCH_WORKLOAD, WORKLOADS


def _out():
    w = WORKLOADS[BENCH_WORKLOAD]
    return {
        "fwd": {"ms_total": 160.0, "launches": 20, "bytes_in": 403e6, "bytes_out": 273e6,
                "clocks": {"sm_mhz": 1700, "sm_max_mhz": 1965, "reasons": ["sw_power_cap"]},
                "e2e": {"ms_per_step": 8.5, "h2d": 402653184, "d2h": 272629760, "steps": 20}},
        "permute": {"workload": "usp", "ms_per_launch": 0.5, "gbs": 6400.0,
                    "bytes_per_launch": 3.2e9, "launches": 25},
        "layout": {"seq_reorder": {"ms": 0.09, "bytes_per_launch": 5.4e8, "gbs": 6000.0},
                   "lse_merge": {"ms": 0.25, "bytes_per_launch": 1.6e9, "gbs": 6500.0}},
        "allgather": {"workload": w.name, "ms_per_step": 8.0, "ms_attention": 7.9,
                      "tflops": 1100.0, "tflops_attention": 1110.0,
                      "flops_per_launch": w.fwd_flops(),
                      "kv_bytes_per_rank": {"ring": 1, "allgather": 4}},
        "steps": {"workload": w.name, "ms_per_step": 10.6, "tflops": 830.0,
                  "launches_per_step": 66, "flops_per_step": w.fwd_flops(),
                  "ms_per_step_two_calls": 12.6, "tflops_two_calls": 698.0},
        "bwdsteps": {"workload": w.name, "ms_per_step": 30.0, "tflops": 733.0,
                     "launches_per_step": 75, "flops_per_step": 2.5 * w.fwd_flops()},
        "exchange": {"workload": "usp", "ms_per_step": 1.0, "gbs": 6400.0,
                     "bytes_per_step": 6.4e9, "launches_per_step": 32},
        "window": {"workload": "win", "window": 4096, "docs": 0, "ms_per_launch": 2.0,
                   "tflops": 1000.0, "flops_per_launch": 2e12, "launches": 25},
        "packed": {"workload": "packed", "window": 0, "docs": 7, "ms_per_launch": 1.5,
                   "tflops": 900.0, "flops_per_launch": 1.4e12, "launches": 25},
        "bwd": {"workload": "bwd64k", "ms_per_step": 100.0, "tflops": 880.0,
                "flops_per_step": 8.8e13, "ms_fused": 140.0, "tflops_fused": 628.0},
    }


@pytest.mark.parametrize("world", [1, 4])
def test_line_carries_the_contract(world):
    w = WORKLOADS[BENCH_WORKLOAD]
    args = types.SimpleNamespace(steps=20, warmup=3, skip_cpu=True, only="all")
    peaks, src = {"hbm_gbs": 6450.3, "bf16_tflops": 1672.7, "bf16_tflops_sustained": 1414.8}, \
        "measured"
    line = bench.build_line(_out(), w, args, world, peaks, src)
    json.dumps(line)                                   # serialisable as one line
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "roofline", "e2e", "clocks", "gpu_launches"):
        assert key in line, key
    assert line["n_gpus"] == world and line["steps"] == 20 and line["warmup"] == 3
    assert line["config"]["workload"] == w.name
    # whole-job throughput: every rank did the workload once per step
    ms_step = 160.0 / 20
    assert line["ms_per_step"] == pytest.approx(ms_step)
    assert line["value"] == pytest.approx(world * w.fwd_flops() / (ms_step * 1e-3) / 1e12)
    r = line["roofline"]
    for key in ("bound", "achieved", "peak", "unit", "frac", "traffic"):
        assert key in r, key
    assert r["frac"] == pytest.approx(r["achieved"] / r["peak"])
    assert r["achieved"] == pytest.approx(w.fwd_flops() / (ms_step * 1e-3) / 1e12)
    e = line["e2e"]
    assert e["h2d_bytes_per_step"] > 0 and e["d2h_bytes_per_step"] > 0
    assert e["value"] == pytest.approx(world * w.fwd_flops() / (8.5e-3) / 1e12)
    extra = line["extra"]
    for name in ("ulysses_permute_qkv", "seq_reorder", "lse_merge", "allgather_attn_fwd",
                 "ring_attn_fwd_step", "ring_attn_fwd_window", "ring_attn_fwd_varlen",
                 "ring_attn_bwd"):
        rf = extra[name]["roofline"]
        assert rf["frac"] == pytest.approx(rf["achieved"] / rf["peak"]), name
    assert extra["ring_attn_bwd"]["roofline"]["peak"] == 1414.8   # a long step: sustained
    bwd = extra["ring_attn_bwd"]
    assert bwd["roofline"]["frac_fused"] == pytest.approx(bwd["TFLOPS_fused"] / 1414.8)


def test_line_without_the_forward_keeps_the_extras():
    w = WORKLOADS[BENCH_WORKLOAD]
    args = types.SimpleNamespace(steps=5, warmup=3, skip_cpu=True, only="permute")
    out = {"permute": _out()["permute"]}
    line = bench.build_line(out, w, args, 1, {"hbm_gbs": 6450.3, "bf16_tflops": 1672.7,
                                             "bf16_tflops_sustained": 1414.8}, "measured")
    assert "value" not in line and list(line["extra"]) == ["ulysses_permute_qkv"]


def test_traffic_only_from_a_summary_of_the_current_source(tmp_path, monkeypatch):
    src = tmp_path / "k.cu"
    src.write_text("kernel v1")
    prof = tmp_path / "profiles"
    prof.mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    digest = bench.source_digest(["k.cu"])
    (prof / "s.txt").write_text(f"source_sha256: {digest}\ndram_bytes_per_launch: 123\n")
    assert bench.profile_traffic("s.txt", ["k.cu"]) == 123.0
    src.write_text("kernel v2")                        # the kernel changed since the capture
    assert bench.profile_traffic("s.txt", ["k.cu"]) is None
    assert bench.profile_traffic("missing.txt", ["k.cu"]) is None
