"""CPU: host-side logic of bench.py's measurement lines (roofline object,
stored DRAM traffic and its staleness check, per-kernel work formulas, the
reference arm's line)."""
import json
import os

import pytest

import bench
from medusa_head_speculative_02_b200 import kernel_bench as KB
from medusa_head_speculative_02_b200.synthetic import CONFIGS

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PK = {"hbm_gbs": 6500.0, "bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0,
      "src": "measured"}


def test_roofline_hbm_and_tensor_bound():
    # 3.25 GB in 1 ms against 6500 GB/s: HBM floor 0.5 ms; 8e11 flop against
    # 1600 TF/s: tensor floor 0.5 ms (ties go to HBM)
    pk = dict(PK, bf16_tflops=1600.0)
    r = bench.classify({"avg_ms": 1.0, "calls": 50, "algorithmic_bytes": 3.25e9,
                        "achieved": 3250.0, "algorithmic_flops": 8e11, "tflops": 800.0,
                        "tensor_frac": 0.5, "tensor_frac_sustained": 800 / 1400}, pk)
    assert r["bound"] == "hbm" and r["floor_ms"] == pytest.approx(0.5)
    line = bench.roofline_of("tree_attention", r, pk, "no_such_workload")
    assert line["unit"] == "GB/s" and line["peak"] == 6500.0
    assert line["frac"] == pytest.approx(0.5) and line["traffic"] is None
    assert line["roofline_frac"] == pytest.approx(0.5)
    # twice the flops: tensor-bound, floor 1.0 ms, frac against the bf16 peak
    r = bench.classify({"avg_ms": 1.25, "calls": 50, "algorithmic_bytes": 3.25e9,
                        "achieved": 2600.0, "algorithmic_flops": 1.6e12, "tflops": 1280.0,
                        "tensor_frac": 0.8, "tensor_frac_sustained": 1280 / 1400}, pk)
    assert r["bound"] == "tensor" and r["floor_ms"] == pytest.approx(1.0)
    assert r["frac"] == pytest.approx(0.8) and r["hbm_frac"] == pytest.approx(0.4)
    line = bench.roofline_of("tree_attention", r, pk, "no_such_workload")
    assert line["unit"] == "TFLOP/s" and line["frac"] == pytest.approx(0.8)
    assert line["hbm_frac"] == pytest.approx(0.4) and line["roofline_frac"] == pytest.approx(0.8)
    # no flops: HBM-bound
    r = bench.classify({"avg_ms": 2.0, "calls": 5, "algorithmic_bytes": 6.5e9,
                        "achieved": 3250.0}, pk)
    assert r["bound"] == "hbm" and r["frac"] == pytest.approx(0.5)


def test_stored_traffic_goes_stale_when_sources_change(tmp_path):
    digest = bench._source_digest(*bench.TRAFFIC_SOURCES["tree_attention"])
    path = tmp_path / "t.json"
    path.write_text(json.dumps({"w": {"tree_attention": {"bytes_per_call": 123,
                                                         "sources_sha16": digest}}}))
    assert bench.stored_traffic("w", "tree_attention", str(path)) == 123
    path.write_text(json.dumps({"w": {"tree_attention": {"bytes_per_call": 123,
                                                         "sources_sha16": "0" * 16}}}))
    assert bench.stored_traffic("w", "tree_attention", str(path)) is None
    assert bench.stored_traffic("other", "tree_attention", str(path)) is None


def test_work_formulas_at_the_long_context_workload():
    c = CONFIGS["longctx_b4"]
    Lsum = c.B * c.L_hi
    # K and V of prefix + tree slots, Q read and O written
    kv = 2 * (Lsum + c.B * c.N) * c.Hkv * c.dh * 2
    assert KB.attention_bytes(c, Lsum) == kv + 2 * c.B * c.N * c.Hq * c.dh * 2
    assert KB.attention_flops(c, Lsum) == 4 * c.Hq * c.N * (Lsum + c.B * c.N) * c.dh
    assert KB.heads_bytes(c) == 2 * (c.K * c.d * c.d + c.K * c.d + c.K * c.V * c.d + c.B * c.d) \
        + 8 * c.B * c.K * c.s
    assert KB.accept_bytes(c) == c.B * c.N * c.V * 2


def test_rotation_copies():
    assert KB._copies(10 * KB.L2_BYTES) == 1
    assert KB._copies(KB.L2_BYTES // 4) == 12
    assert KB._copies(1) == 16


def test_reference_arm_prints_one_valid_line():
    """`bench.py --impl reference` (the fp64 oracle on the host cores) prints
    one JSON line with the keys the bench contract asks of that arm."""
    import subprocess
    import sys
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--config", "tiny_f32", "--steps", "2", "--warmup", "3"],
                       capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["metric"] == "verify steps/s"
    assert line["value"] > 0 and line["unit"] == "steps/s" and line["higher_is_better"] is True
    assert line["steps"] == 2 and line["warmup"] == 3 and line["n_gpus"] == 1
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["sample"] and cb["value"] == line["value"]
    assert line["e2e"] == {"value": line["value"], "unit": "steps/s", "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}
    assert line["config"]["workload"] == "tiny_f32"
