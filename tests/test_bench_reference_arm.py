"""bench.py --impl reference (the float64 oracle timed on the host cores)
prints one JSON line with the contract's keys; it needs no GPU (CPU)."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_prints_one_contract_line():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "0"], capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["unit"] == "TFLOP/s" and d["value"] > 0
    assert d["config"]["workload"] == "gqa_causal_prefill_4k_d128"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    # the reference arm describes its workload with the GPU arm's config keys and values
    sys.path.insert(0, ROOT)
    import bench
    from gqa_flash_attention_attn_b200.inputs import WORKLOADS
    assert d["config"] == bench.workload_config(WORKLOADS[bench.HEADLINE], 1)


def test_base_configs_are_compact_and_per_step():
    sys.path.insert(0, ROOT)
    import bench
    from gqa_flash_attention_attn_b200.inputs import WORKLOADS
    assert all(n in WORKLOADS for n in bench.BASE_CONFIGS) and len(bench.BASE_CONFIGS) == 5
    r = {"value": 4831.123456, "unit": "GB/s", "ms_per_step": 0.11123456, "kernel_ms": 0.0989123,
         "roofline": {"frac": 0.73912345, "kernel_frac": 0.8312345, "bound": "hbm", "traffic": None}}
    c = bench.compact(r)
    assert c == {"value": 4831.0, "unit": "GB/s", "ms_per_step": 0.1112, "kernel_ms": 0.09891,
                 "roofline_frac": 0.739, "kernel_frac": 0.831, "bound": "hbm", "traffic": None}
    assert len(json.dumps({n: c for n in bench.BASE_CONFIGS})) < 1200


def test_workload_metric_units():
    sys.path.insert(0, ROOT)
    import bench
    from gqa_flash_attention_attn_b200.inputs import WORKLOADS
    for w in WORKLOADS.values():
        unit, work = bench.workload_metric(w)
        assert unit == ("TFLOP/s" if w.kind == "prefill" else "GB/s") and work > 0
    assert bench.prefill_sources(WORKLOADS["prefill_d512_g16_4k"]) == "prefill_wide"
    assert bench.prefill_sources(WORKLOADS["prefill_d192_v128_4k"]) == "prefill"
