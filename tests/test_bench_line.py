"""bench.py's JSON lines (CPU): the keys the bench contract asks for, and the
same "config" in the GPU arm and the CPU oracle arm, so the two lines
describe one workload."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import gqe_synth  # noqa: E402

REQUIRED = ["metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
            "scaling", "vs_baseline", "dtype", "data", "config"]


def fake_result():
    roof = {"bound": "tensor", "achieved": 900.0, "peak": 1725.8, "unit": "TFLOP/s", "frac": 0.5215,
            "traffic": None, "algorithmic_per_launch": 5.5e11}
    return {"value": 850.0, "unit": "TFLOP/s", "ms_per_step": 0.64, "attn_ms": 0.571, "route_ms": 0.0697,
            "roofline": roof, "clocks": {"sm_mhz": 1965, "sm_max_mhz": 1965, "reasons": []},
            "gpu_launches": 60, "e2e": {"value": 42.0, "unit": "TFLOP/s", "h2d_bytes_per_step": 1,
                                        "d2h_bytes_per_step": 1}}


def fake_extras():
    f = {"roofline": {"frac": 0.5}}
    return {"paged_decode": f, "layer_ops": {"routed_qproj": f, "routed_oproj": f, "shared_head": f,
                                             "group_slots": f},
            "backward": {"ms": 0.62, "roofline": {"frac": 0.32}, "router": {"ms": 0.19}}}


def test_gqe_line_keys():
    w = gqe_synth.WORKLOADS["gqe_prefill"]
    line = json.loads(json.dumps(bench.gqe_line("m", w, 2, 20, 5, fake_result(), None, {"x": {}}, fake_extras())))
    for key in REQUIRED + ["roofline", "cpu_baseline", "e2e", "clocks", "gpu_launches"]:
        assert key in line, key
    assert line["config"] == bench.workload_config(w, 2)
    assert line["config"]["global_batch"] == 2 * w.B
    assert line["step_breakdown_ms"] == {"route": 0.0697, "attn": 0.571}
    assert line["extras"]["backward_frac"] == 0.32 and "configs" in line


def test_reference_arm_prints_the_same_config():
    w = gqe_synth.WORKLOADS["tiny_f32"]
    proc = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload",
                           w.name, "--steps", "1", "--warmup", "3"],
                          capture_output=True, text=True, timeout=600, cwd=ROOT,
                          env={k: v for k, v in os.environ.items() if k not in ("RANK", "WORLD_SIZE")})
    assert proc.returncode == 0, proc.stderr[-2000:]
    line = json.loads(proc.stdout.strip().splitlines()[-1])
    for key in REQUIRED + ["impl", "cpu_baseline", "e2e"]:
        assert key in line, key
    assert line["impl"] == "reference"
    assert line["config"] == bench.workload_config(w, 1)
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["value"] > 0
