"""Host logic of bench.py that needs no GPU.

- The profiled DRAM traffic is reported only for the kernel source it was captured from.
- The reference arm (the float64 oracle on the host cores) reports the time it actually ran,
  keeps its extrapolation to the whole batch in a key of its own, and carries the same
  `config` as the GPU arm.
"""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_code_hash_ignores_comments_and_whitespace(tmp_path):
    a, b, c = tmp_path / "a.cu", tmp_path / "b.cu", tmp_path / "c.cu"
    a.write_text("int f(int x) { return x + 1; }  // one\n")
    b.write_text("/* block\n   comment */\nint f(int x)\n{\n  return x + 1;\n}\n")
    c.write_text("int f(int x) { return x + 2; }\n")
    assert bench.code_sha256_16(str(a)) == bench.code_sha256_16(str(b))
    assert bench.code_sha256_16(str(a)) != bench.code_sha256_16(str(c))


def test_traffic_is_used_only_for_the_profiled_source(tmp_path, monkeypatch):
    src = tmp_path / "tree_speculative_decoding_kd_b200" / "csrc"
    src.mkdir(parents=True)
    kernel = src / "kd_attn_tc.cu"
    kernel.write_text("__global__ void k() {}\n")
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "attn_loop_traffic.json").write_text(json.dumps(
        {"traffic_bytes_per_launch": 123, "kernel_code_sha256_16": bench.code_sha256_16(str(kernel))}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.profiled_traffic() == 123
    kernel.write_text("__global__ void k() {}  // a comment changes nothing\n")
    assert bench.profiled_traffic() == 123
    kernel.write_text("__global__ void k() { int x = 0; (void)x; }\n")
    assert bench.profiled_traffic() is None


def test_committed_traffic_belongs_to_the_committed_kernel():
    # profiles/attn_loop_traffic.json is re-captured whenever the attention's code changes
    assert bench.profiled_traffic() is not None


def test_reference_arm_reports_what_it_ran():
    run = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--steps", "1", "--warmup", "0"],
                         capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert run.returncode == 0, run.stderr[-2000:]
    line = json.loads(run.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0 and line["dtype"] == "f64"
    # the time measured per step, and (larger) the extrapolation to every request
    assert 0 < line["ms_per_step"] < line["extrapolated_ms_per_step"]
    assert line["e2e"] == {"value": line["value"], "unit": line["unit"], "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    # the GPU arm builds its config from the same function and workload
    assert line["config"] == json.loads(json.dumps(bench.config_json(bench.workload_cfg(0, 1))))
    assert "parallelism" not in line["config"]
