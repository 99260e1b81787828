"""bench.py's reference arm (the fp64 oracle on the host cores) on the CPU: one JSON line
with the contract's keys for each kind of workload, and nothing from ranks other than 0."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(args, env_extra=None):
    env = dict(os.environ)
    env.update(env_extra or {})
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py")] + args, capture_output=True, text=True,
                       env=env, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    return [ln for ln in r.stdout.splitlines() if ln.startswith("{")]


@pytest.mark.parametrize("workload", ["mha2k", "decode8k", "fp8_mha2k"])
def test_reference_arm_prints_one_contract_line(workload):
    lines = _run(["--impl", "reference", "--workload", workload, "--steps", "1", "--warmup", "3"])
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["value"] > 0 and d["steps"] == 1
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["cpu_baseline"]["cores"] >= 1 and d["cpu_baseline"]["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert "workload" in d["config"]


def test_reference_arm_is_silent_on_other_ranks():
    lines = _run(["--impl", "reference", "--steps", "1", "--warmup", "3", "--gpus", "2"],
                 {"RANK": "1", "LOCAL_RANK": "1", "WORLD_SIZE": "2"})
    assert lines == []


def test_warmup_below_three_is_refused():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--warmup", "2"],
                       capture_output=True, text=True, timeout=120, cwd=ROOT)
    assert r.returncode != 0


def test_traffic_record_follows_the_code_not_the_comments(tmp_path):
    """bench.py reports an ncu traffic figure only while the kernel's code is the one the
    counters were taken on: comment and whitespace edits keep the hash, code edits do not."""
    sys.path.insert(0, ROOT)
    import bench
    src = tmp_path / "k.cu"
    src.write_text("// header\n__global__ void k(int* p) {\n  p[0] = 1;  /* store */\n}\n")
    h0 = bench.code_hash(str(src))
    src.write_text("// a longer header\n// over two lines\n__global__ void k(int* p) {\n    p[0] = 1;\n}\n")
    assert bench.code_hash(str(src)) == h0
    src.write_text("__global__ void k(int* p) {\n  p[0] = 2;\n}\n")
    assert bench.code_hash(str(src)) != h0
    # a record applies only to its kernel's current code and to its own workload
    csrc = os.path.join(ROOT, "io_aware_exact_qk_b200", "csrc")
    table = tmp_path / "records.json"
    rec = {"source": "bwd_sm100.cu", "source_code_sha256_16": bench.code_hash(os.path.join(csrc, "bwd_sm100.cu")),
           "dram_bytes_per_launch": 123, "tensor_pipe_active": 0.5}
    stale = dict(rec, source_code_sha256_16="0" * 16)
    table.write_text(json.dumps({"bwd_bf16_sm100@wl_a": rec, "fwd_bf16_sm100@wl_a": dict(stale, source="fwd_sm100.cu")}))
    assert bench.traffic_record("bwd_bf16_sm100", "wl_a", path=str(table))["dram_bytes_per_launch"] == 123
    assert bench.traffic_record("bwd_bf16_sm100", "wl_b", path=str(table)) is None
    assert bench.traffic_record("fwd_bf16_sm100", "wl_a", path=str(table)) is None
    assert bench.traffic_record("no_such_kernel", "wl_a", path=str(table)) is None
    # every committed record names a source file and the workload it was captured on
    committed = json.load(open(os.path.join(ROOT, "profiles", "roofline_traffic.json")))
    for key, r in committed.items():
        if key.startswith("_"):
            continue
        assert "@" in key and os.path.exists(os.path.join(csrc, r["source"])), key
