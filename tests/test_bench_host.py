"""Host-side pieces of the benchmark (no GPU): the decode-kernel code hash
that keys the recorded DRAM traffic ignores comments and layout but not
code, and the recorded traffic file parses."""
import bench


def test_code_hash_ignores_comments_and_layout_only():
    a = "int f(int x) {\n  return x + 1;  // one more\n}\n/* block\n comment */\n"
    b = "int f(int x) { return x + 1; }\n// another comment\n"
    c = "int f(int x) { return x + 2; }\n"
    assert bench._code_only(a) == bench._code_only(b)
    assert bench._code_only(a) != bench._code_only(c)
    assert "//" not in bench._code_only(a) and "/*" not in bench._code_only(a)


def test_recorded_traffic_is_a_byte_count_or_absent():
    v = bench.recorded_traffic("b16_h40_L32k_bs64_s90")
    assert v is None or v > 200e6      # the headline reads >= 218 MB of K/V per launch
    assert bench.recorded_traffic("no_such_workload") is None


def test_reference_arm_prints_one_contract_line():
    """`bench.py --impl reference` (the oracle on the host cores) prints one
    JSON line with the contract's keys, the same metric as the GPU arm, and
    its own e2e/cpu_baseline objects."""
    import json
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1",
                        "--warmup", "3", "--ref-rows", "1"], cwd=root, capture_output=True,
                       text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC and d["unit"] == bench.UNIT
    for key in ("value", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "config", "e2e", "cpu_baseline", "dtype"):
        assert key in d, key
    assert d["value"] > 0 and d["steps"] == 1 and d["higher_is_better"] is True
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
