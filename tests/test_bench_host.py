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
