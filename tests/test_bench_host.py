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
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "2",
                        "--warmup", "3", "--workload", "b8_h32_L8k_bs64_s90_newest"], cwd=root,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC and d["unit"] == bench.UNIT
    for key in ("value", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "config", "e2e", "cpu_baseline", "dtype"):
        assert key in d, key
    assert d["value"] > 0 and d["steps"] == 2 and d["higher_is_better"] is True
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    # every row of the batch in each step: measured, not extrapolated
    assert d["extrapolated"] is False and d["rows_per_step"] == 64
    cfg = d["config"]
    assert cfg["workload"] == "b8_h32_L8k_bs64_s90_newest" and cfg["k_max"] == 13
    assert cfg["num_splits"] >= 1 and cfg["kv_layout"] == "nhd"
    assert d["cpu_baseline"]["cores"] >= 1 and d["cpu_baseline"]["nproc"] >= 1


def test_oracle_pool_computes_what_the_oracle_computes():
    """The spawned oracle processes return the oracle's own results for their
    rows (same inputs, same function), whatever the process count."""
    import numpy as np
    import torch
    from block_sparse_attention_step_b200 import workloads as W
    from oracle import seer_oracle as O
    w = W.WORKLOADS["b64_ragged_h64_paged_bs64"].replace(batch=3, q_heads=8, kv_heads=2,
                                                          seqlen_range=(100, 900))
    data = W.generate(w, 5, "cpu")
    kps = bench.cpu_k_per_seq(w, data["seqlens"].tolist())
    rows = [(b, h) for b in range(3) for h in range(2)]
    inputs = bench.oracle_decode_rows(w, data, rows, kps, w.force_newest)
    pool = bench.OraclePool(2)
    try:
        pool.load(inputs, [float(data["seqlens"][b]) for (b, _) in rows])
        assert pool.step() > 0
        got = pool.results()
    finally:
        pool.close()
    for (b, h), r in zip(rows, got):
        L = int(data["seqlens"][b])
        G = w.group
        q = data["q"][b, h * G:(h + 1) * G].double().numpy()
        K = W.gather_rows(data["k_pool"], data["page_table"], b, h, L, 64).double().numpy()
        V = W.gather_rows(data["v_pool"], data["page_table"], b, h, L, 64).double().numpy()
        ref = O.decode_row(q, data["w_gate"][h].double().numpy(), K, V, L, 64, kps[b], False,
                           0.125 / 2 ** 0.5, 0.125 / 2 ** 0.5)
        assert r["indices"].tolist() == ref["indices"].tolist()
        np.testing.assert_array_equal(r["out"], ref["out"])


def test_row_sample_respects_the_byte_budget():
    from block_sparse_attention_step_b200 import workloads as W
    w = W.WORKLOADS["b64_ragged_h64_paged_bs64"]
    seqlens = [4096 + 1000 * i for i in range(64)]
    rows, sampled = bench.pick_rows(w, seqlens, 1e9)
    assert sampled and sum(4 * 128 * seqlens[b] for b, _ in rows) <= 1e9
    rows, sampled = bench.pick_rows(w, seqlens, 1e12)
    assert not sampled and len(rows) == 64 * 8
