"""bench.py's reference arm runs on the host alone: its JSON line carries the
keys the benchmark contract names, for a small workload."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_prints_one_json_line_with_the_contract_keys():
    out = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload", "tiny", "--steps", "2",
                          "--warmup", "1"], cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "steps/s" and d["value"] > 0
    assert d["higher_is_better"] is True and d["n_gpus"] == 1 and d["steps"] == 2 and d["warmup"] == 1
    assert d["config"]["workload"].startswith("tiny:")
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def _bench():
    import importlib.util
    spec = importlib.util.spec_from_file_location("bench_module", os.path.join(ROOT, "bench.py"))
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    return m


def test_bench_defaults_and_config_keys():
    b = _bench()
    from medusa_tree_speculative_heads_b200 import inputs as I
    assert b.METRIC.startswith("Medusa verify steps/s") and b.UNIT == "steps/s"
    assert b.WORKLOAD == "llama8b"
    for name, w in I.WORKLOADS.items():
        c = b.config_dict(w, 1)
        assert {"workload", "global_batch", "seq_len", "parallelism", "l2"} <= set(c)
        assert c["workload"].startswith(name + ":") and c["global_batch"] == w.B
        assert b.config_dict(w, 4)["global_batch"] == 4 * w.B          # replicas: weak scaling


def test_bench_counts_the_library_launches_of_a_step():
    # the kernels one step launches (the launch list in profiles/ shows four at llama8b)
    b = _bench()
    from medusa_tree_speculative_heads_b200 import inputs as I
    W = I.WORKLOADS
    assert b.launches_per_step(W["llama8b"]) == 4       # heads, attention, argmax, walk + commit
    assert b.launches_per_step(W["stoch_b64"]) == 4     # heads, attention, stochastic verify, commit
    assert b.launches_per_step(W["tiny"]) == 4          # fp32: fused heads, one attention kernel, argmax, walk + commit
    assert b.launches_per_step(W["llama8b_incache"]) == 5   # the walk without commit, then the compaction
    assert b.launches_per_step(I.scaled(W["llama8b"], Hq=24)) == 5   # G = 3: the mma.sync kernel and its combine
    assert b._is_anc([-1, 0, 1, 0], 2, 0) and b._is_anc([-1, 0, 1, 0], 2, 2) and not b._is_anc([-1, 0, 1, 0], 3, 1)
