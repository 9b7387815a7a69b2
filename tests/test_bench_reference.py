"""bench.py's reference arm (the CPU oracle, no GPU needed) prints one JSON line with the
keys the benchmark contract asks for."""

import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_json_line():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "3"],
                       capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout[-2000:]
    d = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["steps"] == 1 and d["warmup"] == 3
    assert d["value"] > 0 and d["higher_is_better"] is True
    assert "workload" in d["config"]
    for key in ("value", "unit", "cores", "kind", "sample"):
        assert key in d["cpu_baseline"], key
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert d["e2e"]["value"] == d["value"] and d["e2e"]["unit"] == d["unit"]


def _bench_module():
    import importlib.util

    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_traffic_hash_ignores_comments_and_whitespace_only():
    bench = _bench_module()
    src = "int f(int a) {  // add one\n  return a + 1; /* done\n  here */\n}\n"
    same = "int f(int a)\n{\n\treturn a+1;  // different words\n}"
    other = "int f(int a) { return a + 2; }"
    assert bench.code_only(src) == bench.code_only(same) == "intf(inta){returna+1;}"
    assert bench.code_only(other) != bench.code_only(src)
    # every recorded capture names a kernel that bench.py times and a full SHA-256
    for kernel, rec in bench.ATTN_TRAFFIC.items():
        assert kernel.startswith("attn_fwd_sm100_kernel<")
        assert len(rec["sources_sha256"]) == 64 and rec["bytes"] > 0
