"""The benchmark's reference arm (the fp64 oracle on the host cores) prints one JSON line with
the keys the benchmark contract fixes, in both offset-combination modes; it runs on the CPU."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("combine", ["mean", "max"])
def test_reference_arm_json_line(combine):
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    out = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload", "tiny_d64_n256",
                          "--steps", "2", "--warmup", "3", "--combine", combine],
                         cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, out.stdout[-2000:]
    j = json.loads(lines[0])
    for k in ("metric", "value", "unit", "impl", "n_gpus", "steps", "warmup", "higher_is_better", "scaling",
              "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert k in j, k
    assert j["impl"] == "reference" and j["n_gpus"] == 1 and j["steps"] == 2 and j["warmup"] >= 3
    assert j["value"] > 0 and j["higher_is_better"] is True
    assert j["config"]["workload"] == "tiny_d64_n256" and j["config"]["offsets_combine"] == combine
    cb = j["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == j["value"]
    e2e = j["e2e"]
    assert e2e["value"] == j["value"] and e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0


def test_traffic_figure_follows_the_code_not_its_comments():
    """roofline.traffic comes from a committed ncu summary only while the prune kernel's code is
    the one the counters were taken on: the hash ignores comments and layout, not code."""
    sys.path.insert(0, ROOT)
    import bench
    a = "int f(int x) { // doubles x\n  return 2 * x; /* fast */ }\nconst char *s = \"a//b\";"
    b = "int f(int x)\n{\n  return 2 * x;\n}\nconst char *s = \"a//b\";  // other words"
    c = "int f(int x) { return 3 * x; } const char *s = \"a//b\";"
    assert bench._code_only(a) == bench._code_only(b)
    assert bench._code_only(a) != bench._code_only(c)
    assert "a//b" in bench._code_only(a)
    assert len(bench.kernel_source_hash()) == 16
