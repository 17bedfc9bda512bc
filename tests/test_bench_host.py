"""Host-side checks of bench.py that need no GPU: the ncu traffic figures go
null once the sources of their kernels change, and the reference arm (the
oracle on the host cores) prints the JSON line the driver reads."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_traffic_is_reported_only_for_the_captured_sources(monkeypatch):
    assert bench.traffic_for("decode_b8_32k_4layers", "attn") == bench.NCU_TRAFFIC["decode_b8_32k_4layers"]["attn"]
    assert bench.traffic_for("no_such_workload", "attn") is None
    assert bench.traffic_for("prefill_2k_1layer", "index") is None          # no capture of that kind
    monkeypatch.setitem(bench.NCU_SOURCES, "attn", "0000000000000000")     # sources changed since
    assert bench.traffic_for("decode_b8_32k_4layers", "attn") is None
    assert bench.traffic_for("decode_b8_32k_4layers", "index") is not None  # other kinds unaffected


def test_every_workload_is_a_recipe_with_a_unique_name():
    names = [c.name for c in bench.CONFIGS.values()]
    assert len(set(names)) == len(names)
    assert set(bench.SUB_WORKLOADS) <= set(bench.CONFIGS)
    assert "decode_32k" not in bench.SUB_WORKLOADS


@pytest.mark.timeout(300)
def test_reference_arm_prints_the_contract_line():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--config",
                          "prefill_2k", "--steps", "1", "--warmup", "3"],
                         capture_output=True, text=True, timeout=280, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    line = json.loads(out.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference"
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "config", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["metric"] == "prefill tokens/s" and line["value"] > 0
    assert line["config"]["workload"] == "prefill_2k_1layer"
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1


def test_source_hash_ignores_comments_but_not_code(tmp_path, monkeypatch):
    a = "int f(int x) {  // doubles\n  return 2 * x; /* plain */\n}\n"
    b = "int f(int x) {\n  // a longer, reflowed\n  // comment\n  return 2 * x;\n}\n"
    c = "int f(int x) {  // doubles\n  return 3 * x;\n}\n"
    for name, text in (("a.cu", a), ("b.cu", b), ("c.cu", c)):
        (tmp_path / name).write_text(text)
    monkeypatch.setattr(bench, "CSRC", str(tmp_path))
    ha, hb, hc = (bench.sources_sha16([n]) for n in ("a.cu", "b.cu", "c.cu"))
    assert bench._code_only(a) == bench._code_only(b)
    assert bench._code_only(a) != bench._code_only(c)
    assert ha != hc
