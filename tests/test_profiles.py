"""The tracked measurement records under profiles/, on CPU: every bench line
keeps the JSON contract and its own identities, was taken with clean clocks,
and the recorded DRAM traffic still belongs to the kernel sources it was
measured on (bench.py reports it only then)."""
import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402

PROFILES = os.path.join(ROOT, "profiles")
KEYS = ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
        "vs_baseline", "dtype", "data", "config")
BAD_REASONS = {"hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"}


def _lines():
    with open(os.path.join(PROFILES, "bench_lines.jsonl")) as f:
        return [json.loads(l) for l in f if l.strip()]


def test_bench_lines_keep_the_contract():
    recs = _lines()
    assert recs
    for r in recs:
        assert r["cmd"].split()[:2] == ["python", "bench.py"] or "python bench.py" in r["cmd"], r["cmd"]
        d = r["line"]
        for k in KEYS:
            assert k in d, (r["cmd"], k)
        assert d["value"] > 0 and d["n_gpus"] == 1 and d["warmup"] >= 1
        if d.get("impl") == "reference":
            assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
            continue
        assert d["warmup"] >= 3, r["cmd"]
        assert "workload" in d["config"]
        # one step is one batch of config.batch tokens: value and ms_per_step agree
        batch = d["config"].get("batch", 1)
        if d["config"]["workload"] in ("decode_stream", "decode_resident"):
            assert abs(d["value"] * d["ms_per_step"] / 1e3 - batch) < 1e-6 * batch, r["cmd"]


def test_bench_lines_clocks_are_clean():
    """Numbers quoted from these lines were taken at the full SM clock with no
    thermal or hardware slowdown active."""
    for r in _lines():
        c = r["line"].get("clocks")
        if c is None:
            continue
        assert not BAD_REASONS & set(c.get("reasons", [])), r["cmd"]
        assert c["sm_mhz"] >= 0.9 * c["sm_max_mhz"], r["cmd"]


def test_bench_lines_rooflines_are_consistent():
    for r in _lines():
        rf = r["line"].get("roofline")
        if not rf or "frac" not in rf:
            continue
        assert abs(rf["frac"] - rf["achieved"] / rf["peak"]) < 1e-9, r["cmd"]
        if rf["bound"] == "pcie":
            d = r["line"]
            assert abs(rf["achieved"] - d["miss_bytes_per_token"] * d["value"] / 1e9) < 1e-6 * rf["achieved"]
            assert d["miss_bytes_check"]["holds"], r["cmd"]


@pytest.mark.parametrize("name", ["traffic.json", "traffic_attn.json"])
def test_recorded_traffic_matches_the_sources(name):
    rec = json.load(open(os.path.join(PROFILES, name)))
    assert rec["source_sha256"] == bench.csrc_sha256(tuple(rec["sources"])), name
