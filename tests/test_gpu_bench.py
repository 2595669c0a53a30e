"""bench.py end to end on a B200 at small sizes: the JSON line it prints keeps
its contract (keys, units, the identities between its own numbers) for the
streamed decode and for resident decode.  The numbers themselves are not
judged here; only that they are consistent."""
import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _line(*argv):
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *argv], capture_output=True, text=True,
                       timeout=900, cwd=ROOT)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout[-2000:]
    return json.loads(lines[0])


def _common(d, steps, warmup):
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
              "vs_baseline", "dtype", "data", "config", "roofline", "e2e", "gpu_launches", "clocks"):
        assert k in d, k
    assert d["unit"] == "tokens/s" and d["n_gpus"] == 1 and d["higher_is_better"] is True
    assert (d["steps"], d["warmup"]) == (steps, warmup)
    assert d["value"] > 0 and d["gpu_launches"] > 0
    # tokens/s and ms per step describe the same timed region (one token per step)
    assert abs(d["value"] * d["ms_per_step"] / 1e3 - d["config"]["batch"]) < 1e-6 * d["config"]["batch"] + 1e-9
    e = d["e2e"]
    assert e["value"] > 0 and e["unit"] == "tokens/s" and e["h2d_bytes_per_step"] > 0 and e["d2h_bytes_per_step"] > 0
    r = d["roofline"]
    assert r["achieved"] > 0 and r["peak"] > 0 and abs(r["frac"] - r["achieved"] / r["peak"]) < 1e-9


def test_bench_streamed_decode_line():
    """Two layers of the streamed decode: the host-link roofline, the miss
    counters and their identity with the hit rate, the look-ahead figures."""
    d = _line("--layers", "2", "--steps", "6", "--warmup", "3", "--no-cpu")
    _common(d, 6, 3)
    r = d["roofline"]
    assert r["bound"] == "pcie" and r["unit"] == "GB/s" and "hbm_kernel" in r
    assert 0.0 <= d["hit_rate"] <= 1.0
    assert d["miss_bytes_check"]["holds"], d["miss_bytes_check"]
    # useful link bytes per token x tokens/s is the achieved rate
    assert abs(r["achieved"] - d["miss_bytes_per_token"] * d["value"] / 1e9) < 1e-6 * r["achieved"] + 1e-9
    pf = d["prefetch"]
    assert pf["used_bytes_per_token"] <= pf["issued_bytes_per_token"]
    assert abs(r["traffic"] - (d["miss_bytes_per_token"] + pf["wasted_bytes_per_token"])) <= 1.0


def test_bench_resident_decode_line():
    """Two resident layers, one token per step: the HBM roofline of the
    dominant kernel with the step-level rate beside it."""
    d = _line("--workload", "decode_resident", "--layers", "2", "--steps", "8", "--warmup", "3", "--no-cpu")
    _common(d, 8, 3)
    r = d["roofline"]
    assert r["bound"] == "hbm" and r["unit"] == "GB/s"
    sl = r["step_level"]
    assert abs(sl["achieved"] - sl["bytes_per_step"] / (d["ms_per_step"] * 1e-3) / 1e9) < 1e-6 * sl["achieved"]
