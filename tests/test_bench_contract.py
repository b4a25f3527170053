"""The host side of bench.py, on the CPU: the algorithmic byte counts behind
the roofline, the gate that reports an ncu traffic figure only while the
captured kernel's sources are unchanged, and the JSON line of the reference
arm (the fp64 oracle timed on the host cores)."""
import importlib.util
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_algorithmic_bytes_of_the_bench_workload(bench):
    """8x12x2048 tokens of q, k, v, out (64 bf16 each) and beta (one bf16),
    the fp32 64x64 final state of 96 heads and 12 fp32 lambdas."""
    tok = 8 * 12 * 2048
    expect = tok * (64 + 64 + 64 + 64) * 2 + tok * 2 + 96 * 64 * 64 * 4 + 12 * 4
    assert expect == 102_629_424
    assert bench.algorithmic_bytes_fwd(8, 12, 2048, 64, 64) == expect
    # per-channel beta (Falcon-2/2A) carries d_v values per token
    assert bench.algorithmic_bytes_fwd(1, 1, 10, 128, 128, per_channel=True) == \
        10 * (128 * 4 + 128) * 2 + 128 * 128 * 4 + 4


def test_window_walk_flops_count_each_dot_product(bench):
    """The Falcon-3 window solve's flop count against a direct loop over
    tokens, window slots and value channels: the dot product of token t,
    slot m covers the rows 0 .. t+B_w-2 finished so far (two flops per row),
    plus eight for the rest of the update; a partial last chunk counts as
    full."""
    C, w, dv = 8, 3, 5
    direct = 0
    for t in range(C):
        for m in range(w):
            for j in range(dv):
                direct += 2 * (t + w - 1) + 8
    assert bench.window_walk_flops(1, 1, C, C, w, dv) == direct
    assert bench.window_walk_flops(2, 3, 2 * C + 1, C, w, dv) == 2 * 3 * 3 * direct
    assert abs(bench.FP32_ALU_TFLOPS - 74.44992) < 1e-6


def test_profiled_traffic_follows_the_sources(bench, monkeypatch, tmp_path):
    """A summary's traffic figure counts while the captured kernel's sources
    hash to the value it records, and not after any of them changes."""
    name, files = bench.PROFILED["chunk"]
    (tmp_path / "profiles").mkdir()
    csrc = tmp_path / "csrc"
    csrc.mkdir()
    for f in files:
        (csrc / f).write_text(open(os.path.join(bench.CSRC, f)).read())
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "CSRC", str(csrc))
    assert bench.profiled_traffic("chunk") is None  # no summary
    (tmp_path / "profiles" / name).write_text(
        "source sha256: %s\n\ntraffic per launch: 123456 B\n" % bench.source_hash(files))
    assert bench.profiled_traffic("chunk") == 123456
    (csrc / files[-1]).write_text((csrc / files[-1]).read_text() + "\n// edited\n")
    assert bench.profiled_traffic("chunk") is None


def test_reference_arm_json_line():
    """bench.py --impl reference prints one JSON line with the contract's
    keys; its e2e and cpu_baseline repeat its own value."""
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                          "--warmup", "1"], capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["unit"] == "tokens/s" and d["value"] > 0
    assert d["e2e"]["value"] == d["value"] and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert d["config"]["workload"] == "falcon1-1A-chunk-bf16-8x12x2048x64"
