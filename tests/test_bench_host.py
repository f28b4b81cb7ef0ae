"""Host logic of bench.py that needs no GPU: the reference arm's JSON line,
the algorithmic byte counts and the L2 rotation rule."""
import json
import os
import subprocess
import sys

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

KEYS = ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
        "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config")


def test_headline_algorithmic_bytes():
    # read Q and K of both streams + write joint Q and K + 4 gammas + the cos/sin rows
    assert bench.fused_bytes(512, 4096, 24, 128, 64) == 115_606_528
    assert 4 * 4608 * 24 * 128 * 2 + 4 * 128 * 2 + 2 * 4608 * 64 * 4 == 115_606_528


def test_rotating_sets_exceed_twice_l2():
    for nbytes in (2 ** 20, 8_329_604, 67_125_248, 115_606_528, 1_073_758_208):
        n = bench.n_sets_for(nbytes)
        assert 1 <= n <= 64
        if n < 64:
            assert n * nbytes > 2 * bench.L2_BYTES


def test_reference_arm_json_line():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--steps", "2", "--warmup", "1"], capture_output=True, text=True,
                         cwd=ROOT, timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    line = json.loads(out.stdout.strip().splitlines()[-1])
    for k in KEYS:
        assert k in line, k
    assert line["impl"] == "reference" and line["metric"] == bench.METRIC
    assert line["value"] > 0 and line["higher_is_better"] is True
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["value"] == line["value"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
