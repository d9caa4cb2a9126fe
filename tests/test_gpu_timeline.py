"""The per-CTA timeline build (libpc_timeline.so) on the GPU: one key switch
records every CTA of each of its six kernels, with the grids the launchers
use, and each kernel's last CTA ends after the last CTA of the kernels it
depends on."""
import json
import os
import subprocess
import sys

import pytest

from tests.conftest import ROOT

pytestmark = pytest.mark.gpu


def _timeline(tmp_path, workload):
    out = tmp_path / f"{workload}.json"
    env = dict(os.environ, PC_TIMELINE="1")
    r = subprocess.run([sys.executable, "-m", "key_switching_b200.timeline", "--workload", workload, "--steps", "8",
                        "--json", str(out)], cwd=ROOT, env=env, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stderr[-2000:]
    return json.load(open(out))["summary"]


def _check_order(s):
    for k, d in s.items():
        assert 0 < d["cta_us_min"] <= d["cta_us_median"] <= d["cta_us_max"] < 1e4, k
        assert d["first_start_us"] >= 0 and d["last_end_us"] >= d["first_end_us"], k
    assert s["row_c1"]["first_start_us"] == 0.0
    assert s["conv_up"]["last_end_us"] >= s["row_c1"]["last_end_us"]
    for k in ("inner_special", "inner_ct"):
        assert s[k]["last_end_us"] >= s["conv_up"]["last_end_us"]
    assert s["conv_down"]["last_end_us"] >= s["inner_special"]["last_end_us"]
    fin = s["moddown_finish"]["last_end_us"]
    assert fin >= s["inner_ct"]["last_end_us"] and fin >= s["conv_down"]["last_end_us"]


def test_timeline_n16(tmp_path):
    s = _timeline(tmp_path, "rot1_n16")  # N=2^16, l=24, alpha=4: 32 row blocks, 128 column strips, 6 digits
    assert set(s) == {"row_c1", "conv_up", "inner_special", "inner_ct", "conv_down", "moddown_finish"}
    assert s["row_c1"]["ctas"] == 32 * 24
    assert s["conv_up"]["ctas"] == 128 * 6
    assert s["inner_special"]["ctas"] == 32 * 4 and s["inner_ct"]["ctas"] == 32 * 24
    assert s["conv_down"]["ctas"] == 128 * 2
    assert s["moddown_finish"]["ctas"] == 32 * 24
    assert s["inner_ct"]["sms"] == 148
    _check_order(s)


def test_timeline_n12(tmp_path):
    s = _timeline(tmp_path, "relin_n12")  # N=2^12, l=4, alpha=2: 2 row blocks, 8 strips, 2 digits
    assert s["row_c1"]["ctas"] == 2 * 4
    # small calls split each item's targets over several CTAs
    assert s["conv_up"]["ctas"] % (8 * 2) == 0 and s["conv_up"]["ctas"] > 8 * 2
    assert s["conv_down"]["ctas"] % (8 * 2) == 0
    assert s["inner_special"]["ctas"] == 2 * 2 and s["inner_ct"]["ctas"] == 2 * 4
    assert s["moddown_finish"]["ctas"] == 2 * 4
    _check_order(s)
