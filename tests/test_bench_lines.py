"""The objects bench.py builds for each leg of its JSON line, on CPU with
synthetic timings: the roofline object's keys and arithmetic (frac =
achieved / peak), the metric's value from the timed steps, and the legs'
stated timing method."""
import math
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402
from causal_gqa_attention_03_b200 import inputs  # noqa: E402

PEAKS = {"hbm_gbs": 6531.9, "bf16_tflops": 1607.7, "bf16_tflops_sustained": 1369.5}
ROOF_KEYS = {"bound", "achieved", "peak", "unit", "frac", "traffic"}


def check_roofline(r, bound, unit, peak):
    assert ROOF_KEYS <= set(r)
    assert r["bound"] == bound and r["unit"] == unit and r["peak"] == peak
    assert r["frac"] == pytest.approx(r["achieved"] / r["peak"], abs=1e-4)


def test_backward_line():
    w = inputs.WORKLOADS[inputs.LARGEST]
    times = [7.0, 7.2, 7.1]
    line = bench.backward_line(w, times, sum(times), 3, 9, 2 << 20, 1, PEAKS, "measured")
    assert line["value"] == pytest.approx(2.5 * w.flops * 3 / (sum(times) * 1e-3) / 1e12, rel=1e-3)
    assert line["gpu_launches"] == 9 and line["workspace_bytes"] == 2 << 20
    r = line["roofline"]
    check_roofline(r, "tensor", "TFLOP/s", 1607.7)
    assert r["achieved"] == pytest.approx(2.5 * w.flops / (7.1 * 1e-3) / 1e12, rel=1e-3)
    assert r["issued_frac"] == pytest.approx(1.4 * r["frac"], abs=2e-4)


def test_decode_line_back_to_back_with_flushed_reference():
    wd = inputs.DECODE
    times = [0.36] * 10
    line = bench.decode_line(wd, times, 3.6, 10, 20, 1 << 20, 1, PEAKS, "measured",
                             flushed=[0.40, 0.39, 0.41])
    nbytes = wd.io_bytes()
    assert line["value"] == pytest.approx(nbytes * 10 / 3.6e-3 / 1e9, rel=1e-3)
    check_roofline(line["roofline"], "hbm", "GB/s", 6531.9)
    assert line["roofline"]["bytes_per_step"] == nbytes
    assert line["l2"].startswith("no flush") and nbytes > 10 * bench.L2_BYTES
    assert line["ms_per_step_write_flush"] == pytest.approx(0.40)


def test_varlen_and_prologue_lines():
    wv = inputs.VARLEN
    vl = bench.varlen_line(wv, [8.0, 8.2, 8.1], 3, PEAKS, "measured")
    assert vl["value"] == pytest.approx(wv.flops / 8.1e-3 / 1e12, rel=1e-3)
    check_roofline(vl["roofline"], "tensor", "TFLOP/s", 1607.7)
    w = inputs.WORKLOADS[inputs.LARGEST]
    res = {"rmsnorm": ([0.055, 0.054], 268443648, 2), "rope_qkv": ([0.076], 402653184, 1)}
    pl = bench.prologue_line(w, res, PEAKS, "measured")
    for name, (ts, nbytes, launches) in res.items():
        obj = pl[name]
        med = sorted(ts)[len(ts) // 2] if len(ts) % 2 else sum(ts) / 2
        assert obj["value"] == pytest.approx(nbytes / (med * 1e-3) / 1e9, rel=1e-3)
        assert obj["gpu_launches"] == launches
        check_roofline(obj["roofline"], "hbm", "GB/s", 6531.9)
    assert not math.isnan(pl["rmsnorm"]["roofline"]["frac"])
