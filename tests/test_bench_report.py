"""Host-side arithmetic of bench.py's report on CPU: the roofline of each
workload (the measured bf16 peak; the block-scaled kernels' mixed peak
2 / (1/r + 1) x bf16 with r = 2 for E4M3 and 4 for E2M1 score operands),
and the config object both arms print (the same keys for every workload)."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from exact_tiled_attention_39_b200 import workloads  # noqa: E402

PEAKS = {"bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0}


def _m(name, kernel_ms, ms_total=10.0):
    return {"w": workloads.get(name), "flops": 2.0e11, "kernel_ms": kernel_ms,
            "ms_total": ms_total, "prepass_ms": 0.01, "launches_timed": 50}


@pytest.mark.parametrize("name,mix", [("dense_causal", 1.0), ("mxfp8_packed", 4.0 / 3.0),
                                      ("nvfp4_packed", 1.6), ("mxfp8_incoherent", 4.0 / 3.0)])
def test_roofline_peak_and_fraction(name, mix):
    r = bench.roofline_for(_m(name, 0.25), PEAKS, "measured")
    achieved = 2.0e11 / 0.25e-3 / 1e12
    assert r["achieved"] == pytest.approx(achieved, rel=1e-4)
    assert r["peak"] == pytest.approx(1600.0 * mix, rel=1e-3)
    assert r["frac"] == pytest.approx(achieved / (1600.0 * mix), rel=1e-3)
    lowp = {"mxfp8_packed": 2.0, "nvfp4_packed": 4.0, "mxfp8_incoherent": 2.0}.get(name)
    if lowp is None:
        assert not any(k.startswith("frac_of_") for k in r)
    else:
        key = f"frac_of_{workloads.get(name).dtype}_peak"
        assert r[key] == pytest.approx(achieved / (1600.0 * lowp), rel=1e-3)


def test_sustained_peak_for_long_timed_regions():
    r = bench.roofline_for(_m("dense_causal", 0.25, ms_total=2000.0), PEAKS, "measured")
    assert r["peak"] == pytest.approx(1400.0)


def test_config_keys_identical_across_workloads():
    keys = None
    for name in ("dense_causal", "packed_causal", "mxfp8_packed"):
        inp = workloads.make_inputs(name, heads=1)
        cfg = bench.workload_config(workloads.get(name), inp, 1)
        assert cfg["workload"].startswith(name)
        keys = keys or set(cfg)
        assert set(cfg) == keys
