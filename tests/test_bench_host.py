"""Host-side pieces of bench.py that run without a GPU: the JSON line's
config (one builder for both arms) and the oracle's timed sample in every
configuration the step can be run in."""
import pytest

import bench


def test_both_arms_share_the_config():
    nv = bench.step_config("nvfp4", False, 1, False)
    assert nv["format"] == "nvfp4" and nv["rht"] == "off" and nv["weights"] == "16x16 tiles"
    assert nv["parallelism"] == "replicas x1" and "32768" in nv["workload"]
    assert bench.step_config("nvfp4", True, 1, False)["rht"] == "wgrad 16-pt"
    mx = bench.step_config("mxfp4", False, 8, True)
    assert mx["rht"] == "all GEMMs 32-pt" and mx["rounding"] == "RTN fwd/bwd"
    assert mx["parallelism"].startswith("dp x8")


@pytest.fixture(scope="module")
def layer_cache():
    return {}            # the synthetic 7B layers, generated once for the module


@pytest.mark.parametrize("fmt,wgrad_rht", [("nvfp4", False), ("nvfp4", True), ("mxfp4", False)])
def test_cpu_baseline_sample_runs(layer_cache, fmt, wgrad_rht):
    out = bench.cpu_baseline(64, 128, seed=0, cache=layer_cache, fmt=fmt, wgrad_rht=wgrad_rht)
    assert out["kind"] == "oracle" and out["unit"] == "TFLOP/s"
    assert out["value"] > 0 and out["cores"] >= 1
    assert fmt.upper() in out["sample"]
