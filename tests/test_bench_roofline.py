"""bench.py's per-call roofline: the fused path divides by the launch time of
its one kernel, the other paths by the whole call's time."""
import importlib.util
import os

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_fused_uses_the_kernel_launch_time(bench):
    r = bench.call_roofline("fused", 340e6, 0.174, 0.180, 6650.0, "fallback")
    assert r["kernel"] == "k_decode_fused" and r["ms_per_launch"] == 0.180
    assert r["achieved"] == pytest.approx(340e6 / 0.180e-3 / 1e9)
    assert r["frac"] == pytest.approx(r["achieved"] / 6650.0)


def test_other_paths_use_the_whole_call(bench):
    r = bench.call_roofline("general", 676e6, 0.318, 0.175, 6650.0, "measured")
    assert "general" in r["kernel"] and r["ms_per_call"] == 0.318 and "ms_per_launch" not in r
    assert r["achieved"] == pytest.approx(676e6 / 0.318e-3 / 1e9)
    assert r["peak_kind"] == "measured" and r["unit"] == "GB/s"
