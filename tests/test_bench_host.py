"""Host-side arithmetic of bench.py's measurement: the algorithmic bytes behind the
per-kernel HBM fractions, the fractions themselves, and the rule that the mixing's
DRAM traffic is reported only for the sources it was captured on.  No GPU."""
import hashlib
import os

import bench


def test_alg_bytes_per_edge_follow_the_rows_each_kernel_moves():
    C = 128
    row, d = 16 * C * 4, 84 * 4
    # layers after the first: full [16][C] rows
    assert bench.alg_bytes("rotate_in", C, False) == 4 * C * 4 + 2 * row + d            # R in; x~ hi/lo out
    assert bench.alg_bytes("bwd_prep", C, False) == 4 * C * 4 + 4 * row + d             # + g_y hi/lo out
    assert bench.alg_bytes("bwd_edge", C, False) == 2 * row + 4 * C * 4 + d + 8 * C * 4  # y, g_x~, R, D; dE/dR hi/lo
    assert bench.alg_bytes("rotate_back_scatter", C, False) == row + d
    # the first layer (degree-0 input) moves only its m = 0 / l = 0 columns
    for k in ("rotate_in", "bwd_prep", "bwd_edge", "rotate_back_scatter"):
        assert bench.alg_bytes(k, C, True) < bench.alg_bytes(k, C, False)
    # the radial products do not depend on the layer
    assert bench.alg_bytes("radial_head", C, True) == bench.alg_bytes("radial_head", C, False) == 2 * 64 * 4 + 4 * C * 4


def test_hbm_fraction_is_bytes_over_time_over_peak():
    C, T, E, steps = 128, 3, 1000, 4
    fam = {"rotate_back_scatter": (steps * 2.0, 0)}          # 2 ms per step
    out = bench.hbm_fractions(fam, steps, E, C, T, hbm_gbs=1000.0)
    r = out["rotate_back_scatter"]
    want = E * (bench.alg_bytes("rotate_back_scatter", C, True) + 2 * bench.alg_bytes("rotate_back_scatter", C, False))
    assert r["alg_bytes_per_step"] == want
    assert abs(r["achieved_gbs"] - want / 2e-3 / 1e9) < 0.1
    assert abs(r["frac_of_hbm"] - r["achieved_gbs"] / 1000.0) < 1e-3
    assert "bwd_prep" not in out                              # kernels not timed are left out


def test_traffic_is_reported_only_for_the_captured_sources(monkeypatch):
    h = hashlib.sha1()
    for f in ("so2_tc.cuh", "emp_lib.cu"):
        h.update(open(os.path.join(bench.ROOT, "edge_message_passing_b200", "csrc", f), "rb").read())
    monkeypatch.setattr(bench, "SO2_TRAFFIC", {"source_sha1": h.hexdigest(), "bytes_per_launch": 123.0})
    assert bench.so2_traffic_per_launch() == 123.0
    monkeypatch.setattr(bench, "SO2_TRAFFIC", {"source_sha1": "0" * 40, "bytes_per_launch": 123.0})
    assert bench.so2_traffic_per_launch() is None
    monkeypatch.setattr(bench, "SO2_TRAFFIC", {"source_sha1": None, "bytes_per_launch": None})
    assert bench.so2_traffic_per_launch() is None
