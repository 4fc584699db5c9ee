"""Host-side arithmetic of bench.py's measurement: the algorithmic bytes behind the
per-kernel HBM fractions, the fractions themselves, and the rule that the mixing's
DRAM traffic is reported only for the sources it was captured on.  No GPU."""
import os

import bench


def test_alg_bytes_follow_the_rows_each_kernel_moves():
    C, T, E, N = 128, 3, 1000, 10
    row, d, d0 = 16 * C * 4, 84 * 4, 16 * 4
    # the per-edge cohort kernels run only in the layers between the first and the last
    assert bench.alg_bytes_step("rotate_in", C, T, E, N) == E * (4 * C * 4 + 2 * row + d)      # R in; x~ hi/lo out
    assert bench.alg_bytes_step("bwd_prep", C, T, E, N) == E * (2 * row + d)                   # D in; g_y hi/lo out
    assert bench.alg_bytes_step("bwd_edge", C, T, E, N) == E * (2 * row + 4 * C * 4 + d + 8 * C * 4)
    assert bench.alg_bytes_step("rotate_back_scatter", C, T, E, N) == E * (row + d)
    for k in ("rotate_in", "bwd_prep", "bwd_edge", "rotate_back_scatter"):
        assert bench.alg_bytes_step(k, C, 2, E, N) == 0                                        # no such layer
        assert bench.alg_bytes_step(k, C, 5, E, N) == 3 * bench.alg_bytes_step(k, C, 3, E, N)
    # end layers: one pass each; a single-layer model has no last-layer kernels
    assert bench.alg_bytes_step("first_fwd", C, T, E, N) == E * (C * 4 + d0) + N * row
    assert bench.alg_bytes_step("last_fwd", C, 1, E, N) == 0
    assert bench.alg_bytes_step("last_bwd", C, T, E, N) == E * (4 * C * 4 + d + 12 + 8 * C * 4 + 24) + N * 2 * row
    # the first layer's radial head writes (and its backward reads) the degree-0 columns only
    assert bench.alg_bytes_step("radial_head", C, 1, E, N) == E * (2 * 64 * 4 + C * 4)
    assert bench.alg_bytes_step("radial_head", C, T, E, N) == E * (2 * 64 * 4 + C * 4) + 2 * E * (2 * 64 * 4 + 4 * C * 4)
    assert bench.alg_bytes_step("radial_h2", C, T, E, N) == 3 * E * (4 + 2 * 64 * 4)
    # the fused network kernels: d in, R out (forward); dE/dR hi/lo, d, r in, g_r updated (backward)
    assert bench.alg_bytes_step("radial_fwd", C, T, E, N) == E * (4 + C * 4) + 2 * E * (4 + 4 * C * 4)
    assert bench.alg_bytes_step("radial_bwd", C, T, E, N) == E * (2 * C * 4 + 40) + 2 * E * (2 * 4 * C * 4 + 40)


def test_hbm_fraction_is_bytes_over_time_over_peak():
    C, T, E, N, steps = 128, 3, 1000, 10, 4
    fam = {"rotate_back_scatter": (steps * 2.0, 0)}          # 2 ms per step
    out = bench.hbm_fractions(fam, steps, E, N, C, T, hbm_gbs=1000.0)
    r = out["rotate_back_scatter"]
    want = bench.alg_bytes_step("rotate_back_scatter", C, T, E, N)
    assert r["alg_bytes_per_step"] == want
    assert abs(r["achieved_gbs"] - want / 2e-3 / 1e9) < 0.1
    assert abs(r["frac_of_hbm"] - r["achieved_gbs"] / 1000.0) < 1e-3
    assert "bwd_prep" not in out                              # kernels not timed are left out


def test_traffic_is_reported_only_for_the_captured_sources(monkeypatch):
    h = bench.so2_source_hash()
    assert h is not None
    monkeypatch.setattr(bench, "SO2_TRAFFIC", {"source_sha1": h, "bytes_per_launch": 123.0})
    assert bench.so2_traffic_per_launch() == 123.0
    monkeypatch.setattr(bench, "SO2_TRAFFIC", {"source_sha1": "0" * 40, "bytes_per_launch": 123.0})
    assert bench.so2_traffic_per_launch() is None
    monkeypatch.setattr(bench, "SO2_TRAFFIC", {"source_sha1": None, "bytes_per_launch": None})
    assert bench.so2_traffic_per_launch() is None


def test_traffic_hash_covers_the_kernel_and_the_marked_launch_code():
    """Edits outside the marked launch code of emp_lib.cu leave the hash alone; edits inside it or
    in so2_tc.cuh change it."""
    import hashlib
    csrc = os.path.join(bench.ROOT, "edge_message_passing_b200", "csrc")
    text = open(os.path.join(csrc, "emp_lib.cu")).read()
    assert text.count("// [per-edge product launches: begin]") == 2
    assert text.count("// [per-edge product launches: end]") == 2


def test_mixing_flops_count_two_mixings_per_middle_layer():
    # 72 C^2 multiply-adds per edge and mixing (m-blocks of widths 4, 6, 4, 2 channel blocks:
    # 16 + 36 + 16 + 4), forward and backward transpose, middle layers only
    assert sum(w * w for w in (4, 6, 4, 2)) == 72
    C, E = 128, 1000
    assert bench.mixing_flops_step(C, 3, E) == E * 2 * 72 * C * C * 2
    assert bench.mixing_flops_step(C, 2, E) == 0
    assert bench.mixing_flops_step(C, 5, E) == 3 * bench.mixing_flops_step(C, 3, E)
