"""Host-side accounting of bench.py: algorithmic bytes / flops per LUT launch
and the roofline entry of the dominant kernel."""
import pytest

import bench
import synth


def test_dense_layer_launches():
    s = synth.cfg1(4, 8)   # H=2560, I=9728, one shared (dense) expert
    la = bench.lut_launches(s)
    assert len(la) == 2    # gate||up, down
    (b_gu, f_gu), (b_dn, f_dn) = la
    assert b_gu == bench.lut_alg_bytes(4, 2 * 9728, 2560, 8)
    assert b_dn == bench.lut_alg_bytes(4, 2560, 9728, 8)
    assert f_gu == 2 * 4 * 2 * 9728 * 2560 and f_dn == 2 * 4 * 2560 * 9728
    # indices + codebooks + codes + scales + fp32 out
    assert bench.lut_alg_bytes(1, 2048, 2048, 4) == 2048 * 1024 + 32 * 2048 + 1024 + 4 + 4 * 2048


def test_routed_launches_count_active_experts_only():
    s = synth.CFG2
    counts = [0] * s.E
    counts[3], counts[7] = 5, 2
    la = bench.lut_launches(s, counts)
    assert len(la) == 2
    assert la[0][0] == (bench.lut_alg_bytes(5, 2 * s.I, s.H, 4) +
                        bench.lut_alg_bytes(2, 2 * s.I, s.H, 4))
    assert la[1][1] == 2 * 7 * s.H * s.I


def test_roofline_picks_the_dominant_kernel():
    launch_alg = [(100e6, 1e9), (50e6, 4e12)]   # per step: an HBM-ish and a flop-heavy launch
    timed = [("k_lut_mma", 0.02), ("k_lut_tc", 5.0)] * 3
    r, src = bench.lut_roofline(launch_alg, timed, 3, 20.0, 6547.8, 1646.9, "measured")
    assert r["kernel"] == "k_lut_tc" and src == "kernels_lut_tc.cu"
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    assert r["achieved"] == pytest.approx(3 * 4e12 / (15.0 / 1e3) / 1e12)
    assert r["frac"] == pytest.approx(r["achieved"] / 1646.9)
    timed = [("k_lut_mma", 0.05), ("k_lut_tc", 0.01)] * 2
    r, src = bench.lut_roofline(launch_alg, timed, 2, 1.0, 6547.8, 1646.9, "measured")
    assert r["kernel"] == "k_lut_mma" and r["bound"] == "hbm"
    assert r["achieved"] == pytest.approx(2 * 100e6 / (0.1 / 1e3) / 1e9)
    assert r["launches_timed"] == 2
