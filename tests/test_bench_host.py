"""Host-side arithmetic of bench.py (no GPU): the per-phase roofline fractions."""
import bench


def test_phase_rooflines_by_hand():
    peaks = {"bf16_tflops_sustained": 1000.0, "hbm_gbs": 5000.0}
    m = n = 4096
    T = 131072
    ph = {"accumulate_HX_HG": 2.0, "sensitivity": 0.01, "biip_forward": 0.5, "quantize_and_pack": 3.0,
          "other": 1.0}
    r = bench.phase_rooflines(ph, m, n, T, peaks)
    assert set(r) == {"accumulate_HX_HG", "sensitivity", "biip_forward", "quantize_and_pack"}
    # 2 T n (n + 1) flop in 2 ms
    acc = 2 * T * n * (n + 1) / 2e-3 / 1e12
    assert abs(r["accumulate_HX_HG"]["achieved"] - acc) < 1e-9 * acc
    assert abs(r["accumulate_HX_HG"]["frac"] - acc / 1000.0) < 1e-12
    # 48 n^2 bytes in 0.5 ms
    b = 48 * n * n / 0.5e-3 / 1e9
    assert abs(r["biip_forward"]["achieved"] - b) < 1e-9 * b and r["biip_forward"]["unit"] == "GB/s"
    q = (2 * n ** 3 / 3 + m * n * n) / 3e-3 / 1e12
    assert abs(r["quantize_and_pack"]["achieved"] - q) < 1e-9 * q
    assert r["quantize_and_pack"]["peak_source"] == "measured"


def test_phase_rooflines_fallback_peaks():
    r = bench.phase_rooflines({"biip_forward": 1.0}, 256, 256, 2048, None)
    assert r["biip_forward"]["peak"] == 6650.0 and r["biip_forward"]["peak_source"] == "fallback"
