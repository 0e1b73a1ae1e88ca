"""Host-side arithmetic of bench.py (no GPU): the per-phase roofline
fractions and the choice of the tensor peak."""
import bench

PEAKS = {"bf16_tflops": 1600.0, "bf16_tflops_sustained": 1000.0, "hbm_gbs": 5000.0}


def test_phase_rooflines_by_hand():
    m = n = 4096
    T = 131072
    ph = {"accumulate_HX_HG": 2.0, "sensitivity": 0.01, "biip_forward": 0.5, "quantize_and_pack": 3.0,
          "other": 1.0}
    r = bench.phase_rooflines(ph, [(m, n)], T, 1000.0, 5000.0, "measured")
    assert set(r) == {"accumulate_HX_HG", "sensitivity", "biip_forward", "quantize_and_pack"}
    # 2 T n (n + 1) flop in 2 ms
    acc = 2 * T * n * (n + 1) / 2e-3 / 1e12
    assert abs(r["accumulate_HX_HG"]["achieved"] - acc) < 1e-9 * acc
    assert abs(r["accumulate_HX_HG"]["frac"] - acc / 1000.0) < 1e-12
    # 48 n^2 bytes in 0.5 ms
    b = 48 * n * n / 0.5e-3 / 1e9
    assert abs(r["biip_forward"]["achieved"] - b) < 1e-9 * b and r["biip_forward"]["unit"] == "GB/s"
    q = (n ** 3 / 3 + m * n * n) / 3e-3 / 1e12
    assert abs(r["quantize_and_pack"]["achieved"] - q) < 1e-9 * q
    assert r["quantize_and_pack"]["peak_source"] == "measured"


def test_phase_work_sums_layers():
    T = 262144
    one = bench.phase_work([(28672, 8192)], T)
    two = bench.phase_work([(28672, 8192), (8192, 28672)], T)
    # gate and down have the same two factor sizes: the SYRK work doubles
    assert two["accumulate_HX_HG"] == 2 * one["accumulate_HX_HG"] == 2 * T * (8192 * 8193 + 28672 * 28673)
    assert two["biip_forward"] == 2 * one["biip_forward"]
    want = 8192 ** 3 / 3 + 28672 * 8192 ** 2 + 28672 ** 3 / 3 + 8192 * 28672 ** 2
    assert abs(two["quantize_and_pack"] - want) <= 1e-12 * want


def test_peak_choice_follows_the_clocks():
    free = {"sm_mhz": 1950.0, "sm_max_mhz": 1965.0, "reasons": []}
    capped = {"sm_mhz": 1500.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"]}
    low = {"sm_mhz": 1500.0, "sm_max_mhz": 1965.0, "reasons": []}
    assert bench.choose_peak(PEAKS, free)[0] == 1600.0
    assert bench.choose_peak(PEAKS, capped)[0] == 1000.0
    assert bench.choose_peak(PEAKS, low)[0] == 1000.0
    assert bench.choose_peak(None, free)[2].startswith("fallback")


def test_workloads_name_the_configured_shapes():
    wl = bench.WORKLOADS["llama3_70b_mlp"]
    assert wl["tokens"] == 262144 and wl["chunk"] == 16384 and wl["bits"] == 2 and wl["group"] == 128
    assert [(m, n) for _, m, n, _ in wl["layers"]] == [(28672, 8192), (8192, 28672)]
    q = bench.WORKLOADS["llama2_7b_q_proj"]
    assert q["tokens"] == 131072 and [(m, n) for _, m, n, _ in q["layers"]] == [(4096, 4096)]


def test_syrk_launch_rule():
    # d >= 16384: a 16384-token call is two 8192-token launches; smaller d one launch
    assert bench.syrk_launches(28672, 16384) == (2, 8192)
    assert bench.syrk_launches(28672, 8192) == (1, 8192)
    assert bench.syrk_launches(28672, 20000) == (3, 8192)
    assert bench.syrk_launches(8192, 16384) == (1, 16384)
    assert bench.syrk_launches(14336, 65536) == (1, 65536)
