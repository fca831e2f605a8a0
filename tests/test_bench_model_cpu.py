"""The algorithmic-work model behind the key-switch roofline fractions, checked
against an independent derivation of the same counts (the per-configuration
totals worked out by hand from the algorithm: hybrid key switching with
contiguous digits, n = 2048, 11 264 modular products per limb transform)."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _ops(w):
    return w["bfly"] + w["mm"] + w["mac"]


def test_boot_rotation_counts():
    up, inner, down = bench.ks_work_keyswitch_parts(2100, 60, 60)
    # ModUp of one ciphertext: 35 digits x 60 sources x 2100 targets x 2048 multiply-adds
    assert up["mac"] == 35 * 60 * 2100 * 2048
    # its transforms: 2100 INTTs and 35 x 2160 - 2100 NTTs of 11 x 1024 butterflies
    assert up["bfly"] == (2100 + 35 * 2160 - 2100) * 11 * 1024
    assert _ops(up) == pytest.approx(9.89e9, rel=0.01)
    assert _ops(inner) + _ops(down) == pytest.approx(8.88e8, rel=0.01)
    w = bench.work_rotation(2100, 60, 60, 1, 4)
    assert _ops(w) == pytest.approx(1.344e10, rel=0.01)
    # 60-prime digits and 60 special primes: every conversion runs on the tensor cores
    assert w["conv_tc"] == up["mac"] + 4 * down["mac"]
    assert bench.work_rotation(2100, 60, 60, 1, 4, engine="integer")["conv_tc"] == 0
    # key bytes: 4 keys of 35 x 2 x 2160 limbs
    assert w["bytes"] == 4 * 35 * 2 * 2160 * 2048 * 8 + 2 * 2100 * 2048 * 8 * 5


def test_layer_and_bsgs_counts():
    assert _ops(bench.work_mrr(112, 8, 8, 1)) == pytest.approx(6.30e7, rel=0.02)
    assert _ops(bench.work_bsgs(112, 8, 8, 1, 32, 32)) == pytest.approx(2.78e9, rel=0.02)
    # alpha = 1, K = 1: below the tensor cores' 8 sources
    assert bench.work_rotation(4, 1, 1, 1, 1)["conv_tc"] == 0


def test_model_charges_the_engine_that_ran():
    """With the conversion on the tensor cores the roofline charges it at the
    int8 rate (64 byte-plane products per multiply-add); the integer-pipe
    model is reported beside it."""
    rates = {"bfly": 1e12, "mm": 1e12, "mac": 1e12, "int8_mac": 64e12}
    w = bench.work(mac=10**12, conv_tc=10**12)
    t_tc, _ = bench.model_seconds(w, rates, 1e3, engine_tc=True)
    t_int, _ = bench.model_seconds(w, rates, 1e3, engine_tc=False)
    assert t_tc == pytest.approx(1.0) and t_int == pytest.approx(1.0)
    e = bench.ks_entry(1, 2000.0, w, 1e3, rates)
    assert e["roofline_frac"] == pytest.approx(0.5) and e["integer_pipe_model_frac"] == pytest.approx(0.5)
    w2 = bench.work(bfly=2 * 10**12, mac=10**12, conv_tc=10**12, bytes=0)
    e2 = bench.ks_entry(1, 3000.0, w2, 1e3, rates)
    assert e2["roofline_frac"] == pytest.approx(1.0)


def test_key_inner_products_charged_at_their_own_rate():
    """The key inner product's multiply-adds (kmac, part of mac) are charged at the
    rate of its split-form product; the other multiply-adds stay at the 128-bit rate."""
    up, inner, down = bench.ks_work_keyswitch_parts(2100, 60, 60)
    assert inner["kmac"] == inner["mac"] == 2 * 35 * 2160 * 2048
    assert up["kmac"] == 0 and down["kmac"] == 0
    rates = {"bfly": 1e12, "mm": 1e12, "mac": 1e12, "int8_mac": 64e12, "kmac": 2e12}
    w = bench.work(mac=3 * 10**12, kmac=2 * 10**12)
    t, _ = bench.model_seconds(w, rates, 1e3)
    assert t == pytest.approx(1.0 + 1.0)
    assert bench.ks_entry(1, 4000.0, w, 1e3, rates)["macs_key_inner"] == 2 * 10**12
    # without a measured split-form rate, kmac falls back to the 128-bit rate
    del rates["kmac"]
    assert bench.model_seconds(w, rates, 1e3)[0] == pytest.approx(3.0)
    assert bench.rates_from({"ntt_butterfly_per_s": 1, "shoup_mulmod_per_s": 1, "mac128_per_s": 5,
                             "int8_mma_n256_ops_per_s": 2})["kmac"] == 5


def test_ntt_launch_bytes_and_products():
    bytes_, mm = bench.ntt_launch_work(2100)
    assert bytes_ == 33600 * 2 * 2048 * 8 + 2100 * 2048 * 16
    assert mm == 33600 * 1024 * 11


def test_traffic_is_reported_only_for_unchanged_sources(tmp_path, monkeypatch):
    """roofline.traffic comes from the committed ncu figure only while the
    kernel's sources hash to what they were at capture; after any change it
    is null."""
    import hashlib
    import json
    import os

    src = tmp_path / "k.cu"
    src.write_bytes(b"kernel v1")
    (tmp_path / "profiles").mkdir()
    entry = {"sources": ["k.cu"], "dram_bytes_per_launch": 12345,
             "sources_sha256_16": hashlib.sha256(b"kernel v1").hexdigest()[:16]}
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps({"k": entry}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.traffic_for("k") == 12345
    assert bench.traffic_for("other") is None
    src.write_bytes(b"kernel v2")
    assert bench.traffic_for("k") is None
    os.remove(tmp_path / "profiles" / "traffic.json")
    assert bench.traffic_for("k") is None


def test_clock_summary_decodes_the_nvml_reasons():
    """Median SM clock under load and the named clock-event reasons (NVML bit
    values: sw_power_cap 0x4, hw_slowdown 0x8, sw_thermal 0x20, hw_thermal 0x40,
    power brake 0x80); idle and application-clock bits are not reasons."""
    cs = bench.ClockSampler(None)
    cs.max_mhz = 1965
    cs.samples = [(1965, 0x0), (1900, 0x4), (1965, 0x4 | 0x8), (1950, 0x1 | 0x2)]
    s = cs.summary()
    assert s["sm_mhz"] == 1957.5 and s["sm_max_mhz"] == 1965 and s["samples"] == 4
    assert s["reasons"] == ["hw_slowdown", "sw_power_cap"]
    cs.samples = [(1965, 0x20 | 0x40 | 0x80)]
    assert cs.summary()["reasons"] == ["hw_power_brake_slowdown", "hw_thermal_slowdown",
                                       "sw_thermal_slowdown"]
    empty = bench.ClockSampler(None)
    assert empty.summary()["reasons"] == ["unsampled"]
