"""Host-side pieces of bench.py: the peak-source naming of the fraction keys and the
kernel-source fingerprint that gates the recorded DRAM traffic."""
import json

import bench


def test_fraction_keys_name_their_peak():
    assert bench.frac_key("measured") == "frac_of_measured"
    assert bench.frac_key("fallback") == "frac_of_fallback"
    assert bench.frac_key("measured", "_bf16") == "frac_of_measured_bf16"
    assert bench.frac_key("fallback", "_bf16") == "frac_of_fallback_bf16"


def test_measured_peaks_file_or_fallback(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    peaks, src = bench.measured_peaks()
    assert src == "fallback" and peaks == bench.FALLBACK_PEAKS
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps({"bf16_tflops": 1668.1, "hbm_gbs": 6555.8}))
    peaks, src = bench.measured_peaks()
    assert src == "measured" and peaks["bf16_tflops"] == 1668.1


def test_recorded_traffic_is_tied_to_the_kernel_sources(tmp_path, monkeypatch):
    # a value is reported only while the sources still hash to the one recorded with it
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    csrc = tmp_path / "attention_attn_fwd_10_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "a.cuh").write_text("one")
    prof = tmp_path / "profiles"
    prof.mkdir()
    import hashlib

    sha = hashlib.sha1(b"one").hexdigest()
    (prof / "roofline_traffic.txt").write_text(f"# header\nattn_bwd_kernel 123 {sha}\nattn_fwd_kernel 45 0000\n")
    assert bench.captured_traffic("attn_bwd_kernel") == 123
    assert bench.captured_traffic("attn_fwd_kernel") is None  # recorded for other sources
    (csrc / "a.cuh").write_text("two")
    assert bench.captured_traffic("attn_bwd_kernel") is None
