"""CPU checks of bench.py's host-side helpers: the peaks file, the ncu-summary lookup keyed by the
kernel source's hash, and the clock-sample parser (no GPU, no nvidia-smi needed)."""
import hashlib
import os

import bench


def test_load_peaks_has_the_roofline_denominators():
    p = bench.load_peaks()
    assert p["hbm_gbs"] > 0 and p["bf16_tflops"] > 0
    assert p["source"] in ("measured", "fallback")


def test_traffic_lookup_follows_the_source_hash(tmp_path, monkeypatch):
    src_dir = tmp_path / "discrete_diffusion_lm_b200" / "csrc"
    src_dir.mkdir(parents=True)
    (tmp_path / "profiles").mkdir()
    src = src_dir / "k.cu"
    src.write_text("// kernel v1\n")
    digest = hashlib.sha256(src.read_bytes()).hexdigest()[:16]
    (tmp_path / "profiles" / "k.md").write_text(
        f"# summary\n\nsource_sha256_16: {digest}\ntraffic_bytes_per_launch: 123456\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.traffic_from_profiles("k.cu", "k.md") == 123456
    src.write_text("// kernel v2\n")  # the counters no longer describe this source
    assert bench.traffic_from_profiles("k.cu", "k.md") is None
    assert bench.traffic_from_profiles("missing.cu", "k.md") is None


def test_committed_summaries_parse():
    # each committed kernel summary names a 16-hex-digit source hash and a byte count
    for name in ("selfcond_full_vocab.md", "logits_pass_full_vocab.md"):
        text = open(os.path.join(bench.ROOT, "profiles", name)).read()
        assert "source_sha256_16:" in text and "traffic_bytes_per_launch:" in text


def test_clock_summary_parses_samples():
    cs = bench.ClockSampler(0)
    cs.lines = [
        "0, 1965, 1965, 700.1, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
        "0, 1800, 1965, 990.5, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "0, 1900, 1965, 950.0, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
        "garbage line",
    ]
    s = cs.summary()
    assert s["samples"] == 3
    assert s["sm_mhz"] == 1900 and s["sm_max_mhz"] == 1965
    assert s["reasons"] == ["sw_power_cap"]
    empty = bench.ClockSampler(0)
    assert empty.summary()["samples"] == 0
