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
    # NVML samples: (time, SM MHz, max SM MHz, clock-event reason bits); only those inside the region
    nv = bench.ClockSampler(0)
    nv.nvml = True
    nv.samples = [(0.5, 900, 1965, 0x1), (1.0, 1965, 1965, 0x1), (1.1, 1500, 1965, 0x4),
                  (1.2, 1400, 1965, 0x4 | 0x40), (1.3, 1600, 1965, 0x0), (2.5, 1965, 1965, 0x8)]
    nv.t0, nv.t1 = 1.0, 2.0
    s = nv.summary()
    assert s["samples"] == 4 and s["sm_mhz"] == 1550 and s["sm_max_mhz"] == 1965
    assert s["reasons"] == ["hw_thermal_slowdown", "sw_power_cap"]  # 0x1 (idle) is not a slowdown
    assert s["source"].startswith("nvml")


def test_oracle_sample_single_and_threaded_on_tiny():
    from discrete_diffusion_lm_b200 import workloads as W
    samp = bench.OracleSample(rows1=16, rows2=16, vfrac=1, cfg=W.TINY)
    one = samp.run(rows2=4)
    many = samp.run_threads(3)  # 16 rows over 3 threads: ragged blocks of 5, 5, 6
    assert one["cores"] == 1 and many["cores"] == 3
    assert one["value"] > 0 and many["value"] > 0
    assert "tiny workload" in one["sample"] and "3 threads" in many["sample"]
    more_threads_than_rows = samp.run_threads(40)
    assert more_threads_than_rows["value"] > 0


def test_reference_arm_prints_one_json_line():
    import json
    import subprocess
    import sys
    out = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1", "--warmup", "3"],
                         cwd=bench.ROOT, capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["unit"] == "steps/s" and rec["value"] > 0
    assert rec["cpu_baseline"]["kind"] == "oracle" and rec["cpu_baseline"]["value"] == rec["value"]
    assert rec["e2e"]["h2d_bytes_per_step"] == 0 and rec["warmup"] >= 3
    # the same config dict as the GPU arm's line (same workload, layout and rotation)
    nbuf, lbytes = bench.rotation(bench_cfg())
    assert rec["config"] == bench.workload_config(1, nbuf, lbytes)


def bench_cfg():
    from discrete_diffusion_lm_b200 import workloads as W
    return W.FULL


def test_parity_leg_compares_the_oracle_with_a_probe_step():
    # the CPU-baseline leg's comparison, fed a probe whose "GPU" outputs are the oracle's own on the
    # same inputs: nothing differs; a planted wrong token (in a copy of the outputs) is counted
    import numpy as np
    import torch
    from discrete_diffusion_lm_b200 import workloads as W
    from oracle import oracle as O
    cfg = W.TINY
    L = W.make_logits(cfg, "cpu")
    E = W.make_embedding(cfg, "cpu")
    x_t = W.make_canvas(cfg, "cpu").numpy()
    t, dt = cfg.times(3)
    ref = O.sampler_step(L.numpy(), x_t, 1, cfg.R, cfg.V, cfg.schedule, t[:1], dt[:1], None, 0, 3, "sample")
    zr = O.selfcond_rows(L.numpy(), E.numpy(), list(range(cfg.R)))
    probe = {"step": 3, "t": t, "dt": dt, "logits": L, "x_t": x_t, "E": E,
             "out": {k: np.asarray(ref[k]).astype(np.float32 if k in ("lse", "max_prob", "entropy") else np.int32)
                     for k in ("x_next", "x0_hat", "argmax", "lse", "max_prob", "entropy")},
             "z": zr.astype(np.float32)}
    samp = bench.OracleSample(rows1=cfg.R, rows2=4, vfrac=1, cfg=cfg, probe=probe)
    samp.run(rows2=4)
    par = samp.parity()
    assert par["rows"] == cfg.R and par["argmax_mismatches"] == 0 and par["x0_hat_mismatches"] == 0
    assert par["x_next_mismatches_where_x0_hat_agrees"] == 0 and par["max_stat_abs_err"] < 1e-6
    assert par["z_rows"] == 4 and par["z_rel_fro_max_row"] < 1e-6
    probe["out"]["argmax"] = probe["out"]["argmax"].copy()
    probe["out"]["argmax"][5] += 1
    assert samp.parity()["argmax_mismatches"] == 1
    assert torch.is_tensor(L)


def test_host_cores_honours_a_cgroup_quota(tmp_path):
    f = tmp_path / "cpu.max"
    f.write_text("max 100000\n")
    free = bench.host_cores(str(f))
    assert free >= 1
    f.write_text("150000 100000\n")  # 1.5 CPUs of quota -> 2 threads at most
    assert bench.host_cores(str(f)) == min(free, 2)
    assert bench.host_cores(str(tmp_path / "absent")) == free


def test_oracle_routines_give_the_same_results_from_threads():
    # the all-cores timings call the C oracle from several threads at once: each call must depend
    # only on its own arguments
    from concurrent.futures import ThreadPoolExecutor

    import numpy as np
    from discrete_diffusion_lm_b200 import workloads as W
    from oracle import oracle as O
    cfg = W.TINY
    L = W.make_logits(cfg, "cpu").numpy()
    E = W.make_embedding(cfg, "cpu").numpy()
    x_t = W.make_canvas(cfg, "cpu").numpy()
    t, dt = cfg.times(2)

    def step(r):
        return O.sampler_step(L[r:r + 1], x_t[r:r + 1], 1, 1, cfg.V, cfg.schedule, t, dt, None, 7, 2, "sample")

    def z(r):
        return O.selfcond_rows(L, E, [r])

    serial = [step(r) for r in range(cfg.R)], [z(r) for r in range(cfg.R)]
    with ThreadPoolExecutor(max_workers=8) as pool:
        threaded = list(pool.map(step, range(cfg.R))), list(pool.map(z, range(cfg.R)))
    for a, b in zip(serial[0], threaded[0]):
        for k in ("x_next", "x0_hat", "argmax", "lse", "entropy"):
            assert np.array_equal(a[k], b[k]), k
    for a, b in zip(serial[1], threaded[1]):
        assert np.array_equal(a, b)
