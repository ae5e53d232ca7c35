"""Benchmark of the per-step sampler hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

A step is one sampler step of the full-vocabulary workload (one canvas of C = 256 tokens,
V = 262144, d = 2048, bf16 logits and embeddings, cosine schedule, 12 denoising steps per
block), made through the public fused entry point dg_sampler_selfcond_step: the logits pass
(softmax statistics, argmax, two-level Gumbel-max draw of x0_hat, Step posterior) followed by
the self-conditioning contraction z = softmax(L) E, which starts while the pass finishes.  The
metric is sampler steps/s (and canvas tokens/s = 256 x steps/s), whole job over N GPUs.

Timing: W untimed warm-up steps, then exactly K steps between a barrier + synchronize on
both sides, on the device with CUDA events, max over ranks.  Each step reads its own logits
buffer out of a rotation whose total size is well above the 126 MB L2 (inputs larger than
L2).  The K steps are one CUDA graph captured beforehand (a denoising loop as a sampler would
run it), replayed once.  N > 1 runs independent replicas, one per GPU (the path has no data
exchange): weak scaling.

Also reported: the dominant kernel's roofline (measured burst peaks), an end-to-end figure
through the public API with host buffers (host->device logits copy and device->host read
of x_next and z inside the timed region), the training-side kernels (forward noise and
canvas cross-entropy on the training workload), the CPU oracle timed on a bounded sample
(rank 0, N = 1; on one thread, and over row blocks on every host core) together with its
comparison against one GPU step on the same inputs (`parity`), SM clocks sampled during the
timed region, and the number of library kernel launches in the timed region.

--impl reference times the CPU oracle (the plain C reference of the same computation) on a
bounded sample of the same workload, its rows split over every host core.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

L2_BYTES = 126 * 2**20
METRIC = "sampler steps/s and canvas tokens/s at C=256,V=262144,d=2048; % of roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        d["source"] = "measured"
        return d
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS)


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def whole_job_rate(local_ms: float, units_per_rank: int, world: int, device="cpu"):
    """Max over ranks of the per-rank device time (ms) and the whole-job rate: every rank
    processed `units_per_rank` units, so the job did world * units_per_rank in the slowest
    rank's time.  Collective only when world > 1 (the data path itself exchanges nothing)."""
    import torch
    ms = float(local_ms)
    if world > 1:
        t = torch.tensor([ms], dtype=torch.float64, device=device)
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
        ms = float(t.item())
    return ms, world * units_per_rank / (ms / 1e3)


# ------------------------------------------------------------------------------ clocks
# NVML poller run as a child process (no GIL shared with the timing thread): prints
# "time sm_mhz max_sm_mhz reason_bits" lines about every 0.2 ms until it is terminated.
_NVML_POLLER = r"""
import sys, time
import pynvml
pynvml.nvmlInit()
h = pynvml.nvmlDeviceGetHandleByUUID(sys.argv[1])
reasons = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
    pynvml.nvmlDeviceGetCurrentClocksThrottleReasons
mx = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
out = sys.stdout
while True:
    out.write("%.6f %d %d %d\n" % (time.time(), pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM), mx,
                                    int(reasons(h))))
    out.flush()
    time.sleep(0.0002)
"""


class ClockSampler:
    """SM clock and clock-event (throttle) reasons sampled while the timed region runs.

    An NVML poller in a child process samples about every 0.2 ms; the samples kept are those whose
    time lies between mark_start() and mark_end(), which bracket the timed region, so even a region
    of a few milliseconds is sampled from inside.  Without NVML: nvidia-smi every 200 ms around the
    region."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    # NVML clock-event reason bits
    REASON_BITS = {"sw_power_cap": 0x4, "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20,
                   "hw_thermal_slowdown": 0x40}

    def __init__(self, gpu_index: int):
        self.gpu = str(gpu_index)
        try:
            import torch
            u = str(torch.cuda.get_device_properties(gpu_index).uuid)
            self.gpu = u if u.startswith("GPU-") else "GPU-" + u
        except Exception:
            pass
        self.proc = None
        self.lines = []
        self.nvml = False
        self.samples = []  # (time, sm MHz, max sm MHz, reason bits) from NVML
        self.t0 = self.t1 = None

    def mark_start(self):
        self.t0 = time.time()

    def mark_end(self):
        self.t1 = time.time()

    def _start_nvml(self) -> bool:
        try:
            import pynvml  # noqa: F401  (the poller needs it)
        except ImportError:
            return False
        try:
            self.proc = subprocess.Popen([sys.executable, "-c", _NVML_POLLER, self.gpu], stdout=subprocess.PIPE,
                                         stderr=subprocess.DEVNULL, text=True)
        except OSError:
            return False
        first = self.proc.stdout.readline()  # wait until it samples
        if not first:
            self.proc.wait(timeout=5)
            self.proc = None
            return False
        self.lines.append(first.strip())
        return True

    def __enter__(self):
        self.nvml = self._start_nvml()
        if not self.nvml:
            try:
                self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.QUERY}",
                                              "--format=csv,noheader,nounits", "-lms", "200"],
                                             stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            except OSError:
                self.proc = None
        if self.proc is not None:
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        if not self.nvml:
            time.sleep(0.3)
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        time.sleep(0.01 if self.nvml else 0.25)
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.thread.join(timeout=5)
        if self.nvml:
            for line in self.lines:
                f = line.split()
                if len(f) == 4:
                    try:
                        self.samples.append((float(f[0]), float(f[1]), float(f[2]), int(f[3])))
                    except ValueError:
                        pass

    def summary(self):
        sm, mx, reasons = [], [], set()
        if self.nvml:
            for t, clk, m, bits in self.samples:
                if self.t0 is not None and t < self.t0:
                    continue
                if self.t1 is not None and t > self.t1:
                    continue
                sm.append(clk)
                mx.append(m)
                reasons.update(name for name, bit in self.REASON_BITS.items() if bits & bit)
            src = "nvml (child process, every ~0.2 ms), samples inside the timed region"
        else:
            names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
            for line in self.lines:
                f = [x.strip() for x in line.split(",")]
                if len(f) < 9:
                    continue
                try:
                    sm.append(float(f[1]))
                    mx.append(float(f[2]))
                except ValueError:
                    continue
                for name, val in zip(names, f[5:9]):
                    if val.lower().startswith("active"):
                        reasons.add(name)
            src = "nvidia-smi every 200 ms around the timed region"
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0, "source": src}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm), "source": src}


# ------------------------------------------------------------------------------ roofline helpers
def traffic_from_profiles(kernel_file: str, summary_name: str):
    """Per-launch DRAM bytes from the committed ncu summary, if it was taken on this source."""
    path = os.path.join(ROOT, "profiles", summary_name)
    src = os.path.join(ROOT, "discrete_diffusion_lm_b200", "csrc", kernel_file)
    try:
        text = open(path).read()
        digest = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    except OSError:
        return None
    m_hash = re.search(r"source_sha256_16:\s*([0-9a-f]{16})", text)
    m_bytes = re.search(r"traffic_bytes_per_launch:\s*([0-9]+)", text)
    if not m_hash or not m_bytes or m_hash.group(1) != digest:
        return None
    return int(m_bytes.group(1))


# ------------------------------------------------------------------------------ our arm
def workload_config(world: int, nbuf: int, lbytes: int, cfg=None) -> dict:
    """The `config` of the JSON line: the same dict on both arms."""
    if cfg is None:
        from discrete_diffusion_lm_b200 import workloads as W
        cfg = W.FULL
    return {"workload": "full-vocab sampler step: 1 canvas, C=256, V=262144, d=2048, bf16, cosine, 12 steps per "
                        "block; step = logits pass + self-conditioning contraction (fused entry point)",
            "B": cfg.B, "C": cfg.C, "V": cfg.V, "d": cfg.d, "parallelism": f"replicas x{world}",
            "l2": f"inputs larger than L2: {nbuf} rotating logits buffers of {lbytes / 1e6:.1f} MB "
                  f"+ E {cfg.V * cfg.d * 2 / 1e9:.2f} GB"}


def rotation(cfg) -> tuple:
    """Number of identical-content logits buffers cycled so that the step's inputs exceed L2."""
    lbytes = cfg.R * cfg.V * 2
    return max(2, math.ceil(3 * L2_BYTES / lbytes) + 1), lbytes


def graph_of(fn, ks, stream):
    """One CUDA graph holding fn(k) for every k in ks, in order."""
    import torch
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for k in ks:
            fn(k)
    return g


def timed_replay(g, stream) -> float:
    """Device time (ms) of one replay of g, CUDA events on the launching stream."""
    import torch
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        a.record(stream)
        g.replay()
        b.record(stream)
    stream.synchronize()
    return a.elapsed_time(b)


def settle(stream, seconds: float = 0.5) -> None:
    """Idle the GPU briefly between independent measurement blocks."""
    stream.synchronize()
    time.sleep(seconds)


def run_ours(args, rank, world, local):
    import torch
    import discrete_diffusion_lm_b200 as dg
    from discrete_diffusion_lm_b200 import workloads as W

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    cfg = W.FULL
    peaks = load_peaks()
    # One stream for everything: inputs, outputs, library calls and graph captures.  Tensors
    # allocated on one stream and written by kernels on another could be handed out again by the
    # caching allocator while work queued on the first stream still uses the memory.
    stream = torch.cuda.Stream(device=dev)
    torch.cuda.set_stream(stream)

    # inputs resident in HBM: a rotation of identical-content logits buffers (> 3x L2 in total)
    base = W.make_logits(cfg, dev)
    nbuf, lbytes = rotation(cfg)
    bufs = [base] + [base.clone() for _ in range(nbuf - 1)]
    E = W.make_embedding(cfg, dev)
    x0 = W.make_canvas(cfg, dev)
    x_buf = [x0.clone(), torch.empty(cfg.R, dtype=torch.int32, device=dev)]
    outs = [{k: torch.empty(cfg.R, dtype=dt, device=dev) for k, dt in
             (("x0_hat", torch.int32), ("argmax", torch.int32), ("max_prob", torch.float32),
              ("lse", torch.float32), ("entropy", torch.float32), ("branch", torch.uint8))} for _ in range(2)]
    z = torch.empty((cfg.R, cfg.d), dtype=torch.bfloat16, device=dev)
    ws_s = torch.zeros(dg.dg_sampler_step_workspace_size(cfg.R, cfg.V), dtype=torch.uint8, device=dev)
    ws_z = torch.zeros(max(256, dg.dg_selfcond_workspace_size(cfg.R, cfg.V, cfg.d, 1, 1, True)), dtype=torch.uint8,
                       device=dev)

    def step(k):  # one sampler step through the public fused entry point
        t, dt = cfg.times(k % cfg.steps)
        o = outs[k % 2]
        o["x_next"] = x_buf[(k + 1) % 2]
        dg.dg_sampler_selfcond_step(bufs[k % nbuf], x_buf[k % 2], E, cfg.C, t, dt, schedule=cfg.schedule, seed=0,
                                    step=k, out=o, z=z, ws=ws_s, ws_z=ws_z, stream=stream)

    def k1(k):  # the logits pass alone
        t, dt = cfg.times(k % cfg.steps)
        o = outs[k % 2]
        o["x_next"] = x_buf[(k + 1) % 2]
        dg.dg_sampler_step(bufs[k % nbuf], x_buf[k % 2], cfg.C, t, dt, schedule=cfg.schedule, seed=0, step=k,
                           out=o, ws=ws_s, stream=stream)

    def k2(k):  # the contraction alone (lse of the last logits pass)
        dg.dg_selfcond(bufs[k % nbuf], E, cfg.C, lse=outs[k % 2]["lse"], z=z, ws=ws_z, stream=stream)

    with torch.cuda.stream(stream):
        for k in range(2):
            step(k)
    stream.synchronize()
    K, Wm = args.steps, args.warmup
    g_warm = graph_of(step, range(Wm), stream)
    c0 = dg.dg_launch_count()
    g_steps = graph_of(step, range(Wm, Wm + K), stream)
    launches = dg.dg_launch_count() - c0
    g_k1 = graph_of(k1, range(Wm, Wm + K), stream)
    g_k2 = graph_of(k2, range(Wm, Wm + K), stream)
    assert dg.dg_device_error() == 0

    def barrier():
        if world > 1:
            torch.distributed.barrier()

    # W untimed warm-up steps, then exactly K steps (one graph of K fused steps), events on the stream
    with torch.cuda.stream(stream):
        g_warm.replay()
    stream.synchronize()
    barrier()
    torch.cuda.synchronize(dev)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    with ClockSampler(local) as clocks:
        clocks.mark_start()
        with torch.cuda.stream(stream):
            ev[0].record(stream)
            g_steps.replay()
            ev[1].record(stream)
        stream.synchronize()
        clocks.mark_end()
    torch.cuda.synchronize(dev)
    barrier()
    total_ms = ev[0].elapsed_time(ev[1])
    dev_err = dg.dg_device_error()
    total_ms, steps_per_s = whole_job_rate(total_ms, K, world, dev)

    # ---- the two kernels of the step, each in a graph of K back-to-back launches (same inputs)
    settle(stream)
    for g in (g_k1, g_k2):
        timed_replay(g, stream)  # warm
    k1_us = timed_replay(g_k1, stream) * 1e3 / K
    k2_us = timed_replay(g_k2, stream) * 1e3 / K

    # ---- roofline of the dominant kernel (the contraction) against the burst peaks: the timed region
    # lasts milliseconds.  Slower of the tensor and HBM bounds; the other fraction is reported beside.
    flops_k2 = 2.0 * cfg.R * cfg.V * cfg.d
    bytes_k2 = cfg.V * cfg.d * 2 + cfg.R * cfg.V * 2 + cfg.R * cfg.d * 2 + cfg.R * 4
    bytes_k1 = cfg.R * cfg.V * 2 + cfg.R * 4 + cfg.R * 25
    hbm = peaks["hbm_gbs"]
    tc = peaks["bf16_tflops"]
    t_tensor_us = flops_k2 / (tc * 1e12) * 1e6
    t_hbm_us = bytes_k2 / (hbm * 1e9) * 1e6
    tflops = flops_k2 / (k2_us * 1e-6) / 1e12
    gbs = bytes_k2 / (k2_us * 1e-6) / 1e9
    if t_tensor_us >= t_hbm_us:
        roof = {"bound": "tensor", "achieved": round(tflops, 1), "peak": tc, "unit": "TFLOP/s",
                "frac": round(tflops / tc, 4)}
    else:
        roof = {"bound": "hbm", "achieved": round(gbs, 1), "peak": hbm, "unit": "GB/s", "frac": round(gbs / hbm, 4)}
    roof["traffic"] = traffic_from_profiles("selfcond.cu", "selfcond_full_vocab.md")
    roof["kernel"] = "selfcond (z = softmax(L) E, tcgen05), its average over K back-to-back launches"
    roof["peak_source"] = f"{peaks['source']} (burst: HBM copy and bf16 GEMM peaks)"
    roof["slower_bound_us"] = round(max(t_tensor_us, t_hbm_us), 1)
    roof["tensor_frac_burst"] = round(tflops / tc, 4)
    if "bf16_tflops_sustained" in peaks:
        roof["tensor_frac_sustained"] = round(tflops / peaks["bf16_tflops_sustained"], 4)
    k1_gbs = bytes_k1 / (k1_us * 1e-6) / 1e9

    # ---- training-side kernels, entropy-bounded step, FFW, other workloads.  Each block starts after a
    # short idle gap, so that the power controller's state after the previous block's load (the SM
    # clock it settled at under the 1 kW cap) does not carry into the next block's numbers.
    settle(stream)
    train = bench_train(dg, W, dev, stream, hbm)
    settle(stream)
    eb = bench_eb(dg, W, dev, stream, bufs, hbm)
    settle(stream)
    ffw = bench_ffw(dg, W, dev, stream, peaks)
    settle(stream)
    configs = bench_configs(dg, W, dev, stream, peaks)

    # ---- end to end through the public API with host buffers
    e2e = bench_e2e(dg, W, cfg, dev, E, args, world, barrier, stream)

    # ---- one more fused step on the first buffer, for the CPU oracle's comparison (outside the timed
    # region; the oracle runs only in the CPU-baseline leg)
    probe_step = 3
    t, dt = cfg.times(probe_step)
    probe = dg.dg_sampler_selfcond_step(base, x0, E, cfg.C, t, dt, schedule=cfg.schedule, seed=0, step=probe_step,
                                        stream=stream)
    stream.synchronize()
    probe_host = {"step": probe_step, "t": t, "dt": dt, "logits": base, "x_t": x0.cpu().numpy(), "E": E,
                  "out": {k: v.cpu().numpy() for k, v in probe.items() if k != "z"},
                  "z": probe["z"].float().cpu().numpy()}

    line = {
        "metric": METRIC,
        "value": round(steps_per_s, 2),
        "unit": "steps/s",
        "n_gpus": world,
        "steps": K,
        "warmup": Wm,
        "ms_per_step": round(total_ms / K, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded; logits N(0,1.5) + Zipf(1.1) boost on 64 ids per row; E ~ N(0, 0.02))",
        "config": workload_config(world, nbuf, lbytes, cfg),
        "canvas_tokens_per_s": round(steps_per_s * cfg.C, 1),
        "roofline": roof,
        "kernels": {
            "timing": "each kernel in a graph of K back-to-back launches on the step's inputs (CUDA events)",
            "logits_pass_us": round(k1_us, 2), "logits_pass_GBps": round(k1_gbs, 1),
            "logits_pass_frac_hbm": round(k1_gbs / hbm, 4),
            "selfcond_us": round(k2_us, 2),
            "selfcond_TFLOPs": round(tflops, 1),
            "selfcond_frac_hbm": round(gbs / hbm, 4),
            "selfcond_frac_tensor_burst": round(tflops / tc, 4),
            "train": train,
            "entropy_bounded": eb,
            "ffw": ffw,
            "other_workloads": configs,
        },
        "e2e": e2e,
        "gpu_launches": int(launches),
        "device_error": dev_err,
        "clocks": clocks.summary(),
    }
    return line, probe_host


def bench_train(dg, W, dev, stream, hbm):
    import torch
    cfg = W.TRAIN
    x0 = W.make_train_tokens(cfg, dev)
    t = W.make_train_times(cfg)
    logits = W.make_train_logits(cfg, dev)
    xt = torch.empty_like(x0)
    kidx = torch.empty(cfg.n_seq, dtype=torch.int32, device=dev)
    loss = torch.empty(cfg.n_seq * cfg.C, dtype=torch.float32, device=dev)
    seq = torch.empty(cfg.n_seq, dtype=torch.float32, device=dev)
    lse = torch.empty_like(loss)
    ws = torch.zeros(dg.dg_canvas_ce_workspace_size(cfg.n_seq, cfg.C, cfg.V), dtype=torch.uint8, device=dev)
    with torch.cuda.stream(stream):
        gn, gc = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
        dg.dg_forward_noise(x0, cfg.P, cfg.K, cfg.C, cfg.V, t, seed=1, x_t=xt, canvas_idx=kidx, stream=stream)
        dg.dg_canvas_ce(logits, x0, kidx, cfg.P, cfg.K, cfg.C, loss_rows=loss, loss_seq=seq, lse_rows=lse, ws=ws,
                        stream=stream)
    stream.synchronize()
    with torch.cuda.graph(gn, stream=stream):
        dg.dg_forward_noise(x0, cfg.P, cfg.K, cfg.C, cfg.V, t, seed=1, x_t=xt, canvas_idx=kidx, stream=stream)
    with torch.cuda.graph(gc, stream=stream):
        dg.dg_canvas_ce(logits, x0, kidx, cfg.P, cfg.K, cfg.C, loss_rows=loss, loss_seq=seq, lse_rows=lse, ws=ws,
                        stream=stream)
    reps = 20
    e = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    with torch.cuda.stream(stream):
        for _ in range(3):
            gn.replay()
            gc.replay()
        e[0].record(stream)
        for _ in range(reps):
            gn.replay()
        e[1].record(stream)
        for _ in range(reps):
            gc.replay()
        e[2].record(stream)
    stream.synchronize()
    noise_us = e[0].elapsed_time(e[1]) * 1e3 / reps
    ce_us = e[1].elapsed_time(e[2]) * 1e3 / reps
    ce_bytes = cfg.n_seq * cfg.C * cfg.V * 2
    # backward of the canvas CE, in place over the same logits (their values no longer matter for
    # timing), and the self-conditioning drop on a z of the training rows
    z = torch.randn(cfg.n_seq * cfg.C, 2048, device=dev).to(torch.bfloat16)
    gb, gd = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        dg.dg_canvas_ce_backward(logits, lse, x0, kidx, cfg.P, cfg.K, cfg.C, stream=stream)
        dg.dg_selfcond_drop(z, cfg.C, seed=0, step=0, stream=stream)
    stream.synchronize()
    with torch.cuda.graph(gb, stream=stream):
        dg.dg_canvas_ce_backward(logits, lse, x0, kidx, cfg.P, cfg.K, cfg.C, stream=stream)
    with torch.cuda.graph(gd, stream=stream):
        dg.dg_selfcond_drop(z, cfg.C, seed=0, step=1, stream=stream)
    e2 = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    with torch.cuda.stream(stream):
        for _ in range(3):
            gb.replay()
            gd.replay()
        e2[0].record(stream)
        for _ in range(reps):
            gb.replay()
        e2[1].record(stream)
        for _ in range(reps):
            gd.replay()
        e2[2].record(stream)
    stream.synchronize()
    bw_us = e2[0].elapsed_time(e2[1]) * 1e3 / reps
    drop_us = e2[1].elapsed_time(e2[2]) * 1e3 / reps
    bw_bytes = 2 * ce_bytes  # read and write every logit
    return {"workload": "train: 8 seq x (P=512 + K=4 x C=256), V=262144, bf16 CE logits [2048, 262144]",
            "forward_noise_us": round(noise_us, 2), "canvas_ce_us": round(ce_us, 2),
            "canvas_ce_GBps": round(ce_bytes / (ce_us * 1e-6) / 1e9, 1),
            "canvas_ce_frac_hbm": round(ce_bytes / (ce_us * 1e-6) / 1e9 / hbm, 4),
            "ce_backward_us": round(bw_us, 2),
            "ce_backward_GBps": round(bw_bytes / (bw_us * 1e-6) / 1e9, 1),
            "ce_backward_frac_hbm": round(bw_bytes / (bw_us * 1e-6) / 1e9 / hbm, 4),
            "selfcond_drop_us": round(drop_us, 2),
            "note": "canvas CE logits (1.07 GB) exceed L2; repeated on one buffer (the backward in place)"}


def bench_ffw(dg, W, dev, stream, peaks):
    """The feed-forward block on the self-conditioning input at the full size (R=256, d=2048,
    d_ff=8192, random bf16 weights): both layers, each a tcgen05 contraction + split sum."""
    import torch
    cfg = W.FULL
    z, w1, w2 = W.make_ffw(cfg, dev)
    out, hidden = dg.dg_ffw(z, w1, w2, stream=stream)
    stream.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        dg.dg_ffw(z, w1, w2, hidden=hidden, out=out, stream=stream)
    reps = 50
    e = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    with torch.cuda.stream(stream):
        for _ in range(5):
            g.replay()
        e[0].record(stream)
        for _ in range(reps):
            g.replay()
        e[1].record(stream)
    stream.synchronize()
    us = e[0].elapsed_time(e[1]) * 1e3 / reps
    dff = W.FFW_RATIO * cfg.d
    flops = 2.0 * 2 * cfg.R * cfg.d * dff
    nbytes = 2 * cfg.d * dff * 2 + cfg.R * (2 * cfg.d + 2 * dff) * 2
    tc = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])
    bound_us = max(flops / (tc * 1e12), nbytes / (peaks["hbm_gbs"] * 1e9)) * 1e6
    return {"workload": f"FFW gelu(z W1) W2: R={cfg.R}, d={cfg.d}, d_ff={dff}, bf16, weights {nbytes / 1e6:.0f} MB "
                        "(L2-resident across replays)",
            "ffw_us": round(us, 2), "ffw_TFLOPs": round(flops / (us * 1e-6) / 1e12, 1),
            "ffw_frac_of_slower_bound": round(bound_us / us, 4), "slower_bound_us": round(bound_us, 2)}


def bench_configs(dg, W, dev, stream, peaks):
    """Per-kernel times of the other sampler workloads (logits pass incl. merge; contraction incl.
    split sum), graph replays after warm-up; tiny and mid fit in L2 (times only)."""
    import torch
    hbm = peaks["hbm_gbs"]
    tc = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])
    out = {}
    for name in ("tiny", "mid", "batched"):
        cfg = W.SAMPLER_CONFIGS[name]
        logits = W.make_logits(cfg, dev)
        E = W.make_embedding(cfg, dev)
        x_t = W.make_canvas(cfg, dev)
        t, dt = cfg.times(1)
        o = dg.dg_sampler_step(logits, x_t, cfg.C, t, dt, schedule=cfg.schedule, stream=stream)
        z = dg.dg_selfcond(logits, E, cfg.C, lse=o["lse"], stream=stream)
        stream.synchronize()
        g1, g2 = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
        with torch.cuda.graph(g1, stream=stream):
            dg.dg_sampler_step(logits, x_t, cfg.C, t, dt, schedule=cfg.schedule, out=o, stream=stream)
        with torch.cuda.graph(g2, stream=stream):
            dg.dg_selfcond(logits, E, cfg.C, lse=o["lse"], z=z, stream=stream)
        reps = 10
        e = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        with torch.cuda.stream(stream):
            for _ in range(3):
                g1.replay()
                g2.replay()
            e[0].record(stream)
            for _ in range(reps):
                g1.replay()
            e[1].record(stream)
            for _ in range(reps):
                g2.replay()
            e[2].record(stream)
        stream.synchronize()
        k1 = e[0].elapsed_time(e[1]) * 1e3 / reps
        k2 = e[1].elapsed_time(e[2]) * 1e3 / reps
        lbytes = logits.numel() * logits.element_size()
        flops = 2.0 * cfg.R * cfg.V * cfg.d
        out[name] = {"R": cfg.R, "V": cfg.V, "d": cfg.d, "logits_pass_us": round(k1, 2), "selfcond_us": round(k2, 2),
                     "step_us": round(k1 + k2, 2), "selfcond_TFLOPs": round(flops / (k2 * 1e-6) / 1e12, 1)}
        if name == "batched":
            out[name]["logits_pass_frac_hbm"] = round(lbytes / (k1 * 1e-6) / 1e9 / hbm, 4)
            out[name]["selfcond_frac_tensor_sustained"] = round(flops / (k2 * 1e-6) / 1e12 / tc, 4)
        else:
            out[name]["note"] = "inputs fit in L2: times only"
        del logits, E, x_t, o, z, g1, g2
        torch.cuda.empty_cache()
    return out


def bench_eb(dg, W, dev, stream, bufs, hbm):
    """The entropy-bounded sampler step (logits pass + per-canvas acceptance and stopping) on the
    full-vocab workload with the annealed temperature, 24 steps captured back to back in one graph
    (as a multi-step sampler loop runs them), and the per-canvas kernel alone."""
    import torch
    cfg = W.FULL
    nbuf = len(bufs)
    reps = 24
    outs = [dg.dg_sampler_step_eb(bufs[0], cfg.C, eps=64.0, theta=0.5, inv_tau=dg.dg_tau_linear([0.5]), stream=stream)
            for _ in range(2)]
    ws = torch.zeros(dg.dg_sampler_step_workspace_size(cfg.R, cfg.V), dtype=torch.uint8, device=dev)
    stream.synchronize()

    def steps(k0):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for k in range(k0, k0 + reps):
                dg.dg_sampler_step_eb(bufs[k % nbuf], cfg.C, eps=64.0, theta=0.5, argmax_prev=outs[(k + 1) % 2]["argmax"],
                                      inv_tau=dg.dg_tau_linear([1.0 - (k % reps) / reps]), seed=0, step=k,
                                      out=outs[k % 2], ws=ws, stream=stream)
        return g
    g_warm, g_eb = steps(0), steps(reps)
    gdec = torch.cuda.CUDAGraph()
    with torch.cuda.graph(gdec, stream=stream):
        for _ in range(reps):
            dg.dg_entropy_accept(outs[0]["entropy"], outs[0]["x0_hat"], cfg.C, cfg.V, 64.0, stream=stream)
    e = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    with torch.cuda.stream(stream):
        g_warm.replay()
        gdec.replay()
        e[0].record(stream)
        g_eb.replay()
        e[1].record(stream)
        gdec.replay()
        e[2].record(stream)
    stream.synchronize()
    step_us = e[0].elapsed_time(e[1]) * 1e3 / reps
    dec_us = e[1].elapsed_time(e[2]) * 1e3 / reps
    lbytes = cfg.R * cfg.V * 2
    return {"workload": "entropy-bounded step on the full-vocab workload (C=256, V=262144), eps=64, theta=0.5, "
                        "tau annealed 0.8->0.4; 24 steps back to back in one graph", "eb_step_us": round(step_us, 2),
            "eb_step_frac_hbm": round(lbytes / (step_us * 1e-6) / 1e9 / hbm, 4),
            "canvas_decide_us": round(dec_us, 2)}


def bench_e2e(dg, W, cfg, dev, E, args, world, barrier, stream):
    """Same metric through the public API with host buffers: every step copies its logits from
    pinned host memory to the device and reads x_next and z back into pinned host memory.  The
    host-to-device copies run on a copy stream into two alternating device buffers, so step k+1's
    copy overlaps step k's kernels; every copy lies inside the timed region."""
    import torch
    host_logits = W.make_logits(cfg, "cpu").pin_memory()
    dev_logits = [torch.empty_like(host_logits, device=dev) for _ in range(2)]
    x_t = W.make_canvas(cfg, dev)
    host_x = torch.empty(cfg.R, dtype=torch.int32).pin_memory()
    host_z = torch.empty((cfg.R, cfg.d), dtype=torch.bfloat16).pin_memory()
    steps = max(3, min(args.steps, 24))
    copy_stream = torch.cuda.Stream(device=dev)
    copied = [torch.cuda.Event() for _ in range(2)]
    consumed = [torch.cuda.Event() for _ in range(2)]

    def issue_copy(k):
        b = k % 2
        with torch.cuda.stream(copy_stream):
            copy_stream.wait_event(consumed[b])  # the step that last read this buffer has run
            dev_logits[b].copy_(host_logits, non_blocking=True)
            copied[b].record(copy_stream)

    def one(k):
        b = k % 2
        stream.wait_event(copied[b])
        t, dt = cfg.times(k % cfg.steps)
        out = dg.dg_sampler_selfcond_step(dev_logits[b], x_t, E, cfg.C, t, dt, schedule=cfg.schedule, seed=0,
                                          step=k, stream=stream)
        consumed[b].record(stream)
        x_t.copy_(out["x_next"])
        host_x.copy_(out["x_next"], non_blocking=True)
        host_z.copy_(out["z"], non_blocking=True)

    def run(n):
        issue_copy(0)
        for k in range(n):
            if k + 1 < n:
                issue_copy(k + 1)
            one(k)

    with torch.cuda.stream(stream):
        run(3)
    stream.synchronize()
    copy_stream.synchronize()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        copy_stream.wait_stream(stream)  # the first copy starts inside the timed region
        run(steps)
        e1.record(stream)
    stream.synchronize()
    ms, rate = whole_job_rate(e0.elapsed_time(e1), steps, world, dev)
    return {"value": round(rate, 2), "unit": "steps/s",
            "h2d_bytes_per_step": host_logits.numel() * host_logits.element_size(),
            "d2h_bytes_per_step": host_x.numel() * 4 + host_z.numel() * 2, "steps": steps,
            "copies": "host-to-device on a second stream, double-buffered (step k+1's copy overlaps step k)"}


# ------------------------------------------------------------------------------ the oracle
class OracleSample:
    """The CPU oracle (plain C, double precision, as it stands) on a bounded sample of the
    full-vocab workload: the logits-pass work (statistics, argmax, two-level draw, Step) on
    `rows1` rows and the contraction z = softmax(l) E on `rows2` rows over a fraction `vfrac` of
    the vocabulary; the measured time is scaled to one step (256 rows, all of V).  With `probe`
    (the GPU's inputs and outputs of one step) the sample runs on exactly those inputs, and the
    single-thread run's results are compared with the GPU's."""

    def __init__(self, rows1: int, rows2: int, vfrac: int, cfg=None, probe=None):
        import numpy as np
        from discrete_diffusion_lm_b200 import workloads as W
        self.cfg = cfg = cfg or W.FULL
        self.rows1, self.rows2, self.vfrac = rows1, rows2, vfrac
        self.probe = probe
        n = max(rows1, rows2)
        if probe is not None:
            self.L = probe["logits"][:n].float().cpu().numpy()
            self.E = probe["E"][: cfg.V // vfrac].float().cpu().numpy()
            self.x_t = np.ascontiguousarray(probe["x_t"][:rows1])
            self.t, self.dt, self.step = probe["t"], probe["dt"], probe["step"]
        else:
            self.L = W.make_logits(cfg, "cpu", rows=n).float().numpy()
            self.E = W.make_embedding(cfg, "cpu")[: cfg.V // vfrac].float().numpy()
            self.x_t = np.zeros(rows1, dtype=np.int32)
            (self.t, self.dt), self.step = cfg.times(0), 0
        self.Vs = cfg.V // vfrac
        self.Ls = np.ascontiguousarray(self.L[:rows2, : self.Vs])
        self.results = None

    def _pass(self, a: int, b: int):
        from oracle import oracle as O
        cfg = self.cfg
        return O.sampler_step(self.L[a:b], self.x_t[a:b], 1, b - a, cfg.V, cfg.schedule, self.t[:1], self.dt[:1], None,
                              0, self.step, "sample")

    def _z(self, a: int, b: int):
        from oracle import oracle as O
        return O.selfcond_rows(self.Ls, self.E, list(range(a, b)))

    def _what(self) -> str:
        c = self.cfg
        return f"{c.name} workload (C={c.C}, V={c.V}, d={c.d})"

    def _per_step(self, t_pass: float, rows1: int, t_z: float, rows2: int) -> float:
        return self.cfg.R * (t_pass / rows1 + t_z * self.vfrac / rows2)

    def run(self, rows2: int = 0) -> dict:
        """Single thread: the logits pass on all `rows1` rows, z on the first `rows2` rows."""
        rows2 = rows2 or self.rows2
        t0 = time.perf_counter()
        ref = self._pass(0, self.rows1)
        t1 = time.perf_counter()
        zr = self._z(0, rows2)
        t2 = time.perf_counter()
        self.results = (ref, zr)
        step_s = self._per_step(t1 - t0, self.rows1, t2 - t1, rows2)
        return {"value": 1.0 / step_s, "unit": "steps/s", "cores": 1, "kind": "oracle", "cpu_seconds": t2 - t0,
                "sample": f"{self._what()}: logits pass on {self.rows1} rows + z on {rows2} rows over "
                          f"1/{self.vfrac} of V, scaled to {self.cfg.R} rows x full V per step"}

    def run_threads(self, threads: int) -> dict:
        """The same routines over contiguous row blocks, one block per thread, all threads at once
        (the C oracle keeps no global state, and ctypes releases the GIL for each foreign call).
        A block restarts the oracle's row numbering, which changes the random words drawn, not
        the work done."""
        from concurrent.futures import ThreadPoolExecutor

        def blocks(n):
            k = min(threads, n)
            edges = [n * i // k for i in range(k + 1)]
            return list(zip(edges[:-1], edges[1:]))

        with ThreadPoolExecutor(max_workers=threads) as pool:
            t0 = time.perf_counter()
            list(pool.map(lambda ab: self._pass(*ab), blocks(self.rows1)))
            t1 = time.perf_counter()
            list(pool.map(lambda ab: self._z(*ab), blocks(self.rows2)))
            t2 = time.perf_counter()
        step_s = self._per_step(t1 - t0, self.rows1, t2 - t1, self.rows2)
        return {"value": 1.0 / step_s, "unit": "steps/s", "cores": threads, "kind": "oracle",
                "cpu_seconds": t2 - t0,
                "sample": f"{self._what()}: logits pass on {self.rows1} rows + z on {self.rows2} rows over "
                          f"1/{self.vfrac} of V, split into row blocks over {threads} threads, scaled to "
                          f"{self.cfg.R} rows x full V per step"}

    def parity(self, near_tie_rel: float = 1e-5) -> dict:
        """The single-thread run's results against the GPU's outputs of the same step (the probe):
        integer outputs compared exactly, sampled tokens exactly except at near-ties (top-two
        Gumbel-perturbed scores within near_tie_rel relative), statistics by their largest absolute
        difference, z by its relative Frobenius error per row."""
        import numpy as np
        ref, zr = self.results
        g = self.probe["out"]
        n = self.rows1
        near = (ref["gap1"] < near_tie_rel) | (ref["gap2"] < near_tie_rel)
        bad = g["x0_hat"][:n] != ref["x0_hat"]
        same = ~bad
        zg = self.probe["z"][: zr.shape[0]].astype(np.float64)
        zrow = np.linalg.norm(zg - zr, axis=1) / np.maximum(np.linalg.norm(zr, axis=1), 1e-300)
        return {"rows": int(n), "argmax_mismatches": int((g["argmax"][:n] != ref["argmax"]).sum()),
                "near_ties": int(near.sum()), "x0_hat_mismatches": int(bad.sum()),
                "x0_hat_mismatches_off_near_ties": int((bad & ~near).sum()),
                "x_next_mismatches_where_x0_hat_agrees": int((g["x_next"][:n][same] != ref["x_next"][same]).sum()),
                "max_stat_abs_err": float(max(np.abs(g[k][:n].astype(np.float64) - ref[k]).max()
                                              for k in ("lse", "max_prob", "entropy"))),
                "z_rows": int(zr.shape[0]), "z_rel_fro_max_row": float(zrow.max()),
                "z_rel_fro": float(np.linalg.norm(zg - zr) / np.linalg.norm(zr)),
                "source": f"CPU-baseline leg: the oracle on the bench's own logits buffer and canvas, step "
                          f"{self.probe['step']}, against one fused GPU step on the same inputs"}


def host_cores(cpu_max_path: str = "/sys/fs/cgroup/cpu.max") -> int:
    """Cores this process may run on: its affinity mask, capped by a cgroup CPU quota if any."""
    try:
        n = len(os.sched_getaffinity(0))
    except AttributeError:
        n = os.cpu_count() or 1
    try:
        quota, period = open(cpu_max_path).read().split()[:2]
        if quota != "max":
            n = min(n, max(1, math.ceil(int(quota) / int(period))))
    except (OSError, ValueError):
        pass
    return n


def oracle_baseline(probe=None) -> tuple:
    """About 10-20 s of single-threaded oracle work on rank 0, then the same routines on every
    host core (z on up to three rows per thread, at most all 256).  With the GPU's probe step, the
    single-thread run is also compared with the GPU's outputs (the `parity` object)."""
    cores = host_cores()
    single_rows2 = 24
    samp = OracleSample(rows1=256, rows2=min(256, max(single_rows2, 3 * cores)), vfrac=1, probe=probe)
    one = samp.run(rows2=single_rows2)
    par = samp.parity() if probe is not None else None
    many = samp.run_threads(cores)
    for r in (one, many):
        r["value"] = round(r["value"], 6)
        r["cpu_seconds"] = round(r["cpu_seconds"], 1)
    return one, many, par


def run_reference(args, rank, world):
    """The reference arm: the CPU oracle as it stands, one bounded sample per step, its rows split
    over every host core (a few tenths of a second per step)."""
    if rank != 0:
        return None
    cores = host_cores()
    samp = OracleSample(rows1=min(1024, 4 * cores), rows2=min(256, cores), vfrac=8)
    for _ in range(args.warmup):
        samp.run_threads(cores)
    res = [samp.run_threads(cores) for _ in range(args.steps)]
    secs = sum(1.0 / r["value"] for r in res)  # extrapolated seconds for K full steps
    v = args.steps / secs
    cfg = samp.cfg
    nbuf, lbytes = rotation(cfg)
    return {"impl": "reference", "metric": METRIC, "value": round(v, 6), "unit": "steps/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 / v, 1), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded)",
            "config": workload_config(world, nbuf, lbytes, cfg),
            "cpu_baseline": {"value": round(v, 6), "unit": "steps/s", "cores": cores, "kind": "oracle",
                             "sample": res[0]["sample"]},
            "e2e": {"value": round(v, 6), "unit": "steps/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)
    rank, world, local = dist_env()

    if args.impl == "reference":
        line = run_reference(args, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        return

    import torch
    if world > 1:
        torch.distributed.init_process_group("nccl", device_id=torch.device("cuda", local),
                                             timeout=__import__("datetime").timedelta(seconds=120))
    line, probe = run_ours(args, rank, world, local)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"], line["cpu_baseline_all_cores"], line["parity"] = oracle_baseline(probe)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
