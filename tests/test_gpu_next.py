"""GPU-vs-oracle parity of the sampler extensions and the training-side backward pieces,
through the C ABI.

  * entropy-bounded acceptance with uniform re-noising (dg_entropy_accept): bit-exact accepted
    set, count and x_next on seeded entropy vectors -- continuous, heavily tied, zero, negative
    and NaN entropies, C = 1, ragged C, C = DG_MAX_CANVAS_ROWS, several tolerances;
  * adaptive stopping (dg_adaptive_stop): bit-exact flags and mean entropies;
  * the fused entropy-bounded step (dg_sampler_step_eb): equal to the logits pass followed by
    the two decisions on its own outputs, and against the oracle's chain on the mid workload
    with a tolerance placed in a clear gap of the oracle's entropy order (bit-exact sets);
  * canvas CE backward (dg_canvas_ce_backward) against the oracle's float64 gradient within bf16
    rounding, on a small case in full and on sampled rows of the training workload;
  * self-conditioning drop (dg_selfcond_drop): bit-exact coins and zeroed rows.
"""
import zlib

import numpy as np
import pytest
import torch

import discrete_diffusion_lm_b200 as dg
from discrete_diffusion_lm_b200 import workloads as W
from oracle import oracle as O
from tests.parity import NEAR_TIE_REL, host_f32

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _entropies(kind, n, rng):
    if kind == "uniform":
        return rng.uniform(0.0, 5.0, n).astype(np.float32)
    if kind == "tied":  # few distinct values: ties everywhere, order by position decides
        return rng.choice(np.float32([0.0, 0.125, 0.5, 1.0, 3.0]), n).astype(np.float32)
    if kind == "tiny":  # below the fixed-point resolution and around it
        return (rng.uniform(0, 4, n) * 2.0 ** -33).astype(np.float32)
    if kind == "special":
        h = rng.uniform(0.0, 2.0, n).astype(np.float32)
        h[rng.integers(0, n, max(1, n // 10))] = np.nan
        h[rng.integers(0, n, max(1, n // 10))] = -1e-6
        h[rng.integers(0, n, max(1, n // 10))] = 80.0
        return h
    raise ValueError(kind)


@pytest.mark.parametrize("kind", ["uniform", "tied", "tiny", "special"])
@pytest.mark.parametrize("B,C", [(4, 256), (1, 1), (3, 100), (2, 1024), (1, 993)])
@pytest.mark.parametrize("eps", [0.0, 0.3, 7.5, 1e9])
def test_entropy_accept_matches_oracle(kind, B, C, eps):
    rng = np.random.default_rng(zlib.crc32(f"{kind}-{B}-{C}".encode()))
    V = 262144
    H = _entropies(kind, B * C, rng)
    x0 = rng.integers(0, V, B * C).astype(np.int32)
    out = dg.dg_entropy_accept(torch.from_numpy(H).to(DEV), torch.from_numpy(x0).to(DEV), C, V, eps, seed=5, step=9)
    torch.cuda.synchronize()
    x_ref, acc_ref, n_ref = O.entropy_accept(H, x0, B, C, V, eps, 5, 9)
    np.testing.assert_array_equal(out["accepted"].cpu().numpy(), acc_ref)
    np.testing.assert_array_equal(out["n_accepted"].cpu().numpy(), n_ref)
    np.testing.assert_array_equal(out["x_next"].cpu().numpy(), x_ref)


@pytest.mark.parametrize("B,C", [(8, 256), (1, 1), (3, 77), (2, 1024), (5, 33)])
def test_adaptive_stop_matches_oracle(B, C):
    rng = np.random.default_rng(C)
    H = rng.uniform(0.0, 1.0, B * C).astype(np.float32)
    H[:C] *= 0.1  # canvas 0 well below any threshold used
    am = rng.integers(0, 1000, B * C).astype(np.int32)
    prev = am.copy()
    if B > 2:
        prev[2 * C] += 1  # canvas 2 changed its prediction
    for theta in [0.0, 0.05, 0.5, 0.55, 2.0]:
        for p in (prev, None):
            stop, mean = dg.dg_adaptive_stop(torch.from_numpy(H).to(DEV), torch.from_numpy(am).to(DEV),
                                             None if p is None else torch.from_numpy(p).to(DEV), C, theta)
            torch.cuda.synchronize()
            s_ref, m_ref = O.adaptive_stop(H, am, p, B, C, theta)
            np.testing.assert_array_equal(stop.cpu().numpy(), s_ref)
            np.testing.assert_array_equal(mean.cpu().numpy(), m_ref.astype(np.float32))


def test_sampler_step_eb_equals_its_parts():
    cfg = W.MID
    logits = W.make_logits(cfg, DEV)
    inv_tau = dg.dg_tau_linear([0.7])
    prev = torch.from_numpy(np.random.default_rng(0).integers(0, cfg.V, cfg.R).astype(np.int32)).to(DEV)
    fused = dg.dg_sampler_step_eb(logits, cfg.C, eps=20.0, theta=0.5, argmax_prev=prev, inv_tau=inv_tau, seed=3,
                                  step=2)
    torch.cuda.synchronize()
    acc = dg.dg_entropy_accept(fused["entropy"], fused["x0_hat"], cfg.C, cfg.V, 20.0, seed=3, step=2)
    stop, mean = dg.dg_adaptive_stop(fused["entropy"], fused["argmax"], prev, cfg.C, 0.5)
    torch.cuda.synchronize()
    assert torch.equal(fused["x_next"], acc["x_next"]) and torch.equal(fused["accepted"], acc["accepted"])
    assert torch.equal(fused["stop"], stop) and torch.equal(fused["mean_entropy"], mean)
    # the statistics and the draw are those of the plain sampler step
    x_t = W.make_canvas(cfg, DEV)
    plain = dg.dg_sampler_step(logits, x_t, cfg.C, 0.5, 0.1, inv_tau=inv_tau, seed=3, step=2)
    torch.cuda.synchronize()
    for k in ("x0_hat", "argmax", "lse", "entropy", "max_prob"):
        assert torch.equal(fused[k], plain[k]), k


def test_sampler_step_eb_batched_equals_its_parts():
    # 16 canvases with per-canvas temperatures: the step's decisions (its decision kernel after the
    # pass) must equal the standalone decisions on the same outputs
    cfg = W.BATCHED
    rows = 16 * 256
    logits = W.make_logits(cfg, DEV, rows=rows)
    ts = [1.0 - b / 16 for b in range(16)]
    inv_tau = dg.dg_tau_linear(ts)
    prev = torch.from_numpy(np.random.default_rng(1).integers(0, cfg.V, rows).astype(np.int32)).to(DEV)
    for rep in range(2):  # a second call on the cached workspace, the previous argmax as argmax_prev
        fused = dg.dg_sampler_step_eb(logits, cfg.C, eps=40.0, theta=6.0, argmax_prev=prev, inv_tau=inv_tau, seed=7,
                                      step=5 + rep)
        torch.cuda.synchronize()
        acc = dg.dg_entropy_accept(fused["entropy"], fused["x0_hat"], cfg.C, cfg.V, 40.0, seed=7, step=5 + rep)
        stop, mean = dg.dg_adaptive_stop(fused["entropy"], fused["argmax"], prev, cfg.C, 6.0)
        torch.cuda.synchronize()
        assert torch.equal(fused["x_next"], acc["x_next"]) and torch.equal(fused["accepted"], acc["accepted"])
        assert torch.equal(fused["stop"], stop) and torch.equal(fused["mean_entropy"], mean)
        prev = fused["argmax"].clone()
    assert dg.dg_device_error() == 0


@pytest.mark.parametrize("mode", ["sample", "greedy"])
def test_sampler_step_eb_vs_oracle_mid(mode):
    cfg = W.MID
    logits = W.make_logits(cfg, DEV)
    t = 0.6
    it = dg.dg_tau_linear([t])[0]
    L = host_f32(logits)
    ref = O.sampler_step(L, np.zeros(cfg.R, np.int32), 1, cfg.C, cfg.V, cfg.schedule, [t], [0.0], [it], 1, 4, mode)
    H = np.asarray(ref["entropy"], dtype=np.float64)
    srt = np.sort(H)
    csum = np.cumsum(srt)
    k = cfg.C // 2
    eps = float((csum[k - 1] + csum[k]) / 2)  # the oracle accepts the k lowest entropies
    out = dg.dg_sampler_step_eb(logits, cfg.C, eps=eps, theta=10.0, argmax_prev=None, inv_tau=[it], seed=1, step=4,
                                mode=mode)
    torch.cuda.synchronize()
    acc = out["accepted"].cpu().numpy().astype(bool)
    # The GPU decides on its own float entropies (within DELTA of the oracle's), so the accepted set
    # must be a valid acceptance for entropies perturbed by at most DELTA: a prefix of the oracle's
    # entropy order up to 2 DELTA, summing below eps, and maximal.
    DELTA = 1e-4
    n = int(acc.sum())
    assert abs(n - k) <= 2, (n, k)
    if 0 < n < cfg.C:
        assert H[acc].max() <= H[~acc].min() + 2 * DELTA
    assert H[acc].sum() < eps + n * DELTA
    if n < cfg.C:
        assert H[acc].sum() + H[~acc].min() >= eps - (n + 1) * DELTA
    x_next = out["x_next"].cpu().numpy()
    x0 = out["x0_hat"].cpu().numpy()
    near = (ref["gap1"] < NEAR_TIE_REL) | (ref["gap2"] < NEAR_TIE_REL)
    assert np.all((x0 == ref["x0_hat"]) | near)
    np.testing.assert_array_equal(x_next[acc], x0[acc])
    # rejected positions: the oracle's uniform re-noise draw for the same (seed, step, row)
    x_ref, _, _ = O.entropy_accept(np.full(cfg.R, 1.0, np.float32), np.zeros(cfg.R, np.int32), 1, cfg.C, cfg.V, 0.0,
                                   1, 4)
    np.testing.assert_array_equal(x_next[~acc], x_ref[~acc])


def _ce_case(n_seq, P, K, C, V, seed):
    g = torch.Generator().manual_seed(seed)
    x0 = torch.randint(0, V, (n_seq, P + K * C), generator=g, dtype=torch.int32)
    k = torch.randint(0, K, (n_seq,), generator=g, dtype=torch.int32)
    logits = (torch.randn(n_seq * C, V, generator=g) * 2).to(torch.bfloat16)
    gs = torch.rand(n_seq, generator=g) + 0.5
    return x0, k, logits, gs


def _ce_tolerance_check(g_gpu, g_ref, gscale_rows):
    err = np.abs(g_gpu - g_ref)
    # bf16 rounding of the result (half an ulp, 2^-9 relative) plus fp32 exp / lse error
    bound = 2.0 ** -8 * np.abs(g_ref) + 1e-6 * gscale_rows[:, None]
    assert np.all(err <= bound), f"max excess {float((err - bound).max()):.3g}"


def test_canvas_ce_backward_small_in_full():
    n_seq, P, K, C, V = 3, 16, 2, 64, 4096
    x0, k, logits, gs = _ce_case(n_seq, P, K, C, V, 0)
    x0[1, P + int(k[1]) * C + 3] = V + 9  # one out-of-range target -> zero row
    xd, kd, ld, gd = x0.to(DEV), k.to(DEV), logits.to(DEV), gs.to(DEV)
    _, _, lse = dg.dg_canvas_ce(ld, xd, kd, P, K, C)
    torch.cuda.synchronize()
    ref = O.canvas_ce_backward(logits.float().numpy(), x0.numpy(), k.numpy(), n_seq, P, K, C, V, gs.double().numpy())
    dg.dg_canvas_ce_backward(ld, lse, xd, kd, P, K, C, g_seq=gd)
    torch.cuda.synchronize()
    got = ld.float().cpu().numpy()
    assert (got[C + 3] == 0).all()
    _ce_tolerance_check(got, ref, np.repeat(gs.double().numpy(), C))


def test_canvas_ce_backward_train_sampled_rows():
    cfg = W.TRAIN
    x0 = W.make_train_tokens(cfg, DEV)
    _, kidx = dg.dg_forward_noise(x0, cfg.P, cfg.K, cfg.C, cfg.V, W.make_train_times(cfg))
    logits = W.make_train_logits(cfg, DEV)
    rows = np.random.default_rng(3).choice(cfg.n_seq * cfg.C, 8, replace=False)
    host_rows = logits[torch.from_numpy(rows).to(DEV)].float().cpu().numpy()
    _, _, lse = dg.dg_canvas_ce(logits, x0, kidx, cfg.P, cfg.K, cfg.C)
    dg.dg_canvas_ce_backward(logits, lse, x0, kidx, cfg.P, cfg.K, cfg.C)
    torch.cuda.synchronize()
    got = logits[torch.from_numpy(rows).to(DEV)].float().cpu().numpy()
    x0h, kh = x0.cpu().numpy(), kidx.cpu().numpy()
    for j, r in enumerate(rows):
        b, i = divmod(int(r), cfg.C)
        # the row as a one-row, one-canvas sequence with the same target
        tgt = np.array([[x0h[b, cfg.P + kh[b] * cfg.C + i]]], np.int32)
        ref = O.canvas_ce_backward(host_rows[j][None], tgt, np.zeros(1, np.int32), 1, 0, 1, 1, cfg.V)
        _ce_tolerance_check(got[j][None], ref, np.ones(1))
        assert abs(float(got[j].astype(np.float64).sum())) < 2e-2  # softmax minus one-hot sums to ~0


def test_selfcond_drop_matches_oracle():
    n_seq, C, d = 64, 16, 128
    z = torch.randn(n_seq * C, d, generator=torch.Generator().manual_seed(1)).to(torch.bfloat16)
    zd = z.to(DEV)
    keep = dg.dg_selfcond_drop(zd, C, seed=7, step=3)
    torch.cuda.synchronize()
    ref, keep_ref = O.selfcond_drop(z.float().numpy(), n_seq, C, d, 7, 3)
    np.testing.assert_array_equal(keep.cpu().numpy(), keep_ref)
    np.testing.assert_array_equal(zd.float().cpu().numpy(), ref.astype(np.float32))
    assert 0 < keep_ref.sum() < n_seq
