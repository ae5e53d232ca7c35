"""Pins of the CPU oracle against what the pages and the mathematics fix.

Each test checks an oracle function against something other than itself:
published known-answer vectors, closed forms, brute-force Bayes over all
(x_s, x_0) pairs, matrix exponentials of the CTMC generator, chi-square tests
against the defining distribution, and library routines (numpy, scipy, torch).
Pages: DiffusionGemma Technical Report (hyper.ai summary), sections "Method"
(forward path, kappa schedule, Step, softmax / p0 E / Step update, loss) and
"Dataset" (P + K*C layout, one uniformly chosen canvas).
"""
import math
import os

import numpy as np
import pytest
import scipy.linalg
import scipy.special
import scipy.stats
import torch

from oracle import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
P_MIN = 1e-4  # chi-square acceptance (inputs are seeded, so results are fixed)


def chisq_p(observed, expected_probs):
    observed = np.asarray(observed, dtype=np.float64)
    exp = np.asarray(expected_probs, dtype=np.float64) * observed.sum()
    keep = exp > 0
    assert observed[~keep].sum() == 0, "draws landed on a zero-probability outcome"
    return scipy.stats.chisquare(observed[keep], exp[keep]).pvalue


# ----------------------------------------------------------------------------- Philox
def test_philox_known_answers():
    rows = [l.split() for l in open(os.path.join(GOLDEN, "philox4x32_10_kat.txt")) if l.strip()
            and not l.startswith("#")]
    assert len(rows) == 3
    for r in rows:
        v = [int(x, 16) for x in r]
        out = O.philox4x32_10(v[0:4], v[4:6])
        assert [int(x) for x in out] == v[6:10]


def test_philox_words_uniform():
    # 2^18 calls over consecutive counters -> 2^20 words; top byte in 256 bins
    lib = O.lib()
    words = []
    for i in range(1 << 12):
        for j in range(64):
            words.extend(O.philox4x32_10([i, j, 7, 0], [0x1234, 0x5678]))
    w = np.asarray(words, dtype=np.uint64)
    assert chisq_p(np.bincount((w >> 24).astype(np.int64), minlength=256), np.full(256, 1 / 256)) > P_MIN
    assert chisq_p(np.bincount((w & 255).astype(np.int64), minlength=256), np.full(256, 1 / 256)) > P_MIN
    del lib


def test_open_uniform_and_gumbel():
    # u = (2k+1) 2^-24 exactly, strictly inside (0,1); extremes included
    assert O.open_uniform(0) == 2.0 ** -24
    assert O.open_uniform(0xFFFFFFFF) == 1.0 - 2.0 ** -24
    assert O.open_uniform(0x1FF) == 2.0 ** -24  # low 9 bits ignored
    rng = np.random.default_rng(0)
    ws = rng.integers(0, 2 ** 32, size=200000, dtype=np.uint64)
    g = np.array([O.gumbel(int(w)) for w in ws])
    # standard Gumbel: mean = Euler-Mascheroni gamma, variance = pi^2/6
    assert abs(g.mean() - np.euler_gamma) < 0.01
    assert abs(g.var() - math.pi ** 2 / 6) < 0.03
    # Kolmogorov-Smirnov against scipy's Gumbel CDF
    assert scipy.stats.kstest(g, "gumbel_r").pvalue > P_MIN


# ----------------------------------------------------------------------------- schedule
@pytest.mark.parametrize("sched", ["linear", "cosine"])
def test_kappa_boundaries_and_monotone(sched):
    assert O.kappa(sched, 0.0) == 1.0
    assert abs(O.kappa(sched, 1.0)) < 1e-30
    ts = np.linspace(0, 1, 1001)
    ks = np.array([O.kappa(sched, t) for t in ts])
    assert np.all(np.diff(ks) <= 0)
    assert abs(O.kappa(sched, 0.5) - (0.5 if sched == "linear" else 0.5)) < 1e-15


# ----------------------------------------------------------------------------- softmax statistics
def test_row_stats_constant_row():
    for V in (1, 7, 1024, 32768):
        lse, pm, H = O.row_stats(np.full(V, 3.25, dtype=np.float32))
        assert abs(lse - (3.25 + math.log(V))) < 1e-12
        assert abs(pm - 1.0 / V) < 1e-15
        assert abs(H - math.log(V)) < 1e-10


def test_row_stats_one_hot():
    row = np.zeros(4096, dtype=np.float32)
    row[1234] = 100.0
    lse, pm, H = O.row_stats(row)
    assert abs(pm - 1.0) < 1e-38 + 4095 * math.exp(-100) * 1.01
    assert H < 1e-38 + 4095 * 101 * math.exp(-100)
    assert abs(lse - 100.0) < 1e-40 + 4096 * math.exp(-100)


@pytest.mark.parametrize("inv_tau", [1.0, 1.25, 2.5])
def test_row_stats_vs_scipy(inv_tau):
    rng = np.random.default_rng(3)
    row = (rng.standard_normal(5000) * 2).astype(np.float32)
    row[rng.choice(5000, 4, replace=False)] = rng.uniform(8, 12, 4)
    x = row.astype(np.float64) * inv_tau
    lse, pm, H = O.row_stats(row, inv_tau)
    p = scipy.special.softmax(x)
    assert abs(lse - scipy.special.logsumexp(x)) < 1e-12
    assert abs(pm - p.max()) < 1e-14
    assert abs(H - scipy.stats.entropy(p)) < 1e-11
    pr = O.row_probs(row, inv_tau)
    assert abs(pr.sum() - 1.0) < 1e-13
    np.testing.assert_allclose(pr, p, rtol=1e-12, atol=1e-300)


def test_argmax_lowest_index_on_ties():
    rng = np.random.default_rng(4)
    for _ in range(200):
        V = int(rng.integers(1, 300))
        row = rng.integers(-3, 4, size=V).astype(np.float32)  # many ties
        # numpy documents that argmax returns the first occurrence of the maximum
        assert O.argmax(row) == int(np.argmax(row))
    bf = torch.randn(10000, generator=torch.Generator().manual_seed(1)).to(torch.bfloat16).float().numpy()
    assert O.argmax(bf) == int(np.argmax(bf))


# ----------------------------------------------------------------------------- x0 draw
def _draw_freq(row, n, Q, inv_tau=1.0, seed=0, step=0):
    V = len(row)
    L = np.tile(np.asarray(row, dtype=np.float32), (n, 1))
    out = O.sampler_step(L, np.zeros(n, np.int32), 1, n, V, "linear", [0.0], [0.0],
                         None if inv_tau == 1.0 else [inv_tau], seed, step, "sample", Q)
    return np.bincount(out["x0_hat"], minlength=V), out


@pytest.mark.parametrize("Q", [2048, 4, 5, 1])
def test_draw_frequencies_match_softmax(Q):
    # Q = 2048: plain one-level Gumbel-max (V < Q); Q = 4: three full chunks;
    # Q = 5: a ragged last chunk; Q = 1: level 1 alone decides
    row = np.array([0.0, 1.0, -1.0, 2.0, 0.5, 0.5, -2.0, 1.5, 3.0, -0.5, 0.0, 1.0], dtype=np.float32)
    counts, _ = _draw_freq(row, 200000, Q)
    assert chisq_p(counts, scipy.special.softmax(row.astype(np.float64))) > P_MIN


def test_draw_frequencies_with_temperature():
    row = np.array([0.0, 1.0, 2.0, -1.0, 0.3, 0.7, 1.9], dtype=np.float32)
    counts, _ = _draw_freq(row, 200000, 3, inv_tau=1.6, seed=5, step=3)
    assert chisq_p(counts, scipy.special.softmax(row.astype(np.float64) * 1.6)) > P_MIN


def test_draw_depends_on_seed_step_row():
    row = np.zeros(64, dtype=np.float32)
    a = O.draw_x0(row, 1.0, 0, 0, 5, 16)[0]
    draws = {O.draw_x0(row, 1.0, s, st, r, 16)[0] for s in range(3) for st in range(3) for r in range(3)}
    assert len(draws) > 10
    assert O.draw_x0(row, 1.0, 0, 0, 5, 16)[0] == a  # deterministic


def test_draw_gumbel_max_identity_single_level():
    # with V <= Q the draw is literally argmax_v l_v + G_v with G_v from the token domain
    rng = np.random.default_rng(6)
    row = rng.standard_normal(40).astype(np.float32)
    x, g1, g2 = O.draw_x0(row, 1.0, 11, 2, 9, 2048)
    scores = []
    for v in range(40):
        w = O.philox4x32_10([v >> 2, 9, 2, 0], [11, 0])[v & 3]
        u = (2 * (int(w) >> 9) + 1) * 2.0 ** -24
        scores.append(float(row[v]) - math.log(-math.log(u)))
    assert x == int(np.argmax(scores))
    assert math.isinf(g1)
    s = sorted(scores)
    assert abs(g2 - (s[-1] - s[-2]) / max(abs(s[-1]), 1.0)) < 1e-12


# ----------------------------------------------------------------------------- Step posterior
def _forward_marginal(kappa, x0, V):
    m = np.full(V, (1 - kappa) / V)
    m[x0] += kappa
    return m


def _bayes_brute_force(x_t, x0, kt, ks, V):
    """P(x_s | x_t, x0) by enumerating x_s, with the s->t kernel obtained from the
    CTMC generator by a matrix exponential (scipy), not from the closed form."""
    # generator of the uniform-noise CTMC: rate beta(u) (1/V 11^T - I); integrating
    # beta from s to t gives log(kappa_s / kappa_t) because kappa' = -beta kappa
    Q = np.full((V, V), 1.0 / V) - np.eye(V)
    K = scipy.linalg.expm(math.log(ks / kt) * Q)  # K[x_s, x_t]
    joint = np.array([K[xs, x_t] * _forward_marginal(ks, x0, V)[xs] for xs in range(V)])
    return joint / joint.sum()


@pytest.mark.parametrize("V", [2, 3, 5, 7])
def test_step_posterior_matches_brute_force_bayes(V):
    for kt, ks in [(0.1, 0.6), (0.3, 0.31), (0.05, 0.99), (0.5, 0.9), (1e-6, 0.2)]:
        for x_t in range(V):
            for x0 in range(V):
                p = O.step_posterior(x_t, x0, kt, ks, V)
                np.testing.assert_allclose(p, _bayes_brute_force(x_t, x0, kt, ks, V), rtol=1e-10, atol=1e-13)
                assert abs(p.sum() - 1) < 1e-13


@pytest.mark.parametrize("V", [2, 3, 6])
def test_kernel_chapman_kolmogorov(V):
    # the s->t kernel carries the s-marginal into the t-marginal of the forward path
    Q = np.full((V, V), 1.0 / V) - np.eye(V)
    for kt, ks in [(0.2, 0.7), (0.6, 0.65)]:
        K = scipy.linalg.expm(math.log(ks / kt) * Q)
        alpha = kt / ks
        np.testing.assert_allclose(K, alpha * np.eye(V) + (1 - alpha) / V, atol=1e-13)
        for x0 in range(V):
            np.testing.assert_allclose(_forward_marginal(ks, x0, V) @ K, _forward_marginal(kt, x0, V), atol=1e-14)


def _step_batch(x_t, x0_hat, kt, ks, V, n, seed=0, step=0):
    """n independent Step draws for fixed (x_t, x0_hat): greedy mode with a one-hot
    row so x0_hat = argmax; rows differ, so the Philox draws are independent."""
    L = np.zeros((n, V), dtype=np.float32)
    L[:, x0_hat] = 1.0
    sched_t = (1 - kt)  # linear schedule: kappa = 1 - t
    t = [sched_t]
    dt = [sched_t - (1 - ks)]
    out = O.sampler_step(L, np.full(n, x_t, np.int32), 1, n, V, "linear", t, dt, None, seed, step, "greedy")
    return out


@pytest.mark.parametrize("case", [(0, 1, 0.3, 0.7, 3), (2, 2, 0.3, 0.7, 3), (1, 4, 0.05, 0.5, 5),
                                  (4, 4, 0.6, 0.95, 5), (0, 1, 0.0, 0.25, 2)])
def test_step_draws_match_posterior(case):
    x_t, x0, kt, ks, V = case
    out = _step_batch(x_t, x0, kt, ks, V, 300000, seed=3, step=1)
    assert np.all(out["x0_hat"] == x0)
    counts = np.bincount(out["x_next"], minlength=V)
    assert chisq_p(counts, O.step_posterior(x_t, x0, kt, ks, V)) > P_MIN
    br = out["branch"]
    # branch bookkeeping: stay keeps x_t, jump lands on x0_hat
    assert np.all(out["x_next"][br == 0] == x_t)
    assert np.all(out["x_next"][br == 1] == x0)


def test_step_kappa_s_one_returns_x0_exactly():
    for x_t, x0 in [(0, 3), (2, 2), (4, 1)]:
        out = _step_batch(x_t, x0, 0.37, 1.0, 5, 20000)
        assert np.all(out["x_next"] == x0)


def test_step_dt_zero_returns_x_t_exactly():
    V, n = 7, 20000
    L = np.random.default_rng(0).standard_normal((n, V)).astype(np.float32)
    xt = np.random.default_rng(1).integers(0, V, n).astype(np.int32)
    for t in (0.0, 0.4, 1.0):
        out = O.sampler_step(L, xt, 1, n, V, "cosine", [t], [0.0], None, 0, 0, "sample")
        assert np.array_equal(out["x_next"], xt)
        assert np.all(out["branch"] == 0)


def test_step_from_t1_linear():
    # t = 1, kappa_t = 0: x_t carries no information; x_s ~ kappa_s delta(x0) + uniform
    V, n = 4, 300000
    out = _step_batch(1, 3, 0.0, 0.25, V, n, seed=9)
    counts = np.bincount(out["x_next"], minlength=V)
    assert chisq_p(counts, _forward_marginal(0.25, 3, V)) > P_MIN


# ----------------------------------------------------------------------------- self-conditioning z
def test_selfcond_one_hot_and_constant():
    rng = np.random.default_rng(7)
    V, d = 300, 16
    E = (rng.standard_normal((V, d)) * 0.02).astype(np.float32)
    L = np.zeros((3, V), dtype=np.float32)
    L[0, 17] = 200.0           # one-hot: z = E[17]
    L[2] = 5.0                 # constant: z = column mean
    L[1] = rng.standard_normal(V)
    z = O.selfcond_rows(L, E, [0, 1, 2])
    np.testing.assert_allclose(z[0], E[17].astype(np.float64), atol=1e-12)
    np.testing.assert_allclose(z[2], E.astype(np.float64).mean(0), atol=1e-15)
    ref = scipy.special.softmax(L[1].astype(np.float64)) @ E.astype(np.float64)
    np.testing.assert_allclose(z[1], ref, rtol=1e-10, atol=1e-15)


def test_selfcond_temperature_rows():
    rng = np.random.default_rng(8)
    V, d = 100, 8
    E = rng.standard_normal((V, d)).astype(np.float32)
    L = rng.standard_normal((4, V)).astype(np.float32)
    it = np.array([1.0, 0.5, 2.0, 1.25], dtype=np.float32)
    z = O.selfcond_rows(L, E, [0, 1, 2, 3], it)
    for r in range(4):
        ref = scipy.special.softmax(L[r].astype(np.float64) * it[r]) @ E.astype(np.float64)
        np.testing.assert_allclose(z[r], ref, rtol=1e-10)


# ----------------------------------------------------------------------------- forward noise
def test_forward_noise_marginal_and_layout():
    n_seq, P, K, C, V = 3, 16, 2, 100000, 8
    rng = np.random.default_rng(10)
    x0 = rng.integers(0, V, (n_seq, P + K * C)).astype(np.int32)
    t = [0.3, 0.7, 0.95]
    xt, k = O.forward_noise(x0, n_seq, P, K, C, V, "cosine", t, 5)
    assert np.array_equal(xt[:, :P], x0[:, :P])  # prompt is copied
    for b in range(n_seq):
        kap = math.cos(math.pi * t[b] / 2) ** 2
        same = (xt[b, P:] == x0[b, P:])
        # P(x_t = x0) = kappa + (1 - kappa)/V (forward path marginal)
        n = same.size
        assert abs(same.mean() - (kap + (1 - kap) / V)) < 5 * math.sqrt(0.25 / n)
        # conditional on x0 = 0, the distribution of x_t is kappa delta + (1-kappa)/V
        sel = x0[b, P:] == 0
        counts = np.bincount(xt[b, P:][sel], minlength=V)
        assert chisq_p(counts, _forward_marginal(kap, 0, V)) > P_MIN
    assert np.all((k >= 0) & (k < K))


@pytest.mark.parametrize("V", [1024, 262144])
def test_forward_noise_marginal_million_draws(V):
    # The forward path marginal kappa delta(x_t, x0) + (1 - kappa)/V, tested per sequence on 10^6
    # canvas tokens each at four kappa.  Every token counts: its offset (x_t - x0) mod V is 0 with
    # probability kappa + (1 - kappa)/V and each other offset with (1 - kappa)/V.  V = 1024: all
    # V offsets are bins; V = 262144: the zero offset plus 256 equal buckets of the others.
    n_seq, P, K, C = 4, 8, 2, 500_000
    rng = np.random.default_rng(14 + V)
    x0 = rng.integers(0, V, (n_seq, P + K * C)).astype(np.int32)
    t = [0.2, 0.5, 0.8, 1.0]
    xt, _ = O.forward_noise(x0, n_seq, P, K, C, V, "cosine", t, 17)
    assert np.array_equal(xt[:, :P], x0[:, :P])
    for b in range(n_seq):
        kap = math.cos(math.pi * t[b] / 2) ** 2
        off = (xt[b, P:].astype(np.int64) - x0[b, P:]) % V
        assert off.size == 10 ** 6
        if V <= 4096:
            counts = np.bincount(off, minlength=V)
            probs = np.full(V, (1 - kap) / V)
            probs[0] += kap
        else:
            nb = 256
            other = off[off > 0]
            bucket = (other - 1) * nb // (V - 1)
            counts = np.append((off == 0).sum(), np.bincount(bucket, minlength=nb))
            sizes = np.bincount((np.arange(1, V) - 1) * nb // (V - 1), minlength=nb)
            probs = np.append(kap + (1 - kap) / V, sizes * (1 - kap) / V)
        assert chisq_p(counts, probs) > P_MIN


def test_forward_noise_kappa_extremes():
    n_seq, P, K, C, V = 2, 5, 3, 50, 1000
    x0 = np.random.default_rng(11).integers(0, V, (n_seq, P + K * C)).astype(np.int32)
    xt, _ = O.forward_noise(x0, n_seq, P, K, C, V, "linear", [0.0, 0.0], 1)
    assert np.array_equal(xt, x0)  # kappa = 1 keeps everything
    xt, _ = O.forward_noise(x0, n_seq, P, K, C, V, "linear", [1.0, 1.0], 1)
    assert np.array_equal(xt[:, :P], x0[:, :P])
    assert (xt[:, P:] == x0[:, P:]).mean() < 0.02  # kappa = 0: only chance agreement


def test_canvas_choice_uniform():
    n_seq, K = 40000, 4
    x0 = np.zeros((n_seq, 1 + K), dtype=np.int32)
    _, k = O.forward_noise(x0, n_seq, 1, K, 1, 10, "cosine", np.full(n_seq, 0.5), 3)
    assert chisq_p(np.bincount(k, minlength=K), np.full(K, 1 / K)) > P_MIN


# ----------------------------------------------------------------------------- canvas CE
def test_canvas_ce_constant_logits_is_log_v():
    n_seq, P, K, C, V = 2, 3, 2, 4, 50
    x0 = np.random.default_rng(12).integers(0, V, (n_seq, P + K * C)).astype(np.int32)
    loss, seq, lse = O.canvas_ce(np.full((n_seq * C, V), 1.5, np.float32), x0, [0, 1], n_seq, P, K, C, V)
    np.testing.assert_allclose(loss, math.log(V), atol=1e-12)
    np.testing.assert_allclose(seq, C * math.log(V), atol=1e-11)
    np.testing.assert_allclose(lse, 1.5 + math.log(V), atol=1e-12)


def test_canvas_ce_vs_torch():
    n_seq, P, K, C, V = 3, 7, 3, 5, 333
    rng = np.random.default_rng(13)
    x0 = rng.integers(0, V, (n_seq, P + K * C)).astype(np.int32)
    L = (rng.standard_normal((n_seq * C, V)) * 2).astype(np.float32)
    kidx = np.array([2, 0, 1], dtype=np.int32)
    loss, seq, lse = O.canvas_ce(L, x0, kidx, n_seq, P, K, C, V)
    tgt = np.concatenate([x0[b, P + kidx[b] * C: P + (kidx[b] + 1) * C] for b in range(n_seq)])
    ref = torch.nn.functional.cross_entropy(torch.from_numpy(L).double(), torch.from_numpy(tgt).long(),
                                            reduction="none").numpy()
    np.testing.assert_allclose(loss, ref, rtol=1e-12)
    np.testing.assert_allclose(seq, ref.reshape(n_seq, C).sum(1), rtol=1e-12)
    np.testing.assert_allclose(lse, torch.logsumexp(torch.from_numpy(L).double(), 1).numpy(), rtol=1e-13)
