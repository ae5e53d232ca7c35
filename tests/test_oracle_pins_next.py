"""Pins of the oracle's sampler extensions and training-side backward pieces.

Pages: DiffusionGemma Technical Report (hyper.ai summary), section "Method" (the sampler
paragraph: entropy-ordered acceptance under an error tolerance with uniform re-noising of the
rest, a temperature annealed linearly from 0.8 to 0.4, adaptive stopping on the canvas-mean
entropy and two identical consecutive deterministic predictions; the cross-entropy loss
equation) and section "Dataset" (self-conditioning state used for 50% of the batch, zero for the
other 50%).

Each oracle function is checked against something other than itself: exhaustive enumeration
over subsets in exact rational arithmetic, closed forms, chi-square and binomial tests against
the defining distribution, and torch autograd in float64 for the loss gradient.
"""
import itertools
from fractions import Fraction

import numpy as np
import pytest
import scipy.stats
import torch

from oracle import oracle as O

P_MIN = 1e-4


# ----------------------------------------------------------------------------- temperature
def test_tau_linear_endpoints_and_line():
    assert O.tau_linear(1.0) == pytest.approx(0.8, abs=1e-15)
    assert O.tau_linear(0.0) == pytest.approx(0.4, abs=1e-15)
    for t in np.linspace(0, 1, 11):
        assert O.tau_linear(t) == pytest.approx(0.4 + 0.4 * t, abs=1e-15)
    # outside the time range the schedule holds its end values
    assert O.tau_linear(1.5) == pytest.approx(0.8) and O.tau_linear(-0.2) == pytest.approx(0.4)
    assert O.tau_linear(0.5, 1.0, 0.5) == pytest.approx(0.75)


# ----------------------------------------------------------------------------- acceptance
def _exact(h):
    return Fraction(float(np.float32(h)))


def brute_force_accept(H, eps):
    """Largest set that is a prefix of the ascending (entropy, position) order and whose
    entropies sum (exactly) to less than eps, found by enumerating every subset."""
    C = len(H)
    order = sorted(range(C), key=lambda i: (_exact(H[i]), i))
    rank = {i: k for k, i in enumerate(order)}
    best = set()
    for n in range(C + 1):
        for S in itertools.combinations(range(C), n):
            if sorted(rank[i] for i in S) != list(range(n)):
                continue  # not a prefix of the entropy order
            if sum((_exact(H[i]) for i in S), Fraction(0)) < Fraction(eps) and n > len(best):
                best = set(S)
    return best


@pytest.mark.parametrize("seed", range(6))
def test_accept_matches_exhaustive_enumeration(seed):
    rng = np.random.default_rng(seed)
    C = 7
    # entropies >= 2^-9 are whole multiples of 2^-32 in float32, so the oracle's fixed point is
    # exact and the rational sum is the reference; ties and zeros included
    H = rng.uniform(0.01, 3.0, C).astype(np.float32)
    H[rng.integers(0, C)] = H[rng.integers(0, C)]
    H[rng.integers(0, C)] = 0.0
    eps = float(np.float32(rng.uniform(0.5, 6.0)))
    x0 = rng.integers(0, 50, C).astype(np.int32)
    x_next, acc, n = O.entropy_accept(H, x0, 1, C, 50, eps, seed, 3)
    want = brute_force_accept(H, eps)
    assert set(np.nonzero(acc)[0].tolist()) == want
    assert n[0] == len(want)
    for i in range(C):
        if acc[i]:
            assert x_next[i] == x0[i]


def test_accept_closed_forms():
    C, V = 16, 1000
    x0 = np.arange(C, dtype=np.int32)
    h = 0.25
    H = np.full(C, h, np.float32)
    for eps in [0.1, 0.25, 0.3, 1.0, 1.01, 3.9, 4.0, 100.0]:
        _, acc, n = O.entropy_accept(H, x0, 1, C, V, eps, 0, 0)
        k = sum(1 for j in range(1, C + 1) if j * h < eps)  # strictly below the tolerance
        assert n[0] == k
        assert acc[:k].all() and not acc[k:].any()  # equal entropies: lower positions first
    _, acc, _ = O.entropy_accept(np.zeros(C, np.float32), x0, 1, C, V, 1e-9, 0, 0)
    assert acc.all()  # zero entropies always fit a positive tolerance
    _, acc, _ = O.entropy_accept(np.zeros(C, np.float32), x0, 1, C, V, 0.0, 0, 0)
    assert not acc.any()  # a tolerance of zero admits nothing


def test_accept_nan_and_negative_entropies():
    H = np.array([np.nan, -1e-7, 0.5, 0.2], np.float32)
    x0 = np.array([10, 11, 12, 13], np.int32)
    _, acc, n = O.entropy_accept(H, x0, 1, 4, 100, 1.0, 0, 0)
    # a rounding-negative entropy counts as zero, NaN as the largest entropy
    assert acc.tolist() == [0, 1, 1, 1] and n[0] == 3
    _, acc, _ = O.entropy_accept(H, x0, 1, 4, 100, 1e6, 0, 0)
    assert acc.tolist() == [1, 1, 1, 1]


def test_accept_canvases_independent():
    rng = np.random.default_rng(5)
    B, C = 3, 32
    H = rng.uniform(0, 2, B * C).astype(np.float32)
    x0 = rng.integers(0, 99, B * C).astype(np.int32)
    xa, acca, na = O.entropy_accept(H, x0, B, C, 99, 4.0, 7, 2)
    for b in range(B):
        sl = slice(b * C, (b + 1) * C)
        _, accb, nb = O.entropy_accept(H[sl], x0[sl], 1, C, 99, 4.0, 7, 2)
        assert (accb == acca[sl]).all() and nb[0] == na[b]


def test_renoise_uniform_and_keyed():
    V, B, C = 7, 50, 400
    H = np.full(B * C, 1.0, np.float32)
    x0 = np.zeros(B * C, np.int32)
    x_next, acc, _ = O.entropy_accept(H, x0, B, C, V, 0.5, 11, 4)  # nothing accepted
    assert not acc.any()
    assert scipy.stats.chisquare(np.bincount(x_next, minlength=V)).pvalue > P_MIN
    other, _, _ = O.entropy_accept(H, x0, B, C, V, 0.5, 11, 5)
    assert (other != x_next).mean() > 0.8  # a different step draws different noise
    again, _, _ = O.entropy_accept(H, x0, B, C, V, 0.5, 11, 4)
    assert (again == x_next).all()


# ----------------------------------------------------------------------------- stopping
def test_adaptive_stop_definition():
    rng = np.random.default_rng(1)
    B, C = 4, 64
    H = rng.uniform(0.01, 1.0, B * C).astype(np.float32)
    am = rng.integers(0, 1000, B * C).astype(np.int32)
    prev = am.copy()
    prev[C + 5] += 1  # canvas 1 changed its prediction
    means = H.reshape(B, C).astype(np.float64).mean(1)
    theta = float(np.median(means))
    stop, mean = O.adaptive_stop(H, am, prev, B, C, theta)
    assert np.allclose(mean, means, atol=1e-9)
    for b in range(B):
        assert stop[b] == (means[b] < theta and b != 1)
    stop0, _ = O.adaptive_stop(H, am, None, B, C, 10.0)
    assert not stop0.any()  # no previous step: predictions cannot agree yet
    # strict: a mean exactly at the threshold does not stop (0.5 is exact in fixed point)
    stop1, _ = O.adaptive_stop(np.full(C, 0.5, np.float32), am[:C], am[:C], 1, C, 0.5)
    assert stop1[0] == 0
    stop2, _ = O.adaptive_stop(np.full(C, 0.5, np.float32), am[:C], am[:C], 1, C, 0.5 + 1e-6)
    assert stop2[0] == 1


# ----------------------------------------------------------------------------- CE backward
@pytest.mark.parametrize("seed", [0, 1])
def test_canvas_ce_backward_vs_autograd(seed):
    rng = np.random.default_rng(seed)
    n_seq, P, K, C, V = 3, 5, 2, 4, 37
    L = P + K * C
    x0 = rng.integers(0, V, (n_seq, L)).astype(np.int32)
    k = rng.integers(0, K, n_seq).astype(np.int32)
    logits = (rng.standard_normal((n_seq * C, V)) * 3).astype(np.float32)
    g_seq = rng.uniform(0.5, 2.0, n_seq)
    grad = O.canvas_ce_backward(logits, x0, k, n_seq, P, K, C, V, g_seq)
    lt = torch.tensor(logits, dtype=torch.float64, requires_grad=True)
    tgt = torch.tensor([int(x0[b, P + k[b] * C + i]) for b in range(n_seq) for i in range(C)], dtype=torch.long)
    per_row = torch.nn.functional.cross_entropy(lt, tgt, reduction="none")
    w = torch.tensor(np.repeat(g_seq, C))
    (per_row * w).sum().backward()
    assert np.allclose(grad, lt.grad.numpy(), rtol=1e-12, atol=1e-15)
    assert np.allclose(grad.sum(1), 0.0, atol=1e-12)  # softmax minus one-hot sums to zero


def test_canvas_ce_backward_invalid_target_is_zero():
    n_seq, P, K, C, V = 2, 1, 1, 3, 9
    x0 = np.zeros((n_seq, P + K * C), np.int32)
    x0[1, P + 1] = V + 4  # out of range
    logits = np.random.default_rng(0).standard_normal((n_seq * C, V)).astype(np.float32)
    grad = O.canvas_ce_backward(logits, x0, np.zeros(n_seq, np.int32), n_seq, P, K, C, V)
    assert (grad[C + 1] == 0).all() and (grad[C] != 0).any()
    grad_bad_k = O.canvas_ce_backward(logits, x0, np.array([0, 5], np.int32), n_seq, P, K, C, V)
    assert (grad_bad_k[C:] == 0).all()


# ----------------------------------------------------------------------------- self-cond drop
def test_selfcond_drop_fair_coin_and_zeroing():
    n_seq, C, d = 4000, 2, 3
    z = np.random.default_rng(0).standard_normal((n_seq * C, d))
    out, keep = O.selfcond_drop(z, n_seq, C, d, 9, 0)
    assert scipy.stats.binomtest(int(keep.sum()), n_seq, 0.5).pvalue > P_MIN
    zz = out.reshape(n_seq, C, d)
    z0 = z.reshape(n_seq, C, d)
    assert (zz[keep == 0] == 0).all()
    assert (zz[keep == 1] == z0[keep == 1]).all()
    _, keep2 = O.selfcond_drop(z, n_seq, C, d, 9, 1)
    assert 0.4 < (keep2 != keep).mean() < 0.6  # a new coin per step


# ----------------------------------------------------------------------------- FFW
def test_gelu_tanh_against_torch_and_limits():
    xs = np.linspace(-8, 8, 161)
    ref = torch.nn.functional.gelu(torch.tensor(xs, dtype=torch.float64), approximate="tanh").numpy()
    got = np.array([O.gelu_tanh(x) for x in xs])
    assert np.allclose(got, ref, rtol=1e-14, atol=1e-15)
    assert O.gelu_tanh(0.0) == 0.0
    assert O.gelu_tanh(30.0) == pytest.approx(30.0) and abs(O.gelu_tanh(-30.0)) < 1e-30


def test_ffw_against_torch_float64():
    rng = np.random.default_rng(2)
    R, d, dff = 5, 16, 48
    z = rng.standard_normal((R, d)).astype(np.float32)
    W1 = (rng.standard_normal((d, dff)) / 4).astype(np.float32)
    W2 = (rng.standard_normal((dff, d)) / 7).astype(np.float32)
    got = O.ffw(z, W1, W2)
    t = lambda a: torch.tensor(a, dtype=torch.float64)
    ref = (torch.nn.functional.gelu(t(z) @ t(W1), approximate="tanh") @ t(W2)).numpy()
    assert np.allclose(got, ref, rtol=1e-12, atol=1e-14)
    assert np.allclose(O.ffw(np.zeros_like(z), W1, W2), 0.0)
    assert np.allclose(O.ffw(z, W1, 2 * W2), 2 * got, rtol=1e-13)  # linear in the second layer
