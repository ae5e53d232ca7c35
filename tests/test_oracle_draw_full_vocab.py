"""The oracle's x0_hat draw at the full vocabulary size, pinned to plain Gumbel-max.

DiffusionGemma Technical Report (hyper.ai summary), section "Method": the per-iteration update
samples the next state from Step(x_t, p0) with p0 = Softmax(L_t / tau_t), which needs a draw
x0_hat ~ p0.  The definition of that draw is plain Gumbel-max: x0_hat = argmax_v l'_v + G_v
with one Gumbel variate per id.  The sampler computes it in two levels (chunks of 512 ids scored
by their log-sum-exp plus a chunk Gumbel variate, then plain Gumbel-max inside the winning
chunk), which draws from the same law.  These tests pin that at the real size, V = 262144, on
rows built by the full-vocab workload's recipe (an N(0, 1.5) background plus a Zipf-like boost on
64 random ids), with many (seed, step) keys and the sampler's own chunk width:

* the keyed batch routines used for the statistics return exactly the single-draw routines'
  results (so the statistics speak about the oracle the parity tests use);
* the two-level draw's frequencies on the 64 boosted ids plus a tail bucket match softmax;
* the flat draw's frequencies match softmax;
* the two draws' frequencies match each other (two-sample test, independent keys);
* a plausible mistake -- chunks scored by their maximum instead of their log-sum-exp -- is
  rejected by the same goodness-of-fit test at 20,000 draws, fewer than the two-level tests use
  (the test has the power to see it).

CPU only; the flat draw costs about 8 ms per key, so its draws run on every host core.
"""
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import pytest
import scipy.special
import scipy.stats

from discrete_diffusion_lm_b200 import workloads as W
from oracle import oracle as O

P_MIN = 1e-4  # inputs and keys are seeded, so every p-value below is fixed
Q = O.GUMBEL_CHUNK


@pytest.fixture(scope="module")
def rows():
    # two rows of the full-vocab workload (bf16 values widened to float32)
    return W.make_logits(W.FULL, "cpu", rows=2).float().numpy()


def _bins(row):
    """Outcome bins: the 64 most probable ids (the boosted set) one by one, then everything else."""
    p = scipy.special.softmax(row.astype(np.float64))
    top = np.argsort(-p, kind="stable")[:64]
    probs = np.append(p[top], 1.0 - p[top].sum())
    lookup = np.full(row.size, 64, dtype=np.int64)
    lookup[top] = np.arange(64)
    return lookup, probs


def _counts(draws, lookup):
    return np.bincount(lookup[draws], minlength=65)


def _keys(n, seed0):
    # many seeds (Philox keys) and many steps (counter words)
    k = np.arange(n)
    return (seed0 + k // 1000).astype(np.uint64), (k % 1000).astype(np.uint32)


def _draw(row, n, seed0, row_id, flat=False):
    seeds, steps = _keys(n, seed0)
    threads = max(1, min(16, os.cpu_count() or 1))
    edges = np.linspace(0, n, threads + 1).astype(int)
    with ThreadPoolExecutor(threads) as pool:  # ctypes releases the GIL during each call
        parts = pool.map(lambda ab: O.draw_x0_keys(row, 1.0, seeds[ab[0]:ab[1]], steps[ab[0]:ab[1]], row_id, Q,
                                                   flat=flat), zip(edges[:-1], edges[1:]))
        return np.concatenate(list(parts))


def _gof(counts, probs):
    exp = probs * counts.sum()
    return scipy.stats.chisquare(counts, exp).pvalue


def test_keyed_draws_equal_single_draws(rows):
    row = rows[0]
    seeds, steps = _keys(6, 3)
    two = O.draw_x0_keys(row, 1.0, seeds, steps, 7, Q)
    flat = O.draw_x0_keys(row, 1.0, seeds, steps, 7, flat=True)
    for k in range(6):
        assert two[k] == O.draw_x0(row, 1.0, int(seeds[k]), int(steps[k]), 7, Q)[0]
        assert flat[k] == O.draw_x0_flat(row, 1.0, int(seeds[k]), int(steps[k]), 7)[0]
    # a ragged vocabulary (the last chunk shorter than Q) and a temperature
    r = row[: 5 * Q + 77]
    two = O.draw_x0_keys(r, 1.3, seeds, steps, 2, Q)
    for k in range(6):
        assert two[k] == O.draw_x0(r, 1.3, int(seeds[k]), int(steps[k]), 2, Q)[0]


def test_flat_draw_is_gumbel_max_written_out():
    # the flat routine is argmax_v l_v + G_v with G_v = -ln(-ln u) from the token domain's words
    rng = np.random.default_rng(3)
    row = rng.standard_normal(700).astype(np.float32)
    words = np.array([O.philox4x32_10([v >> 2, 4, 9, 0], [21, 0])[v & 3] for v in range(700)], dtype=np.uint64)
    u = (2 * (words >> 9) + 1).astype(np.float64) * 2.0 ** -24
    scores = row.astype(np.float64) - np.log(-np.log(u))
    x, gap = O.draw_x0_flat(row, 1.0, 21, 9, 4)
    assert x == int(np.argmax(scores))
    s = np.sort(scores)
    assert abs(gap - (s[-1] - s[-2]) / max(abs(s[-1]), 1.0)) < 1e-12


@pytest.mark.parametrize("r", [0, 1])
def test_two_level_draw_matches_softmax_at_full_vocab(rows, r):
    lookup, probs = _bins(rows[r])
    counts = _counts(_draw(rows[r], 200_000, 100 * r, r), lookup)
    assert _gof(counts, probs) > P_MIN


def test_flat_draw_matches_softmax_and_the_two_level_draw(rows):
    row = rows[0]
    lookup, probs = _bins(row)
    flat = _counts(_draw(row, 12_000, 5000, 0, flat=True), lookup)
    assert _gof(flat, probs) > P_MIN
    two = _counts(_draw(row, 200_000, 9000, 0), lookup)
    # two-sample chi-square on the 65 bins (independent keys: different seeds)
    table = np.stack([two, flat])
    table = table[:, table.sum(axis=0) > 0]
    assert scipy.stats.chi2_contingency(table).pvalue > P_MIN


def test_chunk_max_instead_of_lse_is_rejected(rows):
    # A planted mistake in a copy of the draw (numpy, CPU): level 1 scores chunks by their maximum
    # logit instead of their log-sum-exp.  At 20,000 draws (fewer than the tests above use) the
    # goodness-of-fit test must reject it, so a mistake of this kind in the oracle could not pass.
    row = rows[0].astype(np.float64)
    lookup, probs = _bins(rows[0])
    rng = np.random.default_rng(11)
    n_chunks = row.size // Q
    chunks = row.reshape(n_chunks, Q)
    cmax = chunks.max(axis=1)
    n = 20_000
    win = np.argmax(cmax[None, :] + rng.gumbel(size=(n, n_chunks)), axis=1)
    inner = np.argmax(chunks[win] + rng.gumbel(size=(n, Q)), axis=1)
    draws = win * Q + inner
    assert _gof(_counts(draws, lookup), probs) < 1e-10
