"""CPU checks that the seeded input generators draw what the input recipe says: shapes, dtypes,
value distributions, peak structure, per-canvas times, determinism (small row subsets)."""
import math

import numpy as np
import pytest
import torch

from discrete_diffusion_lm_b200 import workloads as W


@pytest.mark.parametrize("cfg,rows", [(W.TINY, None), (W.MID, 32)])
def test_set4_rows_have_four_peaks_in_8_12_over_the_background(cfg, rows):
    L = W.make_logits(cfg, "cpu", rows=rows)
    R = cfg.R if rows is None else rows
    assert L.shape == (R, cfg.V) and L.dtype == cfg.logits_dtype
    x = L.float()
    top = x.topk(4, dim=1)
    assert bool(((top.values >= 8.0) & (top.values <= 12.0)).all())
    assert bool(((x >= 8.0).sum(1) >= 4).all())
    bg = x.clone()
    bg.scatter_(1, top.indices, float("nan"))
    v = bg[~torch.isnan(bg)]
    assert abs(float(v.mean())) < 0.05
    assert abs(float(v.std()) / cfg.background_std - 1.0) < 0.03


def test_zipf64_rows_hold_most_mass_in_the_boosted_set():
    cfg = W.FULL
    L = W.make_logits(cfg, "cpu", rows=8).float()
    assert L.shape == (8, cfg.V)
    p = torch.softmax(L.double(), dim=1)
    mass = p.topk(64, dim=1).values.sum(1)
    # expectation 0.71: e^{12} sum_k k^{-1.1} against (V - 64), both lifted by e^{1.5^2 / 2}
    s = sum(k ** -1.1 for k in range(1, 65))
    expect = math.exp(12) * s / (math.exp(12) * s + cfg.V - 64)
    assert abs(expect - 0.7126) < 1e-3
    assert bool((mass > 0.4).all()) and bool((mass < 0.9).all())
    assert abs(float(mass.mean()) - expect) < 0.1
    # the boost's largest term (12 at k = 1) puts every row maximum well above the background
    assert bool((L.max(1).values > 10.0).all())
    bg = L.clone()
    bg.scatter_(1, L.topk(64, dim=1).indices, float("nan"))
    v = bg[~torch.isnan(bg)]
    assert abs(float(v.std()) / 1.5 - 1.0) < 0.02


def test_padding_beyond_v_and_determinism():
    cfg = W.TINY
    a = W.make_logits(cfg, "cpu", ld=1032)
    b = W.make_logits(cfg, "cpu")
    assert a.shape == (16, 1032) and bool((a[:, 1024:] == -7.0).all())
    assert torch.equal(a[:, :1024], b)
    assert not torch.equal(W.make_logits(cfg, "cpu", seed=cfg.seed + 1), b)


@pytest.mark.parametrize("cfg", [W.TINY, W.MID])
def test_embedding_is_normal_002(cfg):
    E = W.make_embedding(cfg, "cpu")
    assert E.shape == (cfg.V, cfg.d) and E.dtype == cfg.embed_dtype
    e = E.float()
    assert abs(float(e.mean())) < 1e-3
    assert abs(float(e.std()) / 0.02 - 1.0) < 0.02


def test_canvas_is_uniform_ids():
    cfg = W.MID
    x = W.make_canvas(cfg, "cpu")
    assert x.shape == (cfg.R,) and x.dtype == torch.int32
    assert int(x.min()) >= 0 and int(x.max()) < cfg.V
    assert torch.equal(x, W.make_canvas(cfg, "cpu"))


def test_step_times():
    t, dt = W.TINY.times(3)
    assert t == [1.0 - 3 / 8] and dt == [1 / 8]
    t, dt = W.MID.times(11)
    assert abs(t[0] - 1.0 / 12) < 1e-15 and dt == [1 / 12]
    t0, _ = W.BATCHED.times(0)
    assert len(t0) == 16 and all(0.0 <= v <= 1.0 for v in t0)
    kappa = np.array([math.cos(math.pi * v / 2) ** 2 for v in t0])
    assert 0.0 <= kappa.min() and kappa.max() <= 1.0 and len(set(t0)) == 16
    for k in (1, 5, 20):
        tk, dtk = W.BATCHED.times(k)
        assert dtk == [1 / 12] * 16
        assert all(abs(a - max(b - k / 12, 0.0)) < 1e-15 for a, b in zip(tk, t0))


def test_training_inputs():
    cfg = W.TRAIN
    x0 = W.make_train_tokens(cfg, "cpu")
    assert x0.shape == (8, 512 + 4 * 256) and x0.dtype == torch.int32
    assert int(x0.min()) >= 0 and int(x0.max()) < cfg.V
    t = W.make_train_times(cfg)
    assert len(t) == 8 and all(0.0 <= v < 1.0 for v in t)
    L = W.make_train_logits(cfg, "cpu", rows=4)
    assert L.shape == (4, cfg.V) and L.dtype == torch.bfloat16
    assert abs(float(L.float().std()) / 2.0 - 1.0) < 0.02


def test_ffw_weights_scale():
    cfg = W.MID
    z, w1, w2 = W.make_ffw(cfg, "cpu")
    d, dff = cfg.d, W.FFW_RATIO * cfg.d
    assert z.shape == (cfg.R, d) and w1.shape == (d, dff) and w2.shape == (dff, d)
    assert abs(float(w1.float().std()) * math.sqrt(d) - 1.0) < 0.02
    assert abs(float(w2.float().std()) * math.sqrt(dff) - 1.0) < 0.02
