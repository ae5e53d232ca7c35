"""GPU-vs-oracle parity of the sampler step (logits pass: statistics, argmax, two-level
Gumbel-max draw, Step posterior) through the C ABI.

Sizes: the tiny and mid sampler workloads in full (every row, every step), the
full-vocabulary workload (C = 256, V = 262144, all rows) and the 16-canvas batched
workload on a row sample, plus edge cases: ragged V, V < 32, V = 1, ld > V, odd C,
per-canvas times and temperatures, -inf logits, dt = 0, the final step (kappa_s = 1).
"""
import math

import numpy as np
import pytest
import torch

from discrete_diffusion_lm_b200 import dg_sampler_step, workloads as W
from oracle import oracle as O
from tests.parity import check_sampler, host_f32

pytestmark = pytest.mark.gpu
DEV = "cuda"


def run_both(logits, x_t, C, t, dt, *, schedule, inv_tau=None, seed=0, step=0, mode="sample", V=None,
             rows=None):
    V = logits.shape[1] if V is None else V
    out = dg_sampler_step(logits, x_t, C, t, dt, V=V, schedule=schedule, inv_tau=inv_tau, seed=seed, step=step,
                          mode=mode)
    torch.cuda.synchronize()
    R = logits.shape[0]
    B = R // C
    L = host_f32(logits)
    xt = x_t.cpu().numpy()
    tl = list(t) if not isinstance(t, (int, float)) else [t] * B
    dl = list(dt) if not isinstance(dt, (int, float)) else [dt] * B
    it = None if inv_tau is None else (list(inv_tau) if not isinstance(inv_tau, (int, float)) else [inv_tau] * B)
    if rows is None:
        ref = O.sampler_step(L[:, :], xt, B, C, V, schedule, tl, dl, it, seed, step, mode)
    else:
        # rows are independent: run the oracle row by row on the sample, each as a 1-row canvas with
        # its own canvas's scalars and its global row id
        ref = {k: [] for k in ("x_next", "x0_hat", "argmax", "max_prob", "lse", "entropy", "branch", "gap1", "gap2")}
        for r in rows:
            b = r // C
            one = _oracle_row(L[r], int(xt[r]), V, schedule, tl[b], dl[b], 1.0 if it is None else it[b], seed, step,
                              int(r), mode)
            for k in ref:
                ref[k].append(one[k])
        ref = {k: np.asarray(v) for k, v in ref.items()}
    return out, ref


def _oracle_row(row, x_t, V, schedule, t, dt, inv_tau, seed, step, r, mode):
    lse, pm, H = O.row_stats(row[:V], inv_tau)
    am = O.argmax(row[:V])
    if mode == "greedy":
        x0, g1, g2 = am, math.inf, math.inf
    else:
        x0, g1, g2 = O.draw_x0(row[:V], inv_tau, seed, step, r)
    kt = O.kappa(schedule, t)
    ks = O.kappa(schedule, max(t - dt, 0.0))
    xn, br = O.step(x_t, x0, kt, ks, V, seed, step, r)
    return dict(x_next=xn, x0_hat=x0, argmax=am, max_prob=pm, lse=lse, entropy=H, branch=br, gap1=g1, gap2=g2)


@pytest.mark.parametrize("mode", ["sample", "greedy"])
def test_tiny_all_steps(mode):
    cfg = W.TINY
    logits = W.make_logits(cfg, DEV)
    x_t = W.make_canvas(cfg, DEV)
    for k in range(cfg.steps):
        t, dt = cfg.times(k)
        out, ref = run_both(logits, x_t, cfg.C, t, dt, schedule=cfg.schedule, step=k, mode=mode)
        check_sampler(out, ref, mode, label=f"tiny step {k}")
        x_t = out["x_next"].clone()
    # the last step reaches kappa_s = 1: the canvas is x0_hat exactly
    np.testing.assert_array_equal(out["x_next"].cpu().numpy(), out["x0_hat"].cpu().numpy())


@pytest.mark.parametrize("mode", ["sample", "greedy"])
def test_mid_all_steps(mode):
    cfg = W.MID
    logits = W.make_logits(cfg, DEV)
    x_t = W.make_canvas(cfg, DEV)
    ties = 0
    for k in range(cfg.steps):
        t, dt = cfg.times(k)
        out, ref = run_both(logits, x_t, cfg.C, t, dt, schedule=cfg.schedule, step=k, seed=7, mode=mode)
        ties += check_sampler(out, ref, mode, label=f"mid step {k}")["mismatches"]
        x_t = out["x_next"].clone()
    assert ties <= 1


def test_full_vocab_all_rows():
    cfg = W.FULL
    logits = W.make_logits(cfg, DEV)
    x_t = W.make_canvas(cfg, DEV)
    for k in (0, 5, 11):
        t, dt = cfg.times(k)
        out, ref = run_both(logits, x_t, cfg.C, t, dt, schedule=cfg.schedule, step=k, seed=3)
        check_sampler(out, ref, "sample", label=f"full step {k}")


def test_batched_row_sample():
    cfg = W.BATCHED
    logits = W.make_logits(cfg, DEV)
    x_t = W.make_canvas(cfg, DEV)
    rng = np.random.default_rng(0)
    rows = np.sort(rng.choice(cfg.R, 96, replace=False))
    rows = np.unique(np.concatenate([rows, [0, cfg.C - 1, cfg.C, cfg.R - 1]]))
    for k in (0, 6):
        t, dt = cfg.times(k)
        out, ref = run_both(logits, x_t, cfg.C, t, dt, schedule=cfg.schedule, step=k, seed=11, rows=rows)
        check_sampler(out, ref, "sample", rows=rows, label=f"batched step {k}")


@pytest.mark.parametrize("V,ld,C,B", [(5000, 5000 + 8, 3, 2), (4096 + 7, 4096 + 8, 17, 1), (31, 32, 5, 3),
                                      (1, 8, 4, 2), (2048, 2048, 1, 1), (2049, 2056, 2, 2), (6 * 2048, 6 * 2048, 9, 4)])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_edge_shapes(V, ld, C, B, dtype):
    g = torch.Generator(device=DEV).manual_seed(V + C)
    R = B * C
    full = torch.full((R, ld), -3.0, device=DEV, dtype=torch.float32)
    full[:, :V] = torch.randn((R, V), device=DEV, generator=g) * 2
    logits = full.to(dtype)
    x_t = torch.randint(0, V, (R,), device=DEV, dtype=torch.int32, generator=g)
    t = [0.9 - 0.2 * b for b in range(B)]
    dt = [0.1 + 0.05 * b for b in range(B)]
    inv_tau = [1.0 + 0.25 * b for b in range(B)]
    for mode in ("sample", "greedy"):
        out, ref = run_both(logits, x_t, C, t, dt, schedule="linear", inv_tau=inv_tau, seed=5, step=2, mode=mode, V=V)
        check_sampler(out, ref, mode, label=f"V={V} ld={ld} C={C} B={B} {dtype}")


@pytest.mark.parametrize("V", [262144 + 6 * 512 + 5, 1 << 20])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_rows_longer_than_512_chunks(V, dtype):
    # past 512 chunks the merge keeps the first 512 records in registers and re-reads the rest
    B, C = 2, 3
    R, ld = B * C, (V + 7) // 8 * 8
    g = torch.Generator(device=DEV).manual_seed(V)
    full = torch.zeros((R, ld), device=DEV, dtype=torch.float32)
    full[:, :V] = torch.randn((R, V), device=DEV, generator=g) * 2
    full[0, V - 1] = 14.0  # the row maximum in the last (ragged) chunk
    far = (V // 512 - 2) * 512 + 9  # ... in a chunk past the first 512
    full[1, far] = 14.0
    full[2, :V] = 0.5  # a constant row: argmax 0
    logits = full.to(dtype)
    x_t = torch.randint(0, V, (R,), device=DEV, dtype=torch.int32, generator=g)
    for mode in ("sample", "greedy"):
        out, ref = run_both(logits, x_t, C, [0.7, 0.3], [0.1, 0.3], schedule="cosine", seed=9, step=4, mode=mode,
                            V=V)
        check_sampler(out, ref, mode, label=f"V={V} {dtype}")
    assert int(out["argmax"][0]) == V - 1 and int(out["argmax"][1]) == far
    assert int(out["argmax"][2]) == 0


def test_masked_logits_and_ties():
    V, C = 3000, 8
    g = torch.Generator(device=DEV).manual_seed(1)
    x = torch.randn((C, V), device=DEV, generator=g)
    x[0, :100] = float("-inf")      # masked tokens
    x[1, :] = float("-inf")
    x[1, 2500] = 0.0                # a single allowed token
    x[2, :] = 1.0                   # all tied: argmax 0
    x[3, ::7] = 5.0                 # many tied maxima
    x[4, 2047:2050] = 9.0           # tie straddling a chunk boundary
    for dtype in (torch.bfloat16, torch.float32):
        logits = x.to(dtype)
        x_t = torch.arange(C, device=DEV, dtype=torch.int32)
        for mode in ("sample", "greedy"):
            out, ref = run_both(logits, x_t, C, 0.5, 0.25, schedule="cosine", mode=mode, seed=9)
            check_sampler(out, ref, mode, label=f"masked {dtype} {mode}")
        assert int(out["argmax"][1]) == 2500 and int(out["x0_hat"][1]) == 2500


def test_dt_zero_and_final_step():
    cfg = W.MID
    logits = W.make_logits(cfg, DEV, rows=64)
    x_t = torch.randint(0, cfg.V, (64,), device=DEV, dtype=torch.int32)
    out = dg_sampler_step(logits, x_t, 64, 0.6, 0.0, schedule="cosine", seed=1)
    assert torch.equal(out["x_next"], x_t) and int(out["branch"].max()) == 0
    out = dg_sampler_step(logits, x_t, 64, 1.0 / 12, 1.0 / 12, schedule="cosine", seed=1)
    assert torch.equal(out["x_next"], out["x0_hat"])


def test_repeatable_and_seed_dependent():
    cfg = W.MID
    logits = W.make_logits(cfg, DEV, rows=128)
    x_t = W.make_canvas(cfg, DEV)[:128].contiguous()
    a = {k: v.clone() for k, v in dg_sampler_step(logits, x_t, 128, 0.5, 0.1, seed=4, step=3).items()}
    b = dg_sampler_step(logits, x_t, 128, 0.5, 0.1, seed=4, step=3)
    for k in a:
        assert torch.equal(a[k], b[k]), k
    c = dg_sampler_step(logits, x_t, 128, 0.5, 0.1, seed=5, step=3)
    assert not torch.equal(a["x0_hat"], c["x0_hat"])


def test_draw_frequencies_on_gpu():
    # many rows with the same logits: the GPU's x0_hat frequencies must match softmax (chi-square),
    # with a ragged multi-chunk vocabulary so both Gumbel levels matter
    V = 8 * 512 + 3
    n = 100000
    base = torch.full((V,), -30.0)
    base[[5, 100, 2047, 2048, 3000, 4098]] = torch.tensor([1.0, 0.5, 0.0, 1.5, -0.5, 1.0])
    logits = torch.full((n, V + 1), -30.0, device=DEV)  # row stride padded to 16 bytes
    logits[:, :V] = base.to(DEV)
    x_t = torch.zeros(n, dtype=torch.int32, device=DEV)
    out = dg_sampler_step(logits, x_t, n // 4, 0.5, 0.1, V=V, seed=123, step=0, schedule="linear")
    x0 = out["x0_hat"].cpu().numpy()
    ids = np.array([5, 100, 2047, 2048, 3000, 4098])
    counts = np.array([(x0 == i).sum() for i in ids])
    p = torch.softmax(base.double(), 0).numpy()[ids]
    from scipy.stats import chisquare
    assert counts.sum() >= n - 5  # the -30 background carries < 1e-9 of the mass
    assert chisquare(counts, p / p.sum() * counts.sum()).pvalue > 1e-4


def test_draw_frequencies_full_vocab_on_gpu():
    # the GPU's two-level draw at the real size: 4096 rows holding the same full-vocab row (each row
    # index keys its own Philox counters, so its draw is independent), 25 steps: 102,400 draws.
    # Frequencies on the 64 most probable ids plus a tail bucket must match softmax (chi-square).
    from scipy.special import softmax
    from scipy.stats import chisquare
    cfg = W.FULL
    row = W.make_logits(cfg, DEV, rows=1)[0]
    n = 4096
    logits = row.unsqueeze(0).expand(n, -1).contiguous()
    x_t = torch.zeros(n, dtype=torch.int32, device=DEV)
    p = softmax(row.double().cpu().numpy())
    top = np.argsort(-p, kind="stable")[:64]
    lookup = np.full(cfg.V, 64, dtype=np.int64)
    lookup[top] = np.arange(64)
    probs = np.append(p[top], 1.0 - p[top].sum())
    counts = np.zeros(65, dtype=np.int64)
    for step in range(25):
        out = dg_sampler_step(logits, x_t, 256, 0.5, 0.1, seed=77, step=step, schedule="cosine")
        counts += np.bincount(lookup[out["x0_hat"].cpu().numpy()], minlength=65)
    assert counts.sum() == 25 * n
    assert chisquare(counts, probs * counts.sum()).pvalue > 1e-4
