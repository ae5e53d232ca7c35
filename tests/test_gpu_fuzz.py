"""Seeded random shapes against the oracle (GPU), beyond the hand-picked edge cases.

Sampler step: 40 draws of (B, C, V, ld, dtype, schedule, mode, per-canvas t, dt and inv_tau, seed,
step) with V from 1 to 9000 (chunk multiples and their neighbours among them), row paddings ld > V,
logits of random scale with a few large peaks and a few masked (-inf) ids per row; the comparison
is tests/parity.py's: exact argmax, statistics within 1e-3, x0_hat and x_next exact off near-ties.
Contraction: 12 draws of (R, C, V, d, logits dtype, embedding dtype) with per-canvas inv_tau, z on
sampled rows within the per-row relative Frobenius bound.  Decisions: 16 draws of (B, C up to 1024,
entropy kind -- continuous, heavily tied, below the fixed-point resolution, with NaN / negative /
large values --, tolerance, threshold, with or without a previous argmax canvas), bit-exact against
the oracle.  Training side: 12 draws of (n_seq, P, K, C, V, dtype, schedule), forward corruption
bit-exact and the canvas cross-entropy within its tolerances.  The draws come from fixed numpy
seeds, so every run checks the same cases.
"""
import numpy as np
import pytest
import torch

import discrete_diffusion_lm_b200 as dg
from oracle import oracle as O
from tests.parity import Z_REL_FRO, check_sampler, host_f32, rel_fro_rows

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _padded(V, elt, rng):
    step = 16 // elt  # ld * elt must be a multiple of 16 bytes
    ld = -(-V // step) * step
    return ld + step * int(rng.integers(0, 3))


def _logits(R, V, ld, dtype, rng):
    scale = float(rng.choice([0.5, 1.0, 2.0, 4.0]))
    L = rng.standard_normal((R, ld)).astype(np.float32) * scale
    L[:, V:] = 0.0
    for r in range(R):
        k = min(V, int(rng.integers(0, 4)))
        if k:
            L[r, rng.choice(V, k, replace=False)] += rng.uniform(4, 12, k).astype(np.float32)
        m = min(V - 1, int(rng.integers(0, 3)))  # masked ids, never the whole row
        if m > 0:
            L[r, rng.choice(V, m, replace=False)] = -np.inf
    t = torch.from_numpy(L).to(DEV)
    return t.to(dtype)


def _sampler_cases():
    rng = np.random.default_rng(20240)
    special = [1, 2, 511, 512, 513, 1024, 2049]
    cases = []
    for i in range(40):
        V = int(special[i]) if i < len(special) else int(rng.integers(1, 9001))
        cases.append(dict(
            i=i, B=int(rng.integers(1, 5)), C=int(rng.integers(1, 41)), V=V,
            dtype=torch.bfloat16 if rng.random() < 0.6 else torch.float32,
            schedule=str(rng.choice(["linear", "cosine"])), mode=str(rng.choice(["sample", "greedy"])),
            seed=int(rng.integers(0, 2 ** 40)), step=int(rng.integers(0, 1000)), rng_seed=int(rng.integers(0, 2 ** 31))))
    return cases


@pytest.mark.parametrize("case", _sampler_cases(), ids=lambda c: f"s{c['i']}")
def test_sampler_step_random_shapes(case):
    rng = np.random.default_rng(case["rng_seed"])
    B, C, V, dtype = case["B"], case["C"], case["V"], case["dtype"]
    R = B * C
    elt = 2 if dtype == torch.bfloat16 else 4
    ld = _padded(V, elt, rng)
    L = _logits(R, V, ld, dtype, rng)
    x_t = torch.from_numpy(rng.integers(0, V, R).astype(np.int32)).to(DEV)
    t = rng.uniform(0.05, 1.0, B)
    dt = t * rng.uniform(0.0, 1.0, B)
    inv_tau = rng.uniform(0.5, 2.0, B).astype(np.float32)
    out = dg.dg_sampler_step(L, x_t, C, list(t), list(dt), V=V, schedule=case["schedule"], inv_tau=list(inv_tau),
                             seed=case["seed"], step=case["step"], mode=case["mode"])
    torch.cuda.synchronize()
    ref = O.sampler_step(host_f32(L), x_t.cpu().numpy(), B, C, V, case["schedule"], t, dt, inv_tau, case["seed"],
                         case["step"], case["mode"])
    check_sampler(out, ref, case["mode"], label=f"case {case['i']} B={B} C={C} V={V} ld={ld} {dtype}")
    assert dg.dg_device_error() == 0


def _selfcond_cases():
    rng = np.random.default_rng(777)
    cases = []
    for i in range(12):
        C = int(rng.integers(1, 97))
        B = int(rng.integers(1, max(2, 320 // C)))
        cases.append(dict(i=i, B=B, C=C, V=int(rng.integers(1, 3001)), d=int(rng.choice([64, 128, 192, 256, 512])),
                          ldt=torch.bfloat16 if rng.random() < 0.7 else torch.float32,
                          edt=torch.bfloat16 if rng.random() < 0.7 else torch.float32,
                          rng_seed=int(rng.integers(0, 2 ** 31))))
    return cases


@pytest.mark.parametrize("case", _selfcond_cases(), ids=lambda c: f"z{c['i']}")
def test_selfcond_random_shapes(case):
    rng = np.random.default_rng(case["rng_seed"])
    B, C, V, d = case["B"], case["C"], case["V"], case["d"]
    R = B * C
    ld = _padded(V, 2 if case["ldt"] == torch.bfloat16 else 4, rng)
    L = _logits(R, V, ld, case["ldt"], rng)
    E = torch.from_numpy((rng.standard_normal((V, d)) * 0.05).astype(np.float32)).to(DEV).to(case["edt"])
    inv_tau = rng.uniform(0.5, 2.0, B).astype(np.float32)
    z = dg.dg_selfcond(L, E, C, V=V, inv_tau=list(inv_tau))
    torch.cuda.synchronize()
    rows = sorted({0, R - 1, R // 2, *rng.integers(0, R, 5).tolist()})
    it_rows = np.array([inv_tau[r // C] for r in range(R)], dtype=np.float32)
    zr = O.selfcond_rows(host_f32(L)[:, :ld], host_f32(E), rows, it_rows)
    err = rel_fro_rows(z.float().cpu().numpy()[rows], zr)
    assert err.max() <= Z_REL_FRO, (case, err.max())
    assert dg.dg_device_error() == 0


def _decision_cases():
    rng = np.random.default_rng(4242)
    cases = []
    for i in range(16):
        cases.append(dict(i=i, B=int(rng.integers(1, 9)), C=int(rng.integers(1, 1025)),
                          kind=str(rng.choice(["uniform", "tied", "tiny", "special"])),
                          eps_frac=float(rng.choice([0.0, 0.1, 0.5, 1.0, 2.0])), theta=float(rng.uniform(0, 3)),
                          prev=bool(rng.random() < 0.7), rng_seed=int(rng.integers(0, 2 ** 31))))
    return cases


def _entropies(kind, n, rng):
    if kind == "uniform":
        return rng.uniform(0.0, 6.0, n).astype(np.float32)
    if kind == "tied":
        return rng.choice(np.float32([0.0, 0.25, 1.0, 2.5]), n).astype(np.float32)
    if kind == "tiny":
        return (rng.uniform(0, 4, n) * 2.0 ** -33).astype(np.float32)
    h = rng.uniform(0.0, 3.0, n).astype(np.float32)  # special values
    for v in (np.nan, -1e-6, 90.0):
        h[rng.integers(0, n, max(1, n // 16))] = v
    return h


@pytest.mark.parametrize("case", _decision_cases(), ids=lambda c: f"d{c['i']}")
def test_decisions_random(case):
    rng = np.random.default_rng(case["rng_seed"])
    B, C, V = case["B"], case["C"], 262144
    H = _entropies(case["kind"], B * C, rng)
    x0 = rng.integers(0, V, B * C).astype(np.int32)
    eps = case["eps_frac"] * float(np.nansum(np.clip(H[:C], 0, 64)))
    seed, step = int(rng.integers(0, 2 ** 40)), int(rng.integers(0, 1000))
    Hd = torch.from_numpy(H).to(DEV)
    acc = dg.dg_entropy_accept(Hd, torch.from_numpy(x0).to(DEV), C, V, eps, seed=seed, step=step)
    am = rng.integers(0, V, B * C).astype(np.int32)
    prev = am.copy()
    prev[rng.integers(0, B * C, max(1, B // 2))] += 1  # some canvases changed their prediction
    p = prev if case["prev"] else None
    stop, mean = dg.dg_adaptive_stop(Hd, torch.from_numpy(am).to(DEV), None if p is None else torch.from_numpy(p).to(DEV),
                                     C, case["theta"])
    torch.cuda.synchronize()
    x_ref, a_ref, n_ref = O.entropy_accept(H, x0, B, C, V, eps, seed, step)
    np.testing.assert_array_equal(acc["accepted"].cpu().numpy(), a_ref)
    np.testing.assert_array_equal(acc["n_accepted"].cpu().numpy(), n_ref)
    np.testing.assert_array_equal(acc["x_next"].cpu().numpy(), x_ref)
    s_ref, m_ref = O.adaptive_stop(H, am, p, B, C, case["theta"])
    np.testing.assert_array_equal(stop.cpu().numpy(), s_ref)
    np.testing.assert_array_equal(mean.cpu().numpy(), m_ref.astype(np.float32))


def _train_cases():
    rng = np.random.default_rng(99)
    return [dict(i=i, n_seq=int(rng.integers(1, 7)), P=int(rng.integers(0, 65)), K=int(rng.integers(1, 5)),
                 C=int(rng.integers(1, 65)), V=int(rng.integers(1, 5001)),
                 dtype=torch.bfloat16 if rng.random() < 0.6 else torch.float32,
                 schedule=str(rng.choice(["linear", "cosine"])), rng_seed=int(rng.integers(0, 2 ** 31)))
            for i in range(12)]


@pytest.mark.parametrize("case", _train_cases(), ids=lambda c: f"t{c['i']}")
def test_forward_noise_and_canvas_ce_random(case):
    rng = np.random.default_rng(case["rng_seed"])
    n_seq, P, K, C, V = case["n_seq"], case["P"], case["K"], case["C"], case["V"]
    x0 = torch.from_numpy(rng.integers(0, V, (n_seq, P + K * C)).astype(np.int32)).to(DEV)
    t = list(rng.uniform(0.0, 1.0, n_seq))
    seed = int(rng.integers(0, 2 ** 40))
    xt, kk = dg.dg_forward_noise(x0, P, K, C, V, t, schedule=case["schedule"], seed=seed)
    torch.cuda.synchronize()
    rx, rk = O.forward_noise(x0.cpu().numpy(), n_seq, P, K, C, V, case["schedule"], t, seed)
    np.testing.assert_array_equal(xt.cpu().numpy(), rx)
    np.testing.assert_array_equal(kk.cpu().numpy(), rk)
    elt = 2 if case["dtype"] == torch.bfloat16 else 4
    L = _logits(n_seq * C, V, _padded(V, elt, rng), case["dtype"], rng)
    loss, seq, lse = dg.dg_canvas_ce(L, x0, kk, P, K, C, V=V)
    torch.cuda.synchronize()
    rl, rs, rlse = O.canvas_ce(host_f32(L), x0.cpu().numpy(), kk.cpu().numpy(), n_seq, P, K, C, V)
    gl = loss.cpu().numpy().astype(np.float64)
    with np.errstate(invalid="ignore"):  # a masked (-inf) target gives +inf loss on both sides
        assert np.all((gl == rl) | (np.abs(gl - rl) <= 1e-3 + 1e-5 * np.abs(rl))), case
    assert np.all(np.abs(lse.cpu().numpy() - rlse) <= 1e-3), case
    np.testing.assert_allclose(seq.cpu().numpy(), rs, rtol=1e-5, atol=1e-2)
    assert dg.dg_device_error() == 0
