"""Seeded random shapes against the oracle (GPU), beyond the hand-picked edge cases.

Sampler step: 40 draws of (B, C, V, ld, dtype, schedule, mode, per-canvas t, dt and inv_tau, seed,
step) with V from 1 to 9000 (chunk multiples and their neighbours among them), row paddings ld > V,
logits of random scale with a few large peaks and a few masked (-inf) ids per row; the comparison
is tests/parity.py's: exact argmax, statistics within 1e-3, x0_hat and x_next exact off near-ties.
Contraction: 12 draws of (R, C, V, d, logits dtype, embedding dtype) with per-canvas inv_tau, z on
sampled rows within the per-row relative Frobenius bound.  The draws come from a fixed numpy seed,
so every run checks the same cases.
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
