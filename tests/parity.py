"""Comparison helpers shared by the GPU-vs-oracle parity tests.

Tolerances (written here, used by every parity test):
  * integer outputs (argmax, greedy x0_hat / x_next, branch, forward-noise
    tokens, loss canvas): bit-exact;
  * sampled x0_hat / x_next: bit-exact except at positions where the oracle's
    top-two Gumbel-perturbed scores (either level of the two-level draw) differ
    by less than 1e-5 relative; mismatches must lie on such positions and
    number at most 1e-4 of the positions checked;
  * softmax statistics (lse, max-prob, entropy): |gpu - oracle| <= 1e-3;
  * z = softmax(l) E in bf16: relative Frobenius error <= 2e-2, over the rows
    checked together and on each row alone;
  * canvas cross-entropy: |gpu - oracle| <= 1e-3 + 1e-5 |oracle| per row and
    <= 1e-5 relative (+1e-2 absolute) for the per-sequence sums.
"""
from __future__ import annotations

import numpy as np
import torch

STAT_ATOL = 1e-3
NEAR_TIE_REL = 1e-5
MAX_TIE_FRACTION = 1e-4
Z_REL_FRO = 2e-2


def host_f32(t: torch.Tensor) -> np.ndarray:
    """Exact widening of bf16/fp32 device logits to a float32 host array."""
    return t.detach().float().cpu().numpy()


def check_sampler(gpu: dict, ref: dict, mode: str, rows=None, label: str = "") -> dict:
    """Compare one sampler step; `rows` selects the rows `ref` was computed on."""
    g = {k: v.detach().cpu().numpy() for k, v in gpu.items()}
    if rows is not None:
        g = {k: v[rows] for k, v in g.items()}
    n = len(ref["argmax"])
    np.testing.assert_array_equal(g["argmax"], ref["argmax"], err_msg=f"{label} argmax")
    for k in ("lse", "max_prob", "entropy"):
        err = np.abs(g[k].astype(np.float64) - ref[k])
        assert err.max() <= STAT_ATOL, f"{label} {k}: max |err| {err.max():.3g} at row {int(err.argmax())}"
    near = (ref["gap1"] < NEAR_TIE_REL) | (ref["gap2"] < NEAR_TIE_REL)
    if mode == "greedy":
        np.testing.assert_array_equal(g["x0_hat"], ref["x0_hat"], err_msg=f"{label} greedy x0_hat")
        np.testing.assert_array_equal(g["x_next"], ref["x_next"], err_msg=f"{label} greedy x_next")
        np.testing.assert_array_equal(g["branch"], ref["branch"], err_msg=f"{label} greedy branch")
        mism = 0
    else:
        bad = g["x0_hat"] != ref["x0_hat"]
        assert not np.any(bad & ~near), (
            f"{label} x0_hat differs off near-ties at rows {np.nonzero(bad & ~near)[0][:10]}")
        mism = int(bad.sum())
        assert mism <= MAX_TIE_FRACTION * n, f"{label} {mism} near-tie mismatches in {n} rows"
        same = ~bad
        np.testing.assert_array_equal(g["x_next"][same], ref["x_next"][same], err_msg=f"{label} x_next")
        np.testing.assert_array_equal(g["branch"][same], ref["branch"][same], err_msg=f"{label} branch")
    return {"rows": n, "near_ties": int(near.sum()), "mismatches": mism,
            "max_stat_err": float(max(np.abs(g[k] - ref[k]).max() for k in ("lse", "max_prob", "entropy")))}


def rel_fro(a: np.ndarray, b: np.ndarray) -> float:
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def rel_fro_rows(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    """Relative Frobenius (Euclidean) error of each row of a against the same row of b."""
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return np.linalg.norm(a - b, axis=1) / np.maximum(np.linalg.norm(b, axis=1), 1e-300)
