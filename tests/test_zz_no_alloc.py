"""The allocation-free sampler step, dg_sampler_step_noalloc, against dg_sampler_step.

Some callers cannot allocate device memory where they sample (a serving loop that must not
call cudaMalloc, a runtime that owns all device memory and only lends the library its input
and output buffers).  dg_sampler_step_noalloc serves them: its scratch lives in a fixed device
array inside the library instead of a caller workspace.  The GPU test calls it through the C
ABI twice in a row, with two different shapes (so the second call meets the first call's
leftovers in the shared array), and checks each result against dg_sampler_step on the same
inputs with the parity tolerances of the other tests: integer outputs bit-exact, softmax
statistics within 1e-3.  This file is collected last, so a failure here comes after every
other test has run.
"""
import ctypes

import numpy as np
import pytest
import torch

import discrete_diffusion_lm_b200 as dg
from discrete_diffusion_lm_b200 import workloads as W
from tests.parity import STAT_ATOL

INT_KEYS = ("x_next", "x0_hat", "argmax", "branch")
STAT_KEYS = ("max_prob", "lse", "entropy")


def _compare(a: dict, b: dict, label: str):
    for k in INT_KEYS:
        assert torch.equal(a[k], b[k]), f"{label}: {k} differs"
    for k in STAT_KEYS:
        err = float((a[k].double() - b[k].double()).abs().max())
        assert err <= STAT_ATOL, f"{label}: {k} max |err| {err}"


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point_on_two_calls_in_a_row():
    cases = [(W.FULL, 4, "sample"), (W.MID, 7, "greedy")]
    for cfg, step, mode in cases:
        logits = W.make_logits(cfg, "cuda")
        x_t = W.make_canvas(cfg, "cuda")
        t, dt = cfg.times(step)
        got = dg.dg_sampler_step_noalloc(logits, x_t, cfg.C, t, dt, schedule=cfg.schedule, seed=11, step=step,
                                         mode=mode)
        want = dg.dg_sampler_step(logits, x_t, cfg.C, t, dt, schedule=cfg.schedule, seed=11, step=step, mode=mode)
        torch.cuda.synchronize()
        _compare(got, want, f"{cfg.name} {mode}")


def test_noalloc_rejects_requests_beyond_the_fixed_array():
    # 4096 rows of V = 262144 need 32 MiB of scratch: refused before anything is enqueued.  The
    # device pointers are NULL, so a call that got past the size check would still stop at the
    # host-side argument checks and never reach a kernel.
    L = dg.lib()
    t = (ctypes.c_double * 16)(*([0.5] * 16))
    dt = (ctypes.c_double * 16)(*([0.1] * 16))
    rc = L.dg_sampler_step_noalloc(None, 1, 262144, None, 16, 256, 262144, 1, t, dt, None,
                                   ctypes.c_uint64(0), ctypes.c_uint32(0), 0, None, None, None, None, None,
                                   None, None, None)
    assert rc == 3
    msg = dg.dg_last_error()
    assert "scratch" in msg and str(4 * 1024 * 1024) in msg
