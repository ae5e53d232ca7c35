"""Failure detection on the GPU without a GPU fault.

Every wait inside the library's kernels is bounded.  These tests make waits run out on purpose
-- a barrier nothing arrives on, a contraction whose copy of one block of E is never issued, and
per-row merges of the logits pass whose rows nothing counts -- and check that the kernels give up, report through dg_device_error() (code 1), free
what they hold and leave the device usable: the next normal call gives the same result as a
call made before the stall.  Limits are about 10 ms so the tests stay short.
"""
import ctypes
import time

import pytest
import torch

import discrete_diffusion_lm_b200 as dg
from discrete_diffusion_lm_b200 import workloads as W

pytestmark = pytest.mark.gpu
LIMIT = 20_000_000  # SM cycles, about 10 ms


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def test_bounded_wait_gives_up_and_device_stays_usable():
    assert dg.dg_device_error() == 0
    t0 = time.time()
    assert dg.lib().dg_test_bounded_wait(ctypes.c_uint32(LIMIT), _stream()) == 0
    assert dg.dg_device_error() == 1
    assert time.time() - t0 < 5.0
    assert dg.dg_device_error() == 0  # read-and-clear
    cfg = W.TINY
    logits = W.make_logits(cfg, "cuda")
    x_t = W.make_canvas(cfg, "cuda")
    out = dg.dg_sampler_step(logits, x_t, cfg.C, 0.5, 0.125, schedule="linear", mode="greedy")
    torch.cuda.synchronize()
    assert torch.equal(out["x0_hat"], logits.argmax(1).to(torch.int32))


def _stall(logits, E, C, lse, block):
    R, V = logits.shape[0], E.shape[0]
    z = torch.empty((R, E.shape[1]), dtype=torch.bfloat16, device="cuda")
    nbytes = dg.dg_selfcond_workspace_size(R, V, E.shape[1], dg._dtype_code(logits), dg._dtype_code(E), True)
    ws = torch.zeros(max(nbytes, 256), dtype=torch.uint8, device="cuda")
    rc = dg.lib().dg_test_selfcond_stall(
        ctypes.c_void_p(logits.data_ptr()), dg._dtype_code(logits), logits.stride(0), R // C, C, V, None,
        ctypes.c_void_p(lse.data_ptr()), ctypes.c_void_p(E.data_ptr()), dg._dtype_code(E), E.shape[1],
        ctypes.c_void_p(z.data_ptr()), ctypes.c_void_p(ws.data_ptr()), ws.numel(), _stream(), block,
        ctypes.c_uint32(LIMIT))
    assert rc == 0, dg.dg_last_error()


@pytest.mark.parametrize("name,block", [("mid", 100), ("tiny", 5)])
def test_contraction_stall_aborts_cleanly(name, block):
    # mid: 256 rows, CTA-pair kernel; tiny: 16 rows, single-CTA kernel
    cfg = W.SAMPLER_CONFIGS[name]
    logits = W.make_logits(cfg, "cuda")
    E = W.make_embedding(cfg, "cuda")
    x_t = W.make_canvas(cfg, "cuda")
    lse = dg.dg_sampler_step(logits, x_t, cfg.C, 1.0, 1.0 / cfg.steps, schedule=cfg.schedule)["lse"]
    before = dg.dg_selfcond(logits, E, cfg.C, lse=lse).clone()
    assert dg.dg_device_error() == 0
    t0 = time.time()
    _stall(logits, E, cfg.C, lse, block)
    assert dg.dg_device_error() == 1
    assert time.time() - t0 < 10.0
    after = dg.dg_selfcond(logits, E, cfg.C, lse=lse)
    torch.cuda.synchronize()
    assert dg.dg_device_error() == 0
    assert torch.equal(before, after)


def test_merge_wait_gives_up_and_device_stays_usable():
    cfg = W.TINY
    logits = W.make_logits(cfg, "cuda")
    x_t = W.make_canvas(cfg, "cuda")
    R, V = logits.shape
    nbytes = dg.dg_sampler_step_workspace_size(R, V)
    ws = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
    lse = torch.empty(R, dtype=torch.float32, device="cuda")
    assert dg.dg_device_error() == 0
    t0 = time.time()
    rc = dg.lib().dg_test_merge_stall(ctypes.c_void_p(logits.data_ptr()), dg._dtype_code(logits), logits.stride(0),
                                      R, V, ctypes.c_void_p(lse.data_ptr()), ctypes.c_void_p(ws.data_ptr()), nbytes,
                                      ctypes.c_uint32(LIMIT), _stream())
    assert rc == 0, dg.dg_last_error()
    assert dg.dg_device_error() == 1
    assert time.time() - t0 < 5.0
    # the device is usable and a normal step (on a fresh workspace) is right
    out = dg.dg_sampler_step(logits, x_t, cfg.C, 0.5, 0.125, schedule="linear", mode="greedy")
    torch.cuda.synchronize()
    assert dg.dg_device_error() == 0
    assert torch.equal(out["x0_hat"], logits.argmax(1).to(torch.int32))
