"""GPU-vs-oracle parity of the feed-forward block on the self-conditioning input
(dg_ffw: gelu(z W1) W2 on the tensor cores, bf16 in and out), through the C ABI.

Tolerance (this file): relative Frobenius error <= 1e-2 for the output and for the hidden
activations.  The expected error is the bf16 rounding of the hidden layer and of the output
(2^-9 relative per element, ~0.3% in Frobenius norm); inputs are bf16 on both sides.
Cases: the tiny, mid and full shapes (d = 64 / 1024 / 2048, d_ff = 4d; all rows, or a row sample
at full size), a ragged row count, a single row, and a non-default hidden width.
"""
import numpy as np
import pytest
import torch

import discrete_diffusion_lm_b200 as dg
from discrete_diffusion_lm_b200 import workloads as W
from oracle import oracle as O
from tests.parity import rel_fro

pytestmark = pytest.mark.gpu
DEV = "cuda"
TOL = 1e-2


def _check(z, w1, w2, rows=None):
    out, hidden = dg.dg_ffw(z, w1, w2)
    torch.cuda.synchronize()
    zh, a, b = z.float().cpu().numpy(), w1.float().cpu().numpy(), w2.float().cpu().numpy()
    if rows is not None:
        zh = zh[rows]
    ref = O.ffw(zh, a, b)
    got = out.float().cpu().numpy() if rows is None else out.float().cpu().numpy()[rows]
    err = rel_fro(got, ref)
    assert err <= TOL, f"output rel Frobenius {err:.3g}"
    h_ref = np.vectorize(O.gelu_tanh)(zh.astype(np.float64) @ a.astype(np.float64))
    h_got = hidden.float().cpu().numpy() if rows is None else hidden.float().cpu().numpy()[rows]
    assert rel_fro(h_got, h_ref) <= TOL
    return err


@pytest.mark.parametrize("name", ["tiny", "mid"])
def test_ffw_all_rows(name):
    cfg = W.SAMPLER_CONFIGS[name]
    z, w1, w2 = W.make_ffw(cfg, DEV)
    _check(z, w1, w2)


def test_ffw_full_sampled_rows():
    cfg = W.FULL
    z, w1, w2 = W.make_ffw(cfg, DEV)
    rows = np.sort(np.random.default_rng(0).choice(cfg.R, 8, replace=False))
    _check(z, w1, w2, rows)


@pytest.mark.parametrize("R,d,dff", [(200, 512, 2048), (1, 128, 512), (130, 256, 768), (300, 256, 512), (256, 384, 1152),
                                      (200, 512, 8192)])  # two K-splits folded, ragged rows
def test_ffw_edge_shapes(R, d, dff):
    g = torch.Generator(device=DEV).manual_seed(R + d)
    z = torch.randn(R, d, generator=g, device=DEV).to(torch.bfloat16)
    w1 = (torch.randn(d, dff, generator=g, device=DEV) * d ** -0.5).to(torch.bfloat16)
    w2 = (torch.randn(dff, d, generator=g, device=DEV) * dff ** -0.5).to(torch.bfloat16)
    _check(z, w1, w2)


def test_ffw_repeated_calls_one_workspace():
    # Successive calls on one workspace: the first layer's two K-splits hand their partial tiles over
    # through counters in the workspace, which the second layer's partial sums must not disturb.
    cfg = W.FULL
    z, w1, w2 = W.make_ffw(cfg, DEV)
    R, d = z.shape
    dff = w1.shape[1]
    ws = torch.zeros(max(256, int(dg.lib().dg_ffw_workspace_size(R, d, dff))), dtype=torch.uint8, device=DEV)
    rows = np.sort(np.random.default_rng(1).choice(R, 6, replace=False))
    a, b = w1.float().cpu().numpy(), w2.float().cpu().numpy()
    for k in range(3):
        zk = (z.float() * (1.0 + 0.5 * k) - 0.25 * k).to(torch.bfloat16)
        out, _ = dg.dg_ffw(zk, w1, w2, ws=ws)
        torch.cuda.synchronize()
        ref = O.ffw(zk.float().cpu().numpy()[rows], a, b)
        assert rel_fro(out.float().cpu().numpy()[rows], ref) <= TOL, k
    assert dg.dg_device_error() == 0
