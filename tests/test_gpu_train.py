"""GPU-vs-oracle parity of the training-side kernels through the C ABI: forward corruption
(bit-exact tokens and loss canvases) and the fused canvas cross-entropy."""
import numpy as np
import pytest
import torch

from discrete_diffusion_lm_b200 import dg_canvas_ce, dg_forward_noise, workloads as W
from oracle import oracle as O
from tests.parity import host_f32

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _noise_both(x0, P, K, C, V, t, schedule, seed):
    xt, k = dg_forward_noise(x0, P, K, C, V, t, schedule=schedule, seed=seed)
    torch.cuda.synchronize()
    rx, rk = O.forward_noise(x0.cpu().numpy(), x0.shape[0], P, K, C, V, schedule, t, seed)
    return xt.cpu().numpy(), k.cpu().numpy(), rx, rk


def test_forward_noise_train_config_exact():
    cfg = W.TRAIN
    x0 = W.make_train_tokens(cfg, DEV)
    t = W.make_train_times(cfg)
    for seed in (0, 1, 2**40 + 3):
        xt, k, rx, rk = _noise_both(x0, cfg.P, cfg.K, cfg.C, cfg.V, t, cfg.schedule, seed)
        np.testing.assert_array_equal(xt, rx)
        np.testing.assert_array_equal(k, rk)


@pytest.mark.parametrize("shape", [(1, 0, 1, 1, 7), (3, 5, 2, 300, 1000), (256, 1, 3, 3, 2), (2, 700, 1, 1, 50)])
def test_forward_noise_edge_shapes(shape):
    n_seq, P, K, C, V = shape
    g = torch.Generator(device=DEV).manual_seed(n_seq * 7 + C)
    x0 = torch.randint(0, V, (n_seq, P + K * C), device=DEV, dtype=torch.int32, generator=g)
    t = list(np.linspace(0.0, 1.0, n_seq))
    for sched in ("linear", "cosine"):
        xt, k, rx, rk = _noise_both(x0, P, K, C, V, t, sched, 9)
        np.testing.assert_array_equal(xt, rx)
        np.testing.assert_array_equal(k, rk)


def test_canvas_ce_train_config():
    cfg = W.TRAIN
    logits = W.make_train_logits(cfg, DEV)
    x0 = W.make_train_tokens(cfg, DEV)
    _, kidx = dg_forward_noise(x0, cfg.P, cfg.K, cfg.C, cfg.V, W.make_train_times(cfg), seed=0)
    loss, seq, lse = dg_canvas_ce(logits, x0, kidx, cfg.P, cfg.K, cfg.C)
    torch.cuda.synchronize()
    # oracle on the first two sequences (512 rows of 262144)
    nb = 2
    L = host_f32(logits[: nb * cfg.C])
    rl, rs, rlse = O.canvas_ce(L, x0[:nb].cpu().numpy(), kidx[:nb].cpu().numpy(), nb, cfg.P, cfg.K, cfg.C, cfg.V)
    gl = loss[: nb * cfg.C].cpu().numpy().astype(np.float64)
    assert np.all(np.abs(gl - rl) <= 1e-3 + 1e-5 * np.abs(rl))
    assert np.all(np.abs(lse[: nb * cfg.C].cpu().numpy() - rlse) <= 1e-3)
    np.testing.assert_allclose(seq[:nb].cpu().numpy(), rs, rtol=1e-5, atol=1e-2)
    # every per-sequence sum equals the sum of its rows
    np.testing.assert_allclose(seq.cpu().numpy(), loss.view(cfg.n_seq, cfg.C).double().sum(1).cpu().numpy(),
                               rtol=1e-5)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_canvas_ce_small_exact_and_torch(dtype):
    n_seq, P, K, C, V = 3, 5, 3, 7, 4099
    g = torch.Generator(device=DEV).manual_seed(2)
    x0 = torch.randint(0, V, (n_seq, P + K * C), device=DEV, dtype=torch.int32, generator=g)
    kidx = torch.tensor([2, 0, 1], device=DEV, dtype=torch.int32)
    padded = torch.zeros((n_seq * C, V + 5), device=DEV, dtype=dtype)  # row stride padded to 16 bytes
    logits = padded[:, :V]
    logits.copy_((torch.randn((n_seq * C, V), device=DEV, generator=g) * 2).to(dtype))
    logits[0, :10] = float("-inf")
    loss, seq, lse = dg_canvas_ce(logits, x0, kidx, P, K, C)
    torch.cuda.synchronize()
    rl, rs, rlse = O.canvas_ce(host_f32(logits), x0.cpu().numpy(), kidx.cpu().numpy(), n_seq, P, K, C, V)
    assert np.all(np.abs(loss.cpu().numpy() - rl) <= 1e-3 + 1e-5 * np.abs(rl))
    assert np.all(np.abs(lse.cpu().numpy() - rlse) <= 1e-3)
    np.testing.assert_allclose(seq.cpu().numpy(), rs, rtol=1e-5, atol=1e-3)
    tgt = torch.stack([x0[b, P + int(kidx[b]) * C: P + (int(kidx[b]) + 1) * C] for b in range(n_seq)]).reshape(-1)
    ref = torch.nn.functional.cross_entropy(logits.double(), tgt.long(), reduction="none")
    torch.testing.assert_close(loss.double(), ref, atol=1e-3, rtol=1e-5)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_canvas_ce_rows_longer_than_512_chunks(dtype):
    n_seq, P, K, C, V = 2, 3, 2, 3, 262144 + 8 * 512 + 3
    g = torch.Generator(device=DEV).manual_seed(3)
    x0 = torch.randint(0, V, (n_seq, P + K * C), device=DEV, dtype=torch.int32, generator=g)
    x0[0, P] = V - 1  # a target in the last, ragged chunk
    kidx = torch.tensor([0, 1], device=DEV, dtype=torch.int32)
    padded = torch.zeros((n_seq * C, V + 5), device=DEV, dtype=dtype)
    logits = padded[:, :V]
    logits.copy_((torch.randn((n_seq * C, V), device=DEV, generator=g) * 2).to(dtype))
    loss, seq, lse = dg_canvas_ce(logits, x0, kidx, P, K, C)
    torch.cuda.synchronize()
    rl, rs, rlse = O.canvas_ce(host_f32(logits), x0.cpu().numpy(), kidx.cpu().numpy(), n_seq, P, K, C, V)
    assert np.all(np.abs(loss.cpu().numpy() - rl) <= 1e-3 + 1e-5 * np.abs(rl))
    assert np.all(np.abs(lse.cpu().numpy() - rlse) <= 1e-3)
    np.testing.assert_allclose(seq.cpu().numpy(), rs, rtol=1e-5, atol=1e-3)


def test_canvas_ce_bad_target_gives_nan_not_fault():
    n_seq, P, K, C, V = 2, 1, 2, 4, 100
    x0 = torch.zeros((n_seq, P + K * C), device=DEV, dtype=torch.int32)
    x0[0, P + 2] = 5000          # target out of range
    kidx = torch.tensor([0, 7], device=DEV, dtype=torch.int32)  # canvas 7 out of range
    logits = torch.zeros((n_seq * C, V), device=DEV)
    loss, seq, _ = dg_canvas_ce(logits, x0, kidx, P, K, C)
    l = loss.cpu().numpy()
    assert np.isnan(l[2]) and np.all(np.isnan(l[4:]))
    assert np.all(np.abs(l[[0, 1, 3]] - np.log(V)) < 1e-5)
