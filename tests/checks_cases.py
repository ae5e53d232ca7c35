"""Cases run against the checks library (DG_LIB=checks, built with DG_CHECKS=1) by
tests/test_gpu_checks.py in a child process.

Part 1, valid inputs on odd shapes (C = 1, 17, 33; V not a multiple of the 512-id chunk; ld > V;
ragged pair tiles; bf16 and fp32 logits): every result matches the oracle as in the parity tests,
and no device-side check fires (device error code 0).

Part 2, inputs the caller got wrong, one at a time: a token id of x_t past V, a canvas CE target
past V, a canvas index past K, a training token below 0.  The normal library already handles each
without an out-of-range access (the token ids are only compared or copied, a bad target gives a NaN
loss); the checks library must also report device error code 2.

Exit status 0 when every case passes; the failures are printed otherwise.
"""
import sys

import numpy as np
import torch

import discrete_diffusion_lm_b200 as dg
from oracle import oracle as O

DEV = "cuda"
failures = []


def expect(cond, what):
    if not cond:
        failures.append(what)
        print("FAIL:", what, flush=True)


def logits(R, V, ld, dtype, seed):
    g = torch.Generator(device=DEV).manual_seed(seed)
    full = torch.zeros((R, ld), device=DEV, dtype=torch.float32)
    full[:, :V] = torch.randn((R, V), device=DEV, generator=g) * 2
    return full.to(dtype)


def host(t):
    return t.float().cpu().numpy()


def sampler_case(B, C, V, ld, dtype, seed):
    L = logits(B * C, V, ld, dtype, seed)
    x_t = torch.randint(0, V, (B * C,), device=DEV, dtype=torch.int32)
    t, dt = [0.7] * B, [0.1] * B
    out = dg.dg_sampler_step(L, x_t, C, t, dt, V=V, schedule="cosine", seed=5, step=2)
    torch.cuda.synchronize()
    ref = O.sampler_step(host(L), x_t.cpu().numpy(), B, C, V, "cosine", t, dt, None, 5, 2, "sample")
    tag = f"sampler B={B} C={C} V={V} ld={ld} {dtype}"
    for k in ("argmax", "x0_hat", "x_next"):
        expect(np.array_equal(out[k].cpu().numpy(), ref[k]), f"{tag}: {k}")
    for k in ("lse", "entropy", "max_prob"):
        expect(np.abs(out[k].cpu().numpy() - ref[k]).max() <= 1e-3, f"{tag}: {k}")
    return out


def main():
    # ---- part 1: valid inputs, odd shapes
    sampler_case(3, 17, 1037, 1040, torch.bfloat16, 1)
    sampler_case(2, 1, 513, 520, torch.float32, 2)
    out = sampler_case(2, 33, 4099, 4104, torch.bfloat16, 3)

    H = out["entropy"]
    eps = float(np.sort(H.cpu().numpy()[:33])[:10].sum())
    acc = dg.dg_entropy_accept(H, out["x0_hat"], 33, 4099, eps, seed=5, step=2)
    torch.cuda.synchronize()
    x_ref, a_ref, n_ref = O.entropy_accept(H.cpu().numpy(), out["x0_hat"].cpu().numpy(), 2, 33, 4099, eps, 5, 2)
    expect(np.array_equal(acc["accepted"].cpu().numpy(), a_ref), "entropy accept: accepted")
    expect(np.array_equal(acc["x_next"].cpu().numpy(), x_ref), "entropy accept: x_next")

    # contraction on ragged CTA-pair tiles
    L = logits(200, 3001, 3008, torch.bfloat16, 4)
    g = torch.Generator(device=DEV).manual_seed(4)
    E = (torch.randn((3001, 256), device=DEV, generator=g) * 0.02).to(torch.bfloat16)
    z = dg.dg_selfcond(L, E, 100, V=3001)
    torch.cuda.synchronize()
    rows = [0, 99, 127, 128, 199]
    zr = O.selfcond_rows(host(L), host(E), rows)
    err = np.linalg.norm(host(z)[rows] - zr) / np.linalg.norm(zr)
    expect(err <= 2e-2, f"contraction: rel Frobenius {err:.3g}")

    # feed-forward block with a 128-column tile
    zf = torch.randn((130, 256), device=DEV, generator=g).to(torch.bfloat16)
    w1 = (torch.randn((256, 768), device=DEV, generator=g) * 256 ** -0.5).to(torch.bfloat16)
    w2 = (torch.randn((768, 256), device=DEV, generator=g) * 768 ** -0.5).to(torch.bfloat16)
    y, _ = dg.dg_ffw(zf, w1, w2)
    torch.cuda.synchronize()
    yr = O.ffw(host(zf), host(w1), host(w2))
    ferr = np.linalg.norm(host(y) - yr) / np.linalg.norm(yr)
    expect(ferr <= 1e-2, f"ffw: rel Frobenius {ferr:.3g}")

    # training side: forward noise, canvas CE and its backward
    n_seq, P, K, C, V = 2, 8, 2, 16, 1000
    x0 = torch.randint(0, V, (n_seq, P + K * C), device=DEV, dtype=torch.int32)
    xt, kk = dg.dg_forward_noise(x0, P, K, C, V, [0.4, 0.8], seed=3)
    torch.cuda.synchronize()
    xr, kr = O.forward_noise(x0.cpu().numpy(), n_seq, P, K, C, V, "cosine", [0.4, 0.8], 3)
    expect(np.array_equal(xt.cpu().numpy(), xr) and np.array_equal(kk.cpu().numpy(), kr), "forward noise")
    Lce = logits(n_seq * C, V, 1000, torch.bfloat16, 6)
    loss, seq, lse = dg.dg_canvas_ce(Lce, x0, kk, P, K, C)
    torch.cuda.synchronize()
    lref, sref, _ = O.canvas_ce(host(Lce), x0.cpu().numpy(), kk.cpu().numpy(), n_seq, P, K, C, V)
    expect(np.abs(loss.cpu().numpy() - lref).max() <= 1e-3 + 1e-5 * np.abs(lref).max(), "canvas CE")
    gref = O.canvas_ce_backward(host(Lce), x0.cpu().numpy(), kk.cpu().numpy(), n_seq, P, K, C, V)
    dg.dg_canvas_ce_backward(Lce, lse, x0, kk, P, K, C)
    torch.cuda.synchronize()
    gerr = np.abs(host(Lce)[:, :V] - gref).max()
    expect(gerr <= 4e-3, f"canvas CE backward: max |err| {gerr:.3g}")  # one bf16 rounding of |g| <= 1

    code = dg.dg_device_error()
    expect(code == 0, f"valid inputs: device error {code}")

    # ---- part 2: inputs the caller got wrong, one at a time
    L = logits(17, 1037, 1040, torch.bfloat16, 7)
    x_bad = torch.randint(0, 1037, (17,), device=DEV, dtype=torch.int32)
    x_bad[5] = 1037 + 5
    dg.dg_sampler_step(L, x_bad, 17, [0.5], [0.1], V=1037)
    code = dg.dg_device_error()
    expect(code == 2, f"token id of x_t past V: device error {code}")

    x0_bad = x0.clone()
    k0 = int(kk[0])
    x0_bad[0, P + k0 * C + 3] = V + 1
    dg.dg_canvas_ce(Lce, x0_bad, kk, P, K, C)
    code = dg.dg_device_error()
    expect(code == 2, f"canvas CE target past V: device error {code}")

    k_bad = kk.clone()
    k_bad[1] = K
    dg.dg_canvas_ce(Lce, x0, k_bad, P, K, C)
    code = dg.dg_device_error()
    expect(code == 2, f"canvas index past K: device error {code}")

    x0_neg = x0.clone()
    x0_neg[1, 2] = -3
    dg.dg_forward_noise(x0_neg, P, K, C, V, [0.4, 0.8], seed=3)
    code = dg.dg_device_error()
    expect(code == 2, f"training token below 0: device error {code}")

    expect(dg.dg_device_error() == 0, "the error word clears on reading")
    print("checks library:", dg.lib()._name)
    print("failures:", len(failures))
    return 1 if failures else 0


if __name__ == "__main__":
    sys.exit(main())
