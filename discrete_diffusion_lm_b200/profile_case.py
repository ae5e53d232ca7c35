"""Run one library kernel a few times on a named workload, for a profiler to capture.

    python -m discrete_diffusion_lm_b200.profile_case --kernel selfcond --workload full --reps 3
    python -m discrete_diffusion_lm_b200.profile_case --kernel sampler_step --workload full --reps 4
    python -m discrete_diffusion_lm_b200.profile_case --kernel canvas_ce --workload train --reps 3
    python -m discrete_diffusion_lm_b200.profile_case --kernel ce_backward --workload train --reps 3
    python -m discrete_diffusion_lm_b200.profile_case --kernel selfcond_drop --workload train --reps 3
    python -m discrete_diffusion_lm_b200.profile_case --kernel entropy_bounded --workload full --reps 3
    python -m discrete_diffusion_lm_b200.profile_case --kernel ffw --workload full --reps 3

Inputs come from the seeded workload generators; the logits pass that provides lse for the
contraction runs once before the contraction launches.  Exits non-zero if a kernel reports a
device error.
"""
from __future__ import annotations

import argparse
import sys

import torch

import discrete_diffusion_lm_b200 as dg
from discrete_diffusion_lm_b200 import workloads as W


def main(argv=None) -> int:
    ap = argparse.ArgumentParser()
    ap.add_argument("--kernel", choices=["sampler_step", "selfcond", "canvas_ce", "forward_noise", "ce_backward",
                                         "selfcond_drop", "entropy_bounded", "ffw"], required=True)
    ap.add_argument("--workload", default="full", choices=sorted(W.SAMPLER_CONFIGS) + ["train"])
    ap.add_argument("--reps", type=int, default=3)
    a = ap.parse_args(argv)
    dev = "cuda"
    if a.kernel in ("canvas_ce", "forward_noise", "ce_backward", "selfcond_drop"):
        cfg = W.TRAIN
        x0 = W.make_train_tokens(cfg, dev)
        t = W.make_train_times(cfg)
        _, kidx = dg.dg_forward_noise(x0, cfg.P, cfg.K, cfg.C, cfg.V, t, seed=0)
        logits = W.make_train_logits(cfg, dev) if a.kernel in ("canvas_ce", "ce_backward") else None
        if a.kernel == "ce_backward":
            lse = dg.dg_canvas_ce(logits, x0, kidx, cfg.P, cfg.K, cfg.C)[2]
        if a.kernel == "selfcond_drop":
            z = torch.randn(cfg.n_seq * cfg.C, 2048, device=dev).to(torch.bfloat16)
        for k in range(a.reps):
            if a.kernel == "canvas_ce":
                dg.dg_canvas_ce(logits, x0, kidx, cfg.P, cfg.K, cfg.C)
            elif a.kernel == "ce_backward":
                dg.dg_canvas_ce_backward(logits, lse, x0, kidx, cfg.P, cfg.K, cfg.C)
            elif a.kernel == "selfcond_drop":
                dg.dg_selfcond_drop(z, cfg.C, seed=0, step=k)
            else:
                dg.dg_forward_noise(x0, cfg.P, cfg.K, cfg.C, cfg.V, t, seed=1)
    elif a.kernel == "ffw":
        cfg = W.SAMPLER_CONFIGS[a.workload]
        zf, w1, w2 = W.make_ffw(cfg, dev)
        y, hidden = dg.dg_ffw(zf, w1, w2)
        for _ in range(a.reps - 1):
            dg.dg_ffw(zf, w1, w2, hidden=hidden, out=y)
    elif a.kernel == "entropy_bounded":
        cfg = W.SAMPLER_CONFIGS[a.workload]
        logits = W.make_logits(cfg, dev)
        prev = None
        for k in range(a.reps):
            o = dg.dg_sampler_step_eb(logits, cfg.C, eps=64.0, theta=0.5, argmax_prev=prev,
                                      inv_tau=dg.dg_tau_linear([1.0 - k / max(1, a.reps)]), seed=0, step=k)
            prev = o["argmax"]
    else:
        cfg = W.SAMPLER_CONFIGS[a.workload]
        logits = W.make_logits(cfg, dev)
        x_t = W.make_canvas(cfg, dev)
        t, dt = cfg.times(0)
        out = dg.dg_sampler_step(logits, x_t, cfg.C, t, dt, schedule=cfg.schedule)
        if a.kernel == "selfcond":
            E = W.make_embedding(cfg, dev)
            for _ in range(a.reps):
                dg.dg_selfcond(logits, E, cfg.C, lse=out["lse"])
        else:
            for _ in range(a.reps - 1):
                dg.dg_sampler_step(logits, x_t, cfg.C, t, dt, schedule=cfg.schedule, out=out)
    torch.cuda.synchronize()
    err = dg.dg_device_error()
    print(f"{a.kernel} on {a.workload}: {a.reps} launches, device error {err}")
    return 1 if err else 0


if __name__ == "__main__":
    sys.exit(main())
