"""Seeded synthetic workloads for the sampler hot path.

This module only draws inputs (logits, embeddings, canvases, per-canvas times);
it holds none of the method's arithmetic, and both the CUDA path and the CPU
oracle are fed the same tensors from here.  No dataset or trained weight
exists for these shapes, so every input is synthetic, with the sizes and value
structure of the DiffusionGemma Technical Report's sampler setting: C = 256
canvases (block-autoregressive generation, section "Method"), a 262k
vocabulary (section "Experiments"), about 12 denoising steps per block.

Notation: N(mu, sigma) has standard deviation sigma.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch


@dataclass(frozen=True)
class SamplerConfig:
    name: str
    B: int                 # canvases
    C: int                 # tokens per canvas
    V: int                 # vocabulary
    d: int                 # embedding width (self-conditioning)
    logits_dtype: torch.dtype
    embed_dtype: torch.dtype
    schedule: str          # "linear" | "cosine"
    steps: int
    peaks: str             # "set4" (4 ids per row set to U[8,12]) | "zipf64"
    background_std: float
    per_canvas_kappa: bool = False
    seed: int = 0          # torch generator seed
    philox_seed: int = 0

    @property
    def R(self) -> int:
        return self.B * self.C

    def times(self, step: int, gen_seed: int | None = None) -> tuple[list[float], list[float]]:
        """Per-canvas (t, dt) of denoising step `step` (0-based), t running 1 -> 0."""
        dt = 1.0 / self.steps
        if not self.per_canvas_kappa:
            t = 1.0 - step * dt
            return [t] * self.B, [dt] * self.B
        g = torch.Generator().manual_seed(self.seed + 1000 if gen_seed is None else gen_seed)
        kappa0 = torch.rand(self.B, generator=g, dtype=torch.float64)
        # each canvas starts at its own kappa_b ~ U(0,1), i.e. t_b = (2/pi) acos(sqrt(kappa_b))
        # on the cosine schedule, and moves by dt per step, clamped at t = 0
        t0 = [(2.0 / math.pi) * math.acos(math.sqrt(float(k))) for k in kappa0]
        return [max(t - step * dt, 0.0) for t in t0], [dt] * self.B


@dataclass(frozen=True)
class TrainConfig:
    name: str
    n_seq: int
    P: int
    K: int
    C: int
    V: int
    logits_std: float
    schedule: str = "cosine"
    seed: int = 4
    philox_seed: int = 0

    @property
    def L(self) -> int:
        return self.P + self.K * self.C


TINY = SamplerConfig("tiny", 1, 16, 1024, 64, torch.float32, torch.float32, "linear", 8, "set4", 2.0, seed=0)
MID = SamplerConfig("mid", 1, 256, 32768, 1024, torch.bfloat16, torch.bfloat16, "cosine", 12, "set4", 2.0, seed=1)
FULL = SamplerConfig("full", 1, 256, 262144, 2048, torch.bfloat16, torch.bfloat16, "cosine", 12, "zipf64", 1.5,
                     seed=2)
BATCHED = SamplerConfig("batched", 16, 256, 262144, 2048, torch.bfloat16, torch.bfloat16, "cosine", 12, "zipf64",
                        1.5, per_canvas_kappa=True, seed=3)
TRAIN = TrainConfig("train", 8, 512, 4, 256, 262144, 2.0, seed=4)

SAMPLER_CONFIGS = {c.name: c for c in (TINY, MID, FULL, BATCHED)}


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


@torch.no_grad()
def make_logits(cfg: SamplerConfig, device="cpu", rows: int | None = None, seed: int | None = None,
                ld: int | None = None) -> torch.Tensor:
    """Logits [R, ld] (view [:, :V] is the data) with the config's peak structure.

    set4:   background N(0, std); 4 distinct ids per row, positions uniform,
            whose values are *set* to U[8, 12].
    zipf64: background N(0, std); on 64 distinct random ids per row a boost
            12 - 1.1 ln k (k = 1..64) is *added*: the log of a Zipf(s = 1.1)
            profile over the top-64 set.  With std = 1.5 the set holds about
            70% of a row's probability mass (0.71 in expectation, since the
            background lifts each boosted id by e^{std^2 / 2} on average).
    """
    R = cfg.R if rows is None else rows
    V = cfg.V
    ld = V if ld is None else ld
    g = _gen(device, cfg.seed if seed is None else seed)
    out = torch.empty((R, ld), dtype=cfg.logits_dtype, device=device)
    if ld > V:
        out[:, V:].fill_(-7.0)  # padding beyond V: never read by a correct kernel
    block = max(1, (1 << 26) // V)
    for r0 in range(0, R, block):
        r1 = min(R, r0 + block)
        n = r1 - r0
        x = torch.randn((n, V), generator=g, device=device, dtype=torch.float32) * cfg.background_std
        if cfg.peaks == "set4":
            ids = torch.rand((n, V), generator=g, device=device).topk(4, dim=1).indices
            vals = 8.0 + 4.0 * torch.rand((n, 4), generator=g, device=device)
            x.scatter_(1, ids, vals)
        else:
            ids = torch.rand((n, V), generator=g, device=device).topk(64, dim=1).indices
            k = torch.arange(1, 65, device=device, dtype=torch.float32)
            boost = (12.0 - 1.1 * torch.log(k)).expand(n, 64)
            x.scatter_add_(1, ids, boost.contiguous())
        out[r0:r1, :V] = x.to(cfg.logits_dtype)
    return out


@torch.no_grad()
def make_embedding(cfg: SamplerConfig, device="cpu", seed: int | None = None) -> torch.Tensor:
    """E [V, d] ~ N(0, 0.02), row-major."""
    g = _gen(device, (cfg.seed if seed is None else seed) + 100)
    out = torch.empty((cfg.V, cfg.d), dtype=cfg.embed_dtype, device=device)
    block = max(1, (1 << 26) // cfg.d)
    for r0 in range(0, cfg.V, block):
        r1 = min(cfg.V, r0 + block)
        out[r0:r1] = (torch.randn((r1 - r0, cfg.d), generator=g, device=device) * 0.02).to(cfg.embed_dtype)
    return out


@torch.no_grad()
def make_canvas(cfg: SamplerConfig, device="cpu", seed: int | None = None) -> torch.Tensor:
    """Initial x_t: uniform over [0, V) (t = 1 is pure uniform noise), int32 [R]."""
    g = _gen(device, (cfg.seed if seed is None else seed) + 200)
    return torch.randint(0, cfg.V, (cfg.R,), generator=g, device=device, dtype=torch.int64).to(torch.int32)


@torch.no_grad()
def make_train_tokens(cfg: TrainConfig, device="cpu") -> torch.Tensor:
    """x0 int32 [n_seq, P + K*C], tokens uniform over [0, V)."""
    g = _gen(device, cfg.seed + 300)
    return torch.randint(0, cfg.V, (cfg.n_seq, cfg.L), generator=g, device=device,
                         dtype=torch.int64).to(torch.int32)


def make_train_times(cfg: TrainConfig) -> list[float]:
    """t_b ~ U(0, 1) per sequence (float64, host)."""
    g = torch.Generator().manual_seed(cfg.seed + 400)
    return [float(x) for x in torch.rand(cfg.n_seq, generator=g, dtype=torch.float64)]


@torch.no_grad()
def make_train_logits(cfg: TrainConfig, device="cpu", rows: int | None = None) -> torch.Tensor:
    """Decoder logits for the chosen canvases: bf16 [n_seq*C, V] ~ N(0, logits_std)."""
    R = cfg.n_seq * cfg.C if rows is None else rows
    g = _gen(device, cfg.seed + 500)
    out = torch.empty((R, cfg.V), dtype=torch.bfloat16, device=device)
    block = max(1, (1 << 26) // cfg.V)
    for r0 in range(0, R, block):
        r1 = min(R, r0 + block)
        out[r0:r1] = (torch.randn((r1 - r0, cfg.V), generator=g, device=device) * cfg.logits_std).to(
            torch.bfloat16)
    return out


# Feed-forward block on the self-conditioning input: hidden width = FFW_RATIO x d.
FFW_RATIO = 4


def make_ffw(cfg: SamplerConfig, device="cpu", seed: int | None = None):
    """Random-init weights of the two-layer feed-forward block and a self-conditioning input:
    z ~ N(0, 1) [R, d], W1 ~ N(0, 1/d) [d, 4d], W2 ~ N(0, 1/(4d)) [4d, d], all bf16."""
    s = cfg.seed if seed is None else seed
    dff = FFW_RATIO * cfg.d
    z = torch.randn(cfg.R, cfg.d, generator=_gen(device, s + 600), device=device)
    w1 = torch.randn(cfg.d, dff, generator=_gen(device, s + 700), device=device) * cfg.d ** -0.5
    w2 = torch.randn(dff, cfg.d, generator=_gen(device, s + 800), device=device) * dff ** -0.5
    return z.to(torch.bfloat16), w1.to(torch.bfloat16), w2.to(torch.bfloat16)
