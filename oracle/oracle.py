"""ctypes shim over the plain-C oracle (``dg_oracle.c``).

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the benchmark's
CPU-baseline leg may import this module; the product path (the CUDA library
and its Python binding) never does.  The oracle shares no code with the CUDA
path.  Every function works on numpy arrays on the host, in double precision.

Citations follow the oracle's C header: DiffusionGemma Technical Report
(hyper.ai summary), sections "Method" and "Dataset"; Salmon et al., SC'11 for
Philox4x32-10.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "dg_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libdg_oracle.so")

# Chunk width of the two-level Gumbel-max draw (level 1 scores chunks of Q ids).
GUMBEL_CHUNK = 512


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (-O2, no fast-math, no FP contraction)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-D_DEFAULT_SOURCE", "-fPIC", "-shared",
               "-ffp-contract=off", "-fno-fast-math", "-o", _LIB_PATH, _SRC, "-lm"]
        subprocess.check_call(cmd)
    return _LIB_PATH


_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        _declare(_lib)
    return _lib


_p = ctypes.c_void_p
_i32 = ctypes.c_int32
_i64 = ctypes.c_int64
_u32 = ctypes.c_uint32
_u64 = ctypes.c_uint64
_f64 = ctypes.c_double


def _declare(L):
    L.dgo_philox4x32_10.argtypes = [_p, _p, _p]
    L.dgo_open_uniform.argtypes = [_u32]
    L.dgo_open_uniform.restype = _f64
    L.dgo_gumbel.argtypes = [_u32]
    L.dgo_gumbel.restype = _f64
    L.dgo_kappa.argtypes = [_i32, _f64]
    L.dgo_kappa.restype = _f64
    L.dgo_row_stats.argtypes = [_p, _i32, _f64, _p, _p, _p]
    L.dgo_row_probs.argtypes = [_p, _i32, _f64, _p]
    L.dgo_argmax.argtypes = [_p, _i32]
    L.dgo_argmax.restype = _i32
    L.dgo_draw_x0.argtypes = [_p, _i32, _f64, _u64, _u32, _u32, _i32, _p, _p]
    L.dgo_draw_x0.restype = _i32
    L.dgo_draw_x0_flat.argtypes = [_p, _i32, _f64, _u64, _u32, _u32, _p]
    L.dgo_draw_x0_flat.restype = _i32
    L.dgo_draw_x0_keys.argtypes = [_p, _i32, _f64, _p, _p, _i32, _u32, _i32, _i32, _p]
    L.dgo_step.argtypes = [_i32, _i32, _f64, _f64, _i32, _u64, _u32, _u32, _p]
    L.dgo_step.restype = _i32
    L.dgo_step_posterior.argtypes = [_i32, _i32, _f64, _f64, _i32, _p]
    L.dgo_sampler_step.argtypes = [_p, _i64, _p, _i32, _i32, _i32, _i32, _p, _p, _p, _u64, _u32,
                                   _i32, _i32, _p, _p, _p, _p, _p, _p, _p, _p, _p]
    L.dgo_selfcond_rows.argtypes = [_p, _i64, _i32, _p, _i32, _p, _p, _i32, _p]
    L.dgo_forward_noise.argtypes = [_p, _i32, _i32, _i32, _i32, _i32, _i32, _p, _u64, _p, _p]
    L.dgo_canvas_ce.argtypes = [_p, _i64, _p, _p, _i32, _i32, _i32, _i32, _i32, _p, _p, _p]
    L.dgo_tau_linear.argtypes = [_f64, _f64, _f64]
    L.dgo_tau_linear.restype = _f64
    L.dgo_entropy_accept.argtypes = [_p, _p, _i32, _i32, _i32, _f64, _u64, _u32, _p, _p, _p]
    L.dgo_adaptive_stop.argtypes = [_p, _p, _p, _i32, _i32, _f64, _p, _p]
    L.dgo_canvas_ce_backward.argtypes = [_p, _i64, _p, _p, _i32, _i32, _i32, _i32, _i32, _p, _p]
    L.dgo_selfcond_drop.argtypes = [_p, _i32, _i32, _i32, _u64, _u32, _p]
    L.dgo_gelu_tanh.argtypes = [_f64]
    L.dgo_gelu_tanh.restype = _f64
    L.dgo_ffw.argtypes = [_p, _p, _p, _i32, _i32, _i32, _p]


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _f32(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float32)


def _i32a(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.int32)


def _f64a(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float64)


SCHEDULES = {"linear": 0, "cosine": 1}


# --------------------------------------------------------------------------- primitives
def philox4x32_10(ctr, key) -> np.ndarray:
    c = np.ascontiguousarray(ctr, dtype=np.uint32)
    k = np.ascontiguousarray(key, dtype=np.uint32)
    out = np.zeros(4, dtype=np.uint32)
    lib().dgo_philox4x32_10(_ptr(c), _ptr(k), _ptr(out))
    return out


def open_uniform(w: int) -> float:
    return lib().dgo_open_uniform(int(w))


def gumbel(w: int) -> float:
    return lib().dgo_gumbel(int(w))


def kappa(schedule: str, t: float) -> float:
    return lib().dgo_kappa(SCHEDULES[schedule], float(t))


def row_stats(row, inv_tau: float = 1.0):
    r = _f32(row)
    out = np.zeros(3, dtype=np.float64)
    lib().dgo_row_stats(_ptr(r), r.size, float(inv_tau), _ptr(out[0:]), _ptr(out[1:]), _ptr(out[2:]))
    return float(out[0]), float(out[1]), float(out[2])


def row_probs(row, inv_tau: float = 1.0) -> np.ndarray:
    r = _f32(row)
    p = np.zeros(r.size, dtype=np.float64)
    lib().dgo_row_probs(_ptr(r), r.size, float(inv_tau), _ptr(p))
    return p


def argmax(row) -> int:
    r = _f32(row)
    return lib().dgo_argmax(_ptr(r), r.size)


def draw_x0(row, inv_tau: float, seed: int, step: int, row_id: int, chunk: int = GUMBEL_CHUNK):
    r = _f32(row)
    g = np.zeros(2, dtype=np.float64)
    x = lib().dgo_draw_x0(_ptr(r), r.size, float(inv_tau), seed, step, row_id, chunk,
                          _ptr(g[0:]), _ptr(g[1:]))
    return x, float(g[0]), float(g[1])


def draw_x0_flat(row, inv_tau: float, seed: int, step: int, row_id: int):
    """Plain Gumbel-max over the whole row (no chunking): (x0_hat, gap)."""
    r = _f32(row)
    g = np.zeros(1, dtype=np.float64)
    x = lib().dgo_draw_x0_flat(_ptr(r), r.size, float(inv_tau), seed, step, row_id, _ptr(g))
    return x, float(g[0])


def draw_x0_keys(row, inv_tau: float, seeds, steps, row_id: int, chunk: int = GUMBEL_CHUNK,
                 flat: bool = False) -> np.ndarray:
    """One draw of the row per (seeds[k], steps[k]) key: the two-level draw (chunk width
    `chunk`), or plain Gumbel-max with flat=True."""
    r = _f32(row)
    sd = np.ascontiguousarray(seeds, dtype=np.uint64)
    st = np.ascontiguousarray(steps, dtype=np.uint32)
    out = np.zeros(sd.size, dtype=np.int32)
    lib().dgo_draw_x0_keys(_ptr(r), r.size, float(inv_tau), _ptr(sd), _ptr(st), sd.size, row_id, chunk,
                           1 if flat else 0, _ptr(out))
    return out


def step(x_t: int, x0_hat: int, kappa_t: float, kappa_s: float, V: int, seed: int, step_idx: int,
         row_id: int):
    br = np.zeros(1, dtype=np.uint8)
    x = lib().dgo_step(x_t, x0_hat, kappa_t, kappa_s, V, seed, step_idx, row_id, _ptr(br))
    return x, int(br[0])


def step_posterior(x_t: int, x0: int, kappa_t: float, kappa_s: float, V: int) -> np.ndarray:
    p = np.zeros(V, dtype=np.float64)
    lib().dgo_step_posterior(x_t, x0, kappa_t, kappa_s, V, _ptr(p))
    return p


# --------------------------------------------------------------------------- whole kernels
def sampler_step(logits, x_t, B: int, C: int, V: int, schedule: str, t, dt, inv_tau, seed: int,
                 step_idx: int, mode: str = "sample", chunk: int = GUMBEL_CHUNK) -> dict:
    """The whole per-step sampler over B canvases of C rows (logits [B*C, ld])."""
    L = _f32(logits)
    ld = L.shape[1]
    xt = _i32a(x_t).reshape(-1)
    R = B * C
    tt, dd = _f64a(t), _f64a(dt)
    it = None if inv_tau is None else _f32(inv_tau)
    out = {k: np.zeros(R, dtype=np.int32) for k in ("x_next", "x0_hat", "argmax")}
    for k in ("max_prob", "lse", "entropy", "gap1", "gap2"):
        out[k] = np.zeros(R, dtype=np.float64)
    out["branch"] = np.zeros(R, dtype=np.uint8)
    lib().dgo_sampler_step(_ptr(L), ld, _ptr(xt), B, C, V, SCHEDULES[schedule], _ptr(tt), _ptr(dd),
                           None if it is None else _ptr(it), seed, step_idx,
                           {"sample": 0, "greedy": 1}[mode], chunk,
                           _ptr(out["x_next"]), _ptr(out["x0_hat"]), _ptr(out["argmax"]),
                           _ptr(out["max_prob"]), _ptr(out["lse"]), _ptr(out["entropy"]),
                           _ptr(out["branch"]), _ptr(out["gap1"]), _ptr(out["gap2"]))
    return out


def selfcond_rows(logits, E, rows, inv_tau_rows=None) -> np.ndarray:
    """z rows = softmax(l * inv_tau) @ E for the listed rows, in double."""
    L = _f32(logits)
    Ea = _f32(E)
    rr = _i32a(rows)
    it = None if inv_tau_rows is None else _f32(inv_tau_rows)
    V = Ea.shape[0]
    assert L.shape[1] >= V
    z = np.zeros((rr.size, Ea.shape[1]), dtype=np.float64)
    lib().dgo_selfcond_rows(_ptr(L), L.shape[1], V, _ptr(Ea), Ea.shape[1],
                            None if it is None else _ptr(it), _ptr(rr), rr.size, _ptr(z))
    return z


def forward_noise(x0, n_seq: int, P: int, K: int, C: int, V: int, schedule: str, t, seed: int):
    x = _i32a(x0)
    tt = _f64a(t)
    out = np.zeros_like(x)
    k = np.zeros(n_seq, dtype=np.int32)
    lib().dgo_forward_noise(_ptr(x), n_seq, P, K, C, V, SCHEDULES[schedule], _ptr(tt), seed,
                            _ptr(out), _ptr(k))
    return out, k


def canvas_ce(logits, x0, canvas_idx, n_seq: int, P: int, K: int, C: int, V: int):
    L = _f32(logits)
    x = _i32a(x0)
    k = _i32a(canvas_idx)
    R = n_seq * C
    loss = np.zeros(R, dtype=np.float64)
    lse = np.zeros(R, dtype=np.float64)
    seq = np.zeros(n_seq, dtype=np.float64)
    lib().dgo_canvas_ce(_ptr(L), L.shape[1], _ptr(x), _ptr(k), n_seq, P, K, C, V, _ptr(loss),
                        _ptr(seq), _ptr(lse))
    return loss, seq, lse


# --------------------------------------------------------------------------- sampler extensions
def tau_linear(t: float, tau_max: float = 0.8, tau_min: float = 0.4) -> float:
    """Linearly annealed temperature: tau(1) = tau_max, tau(0) = tau_min."""
    return lib().dgo_tau_linear(float(t), float(tau_max), float(tau_min))


def entropy_accept(H, x0_hat, B: int, C: int, V: int, eps: float, seed: int, step: int):
    """Entropy-bounded acceptance per canvas; returns (x_next, accepted, n_accepted)."""
    h = _f32(H)
    x = _i32a(x0_hat)
    out = np.zeros(B * C, dtype=np.int32)
    acc = np.zeros(B * C, dtype=np.uint8)
    n = np.zeros(B, dtype=np.int32)
    lib().dgo_entropy_accept(_ptr(h), _ptr(x), B, C, V, float(eps), seed, step, _ptr(out), _ptr(acc), _ptr(n))
    return out, acc, n


def adaptive_stop(H, argmax, argmax_prev, B: int, C: int, theta: float):
    """Adaptive-stopping flags per canvas; returns (stop, mean_entropy)."""
    h = _f32(H)
    a = _i32a(argmax)
    ap = None if argmax_prev is None else _i32a(argmax_prev)
    stop = np.zeros(B, dtype=np.uint8)
    mean = np.zeros(B, dtype=np.float64)
    lib().dgo_adaptive_stop(_ptr(h), _ptr(a), None if ap is None else _ptr(ap), B, C, float(theta), _ptr(stop),
                            _ptr(mean))
    return stop, mean


def canvas_ce_backward(logits, x0, canvas_idx, n_seq: int, P: int, K: int, C: int, V: int, g_seq=None):
    """d(sum_i loss_i of sequence b) * g_seq[b] / d logits, in double: [n_seq*C, V]."""
    L = _f32(logits)
    x = _i32a(x0)
    k = _i32a(canvas_idx)
    g = _f64a(np.ones(n_seq) if g_seq is None else g_seq)
    out = np.zeros((n_seq * C, V), dtype=np.float64)
    lib().dgo_canvas_ce_backward(_ptr(L), L.shape[1], _ptr(x), _ptr(k), n_seq, P, K, C, V, _ptr(g), _ptr(out))
    return out


def selfcond_drop(z, n_seq: int, C: int, d: int, seed: int, step: int):
    """Zero the self-conditioning rows of dropped sequences; returns (z, keep)."""
    zz = np.array(z, dtype=np.float64, copy=True, order="C")
    keep = np.zeros(n_seq, dtype=np.uint8)
    lib().dgo_selfcond_drop(_ptr(zz), n_seq, C, d, seed, step, _ptr(keep))
    return zz, keep


def gelu_tanh(x: float) -> float:
    return lib().dgo_gelu_tanh(float(x))


def ffw(z, W1, W2) -> np.ndarray:
    """Two-layer feed-forward block gelu(z W1) W2 in double: z [R, d], W1 [d, dff], W2 [dff, d]."""
    zz, a, b = _f32(z), _f32(W1), _f32(W2)
    R, d = zz.shape
    dff = a.shape[1]
    assert a.shape == (d, dff) and b.shape == (dff, d)
    out = np.zeros((R, d), dtype=np.float64)
    lib().dgo_ffw(_ptr(zz), _ptr(a), _ptr(b), R, d, dff, _ptr(out))
    return out
