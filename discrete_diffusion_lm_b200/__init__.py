"""Python binding of libdg, the B200 (sm_100a) sampler library for block-parallel
uniform-noise discrete diffusion (DiffusionGemma Technical Report, sections "Method" and
"Dataset").

The binding only marshals arguments: torch tensors supply device memory and
the current CUDA stream; every step of the computation runs in libdg's CUDA
kernels.  There is no CPU fallback: if libdg.so is missing, a tensor is not on
the GPU, or the device is not sm_100, the calls raise.

Functions carry the C ABI's names (include/dg.h):
    sampler:   dg_sampler_step, dg_sampler_selfcond_step, dg_sampler_step_eb,
               dg_entropy_accept, dg_adaptive_stop, dg_tau_linear, dg_sampler_step_noalloc
    self-conditioning input:   dg_selfcond, dg_ffw
    training:  dg_forward_noise, dg_canvas_ce, dg_canvas_ce_backward, dg_selfcond_drop
plus the workspace-size queries, dg_last_error, dg_device_error, dg_launch_count, dg_version.

Typical sampler loop over one 256-token canvas (logits from the model each step):

    import discrete_diffusion_lm_b200 as dg
    x = initial_canvas                                   # int32 [256] on the GPU
    for k in range(steps):
        t, dt = 1 - k / steps, 1 / steps
        logits = model(x, z)                             # [256, V] bf16
        out = dg.dg_sampler_selfcond_step(logits, x, E, 256, t, dt, step=k,
                                          inv_tau=dg.dg_tau_linear([t]))
        x, z = out["x_next"], out["z"]                   # next canvas, self-conditioning input

or, with entropy-bounded acceptance and adaptive stopping instead of the Step posterior:

        out = dg.dg_sampler_step_eb(logits, 256, eps=eps, theta=theta, argmax_prev=prev, step=k,
                                    inv_tau=dg.dg_tau_linear([t]))
        if out["stop"].item(): break
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
# DG_LIB=checks selects the checks library (device-side index and token-id checks, built with
# `python -m discrete_diffusion_lm_b200.build --checks`); anything else, or unset, the normal one.
LIB_PATH = os.path.join(_PKG, "libdg_checks.so" if os.environ.get("DG_LIB") == "checks" else "libdg.so")

DG_OK = 0
DG_F32, DG_BF16 = 0, 1
DG_SCHED = {"linear": 0, "cosine": 1}
DG_X0 = {"sample": 0, "greedy": 1}
DG_GUMBEL_CHUNK = 512
DG_MAX_CANVASES = 256
DG_MAX_CANVAS_ROWS = 1024
DG_MAX_VOCAB = 1 << 30


class DGError(RuntimeError):
    def __init__(self, fn: str, code: int, msg: str):
        super().__init__(f"{fn} failed with status {code}: {msg}")
        self.code = code


_lib = None
_p, _i32, _i64, _u32, _u64, _sz, _int = (ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_uint32,
                                         ctypes.c_uint64, ctypes.c_size_t, ctypes.c_int)


def lib() -> ctypes.CDLL:
    """Load libdg.so (built in-tree by discrete_diffusion_lm_b200.build)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            flag = " --checks" if LIB_PATH.endswith("_checks.so") else ""
            raise ImportError(f"{LIB_PATH} is missing: build it with `python -m discrete_diffusion_lm_b200.build{flag}`")
        L = ctypes.CDLL(LIB_PATH)
        L.dg_last_error.restype = ctypes.c_char_p
        L.dg_version.restype = ctypes.c_char_p
        L.dg_launch_count.restype = _u64
        L.dg_device_error.argtypes = [_p]
        L.dg_test_bounded_wait.argtypes = [_u32, _p]
        L.dg_test_merge_stall.argtypes = [_p, _int, _i64, _i32, _i32, _p, _p, _sz, _u32, _p]
        L.dg_test_selfcond_stall.argtypes = [_p, _int, _i64, _i32, _i32, _i32, _p, _p, _p, _int, _i32, _p, _p, _sz,
                                             _p, _i32, _u32]
        L.dg_sampler_step_workspace_size.argtypes = [_i32, _i32]
        L.dg_sampler_step_workspace_size.restype = _sz
        L.dg_sampler_step.argtypes = [_p, _int, _i64, _p, _i32, _i32, _i32, _int, _p, _p, _p, _u64, _u32, _int,
                                      _p, _p, _p, _p, _p, _p, _p, _p, _sz, _p]
        L.dg_sampler_step_noalloc.argtypes = [_p, _int, _i64, _p, _i32, _i32, _i32, _int, _p, _p, _p, _u64, _u32,
                                              _int, _p, _p, _p, _p, _p, _p, _p, _p]
        L.dg_selfcond_workspace_size.argtypes = [_i32, _i32, _i32, _int, _int, _int]
        L.dg_selfcond_workspace_size.restype = _sz
        L.dg_selfcond.argtypes = [_p, _int, _i64, _i32, _i32, _i32, _p, _p, _p, _int, _i32, _p, _p, _sz, _p]
        L.dg_forward_noise.argtypes = [_p, _i32, _i32, _i32, _i32, _i32, _int, _p, _u64, _p, _p, _p]
        L.dg_canvas_ce_workspace_size.argtypes = [_i32, _i32, _i32]
        L.dg_canvas_ce_workspace_size.restype = _sz
        L.dg_canvas_ce.argtypes = [_p, _int, _i64, _p, _p, _i32, _i32, _i32, _i32, _i32, _p, _p, _p, _p, _sz, _p]
        L.dg_tau_linear.argtypes = [_p, _i32, ctypes.c_double, ctypes.c_double, _p]
        L.dg_entropy_accept.argtypes = [_p, _p, _i32, _i32, _i32, ctypes.c_double, _u64, _u32, _p, _p, _p, _p]
        L.dg_adaptive_stop.argtypes = [_p, _p, _p, _i32, _i32, ctypes.c_double, _p, _p, _p]
        L.dg_sampler_step_eb.argtypes = [_p, _int, _i64, _i32, _i32, _i32, _p, _u64, _u32, _int, ctypes.c_double,
                                         ctypes.c_double, _p, _p, _p, _p, _p, _p, _p, _p, _p, _p, _p, _sz, _p]
        L.dg_canvas_ce_backward.argtypes = [_p, _i64, _p, _p, _p, _i32, _i32, _i32, _i32, _i32, _p, _p]
        L.dg_selfcond_drop.argtypes = [_p, _i32, _i32, _i32, _u64, _u32, _p, _p]
        L.dg_ffw_workspace_size.argtypes = [_i32, _i32, _i32]
        L.dg_ffw_workspace_size.restype = _sz
        L.dg_ffw.argtypes = [_p, _i32, _i32, _i32, _p, _p, _p, _p, _p, _sz, _p]
        L.dg_sampler_selfcond_step.argtypes = [_p, _int, _i64, _p, _i32, _i32, _i32, _int, _p, _p, _p, _u64, _u32,
                                               _int, _p, _p, _p, _p, _p, _p, _p, _p, _sz, _p, _int, _i32, _p, _p,
                                               _sz, _p]
        _lib = L
    return _lib


def dg_last_error() -> str:
    return lib().dg_last_error().decode()


def dg_version() -> str:
    return lib().dg_version().decode()


def dg_launch_count() -> int:
    return int(lib().dg_launch_count())


def dg_device_error() -> int:
    """Synchronize the device and return (and clear) the library's device error word:
    0 = no kernel reported a problem, 1 = a kernel gave up on a bounded wait."""
    code = ctypes.c_int(0)
    _check("dg_device_error", lib().dg_device_error(ctypes.byref(code)))
    return code.value


def _check(fn: str, rc: int):
    if rc != DG_OK:
        raise DGError(fn, rc, dg_last_error())


def _ptr(t: Optional[torch.Tensor]):
    """Device address of a tensor (None stays NULL).  Only CUDA tensors reach the library: a host
    address handed to a kernel would fault the device."""
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("the library takes CUDA tensors only (got a tensor on %s)" % t.device)
    return ctypes.c_void_p(t.data_ptr())


def _vec(t: Optional[torch.Tensor], name: str, dtype, n: Optional[int] = None):
    """Check a contiguous device vector argument: dtype, and at least n elements when given."""
    if t is None:
        return
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if n is not None and t.numel() < n:
        raise ValueError(f"{name} has {t.numel()} elements, {n} are needed")


def _stream(stream) -> ctypes.c_void_p:
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return DG_BF16
    if t.dtype == torch.float32:
        return DG_F32
    raise TypeError(f"unsupported dtype {t.dtype}; use torch.bfloat16 or torch.float32")


def _row_major_2d(t: torch.Tensor, name: str) -> int:
    if t.dim() != 2 or t.stride(1) != 1:
        raise ValueError(f"{name} must be a 2-D tensor with unit stride along the last dim")
    return t.stride(0)


def _host_doubles(vals: Sequence[float], n: int):
    if len(vals) != n:
        raise ValueError(f"expected {n} per-canvas values, got {len(vals)}")
    return (ctypes.c_double * n)(*[float(v) for v in vals])


def _host_floats(vals, n: int):
    if vals is None:
        return None
    if len(vals) != n:
        raise ValueError(f"expected {n} per-canvas values, got {len(vals)}")
    return (ctypes.c_float * n)(*[float(v) for v in vals])


def _expand(v, n):
    if isinstance(v, (int, float)):
        return [float(v)] * n
    return list(v)


# Workspaces are zero-filled once and reused: every successful call leaves their counters at
# zero.  The layout inside a workspace depends on the call's shape, so a cached workspace is
# zero-filled again (on the call's stream) whenever the shape it serves changes.
_WS: dict = {}


def workspace(kind: str, nbytes: int, device, layout=None, stream=None) -> torch.Tensor:
    """A cached zero-filled workspace of at least nbytes for calls of shape `layout`."""
    dev = torch.device(device)
    key = (kind, dev.type, dev.index)
    ws, last = _WS.get(key, (None, None))
    if ws is None or ws.numel() < nbytes:
        ws = torch.zeros(max(nbytes, 256), dtype=torch.uint8, device=dev)
    elif last != layout:
        with torch.cuda.stream(torch.cuda.current_stream(dev) if stream is None else stream):
            ws.zero_()
    _WS[key] = (ws, layout)
    return ws


def dg_sampler_step_workspace_size(rows: int, V: int) -> int:
    return int(lib().dg_sampler_step_workspace_size(rows, V))


def dg_selfcond_workspace_size(rows: int, V: int, d: int, logits_dtype: int, embed_dtype: int, have_lse: bool) -> int:
    return int(lib().dg_selfcond_workspace_size(rows, V, d, logits_dtype, embed_dtype, int(bool(have_lse))))


def dg_canvas_ce_workspace_size(n_seq: int, C: int, V: int) -> int:
    return int(lib().dg_canvas_ce_workspace_size(n_seq, C, V))


_STEP_OUT_DTYPES = {"x_next": torch.int32, "x0_hat": torch.int32, "argmax": torch.int32, "max_prob": torch.float32,
                    "lse": torch.float32, "entropy": torch.float32, "branch": torch.uint8}


def _check_step_vectors(x_t, out: dict, R: int):
    _vec(x_t, "x_t", torch.int32, R)
    for k, dt_ in _STEP_OUT_DTYPES.items():
        _vec(out.get(k), k, dt_, R)


def dg_sampler_step(logits: torch.Tensor, x_t: torch.Tensor, C: int, t, dt, *, V: Optional[int] = None,
                    schedule: str = "cosine", inv_tau=None, seed: int = 0, step: int = 0, mode: str = "sample",
                    out: Optional[dict] = None, ws: Optional[torch.Tensor] = None, stream=None) -> dict:
    """One sampler step over B = rows / C canvases.  Returns the dict of output tensors
    (x_next, x0_hat, argmax, max_prob, lse, entropy, branch); pass `out` to reuse buffers."""
    ld = _row_major_2d(logits, "logits")
    R = logits.shape[0]
    V = logits.shape[1] if V is None else V
    if R % C:
        raise ValueError("rows must be a multiple of C")
    B = R // C
    dev = logits.device
    if out is None:
        out = {
            "x_next": torch.empty(R, dtype=torch.int32, device=dev),
            "x0_hat": torch.empty(R, dtype=torch.int32, device=dev),
            "argmax": torch.empty(R, dtype=torch.int32, device=dev),
            "max_prob": torch.empty(R, dtype=torch.float32, device=dev),
            "lse": torch.empty(R, dtype=torch.float32, device=dev),
            "entropy": torch.empty(R, dtype=torch.float32, device=dev),
            "branch": torch.empty(R, dtype=torch.uint8, device=dev),
        }
    _check_step_vectors(x_t, out, R)
    nbytes = dg_sampler_step_workspace_size(R, V)
    if ws is None:
        ws = workspace("sampler_step", nbytes, dev, (R, V), stream)
    rc = lib().dg_sampler_step(
        _ptr(logits), _dtype_code(logits), ld, _ptr(x_t), B, C, V, DG_SCHED[schedule],
        _host_doubles(_expand(t, B), B), _host_doubles(_expand(dt, B), B),
        _host_floats(None if inv_tau is None else _expand(inv_tau, B), B),
        ctypes.c_uint64(seed), ctypes.c_uint32(step), DG_X0[mode],
        _ptr(out.get("x_next")), _ptr(out.get("x0_hat")), _ptr(out.get("argmax")), _ptr(out.get("max_prob")),
        _ptr(out.get("lse")), _ptr(out.get("entropy")), _ptr(out.get("branch")),
        _ptr(ws), ws.numel() * ws.element_size(), _stream(stream))
    _check("dg_sampler_step", rc)
    return out


def dg_sampler_selfcond_step(logits: torch.Tensor, x_t: torch.Tensor, E: torch.Tensor, C: int, t, dt, *,
                             V: Optional[int] = None, schedule: str = "cosine", inv_tau=None, seed: int = 0,
                             step: int = 0, mode: str = "sample", out: Optional[dict] = None,
                             z: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None,
                             ws_z: Optional[torch.Tensor] = None, stream=None) -> dict:
    """One sampler step and its self-conditioning input z = softmax(L) E in one call (the
    contraction starts while the logits pass finishes).  Returns the dict of dg_sampler_step's
    outputs plus "z"."""
    ld = _row_major_2d(logits, "logits")
    R = logits.shape[0]
    V = logits.shape[1] if V is None else V
    if R % C:
        raise ValueError("rows must be a multiple of C")
    B = R // C
    dev = logits.device
    d = E.shape[1]
    if out is None:
        out = {k: torch.empty(R, dtype=dt_, device=dev) for k, dt_ in
               (("x_next", torch.int32), ("x0_hat", torch.int32), ("argmax", torch.int32),
                ("max_prob", torch.float32), ("lse", torch.float32), ("entropy", torch.float32),
                ("branch", torch.uint8))}
    z = torch.empty((R, d), dtype=torch.bfloat16, device=dev) if z is None else z
    out["z"] = z
    _check_step_vectors(x_t, out, R)
    _vec(z, "z", torch.bfloat16, R * d)
    if ws is None:
        ws = workspace("sampler_step", dg_sampler_step_workspace_size(R, V), dev, (R, V), stream)
    if ws_z is None:
        nz = dg_selfcond_workspace_size(R, V, d, _dtype_code(logits), _dtype_code(E), True)
        ws_z = workspace("selfcond", nz, dev, (R, V, d, False, E.dtype), stream)
    rc = lib().dg_sampler_selfcond_step(
        _ptr(logits), _dtype_code(logits), ld, _ptr(x_t), B, C, V, DG_SCHED[schedule],
        _host_doubles(_expand(t, B), B), _host_doubles(_expand(dt, B), B),
        _host_floats(None if inv_tau is None else _expand(inv_tau, B), B),
        ctypes.c_uint64(seed), ctypes.c_uint32(step), DG_X0[mode],
        _ptr(out.get("x_next")), _ptr(out.get("x0_hat")), _ptr(out.get("argmax")), _ptr(out.get("max_prob")),
        _ptr(out["lse"]), _ptr(out.get("entropy")), _ptr(out.get("branch")),
        _ptr(ws), ws.numel() * ws.element_size(), _ptr(E), _dtype_code(E), d, _ptr(z), _ptr(ws_z),
        ws_z.numel() * ws_z.element_size(), _stream(stream))
    _check("dg_sampler_selfcond_step", rc)
    return out


DG_NOALLOC_SCRATCH_BYTES = 4 * 1024 * 1024


def dg_sampler_step_noalloc(logits: torch.Tensor, x_t: torch.Tensor, C: int, t, dt, *, V: Optional[int] = None,
                            schedule: str = "cosine", inv_tau=None, seed: int = 0, step: int = 0,
                            mode: str = "sample", out: Optional[dict] = None, stream=None) -> dict:
    """The sampler step without a caller workspace: for callers that cannot allocate device
    memory where they sample.  Scratch lives in the library's fixed device array (at most
    DG_NOALLOC_SCRATCH_BYTES); calls share it, so overlapping calls race.  Output tensors are
    the caller's (pass `out` to reuse buffers; otherwise they are created here, as for
    dg_sampler_step)."""
    ld = _row_major_2d(logits, "logits")
    R = logits.shape[0]
    V = logits.shape[1] if V is None else V
    if R % C:
        raise ValueError("rows must be a multiple of C")
    B = R // C
    dev = logits.device
    if out is None:
        out = {k: torch.empty(R, dtype=dt_, device=dev) for k, dt_ in
               (("x_next", torch.int32), ("x0_hat", torch.int32), ("argmax", torch.int32),
                ("max_prob", torch.float32), ("lse", torch.float32), ("entropy", torch.float32),
                ("branch", torch.uint8))}
    _check_step_vectors(x_t, out, R)
    rc = lib().dg_sampler_step_noalloc(
        _ptr(logits), _dtype_code(logits), ld, _ptr(x_t), B, C, V, DG_SCHED[schedule],
        _host_doubles(_expand(t, B), B), _host_doubles(_expand(dt, B), B),
        _host_floats(None if inv_tau is None else _expand(inv_tau, B), B),
        ctypes.c_uint64(seed), ctypes.c_uint32(step), DG_X0[mode],
        _ptr(out.get("x_next")), _ptr(out.get("x0_hat")), _ptr(out.get("argmax")), _ptr(out.get("max_prob")),
        _ptr(out.get("lse")), _ptr(out.get("entropy")), _ptr(out.get("branch")), _stream(stream))
    _check("dg_sampler_step_noalloc", rc)
    return out


def dg_selfcond(logits: torch.Tensor, E: torch.Tensor, C: int, *, V: Optional[int] = None, inv_tau=None,
                lse: Optional[torch.Tensor] = None, z: Optional[torch.Tensor] = None,
                ws: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """z = softmax(logits * inv_tau) @ E in bf16 (tcgen05 tensor cores)."""
    ld = _row_major_2d(logits, "logits")
    if E.dim() != 2 or not E.is_contiguous():
        raise ValueError("E must be a contiguous [V, d] tensor")
    R = logits.shape[0]
    V = E.shape[0] if V is None else V
    d = E.shape[1]
    if R % C:
        raise ValueError("rows must be a multiple of C")
    B = R // C
    dev = logits.device
    if z is None:
        z = torch.empty((R, d), dtype=torch.bfloat16, device=dev)
    _vec(z, "z", torch.bfloat16, R * d)
    _vec(lse, "lse", torch.float32, R)
    nbytes = dg_selfcond_workspace_size(R, V, d, _dtype_code(logits), _dtype_code(E), lse is not None)
    if ws is None:
        ws = workspace("selfcond", nbytes, dev, (R, V, d, lse is None, E.dtype), stream)
    rc = lib().dg_selfcond(
        _ptr(logits), _dtype_code(logits), ld, B, C, V,
        _host_floats(None if inv_tau is None else _expand(inv_tau, B), B), _ptr(lse),
        _ptr(E), _dtype_code(E), d, _ptr(z), _ptr(ws), ws.numel() * ws.element_size(), _stream(stream))
    _check("dg_selfcond", rc)
    return z


def dg_forward_noise(x0: torch.Tensor, P: int, K: int, C: int, V: int, t, *, schedule: str = "cosine",
                     seed: int = 0, x_t: Optional[torch.Tensor] = None, canvas_idx: Optional[torch.Tensor] = None,
                     stream=None):
    """Corrupt the K canvases of each sequence; returns (x_t, canvas_idx)."""
    if x0.dim() != 2 or not x0.is_contiguous() or x0.dtype != torch.int32:
        raise ValueError("x0 must be a contiguous int32 [n_seq, P + K*C] tensor")
    n_seq = x0.shape[0]
    if x_t is None:
        x_t = torch.empty_like(x0)
    if canvas_idx is None:
        canvas_idx = torch.empty(n_seq, dtype=torch.int32, device=x0.device)
    _vec(x_t, "x_t", torch.int32, x0.numel())
    _vec(canvas_idx, "canvas_idx", torch.int32, n_seq)
    rc = lib().dg_forward_noise(_ptr(x0), n_seq, P, K, C, V, DG_SCHED[schedule],
                                _host_doubles(_expand(t, n_seq), n_seq), ctypes.c_uint64(seed), _ptr(x_t),
                                _ptr(canvas_idx), _stream(stream))
    _check("dg_forward_noise", rc)
    return x_t, canvas_idx


def dg_canvas_ce(logits: torch.Tensor, x0: torch.Tensor, canvas_idx: torch.Tensor, P: int, K: int, C: int, *,
                 V: Optional[int] = None, loss_rows=None, loss_seq=None, lse_rows=None,
                 ws: Optional[torch.Tensor] = None, stream=None):
    """Cross-entropy of each sequence's chosen canvas; returns (loss_rows, loss_seq, lse_rows)."""
    ld = _row_major_2d(logits, "logits")
    R = logits.shape[0]
    V = logits.shape[1] if V is None else V
    n_seq = x0.shape[0]
    _vec(x0, "x0", torch.int32)
    _vec(canvas_idx, "canvas_idx", torch.int32, n_seq)
    if R != n_seq * C:
        raise ValueError("logits must have n_seq * C rows")
    dev = logits.device
    loss_rows = torch.empty(R, dtype=torch.float32, device=dev) if loss_rows is None else loss_rows
    loss_seq = torch.empty(n_seq, dtype=torch.float32, device=dev) if loss_seq is None else loss_seq
    lse_rows = torch.empty(R, dtype=torch.float32, device=dev) if lse_rows is None else lse_rows
    nbytes = dg_canvas_ce_workspace_size(n_seq, C, V)
    if ws is None:
        ws = workspace("canvas_ce", nbytes, dev, (n_seq, C, V), stream)
    rc = lib().dg_canvas_ce(_ptr(logits), _dtype_code(logits), ld, _ptr(x0), _ptr(canvas_idx), n_seq, P, K, C, V,
                            _ptr(loss_rows), _ptr(loss_seq), _ptr(lse_rows), _ptr(ws),
                            ws.numel() * ws.element_size(), _stream(stream))
    _check("dg_canvas_ce", rc)
    return loss_rows, loss_seq, lse_rows


# ------------------------------------------------------------------------------ sampler extensions
def dg_tau_linear(t, tau_max: float = 0.8, tau_min: float = 0.4) -> list:
    """Per-canvas inverse temperatures of the linear schedule tau(1) = tau_max, tau(0) = tau_min."""
    tt = _expand(t, 1) if isinstance(t, (int, float)) else list(t)
    n = len(tt)
    out = (ctypes.c_float * n)()
    rc = lib().dg_tau_linear(_host_doubles(tt, n), n, float(tau_max), float(tau_min), out)
    _check("dg_tau_linear", rc)
    return [float(v) for v in out]


def dg_entropy_accept(entropy: torch.Tensor, x0_hat: torch.Tensor, C: int, V: int, eps: float, *, seed: int = 0,
                      step: int = 0, out: Optional[dict] = None, stream=None) -> dict:
    """Entropy-bounded acceptance per canvas; returns {x_next, accepted, n_accepted}."""
    R = entropy.numel()
    if R % C:
        raise ValueError("rows must be a multiple of C")
    B = R // C
    dev = entropy.device
    _vec(entropy, "entropy", torch.float32)
    _vec(x0_hat, "x0_hat", torch.int32, R)
    if out is None:
        out = {"x_next": torch.empty(R, dtype=torch.int32, device=dev),
               "accepted": torch.empty(R, dtype=torch.uint8, device=dev),
               "n_accepted": torch.empty(B, dtype=torch.int32, device=dev)}
    rc = lib().dg_entropy_accept(_ptr(entropy), _ptr(x0_hat), B, C, V, float(eps), ctypes.c_uint64(seed),
                                 ctypes.c_uint32(step), _ptr(out["x_next"]), _ptr(out.get("accepted")),
                                 _ptr(out.get("n_accepted")), _stream(stream))
    _check("dg_entropy_accept", rc)
    return out


def dg_adaptive_stop(entropy: torch.Tensor, argmax: torch.Tensor, argmax_prev: Optional[torch.Tensor], C: int,
                     theta: float, *, stream=None):
    """Adaptive-stopping flags per canvas; returns (stop uint8 [B], mean_entropy float [B])."""
    R = entropy.numel()
    if R % C:
        raise ValueError("rows must be a multiple of C")
    B = R // C
    _vec(entropy, "entropy", torch.float32)
    _vec(argmax, "argmax", torch.int32, R)
    _vec(argmax_prev, "argmax_prev", torch.int32, R)
    stop = torch.empty(B, dtype=torch.uint8, device=entropy.device)
    mean = torch.empty(B, dtype=torch.float32, device=entropy.device)
    rc = lib().dg_adaptive_stop(_ptr(entropy), _ptr(argmax), _ptr(argmax_prev), B, C, float(theta), _ptr(stop),
                                _ptr(mean), _stream(stream))
    _check("dg_adaptive_stop", rc)
    return stop, mean


def dg_sampler_step_eb(logits: torch.Tensor, C: int, *, eps: float, theta: float = 0.0,
                       argmax_prev: Optional[torch.Tensor] = None, V: Optional[int] = None, inv_tau=None,
                       seed: int = 0, step: int = 0, mode: str = "sample", out: Optional[dict] = None,
                       ws: Optional[torch.Tensor] = None, stream=None) -> dict:
    """Entropy-bounded sampler step: statistics and x0_hat draw, then per-canvas acceptance with
    uniform re-noising and the adaptive-stopping flag.  Returns the dict of outputs (x_next,
    x0_hat, argmax, max_prob, lse, entropy, accepted, stop, mean_entropy)."""
    ld = _row_major_2d(logits, "logits")
    R = logits.shape[0]
    V = logits.shape[1] if V is None else V
    if R % C:
        raise ValueError("rows must be a multiple of C")
    B = R // C
    dev = logits.device
    if out is None:
        out = {k: torch.empty(R, dtype=dt, device=dev) for k, dt in
               (("x_next", torch.int32), ("x0_hat", torch.int32), ("argmax", torch.int32),
                ("max_prob", torch.float32), ("lse", torch.float32), ("entropy", torch.float32),
                ("accepted", torch.uint8))}
        out["stop"] = torch.empty(B, dtype=torch.uint8, device=dev)
        out["mean_entropy"] = torch.empty(B, dtype=torch.float32, device=dev)
    _vec(argmax_prev, "argmax_prev", torch.int32, R)
    nbytes = dg_sampler_step_workspace_size(R, V)
    if ws is None:
        ws = workspace("sampler_step", nbytes, dev, (R, V), stream)
    rc = lib().dg_sampler_step_eb(
        _ptr(logits), _dtype_code(logits), ld, B, C, V, _host_floats(None if inv_tau is None else _expand(inv_tau, B), B),
        ctypes.c_uint64(seed), ctypes.c_uint32(step), DG_X0[mode], float(eps), float(theta), _ptr(argmax_prev),
        _ptr(out["x_next"]), _ptr(out["x0_hat"]), _ptr(out.get("argmax")), _ptr(out.get("max_prob")),
        _ptr(out.get("lse")), _ptr(out["entropy"]), _ptr(out.get("accepted")), _ptr(out.get("stop")),
        _ptr(out.get("mean_entropy")), _ptr(ws), ws.numel() * ws.element_size(), _stream(stream))
    _check("dg_sampler_step_eb", rc)
    return out


def dg_canvas_ce_backward(logits: torch.Tensor, lse_rows: torch.Tensor, x0: torch.Tensor, canvas_idx: torch.Tensor,
                          P: int, K: int, C: int, *, V: Optional[int] = None, g_seq: Optional[torch.Tensor] = None,
                          stream=None) -> torch.Tensor:
    """Overwrite bf16 logits with d(sum of each sequence's canvas CE) / d logits (times g_seq)."""
    ld = _row_major_2d(logits, "logits")
    if logits.dtype != torch.bfloat16:
        raise TypeError("the in-place CE backward works on bf16 logits")
    V = logits.shape[1] if V is None else V
    n_seq = x0.shape[0]
    _vec(lse_rows, "lse_rows", torch.float32, logits.shape[0])
    _vec(x0, "x0", torch.int32)
    _vec(canvas_idx, "canvas_idx", torch.int32, n_seq)
    _vec(g_seq, "g_seq", torch.float32, n_seq)
    rc = lib().dg_canvas_ce_backward(_ptr(logits), ld, _ptr(lse_rows), _ptr(x0), _ptr(canvas_idx), n_seq, P, K, C, V,
                                     _ptr(g_seq), _stream(stream))
    _check("dg_canvas_ce_backward", rc)
    return logits


def dg_selfcond_drop(z: torch.Tensor, C: int, *, seed: int = 0, step: int = 0,
                     keep: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Zero, in place, the bf16 self-conditioning rows of sequences whose fair coin drops them;
    returns keep (uint8 [n_seq])."""
    if z.dtype != torch.bfloat16 or not z.is_contiguous():
        raise TypeError("z must be a contiguous bf16 tensor [n_seq*C, d]")
    R, d = z.shape
    if R % C:
        raise ValueError("rows must be a multiple of C")
    n_seq = R // C
    keep = torch.empty(n_seq, dtype=torch.uint8, device=z.device) if keep is None else keep
    rc = lib().dg_selfcond_drop(_ptr(z), n_seq, C, d, ctypes.c_uint64(seed), ctypes.c_uint32(step), _ptr(keep),
                                _stream(stream))
    _check("dg_selfcond_drop", rc)
    return keep


def dg_ffw(z: torch.Tensor, W1: torch.Tensor, W2: torch.Tensor, *, hidden: Optional[torch.Tensor] = None,
           out: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None, stream=None):
    """Two-layer feed-forward block gelu(z W1) W2 on the tensor cores (bf16 in and out).
    Returns (out [R, d], hidden [R, d_ff])."""
    for t, n in ((z, "z"), (W1, "W1"), (W2, "W2")):
        if t.dtype != torch.bfloat16 or not t.is_contiguous():
            raise TypeError(f"{n} must be a contiguous bf16 tensor")
    R, d = z.shape
    dff = W1.shape[1]
    if W1.shape != (d, dff) or W2.shape != (dff, d):
        raise ValueError("W1 must be [d, d_ff] and W2 [d_ff, d]")
    dev = z.device
    hidden = torch.empty(R, dff, dtype=torch.bfloat16, device=dev) if hidden is None else hidden
    out = torch.empty(R, d, dtype=torch.bfloat16, device=dev) if out is None else out
    nbytes = int(lib().dg_ffw_workspace_size(R, d, dff))
    if ws is None:
        ws = workspace("ffw", nbytes, dev, (R, d, dff), stream)
    rc = lib().dg_ffw(_ptr(z), R, d, dff, _ptr(W1), _ptr(W2), _ptr(hidden), _ptr(out), _ptr(ws),
                      ws.numel() * ws.element_size(), _stream(stream))
    _check("dg_ffw", rc)
    return out, hidden
