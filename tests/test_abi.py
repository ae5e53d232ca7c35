"""CPU checks of the C ABI: the library builds for sm_100a, loads, exports every function
include/*.h declares (dg.h, the sampler's interface, and dg_test.h, its failure-detection test
hooks), and rejects bad arguments with a status and a message before any launch (these calls
never reach a device, so they are safe with or without a GPU)."""
import ctypes
import os
import re

import pytest
import torch

import discrete_diffusion_lm_b200 as dg
from discrete_diffusion_lm_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "dg.h")
HEADERS = [os.path.join(ROOT, "include", h) for h in sorted(os.listdir(os.path.join(ROOT, "include"))) if h.endswith(".h")]

FAKE = 1 << 20  # an aligned non-null address that is never dereferenced (calls fail validation first)


@pytest.fixture(scope="module")
def L():
    build.build()
    return dg.lib()


def declared_functions(path=None):
    names = set()
    for h in ([path] if path else HEADERS):
        text = re.sub(r"/\*.*?\*/", "", open(h).read(), flags=re.S)
        names |= set(re.findall(r"\b(dg_[a-z0-9_]+)\s*\(", text))
    return sorted(names)


def test_exports_every_declared_symbol(L):
    names = declared_functions()
    assert {"dg_sampler_step", "dg_selfcond", "dg_forward_noise", "dg_canvas_ce"} <= set(names)
    assert {"dg_test_bounded_wait", "dg_test_merge_stall", "dg_test_selfcond_stall"} <= set(names)
    for n in names:
        assert hasattr(L, n), f"{n} declared in include/ but not exported"
    # the sampler's interface header declares no test hook
    assert not [n for n in declared_functions(HEADER) if n.startswith("dg_test_")]


def test_version_and_launch_count(L):
    assert dg.dg_version().startswith("dg ")
    assert dg.dg_launch_count() >= 0


def _step(L, **kw):
    a = dict(logits=FAKE, dtype=1, ld=1024, x_t=FAKE, B=1, C=16, V=1024, sched=0, t=[0.5], dt=[0.1],
             inv_tau=None, seed=0, step=0, mode=0, x_next=FAKE, ws=FAKE, ws_bytes=1 << 30)
    a.update(kw)
    B = a["B"]
    t = (ctypes.c_double * max(B, 1))(*(a["t"] * max(B, 1))[:max(B, 1)]) if a["t"] is not None else None
    dt = (ctypes.c_double * max(B, 1))(*(a["dt"] * max(B, 1))[:max(B, 1)]) if a["dt"] is not None else None
    it = None if a["inv_tau"] is None else (ctypes.c_float * max(B, 1))(*([a["inv_tau"]] * max(B, 1)))
    rc = L.dg_sampler_step(a["logits"], a["dtype"], a["ld"], a["x_t"], B, a["C"], a["V"], a["sched"], t, dt, it,
                           ctypes.c_uint64(a["seed"]), ctypes.c_uint32(a["step"]), a["mode"], a["x_next"], None,
                           None, None, None, None, None, a["ws"], a["ws_bytes"], None)
    return rc, dg.dg_last_error()


@pytest.mark.parametrize("kw,code,frag", [
    (dict(logits=None), 1, "logits is NULL"),
    (dict(dtype=7), 1, "dtype"),
    (dict(V=0), 1, "V = 0"),
    (dict(V=(1 << 30) + 8, ld=(1 << 30) + 8), 1, "DG_MAX_VOCAB"),
    (dict(ld=1000), 1, "smaller than V"),
    (dict(logits=FAKE + 2), 2, "16-byte"),
    (dict(ld=1028, V=1025), 2, "multiple of 16"),
    (dict(B=0), 1, "B = 0"),
    (dict(B=300), 1, "B = 300"),
    (dict(C=0), 1, "C = 0"),
    (dict(x_next=None), 1, "required"),
    (dict(t=None), 1, "required"),
    (dict(sched=5), 1, "schedule"),
    (dict(mode=3), 1, "x0_mode"),
    (dict(ws=None), 3, "workspace"),
    (dict(ws_bytes=16), 3, "workspace"),
    (dict(t=[1.5]), 1, "outside [0, 1]"),
    (dict(t=[float("nan")]), 1, "outside [0, 1]"),
    (dict(dt=[-0.1]), 1, "dt[0]"),
    (dict(inv_tau=0.0), 1, "inv_tau"),
    (dict(inv_tau=float("inf")), 1, "inv_tau"),
])
def test_sampler_step_rejects(L, kw, code, frag):
    rc, msg = _step(L, **kw)
    assert rc == code, msg
    assert frag in msg


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device path")
def test_valid_call_without_device_reports_cuda_error(L):
    rc, msg = _step(L)
    assert rc in (4, 5), msg  # DG_ERR_CUDA (no device) or DG_ERR_UNSUPPORTED
    assert msg


def test_forward_noise_rejects(L):
    t = (ctypes.c_double * 2)(0.5, 0.5)
    f = L.dg_forward_noise
    assert f(FAKE, 0, 0, 1, 4, 10, 1, t, 0, FAKE + 64, None, None) == 1      # n_seq = 0
    assert f(FAKE, 2, -1, 1, 4, 10, 1, t, 0, FAKE + 64, None, None) == 1     # P < 0
    assert f(FAKE, 2, 0, 1, 4, 10, 7, t, 0, FAKE + 64, None, None) == 1      # schedule
    assert f(FAKE, 2, 0, 1, 4, 10, 1, t, 0, None, None, None) == 1           # x_t missing
    assert f(FAKE, 2, 0, 1, 4, 10, 1, t, 0, FAKE, None, None) == 1           # x_t aliases x0
    bad_t = (ctypes.c_double * 2)(0.5, 2.0)
    assert f(FAKE, 2, 0, 1, 4, 10, 1, bad_t, 0, FAKE + 64, None, None) == 1  # t outside [0, 1]
    assert "t[1]" in dg.dg_last_error()


def test_selfcond_rejects(L):
    it = None
    f = L.dg_selfcond
    assert f(FAKE, 1, 1024, 1, 16, 1024, it, None, FAKE, 1, 100, FAKE, FAKE, 1 << 30, None) == 1  # d % 64
    assert f(FAKE, 1, 1024, 1, 16, 1024, it, None, None, 1, 64, FAKE, FAKE, 1 << 30, None) == 1
    assert f(FAKE, 1, 1024, 1, 16, 1024, it, None, FAKE + 8, 1, 64, FAKE, FAKE, 1 << 30, None) == 2
    assert f(FAKE, 1, 1024, 1, 16, 1024, it, None, FAKE, 1, 64, FAKE, FAKE, 8, None) == 3
    assert f(FAKE, 1, 1024, 1, 16, 1024, it, None, FAKE, 9, 64, FAKE, FAKE, 1 << 30, None) == 1


def test_canvas_ce_rejects(L):
    f = L.dg_canvas_ce
    assert f(FAKE, 1, 1024, FAKE, FAKE, 2, 4, 2, 8, 1024, None, None, None, FAKE, 1 << 30, None) == 1
    assert f(FAKE, 1, 1024, FAKE, FAKE, 2, 4, 0, 8, 1024, FAKE, None, None, FAKE, 1 << 30, None) == 1
    assert f(FAKE, 1, 1024, FAKE, FAKE, 2, 4, 2, 8, 1024, FAKE, None, None, FAKE, 4, None) == 3


def test_workspace_queries(L):
    assert dg.dg_sampler_step_workspace_size(256, 262144) >= 256 * 128 * 16
    assert dg.dg_sampler_step_workspace_size(0, 5) == 0
    assert dg.dg_canvas_ce_workspace_size(8, 256, 262144) >= 2048 * 128 * 16
    assert dg.dg_selfcond_workspace_size(256, 262144, 2048, 1, 1, True) >= 0
    assert dg.dg_selfcond_workspace_size(256, 262144, 2048, 1, 0, True) >= 262144 * 2048 * 2


def test_sampler_extensions_reject(L):
    ea = L.dg_entropy_accept
    assert ea(None, FAKE, 1, 16, 100, ctypes.c_double(1.0), 0, 0, FAKE, None, None, None) == 1
    assert ea(FAKE, FAKE, 1, 16, 100, ctypes.c_double(1.0), 0, 0, None, None, None, None) == 1
    assert ea(FAKE, FAKE, 1, 1025, 100, ctypes.c_double(1.0), 0, 0, FAKE, None, None, None) == 5  # C > max
    assert ea(FAKE, FAKE, 0, 16, 100, ctypes.c_double(1.0), 0, 0, FAKE, None, None, None) == 1
    assert ea(FAKE, FAKE, 1, 16, 100, ctypes.c_double(float("nan")), 0, 0, FAKE, None, None, None) == 1
    st = L.dg_adaptive_stop
    assert st(FAKE, FAKE, None, 1, 16, ctypes.c_double(0.5), None, None, None) == 1  # no output
    assert st(FAKE, None, None, 1, 16, ctypes.c_double(0.5), FAKE, None, None) == 1
    eb = L.dg_sampler_step_eb
    args = [FAKE, 1, 1024, 1, 16, 1024, None, 0, 0, 0, ctypes.c_double(1.0), ctypes.c_double(0.5), None,
            FAKE, FAKE, None, None, None, FAKE, None, FAKE, None, FAKE, 1 << 30, None]
    assert eb(*args) == 1  # stop requested without argmax
    a2 = list(args)
    a2[20] = None
    a2[13] = None
    assert eb(*a2) == 1  # x_next missing
    bw = L.dg_canvas_ce_backward
    assert bw(FAKE, 1028, FAKE, FAKE, FAKE, 2, 4, 2, 8, 1028, None, None) == 2  # V not a multiple of 8
    assert bw(FAKE, 1024, None, FAKE, FAKE, 2, 4, 2, 8, 1024, None, None) == 1
    dr = L.dg_selfcond_drop
    assert dr(FAKE + 8, 2, 4, 8, 0, 0, None, None) == 2
    assert dr(FAKE, 2, 3, 3, 0, 0, None, None) == 2  # C*d not a multiple of 8


def test_tau_linear_host_matches_oracle(L):
    from oracle import oracle as O
    ts = [0.0, 0.1, 0.5, 0.73, 1.0, -0.5, 1.5]
    got = dg.dg_tau_linear(ts)
    for t, g in zip(ts, got):
        assert g == pytest.approx(1.0 / O.tau_linear(t), rel=1e-7)
    out = (ctypes.c_float * 1)()
    assert L.dg_tau_linear((ctypes.c_double * 1)(0.5), 1, ctypes.c_double(0.8), ctypes.c_double(0.0), out) == 1


def test_ffw_rejects(L):
    f = L.dg_ffw
    ws = L.dg_ffw_workspace_size
    ws.restype = ctypes.c_size_t
    assert ws(256, 2048, 8192) > 0 and ws(0, 64, 64) == 0
    assert f(FAKE, 16, 100, 256, FAKE, FAKE, FAKE + 4096, FAKE + 8192, FAKE, 1 << 30, None) == 1  # d % 64
    assert f(FAKE, 16, 64, 256, None, FAKE, FAKE + 4096, FAKE + 8192, FAKE, 1 << 30, None) == 1
    assert f(FAKE, 16, 64, 256, FAKE + 8, FAKE, FAKE + 4096, FAKE + 8192, FAKE, 1 << 30, None) == 2
    assert f(FAKE, 16, 64, 256, FAKE, FAKE, FAKE, FAKE + 8192, FAKE, 1 << 30, None) == 1  # hidden aliases z_in
    assert f(FAKE, 256, 2048, 8192, FAKE, FAKE, FAKE + 4096, FAKE + 8192, FAKE, 8, None) == 3  # workspace


def test_binding_rejects_host_and_mistyped_tensors(L):
    # host tensors never reach the library; wrong dtypes are refused before any call
    logits = torch.zeros(16, 1024, dtype=torch.bfloat16)
    x_t = torch.zeros(16, dtype=torch.int32)
    with pytest.raises(ValueError, match="CUDA tensors only"):
        dg.dg_sampler_step(logits, x_t, 16, 0.5, 0.1, ws=torch.zeros(1))
    with pytest.raises(TypeError, match="x_t must be torch.int32"):
        dg.dg_sampler_step(logits, x_t.long(), 16, 0.5, 0.1)
    with pytest.raises(TypeError, match="entropy must be torch.float32"):
        dg.dg_entropy_accept(torch.zeros(16, dtype=torch.float64), x_t, 16, 1024, 1.0)
    with pytest.raises(TypeError, match="argmax_prev must be torch.int32"):
        dg.dg_adaptive_stop(torch.zeros(16), x_t, x_t.long(), 16, 0.5)


def test_noalloc_binding_checks_vectors_before_any_call(L):
    # the allocation-free step takes the same vector checks as dg_sampler_step: a mistyped or short
    # canvas, or a caller output buffer that is too short, is refused before the library is called
    logits = torch.zeros(16, 1024, dtype=torch.bfloat16)
    x_t = torch.zeros(16, dtype=torch.int32)
    with pytest.raises(TypeError, match="x_t must be torch.int32"):
        dg.dg_sampler_step_noalloc(logits, x_t.long(), 16, 0.5, 0.1)
    with pytest.raises(ValueError, match="x_t has 8 elements, 16 are needed"):
        dg.dg_sampler_step_noalloc(logits, x_t[:8], 16, 0.5, 0.1)
    out = {"x_next": torch.zeros(8, dtype=torch.int32)}
    with pytest.raises(ValueError, match="x_next has 8 elements, 16 are needed"):
        dg.dg_sampler_step_noalloc(logits, x_t, 16, 0.5, 0.1, out=out)
    with pytest.raises(TypeError, match="lse must be torch.float32"):
        dg.dg_sampler_step_noalloc(logits, x_t, 16, 0.5, 0.1, out={"lse": torch.zeros(16, dtype=torch.float64)})


def _int_expr(src: str) -> int:
    """Value of a #define body made of integer literals, *, << and parentheses."""
    import ast
    import operator
    ops = {ast.Mult: operator.mul, ast.LShift: operator.lshift}

    def ev(n):
        if isinstance(n, ast.Constant) and isinstance(n.value, int):
            return n.value
        if isinstance(n, ast.BinOp) and type(n.op) in ops:
            return ops[type(n.op)](ev(n.left), ev(n.right))
        raise ValueError(src)
    return ev(ast.parse(src.strip(), mode="eval").body)


def test_binding_constants_match_the_header():
    text = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    defines = {name: body for name, body in re.findall(r"#define\s+(DG_[A-Z_]+)[ \t]+([^\n]+)", text)}
    for name in ("DG_GUMBEL_CHUNK", "DG_MAX_CANVASES", "DG_MAX_CANVAS_ROWS", "DG_MAX_VOCAB",
                 "DG_NOALLOC_SCRATCH_BYTES"):
        assert getattr(dg, name) == _int_expr(defines[name]), name


def test_checks_library_builds_and_exports_the_same_symbols():
    # the checks build (DG_CHECKS=1): same sources and entry points, device-side checks compiled in
    path = build.build(checks=True)
    assert path.endswith("libdg_checks.so") and os.path.exists(path)
    C = ctypes.CDLL(path)
    for n in declared_functions():
        assert hasattr(C, n), n
    C.dg_version.restype = ctypes.c_char_p
    assert C.dg_version() == dg.lib().dg_version()
