"""ctypes binding of librope_attn.so (see include/rope_attn.h).

Argument marshalling only: every step of the path runs in the library's CUDA
kernels.  PyTorch provides device memory (outputs and workspace) and the
current CUDA stream.  There is no fallback: if the library is missing or a
call fails, a RuntimeError is raised.
"""
import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "librope_attn.so")

RA_F32, RA_BF16 = 0, 1
_DTYPE = {torch.float32: RA_F32, torch.bfloat16: RA_BF16}
STATUS = {0: "RA_OK", 1: "RA_ERR_INVALID_ARG", 2: "RA_ERR_UNSUPPORTED", 3: "RA_ERR_WORKSPACE",
          4: "RA_ERR_CUDA", 5: "RA_ERR_TIMEOUT", 6: "RA_ERR_RANGE"}


class RaProblem(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int64), ("H", ctypes.c_int64), ("n", ctypes.c_int64),
                ("d", ctypes.c_int64), ("dtype", ctypes.c_int32), ("causal", ctypes.c_int32),
                ("base", ctypes.c_double), ("fixed_bands", ctypes.c_int32),
                ("reserved", ctypes.c_int32)]


class RaAdam(ctypes.Structure):
    _fields_ = [("lr", ctypes.c_float), ("beta1", ctypes.c_float), ("beta2", ctypes.c_float),
                ("eps", ctypes.c_float), ("clip_norm", ctypes.c_float), ("step", ctypes.c_int32)]


class RopeAttnError(RuntimeError):
    def __init__(self, fn, code):
        self.code = code
        super().__init__(f"{fn} returned {STATUS.get(code, code)}: "
                         f"{lib().rope_attn_status_string(code).decode()}")


_lib = None


def lib():
    """Load librope_attn.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: run python -m rope_attention_fwd_b200.build")
        L = ctypes.CDLL(LIB_PATH)
        P, vp, sz = ctypes.POINTER(RaProblem), ctypes.c_void_p, ctypes.c_size_t
        L.rope_attn_workspace_bytes.argtypes = [P]
        L.rope_attn_workspace_bytes.restype = sz
        L.rope_attn_fwd_workspace_bytes.argtypes = [P]
        L.rope_attn_fwd_workspace_bytes.restype = sz
        L.rope_attn_fwd.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        L.rope_attn_fwd.restype = ctypes.c_int
        L.rope_attn_loss.argtypes = [P, vp, vp, vp, vp, vp, sz, vp]
        L.rope_attn_loss.restype = ctypes.c_int
        L.rope_attn_bwd.argtypes = [P] + [vp] * 12 + [sz, vp]
        L.rope_attn_bwd.restype = ctypes.c_int
        L.rope_attn_bwd_saved.argtypes = [P] + [vp] * 10 + [sz, vp]
        L.rope_attn_bwd_saved.restype = ctypes.c_int
        L.rope_attn_alpha_adam.argtypes = [ctypes.POINTER(RaAdam), ctypes.c_int64, vp, vp, vp, vp,
                                           vp]
        L.rope_attn_alpha_adam.restype = ctypes.c_int
        L.rope_attn_proj_fwd.argtypes = [P, ctypes.c_int64] + [vp] * 8 + [sz, vp]
        L.rope_attn_proj_fwd.restype = ctypes.c_int
        L.rope_attn_proj_bwd.argtypes = [P, ctypes.c_int64] + [vp] * 12 + [sz, vp]
        L.rope_attn_proj_bwd.restype = ctypes.c_int
        L.rope_attn_proj_workspace_bytes.argtypes = [P]
        L.rope_attn_proj_workspace_bytes.restype = sz
        L.rope_attn_spectrum_workspace_bytes.argtypes = [P]
        L.rope_attn_spectrum_workspace_bytes.restype = sz
        L.rope_attn_spectrum.argtypes = [P] + [vp] * 10 + [sz, vp]
        L.rope_attn_spectrum.restype = ctypes.c_int
        L.rope_attn_fwd_noalloc.argtypes = [P, vp, vp, vp, vp, vp, vp, vp]
        L.rope_attn_fwd_noalloc.restype = ctypes.c_int
        L.rope_attn_noalloc_status.argtypes = [vp, ctypes.POINTER(ctypes.c_int32)]
        L.rope_attn_noalloc_status.restype = ctypes.c_int
        L.rope_attn_device_status.argtypes = [vp, sz, vp, ctypes.POINTER(ctypes.c_int32)]
        L.rope_attn_device_status.restype = ctypes.c_int
        L.rope_attn_status_string.argtypes = [ctypes.c_int]
        L.rope_attn_status_string.restype = ctypes.c_char_p
        L.rope_attn_timing_enable.argtypes = [ctypes.c_int]
        L.rope_attn_timing_enable.restype = None
        L.rope_attn_timing_read.argtypes = [ctypes.POINTER(ctypes.c_int32),
                                            ctypes.POINTER(ctypes.c_double), ctypes.c_int]
        L.rope_attn_timing_read.restype = ctypes.c_int
        L.rope_attn_kernel_name.argtypes = [ctypes.c_int]
        L.rope_attn_kernel_name.restype = ctypes.c_char_p
        _lib = L
    return _lib


def problem(B, H, n, d, dtype, causal, base, fixed_bands=0):
    """fixed_bands: the slowest bands left unrotated (partial RoPE; 0 = all rotate)."""
    if isinstance(dtype, torch.dtype):
        dtype = _DTYPE[dtype]
    return RaProblem(int(B), int(H), int(n), int(d), int(dtype), int(bool(causal)), float(base),
                     int(fixed_bands), 0)


def _problem_of(q, causal, base, fixed_bands=0):
    B, H, n, d = q.shape
    return problem(B, H, n, d, q.dtype, causal, base, fixed_bands)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def _stream(device):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _check(fn, code):
    if code != 0:
        raise RopeAttnError(fn, code)


def _expect(fn, device, *args):
    """The C ABI takes raw pointers to dense row-major buffers on one device: every tensor
    argument (name, tensor, element count or None) must be contiguous, on `device` and,
    where a count is given, hold exactly that many elements."""
    for name, t, count in args:
        if t is None:
            continue
        if t.device != device:
            raise ValueError(f"{fn}: {name} is on {t.device}, expected {device}")
        if not t.is_contiguous():
            raise ValueError(f"{fn}: {name} is not contiguous")
        if count is not None and t.numel() != count:
            raise ValueError(f"{fn}: {name} has {t.numel()} elements, expected {count}")


def rope_attn_workspace_bytes(prob):
    return int(lib().rope_attn_workspace_bytes(ctypes.byref(prob)))


def rope_attn_proj_workspace_bytes(prob):
    return int(lib().rope_attn_proj_workspace_bytes(ctypes.byref(prob)))


def rope_attn_spectrum_workspace_bytes(prob):
    return int(lib().rope_attn_spectrum_workspace_bytes(ctypes.byref(prob)))


def workspace(prob, device):
    """A fresh device workspace for `prob` (uint8 tensor)."""
    nbytes = rope_attn_workspace_bytes(prob)
    if nbytes == 0:
        raise RopeAttnError("rope_attn_workspace_bytes", 1)
    return torch.empty(nbytes, dtype=torch.uint8, device=device)


def rope_attn_fwd(q, k, v, alpha, base, causal, ws=None, o=None, lse=None, fixed_bands=0):
    """(o, lse) = softmax(Q~ K~^T / sqrt(d)) V and its row log-sum-exp."""
    prob = _problem_of(q, causal, base, fixed_bands)
    B, H, n, d = q.shape
    if ws is None:
        ws = workspace(prob, q.device)
    o = torch.empty_like(q) if o is None else o
    lse = torch.empty((B, H, n), dtype=torch.float32, device=q.device) if lse is None else lse
    N = q.numel()
    _expect("rope_attn_fwd", q.device, ("q", q, None), ("k", k, N), ("v", v, N),
            ("alpha", alpha, d // 2), ("o", o, N), ("lse", lse, B * H * n), ("ws", ws, None))
    _check("rope_attn_fwd", lib().rope_attn_fwd(
        ctypes.byref(prob), _ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(o), _ptr(lse),
        _ptr(ws), ws.numel(), _stream(q.device)))
    return o, lse


def rope_attn_fwd_noalloc(q, k, v, alpha, base, causal, o=None, lse=None, fixed_bands=0):
    """rope_attn_fwd without a workspace: scratch comes from the library's static
    RA_NOALLOC_SCRATCH_BYTES device array (problems that need more are rejected)."""
    prob = _problem_of(q, causal, base, fixed_bands)
    B, H, n, d = q.shape
    o = torch.empty_like(q) if o is None else o
    lse = torch.empty((B, H, n), dtype=torch.float32, device=q.device) if lse is None else lse
    N = q.numel()
    _expect("rope_attn_fwd_noalloc", q.device, ("q", q, None), ("k", k, N), ("v", v, N),
            ("alpha", alpha, d // 2), ("o", o, N), ("lse", lse, B * H * n))
    # the library uses the static array of the CURRENT device: make it q's
    with torch.cuda.device(q.device):
        _check("rope_attn_fwd_noalloc", lib().rope_attn_fwd_noalloc(
            ctypes.byref(prob), _ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(o), _ptr(lse),
            _stream(q.device)))
    return o, lse


def rope_attn_noalloc_status(device):
    """Synchronise the device's current stream and return (status code, [kernel, site,
    block]) from the static array's error word (read and cleared)."""
    device = torch.device(device)
    info = (ctypes.c_int32 * 3)()
    with torch.cuda.device(device):
        code = lib().rope_attn_noalloc_status(_stream(device), info)
    return code, list(info)


def rope_attn_loss(o, e, ws=None, L=None, dO=None, causal=False, base=10000.0):
    """(L, dO): L = 1/2 ||o - e||^2 (fp32 scalar tensor on device), dO = o - e."""
    prob = _problem_of(o, causal, base)
    if ws is None:
        ws = workspace(prob, o.device)
    L = torch.empty((), dtype=torch.float32, device=o.device) if L is None else L
    dO = torch.empty_like(o) if dO is None else dO
    N = o.numel()
    _expect("rope_attn_loss", o.device, ("o", o, None), ("e", e, N), ("L", L, 1), ("dO", dO, N),
            ("ws", ws, None))
    _check("rope_attn_loss", lib().rope_attn_loss(
        ctypes.byref(prob), _ptr(o), _ptr(e), _ptr(L), _ptr(dO), _ptr(ws), ws.numel(),
        _stream(o.device)))
    return L, dO


def rope_attn_bwd(q, k, v, o, lse, dO, alpha, base, causal, ws=None, dq=None, dk=None, dv=None,
                  dalpha=None, fixed_bands=0, frozen_alpha=False):
    """(dq, dk, dv, dalpha) of L for upstream gradient dO.  frozen_alpha: the frequencies
    are not trained; no dalpha is computed and None is returned in its place."""
    prob = _problem_of(q, causal, base, fixed_bands)
    if ws is None:
        ws = workspace(prob, q.device)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    if frozen_alpha:
        dalpha = None
    elif dalpha is None:
        dalpha = torch.empty_like(alpha)
    B, H, n, d = q.shape
    N = q.numel()
    _expect("rope_attn_bwd", q.device, ("q", q, None), ("k", k, N), ("v", v, N), ("o", o, N),
            ("lse", lse, B * H * n), ("dO", dO, N), ("alpha", alpha, d // 2), ("dq", dq, N),
            ("dk", dk, N), ("dv", dv, N), ("dalpha", dalpha, d // 2), ("ws", ws, None))
    _check("rope_attn_bwd", lib().rope_attn_bwd(
        ctypes.byref(prob), _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dO),
        _ptr(alpha), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dalpha), _ptr(ws), ws.numel(),
        _stream(q.device)))
    return dq, dk, dv, dalpha


def rope_attn_bwd_saved(v, o, lse, dO, alpha, base, causal, ws, dq=None, dk=None, dv=None,
                        dalpha=None, fixed_bands=0, frozen_alpha=False):
    """rope_attn_bwd from the table, Q~ and K~ the preceding rope_attn_fwd left in ws
    (same problem, q, k and alpha; see include/rope_attn.h)."""
    prob = _problem_of(v, causal, base, fixed_bands)
    dq = torch.empty_like(v) if dq is None else dq
    dk = torch.empty_like(v) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    if frozen_alpha:
        dalpha = None
    elif dalpha is None:
        dalpha = torch.empty_like(alpha)
    B, H, n, d = v.shape
    N = v.numel()
    _expect("rope_attn_bwd_saved", v.device, ("v", v, None), ("o", o, N), ("lse", lse, B * H * n),
            ("dO", dO, N), ("alpha", alpha, d // 2), ("dq", dq, N), ("dk", dk, N), ("dv", dv, N),
            ("dalpha", dalpha, d // 2), ("ws", ws, None))
    _check("rope_attn_bwd_saved", lib().rope_attn_bwd_saved(
        ctypes.byref(prob), _ptr(v), _ptr(o), _ptr(lse), _ptr(dO), _ptr(alpha), _ptr(dq),
        _ptr(dk), _ptr(dv), _ptr(dalpha), _ptr(ws), ws.numel(), _stream(v.device)))
    return dq, dk, dv, dalpha


def rope_attn_proj_fwd(x, wq, wk, wv, H, q=None, k=None, v=None, ws=None):
    """q, k, v [B, H, n, d] = x [B, n, d_model] @ W [d_model, H*d], head h in columns h*d..
    ws: a workspace of at least 1024 bytes (its first 64 bytes are the error word)."""
    B, n, dm = x.shape
    d = wq.shape[1] // H
    prob = problem(B, H, n, d, x.dtype, False, 1.0)
    out = [torch.empty((B, H, n, d), dtype=x.dtype, device=x.device) if t is None else t
           for t in (q, k, v)]
    if ws is None:
        ws = torch.empty(1024, dtype=torch.uint8, device=x.device)
    W, Y = dm * H * d, B * H * n * d
    _expect("rope_attn_proj_fwd", x.device, ("x", x, None), ("wq", wq, W), ("wk", wk, W),
            ("wv", wv, W), ("q", out[0], Y), ("k", out[1], Y), ("v", out[2], Y), ("ws", ws, None))
    _check("rope_attn_proj_fwd", lib().rope_attn_proj_fwd(
        ctypes.byref(prob), dm, _ptr(x), _ptr(wq), _ptr(wk), _ptr(wv), *[_ptr(t) for t in out],
        _ptr(ws), ws.numel(), _stream(x.device)))
    return tuple(out)


def rope_attn_proj_bwd(x, wq, wk, wv, dq, dk, dv):
    """(dW_Q, dW_K, dW_V [d_model, H*d], dx [B, n, d_model]), all fp32, from the path's
    dq, dk, dv [B, H, n, d]."""
    B, H, n, d = dq.shape
    dm = x.shape[2]
    prob = problem(B, H, n, d, x.dtype, False, 1.0)
    f32 = dict(dtype=torch.float32, device=x.device)
    dws = [torch.empty((dm, H * d), **f32) for _ in range(3)]
    dx = torch.empty((B, n, dm), **f32)
    ws = torch.empty(int(lib().rope_attn_proj_workspace_bytes(ctypes.byref(prob))),
                     dtype=torch.uint8, device=x.device)
    W, Y = dm * H * d, dq.numel()
    _expect("rope_attn_proj_bwd", x.device, ("x", x, B * n * dm), ("wq", wq, W), ("wk", wk, W),
            ("wv", wv, W), ("dq", dq, None), ("dk", dk, Y), ("dv", dv, Y))
    _check("rope_attn_proj_bwd", lib().rope_attn_proj_bwd(
        ctypes.byref(prob), dm, _ptr(x), _ptr(wq), _ptr(wk), _ptr(wv), _ptr(dq), _ptr(dk),
        _ptr(dv), *[_ptr(t) for t in dws], _ptr(dx), _ptr(ws), ws.numel(), _stream(x.device)))
    return dws[0], dws[1], dws[2], dx


def rope_attn_spectrum(q, k, v, o, lse, dO, alpha, base, causal, fixed_bands=0):
    """(g [d/2, 2n-1] complex64, dalpha [d/2] fp32): the offset-aggregated gradient signal of
    every band and the frequency gradient from its DTFT surrogate (see include/rope_attn.h)."""
    prob = _problem_of(q, causal, base, fixed_bands)
    B, H, n, d = q.shape
    ws = torch.empty(int(lib().rope_attn_spectrum_workspace_bytes(ctypes.byref(prob))),
                     dtype=torch.uint8, device=q.device)
    g = torch.empty((d // 2, 2 * n - 1, 2), dtype=torch.float32, device=q.device)
    dalpha = torch.empty(d // 2, dtype=torch.float32, device=q.device)
    N = q.numel()
    _expect("rope_attn_spectrum", q.device, ("q", q, None), ("k", k, N), ("v", v, N), ("o", o, N),
            ("lse", lse, B * H * n), ("dO", dO, N), ("alpha", alpha, d // 2))
    _check("rope_attn_spectrum", lib().rope_attn_spectrum(
        ctypes.byref(prob), _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dO), _ptr(alpha),
        _ptr(g), _ptr(dalpha), _ptr(ws), ws.numel(), _stream(q.device)))
    return torch.view_as_complex(g), dalpha


def rope_attn_alpha_adam(alpha, dalpha, m1, m2, step, lr, beta1=0.9, beta2=0.999, eps=1e-8,
                         clip_norm=1.0):
    """One in-place Adam step (weight decay 0) of the fp32 device tensors alpha, m1, m2 from
    dalpha clipped to L2 norm clip_norm (clip_norm <= 0: no clipping); step is 1-based."""
    opt = RaAdam(float(lr), float(beta1), float(beta2), float(eps), float(clip_norm), int(step))
    M = alpha.numel()
    _expect("rope_attn_alpha_adam", alpha.device, ("alpha", alpha, None), ("dalpha", dalpha, M),
            ("m1", m1, M), ("m2", m2, M))
    _check("rope_attn_alpha_adam", lib().rope_attn_alpha_adam(
        ctypes.byref(opt), alpha.numel(), _ptr(alpha), _ptr(dalpha), _ptr(m1), _ptr(m2),
        _stream(alpha.device)))
    return alpha, m1, m2


def rope_attn_device_status(ws):
    """Synchronise the current stream and return (status code, [kernel, site, block])."""
    _expect("rope_attn_device_status", ws.device, ("ws", ws, None))
    info = (ctypes.c_int32 * 3)()
    code = lib().rope_attn_device_status(_ptr(ws), ws.numel(), _stream(ws.device), info)
    return code, list(info)


def rope_attn_timing_enable(on=True):
    lib().rope_attn_timing_enable(1 if on else 0)


def rope_attn_timing_read():
    """{kernel name: (launches, total ms)} since the last read."""
    n = 32
    launches = (ctypes.c_int32 * n)()
    total = (ctypes.c_double * n)()
    k = lib().rope_attn_timing_read(launches, total, n)
    return {lib().rope_attn_kernel_name(i).decode(): (launches[i], total[i])
            for i in range(k) if launches[i] > 0}
