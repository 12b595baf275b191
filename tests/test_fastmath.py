"""The packed fp32-pair helpers of the softmax loops (csrc/fastmath.cuh): ffma2, fmul2,
fadd2 and fsub2 must round each lane exactly as the scalar instruction does (the dQ kernel
relies on this for bit-identical results), on random, tiny, huge and signed-zero inputs.
The forward's FMA-pipe 2^x (exp2_poly2: Cody-Waite range reduction and a degree-3
polynomial) must stay within its stated relative error of 2^x, checked on the CPU by
replaying its float32 steps and on the GPU against float64 exp2."""
import ctypes
import os
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "rope_attention_fwd_b200", "csrc")


@pytest.fixture(scope="module")
def probe():
    out = os.path.join(ROOT, "_build", "fastmath_probe.so")
    os.makedirs(os.path.dirname(out), exist_ok=True)
    src = os.path.join(ROOT, "tests", "csrc", "fastmath_probe.cu")
    subprocess.run(["/usr/local/cuda/bin/nvcc", "-gencode", "arch=compute_100a,code=sm_100a",
                    "-O3", "-std=c++17", "-shared", "-Xcompiler", "-fPIC", "-I" + CSRC, src,
                    "-o", out], check=True)
    lib = ctypes.CDLL(out)
    lib.fastmath_probe.argtypes = [ctypes.c_void_p] * 7 + [ctypes.c_int, ctypes.c_void_p]
    lib.addsub_probe.argtypes = [ctypes.c_void_p] * 6 + [ctypes.c_int, ctypes.c_void_p]
    lib.exp2_probe.argtypes = [ctypes.c_void_p] * 2 + [ctypes.c_int, ctypes.c_void_p]
    return lib


def test_probe_builds(probe):
    assert hasattr(probe, "fastmath_probe")


@pytest.mark.gpu
def test_packed_pairs_round_like_scalars(probe):
    import torch
    g = torch.Generator().manual_seed(5)
    n = 1 << 20
    a = torch.randn(n, generator=g) * torch.exp2(torch.randint(-60, 60, (n,), generator=g).float())
    b = torch.randn(n, generator=g) * torch.exp2(torch.randint(-60, 60, (n,), generator=g).float())
    c = torch.randn(n, generator=g) * torch.exp2(torch.randint(-60, 60, (n,), generator=g).float())
    a[:4] = torch.tensor([0.0, -0.0, 1e-40, -3e38])
    a, b, c = a.cuda(), b.cuda(), c.cuda()
    outs = [torch.empty_like(a) for _ in range(4)]
    ptr = lambda t: ctypes.c_void_p(t.data_ptr())
    assert probe.fastmath_probe(ptr(a), ptr(b), ptr(c), *[ptr(t) for t in outs], n,
                                ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)) == 0
    torch.cuda.synchronize()
    fma2, fma1, mul2, mul1 = outs
    assert torch.equal(fma2.view(torch.int32), fma1.view(torch.int32))
    assert torch.equal(mul2.view(torch.int32), mul1.view(torch.int32))


# ---------------------------------------------------------------- exp2_poly2
EXP2_REL_ERR = 7.6e-5   # the minimax cubic's bound (7.48e-5) plus float32 rounding


def _poly_coefficients():
    """c0..c3 as written in fastmath.cuh."""
    import re
    text = open(os.path.join(CSRC, "fastmath.cuh")).read()
    body = text[text.index("float2 exp2_poly2"):]
    return [float(re.search(rf"c{k} = ([0-9.eE+-]+)f", body).group(1)) for k in range(4)]


def _exp2_poly_cpu(x):
    """The float32 steps of exp2_poly2 replayed in numpy: each add / sub rounded to float32,
    each fused multiply-add formed exactly in float64 (float32 operands of these magnitudes)
    and rounded once, the exponent inserted with 32-bit integer arithmetic."""
    import numpy as np
    c0, c1, c2, c3 = (np.float32(c) for c in _poly_coefficients())
    r = np.float32(12582912.0)
    x = np.maximum(x.astype(np.float32), np.float32(-126.0))
    t = (x + r).astype(np.float32)
    f = (x - (t - r).astype(np.float32)).astype(np.float32)
    fma = lambda a, b, c: (a.astype(np.float64) * b.astype(np.float64) + np.float64(c)).astype(np.float32)
    p = fma(f, np.full_like(f, c3), c2)
    p = fma(p, f, c1)
    p = fma(p, f, c0)
    bits = p.view(np.int32).astype(np.int64) + (t.view(np.int32).astype(np.int64) << 23)
    return (bits & 0xFFFFFFFF).astype(np.uint32).view(np.float32)


def test_exp2_poly_relative_error_cpu():
    import numpy as np
    x = np.concatenate([np.linspace(-120.0, 8.0, 2_000_001), np.arange(-120.0, 8.5, 0.5),
                        np.arange(-120.0, 8.0) + 0.49999997]).astype(np.float32)
    y = _exp2_poly_cpu(x).astype(np.float64)
    rel = np.abs(y / np.exp2(x.astype(np.float64)) - 1.0)
    assert rel.max() <= EXP2_REL_ERR, rel.max()


def _remez_relative(deg, a, b, grid_points=200_001, iters=30):
    """Best uniform (minimax) polynomial approximation of 2^x on [a, b] in relative error,
    by the Remez exchange algorithm: solve p(x_i) - 2^x_i = (-1)^i E 2^x_i on deg + 2
    reference points, move each point to the extremum of the error on its sign-alternating
    segment, repeat.  Returns the coefficients (constant first) and the maximum error."""
    import numpy as np
    n = deg + 2
    k = np.arange(n)
    xs = (a + b) / 2 + (b - a) / 2 * np.cos(np.pi * k[::-1] / (n - 1))
    grid = np.linspace(a, b, grid_points)
    fg = np.exp2(grid)
    for _ in range(iters):
        f = np.exp2(xs)
        m = np.hstack([np.stack([xs ** j for j in range(deg + 1)], 1),
                       ((-1.0) ** k * f)[:, None]])
        c = np.linalg.solve(m, f)[:-1]
        e = np.polyval(c[::-1], grid) / fg - 1.0
        sign = np.sign(e)
        cuts = np.flatnonzero(sign[1:] != sign[:-1]) + 1
        idx = np.array([s0 + np.argmax(np.abs(e[s0:s1]))
                        for s0, s1 in zip(np.r_[0, cuts], np.r_[cuts, len(e)])])
        while len(idx) > n:
            idx = idx[1:] if abs(e[idx[0]]) < abs(e[idx[-1]]) else idx[:-1]
        if len(idx) < n:
            break
        xs = grid[idx]
    return c, np.abs(e).max()


def test_exp2_poly_coefficients_are_the_minimax_cubic():
    """The constants of exp2_poly2 are the degree-3 minimax approximation of 2^f in relative
    error on [-1/2, 1/2] (the range the round-to-nearest split leaves), re-derived here from
    the definition; their own error is that minimax error."""
    import numpy as np
    c, err = _remez_relative(3, -0.5, 0.5)
    got = np.array(_poly_coefficients())
    assert np.abs(got - c).max() <= 1e-6, (got, c)
    x = np.linspace(-0.5, 0.5, 200_001)
    own = np.abs(np.polyval(got[::-1], x) / np.exp2(x) - 1.0).max()
    assert own <= err * 1.001 and err <= 7.5e-5, (own, err)


def test_exp2_poly_clamp_cpu():
    """Below -126 (and at -inf, a masked score) the result is a tiny non-negative number."""
    import numpy as np
    x = np.array([-126.0, -126.4, -130.0, -1e30, -np.inf, -125.6], dtype=np.float32)
    y = _exp2_poly_cpu(x)
    assert np.all(np.isfinite(y)) and np.all(y >= 0) and np.all(y <= 2.0 ** -125)


@pytest.mark.gpu
def test_packed_add_sub_round_like_scalars(probe):
    import torch
    g = torch.Generator().manual_seed(6)
    n = 1 << 20
    a = torch.randn(n, generator=g) * torch.exp2(torch.randint(-60, 60, (n,), generator=g).float())
    b = torch.randn(n, generator=g) * torch.exp2(torch.randint(-60, 60, (n,), generator=g).float())
    a[:4] = torch.tensor([0.0, -0.0, 1e-40, -3e38])
    a, b = a.cuda(), b.cuda()
    outs = [torch.empty_like(a) for _ in range(4)]
    ptr = lambda t: ctypes.c_void_p(t.data_ptr())
    assert probe.addsub_probe(ptr(a), ptr(b), *[ptr(t) for t in outs], n,
                              ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)) == 0
    torch.cuda.synchronize()
    add2, add1, sub2, sub1 = outs
    assert torch.equal(add2.view(torch.int32), add1.view(torch.int32))
    assert torch.equal(sub2.view(torch.int32), sub1.view(torch.int32))


@pytest.mark.gpu
def test_exp2_poly_on_device(probe):
    """The device function against float64 exp2 and against its CPU replay."""
    import numpy as np
    import torch
    g = torch.Generator().manual_seed(7)
    n = 1 << 20
    x = torch.rand(n, generator=g, dtype=torch.float64) * 128.0 - 120.0
    x[:8] = torch.tensor([0.0, 8.0, -0.5, 0.5, -120.0, -126.0, -200.0, -float("inf")],
                         dtype=torch.float64)
    x = x.float()
    xd = x.cuda()
    y = torch.empty_like(xd)
    assert probe.exp2_probe(ctypes.c_void_p(xd.data_ptr()), ctypes.c_void_p(y.data_ptr()), n,
                            ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)) == 0
    torch.cuda.synchronize()
    y = y.cpu().numpy()
    xs = x.numpy()
    # within one unit in the last place of the replay (its float64 fma can round twice)
    assert np.max(np.abs(y.view(np.int32).astype(np.int64) -
                         _exp2_poly_cpu(xs).view(np.int32).astype(np.int64))) <= 1
    ok = xs >= -120.0
    rel = np.abs(y[ok].astype(np.float64) / np.exp2(xs[ok].astype(np.float64)) - 1.0)
    assert rel.max() <= EXP2_REL_ERR, rel.max()
    assert np.all(y[~ok] >= 0) and np.all(y[~ok] <= 2.0 ** -125)
