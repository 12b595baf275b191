"""The softmax loops' replacements for XU-pipe operations (csrc/fastmath.cuh).

CPU: the header's exp2 coefficients are the ones gen_exp2_poly.py derives (Chebyshev
interpolation of 2^f on [-1/2, 1/2]), and an fp32 emulation of the whole evaluation
(magic-number range reduction, Horner, exponent insertion) stays within 1.2e-4 of 2^x.
GPU: the device functions against CUDA's exp2f and round-to-nearest-even packing."""
import ctypes
import os
import re
import subprocess
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "rope_attention_fwd_b200", "csrc")
sys.path.insert(0, CSRC)


def header_coefficients():
    text = open(os.path.join(CSRC, "fastmath.cuh")).read()
    return [float(v) for v in re.findall(r"kExp2C\d = ([0-9.e+-]+)f;", text)]


def emulate_exp2_poly(x):
    x = np.maximum(np.float32(x), np.float32(-125.0)).astype(np.float32)
    magic = np.float32(12582912.0)
    t = (x + magic).astype(np.float32)
    f = (x - (t - magic).astype(np.float32)).astype(np.float32)
    c = [np.float32(v) for v in header_coefficients()]
    p = np.float32(c[3])
    for a in (c[2], c[1], c[0]):
        p = (p * f + a).astype(np.float32)   # fmaf rounds once; this rounds twice (bound below)
    bits = (p.view(np.uint32).astype(np.uint64) + (t.view(np.uint32).astype(np.uint64) << 23))
    return (bits & 0xFFFFFFFF).astype(np.uint32).view(np.float32)


def test_coefficients_match_derivation():
    import gen_exp2_poly
    c = gen_exp2_poly.coefficients(3)
    assert np.array_equal(np.float32(header_coefficients()), np.float32(c))  # fp32 rounding
    assert gen_exp2_poly.max_rel_err_fp32(c) < 1.1e-4


def test_emulated_evaluation_error():
    x = np.linspace(-124.0, 10.0, 2_000_001, dtype=np.float32)
    y = emulate_exp2_poly(x).astype(np.float64)
    rel = np.abs(y / np.exp2(x.astype(np.float64)) - 1.0)
    assert rel.max() < 1.2e-4
    assert emulate_exp2_poly(np.float32(-np.inf)) < 2.0 ** -124


@pytest.fixture(scope="module")
def probe():
    out = os.path.join(ROOT, "_build", "fastmath_probe.so")
    os.makedirs(os.path.dirname(out), exist_ok=True)
    src = os.path.join(ROOT, "tests", "csrc", "fastmath_probe.cu")
    subprocess.run(["/usr/local/cuda/bin/nvcc", "-gencode", "arch=compute_100a,code=sm_100a",
                    "-O3", "-std=c++17", "-shared", "-Xcompiler", "-fPIC", "-I" + CSRC, src,
                    "-o", out], check=True)
    lib = ctypes.CDLL(out)
    lib.fastmath_probe.argtypes = [ctypes.c_void_p] * 5 + [ctypes.c_int, ctypes.c_void_p]
    return lib


@pytest.mark.gpu
def test_device_functions_against_cuda(probe):
    import torch
    x = torch.cat([torch.linspace(-124.0, 10.0, 1_000_001),
                   torch.tensor([0.0, -0.5, 0.5, -1e-30, float("-inf")])]).float().cuda()
    n = x.numel()
    poly, ref = torch.empty_like(x), torch.empty_like(x)
    pa = torch.empty(n, dtype=torch.int32, device="cuda")
    pr = torch.empty_like(pa)
    ptr = lambda t: ctypes.c_void_p(t.data_ptr())
    assert probe.fastmath_probe(ptr(x), ptr(poly), ptr(ref), ptr(pa), ptr(pr), n,
                                ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)) == 0
    torch.cuda.synchronize()
    fin = torch.isfinite(x)
    rel = ((poly[fin].double() / ref[fin].double()) - 1).abs().max().item()
    assert rel < 1.2e-4, rel
    assert poly[-1].item() < 2.0 ** -124   # -inf
    # packing: identical to round-to-nearest-even except at exact ties, never off by
    # more than one bf16 ulp in either half
    a, b = pa.cpu().numpy().view(np.uint32), pr.cpu().numpy().view(np.uint32)
    for shift in (0, 16):
        ha = ((a >> shift) & 0xFFFF).astype(np.int64)
        hb = ((b >> shift) & 0xFFFF).astype(np.int64)
        assert np.max(np.abs(ha - hb)) <= 1
    assert np.mean(a == b) > 0.99
