"""The packed fp32-pair helpers of the softmax loops (csrc/fastmath.cuh): ffma2 and fmul2
must round each lane exactly as the scalar fmaf and multiply do (the dQ kernel relies on
this for bit-identical results), on random, tiny, huge and signed-zero inputs."""
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
