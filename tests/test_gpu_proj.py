"""GPU parity of the projections around the path ("RoPE attention can be trained in
almost-linear time", Lemma 4.1: the loss gradient with respect to the weights): q, k, v =
x W through the library's GEMMs (tcgen05 for bf16, CUDA cores for fp32) into the path's
layout, and dW_Q, dW_K, dW_V, dx back from the path's dq, dk, dv; then the whole layer
x -> projections -> attention -> loss -> gradients."""
import numpy as np
import pytest
import torch

from helpers import TOL, rel_frob, to64
from oracle import rope_attn_ref as ref
from rope_attention_fwd_b200 import binding as rb

pytestmark = pytest.mark.gpu


def _rand(shape, dtype, scale, gen):
    return (torch.randn(shape, generator=gen, dtype=torch.float64) * scale).to(dtype).cuda()


@pytest.mark.parametrize("dtype,B,H,n,d,dm", [
    (torch.float32, 2, 3, 200, 64, 96),
    (torch.bfloat16, 2, 3, 200, 64, 96),      # ragged tiles in M, N and K
    (torch.bfloat16, 2, 4, 512, 128, 256),    # several 128 x 256 tiles in every direction
    (torch.bfloat16, 1, 2, 130, 128, 520),    # a K chunk and a d_model tail that are partial
])
def test_proj_fwd_and_bwd_match_oracle(dtype, B, H, n, d, dm):
    g = torch.Generator().manual_seed(71)
    x = _rand((B, n, dm), dtype, 1.0, g)
    w = [_rand((dm, H * d), dtype, 0.1, g) for _ in range(3)]
    q, k, v = rb.rope_attn_proj_fwd(x, *w, H)
    want = ref.proj_forward(to64(x), *[to64(t) for t in w], H)
    tol = 1e-5 if dtype == torch.float32 else 4e-3   # the outputs are rounded to the dtype
    for got, exp in zip((q, k, v), want):
        assert rel_frob(to64(got), exp) <= tol
    dq, dk, dv = (_rand((B, H, n, d), dtype, 1.0, g) for _ in range(3))
    got = rb.rope_attn_proj_bwd(x, *w, dq, dk, dv)
    want = ref.proj_backward(to64(x), *[to64(t) for t in w], to64(dq), to64(dk), to64(dv))
    for a, b in zip(got, want):
        assert rel_frob(to64(a), b) <= 1e-5   # fp32 accumulation of exact products


def test_whole_layer_bf16():
    """x, W -> q, k, v -> fwd -> loss -> bwd -> dW, dx through the library, against the oracle
    chain on the same (bf16-rounded) q, k, v."""
    B, H, n, d, dm, base = 1, 2, 256, 128, 128, 1e4
    g = torch.Generator().manual_seed(73)
    x = _rand((B, n, dm), torch.bfloat16, 1.0, g)
    w = [_rand((dm, H * d), torch.bfloat16, dm ** -0.5, g) for _ in range(3)]
    e = _rand((B, H, n, d), torch.bfloat16, 1.0, g)
    alpha = (0.3 * torch.randn(d // 2, generator=g)).float().cuda()
    q, k, v = rb.rope_attn_proj_fwd(x, *w, H)
    ws = rb.workspace(rb.problem(B, H, n, d, torch.bfloat16, True, base), "cuda")
    o, lse = rb.rope_attn_fwd(q, k, v, alpha, base, True, ws=ws)
    _, dO = rb.rope_attn_loss(o, e, ws=ws)
    dq, dk, dv, _ = rb.rope_attn_bwd_saved(v, o, lse, dO, alpha, base, True, ws)
    got = rb.rope_attn_proj_bwd(x, *w, dq, dk, dv)
    assert rb.rope_attn_device_status(ws)[0] == 0
    r = ref.forward_backward(to64(q), to64(k), to64(v), to64(e), to64(alpha), base, True)
    want = ref.proj_backward(to64(x), *[to64(t) for t in w], r["dq"], r["dk"], r["dv"])
    for a, b in zip(got, want):
        assert rel_frob(to64(a), b) <= TOL["bf16"]["grad"]


def test_proj_launches_are_timed_per_product():
    """With the library's timing on, each projection product is recorded under its own
    kernel id: one q/k/v GEMM, three head merges, one dW and one dx GEMM per call pair."""
    g = torch.Generator().manual_seed(5)
    B, H, n, d, dm = 1, 2, 256, 128, 256
    x = _rand((B, n, dm), torch.bfloat16, 1.0, g)
    w = [_rand((dm, H * d), torch.bfloat16, 0.1, g) for _ in range(3)]
    rb.rope_attn_timing_read()
    rb.rope_attn_timing_enable(True)
    try:
        q, k, v = rb.rope_attn_proj_fwd(x, *w, H)
        rb.rope_attn_proj_bwd(x, *w, q, k, v)
        torch.cuda.synchronize()
    finally:
        rb.rope_attn_timing_enable(False)
    rec = rb.rope_attn_timing_read()
    assert {name: cnt for name, (cnt, _) in rec.items()} == {
        "proj_gemm": 1, "merge_heads": 3, "proj_dw_gemm": 1, "proj_dx_gemm": 1}
    assert all(ms > 0 for _, ms in rec.values())
