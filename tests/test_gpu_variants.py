"""GPU parity of the LeRoPE variants the kernels support ("LeRoPE: learnable RoPE
frequencies", Configuracao Experimental, Ablacao and Escolhas de Design Principais):
partial RoPE with the slowest bands unrotated (p-RoPE), frozen frequencies (no dalpha), and
the optimiser step for alpha (Adam, weight decay 0, its own gradient clipping)."""
import numpy as np
import pytest
import torch

from helpers import TOL, compare, gpu_run, make, oracle_run, small_workload
from oracle import rope_attn_ref as ref
from rope_attention_fwd_b200 import binding as rb

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype,d", [("f32", 64), ("bf16", 64), ("bf16", 128)])
@pytest.mark.parametrize("causal", [False, True])
def test_fixed_bands_match_oracle(dtype, d, causal):
    """p = 0.75: the slowest quarter of the bands not rotated; their dalpha is exactly 0."""
    wl = small_workload(2, 2, 201, d, dtype, causal, seed=31)
    inp = make(wl)
    f = d // 8  # a quarter of the d/2 bands
    g = gpu_run(inp, fixed_bands=f)
    compare(g, oracle_run(inp, fixed_bands=f), dtype)
    assert np.all(g["dalpha"][d // 2 - f:] == 0.0)


def test_fixed_bands_all_is_unrotated_attention():
    """Every band fixed: the forward equals the plain-attention forward with alpha -> -inf,
    i.e. torch's scaled_dot_product_attention of the unrotated inputs, to bf16 rounding."""
    wl = small_workload(1, 2, 160, 64, "bf16", True, seed=33)
    inp = make(wl)
    g = gpu_run(inp, fixed_bands=32)
    sd = torch.nn.functional.scaled_dot_product_attention(
        inp.q.double(), inp.k.double(), inp.v.double(), is_causal=True).numpy()
    assert np.max(np.abs(g["o"] - sd)) <= TOL["bf16"]["o"]
    assert np.all(g["dalpha"] == 0.0)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_frozen_alpha_skips_dalpha_only(dtype):
    """Frozen frequencies: no dalpha; dq, dk, dv bit for bit those of the full backward."""
    wl = small_workload(2, 2, 190, 64, dtype, True, seed=35)
    inp = make(wl)
    q, k, v, e, alpha = (getattr(inp, x).cuda() for x in ("q", "k", "v", "e", "alpha"))
    ws = rb.workspace(rb.problem(wl.B, wl.H, wl.n, wl.d, q.dtype, True, wl.base), "cuda")
    o, lse = rb.rope_attn_fwd(q, k, v, alpha, wl.base, True, ws=ws)
    _, dO = rb.rope_attn_loss(o, e, ws=ws)
    full = rb.rope_attn_bwd(q, k, v, o, lse, dO, alpha, wl.base, True, ws=ws)
    frozen = rb.rope_attn_bwd(q, k, v, o, lse, dO, alpha, wl.base, True, ws=ws,
                              frozen_alpha=True)
    saved = rb.rope_attn_bwd_saved(v, o, lse, dO, alpha, wl.base, True, ws, frozen_alpha=True)
    assert rb.rope_attn_device_status(ws)[0] == 0
    assert frozen[3] is None and saved[3] is None
    for i in range(3):
        assert torch.equal(frozen[i], full[i]) and torch.equal(saved[i], full[i])


@pytest.mark.parametrize("clip", [0.0, 0.5, 1e3])
def test_alpha_adam_matches_oracle(clip):
    """Three fused alpha steps (clipping off, active, inactive) against the oracle's update."""
    M = 64
    rng = np.random.default_rng(37)
    a64 = 0.3 * rng.standard_normal(M)
    m1_64, m2_64 = np.zeros(M), np.zeros(M)
    alpha = torch.tensor(a64, dtype=torch.float32, device="cuda")
    m1 = torch.zeros(M, dtype=torch.float32, device="cuda")
    m2 = torch.zeros(M, dtype=torch.float32, device="cuda")
    a64 = alpha.double().cpu().numpy()
    for t in (1, 2, 3):
        g = torch.tensor(rng.standard_normal(M) * (0.1 * t), dtype=torch.float32, device="cuda")
        rb.rope_attn_alpha_adam(alpha, g, m1, m2, t, 1e-2, 0.9, 0.95, 1e-8, clip)
        a64, m1_64, m2_64 = ref.alpha_adam_step(a64, g.double().cpu().numpy(), m1_64, m2_64, t,
                                                1e-2, 0.9, 0.95, 1e-8, clip)
    torch.cuda.synchronize()
    np.testing.assert_allclose(alpha.double().cpu().numpy(), a64, rtol=0, atol=2e-6)
    np.testing.assert_allclose(m1.double().cpu().numpy(), m1_64, rtol=1e-5, atol=1e-8)
    np.testing.assert_allclose(m2.double().cpu().numpy(), m2_64, rtol=1e-5, atol=1e-10)
