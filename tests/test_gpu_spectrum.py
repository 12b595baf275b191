"""GPU parity of the frequency-spectrum diagnostic ("LeRoPE: learnable RoPE frequencies",
Analise Teorica): the offset-aggregated gradient signal g_m(D) against the oracle, and the
frequency gradient from its DTFT surrogate against both the oracle and the backward's own
dalpha (two routes to the same number)."""
import numpy as np
import pytest
import torch

from helpers import make, small_workload, to64
from oracle import rope_attn_ref as ref
from rope_attention_fwd_b200 import binding as rb

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype,d,n", [("f32", 16, 96), ("bf16", 64, 96), ("bf16", 128, 300),
                                       ("f32", 128, 200), ("bf16", 128, 1100)])
@pytest.mark.parametrize("causal", [False, True])
def test_spectrum_matches_oracle_and_backward(dtype, d, n, causal):
    """Several 64-row blocks (the last one ragged), d up to 128."""
    wl = small_workload(1, 2, n, d, dtype, causal, base=500.0, seed=81)
    inp = make(wl)
    q, k, v, e, alpha = (getattr(inp, x).cuda() for x in ("q", "k", "v", "e", "alpha"))
    ws = rb.workspace(rb.problem(wl.B, wl.H, wl.n, wl.d, q.dtype, causal, wl.base), "cuda")
    o, lse = rb.rope_attn_fwd(q, k, v, alpha, wl.base, causal, ws=ws)
    _, dO = rb.rope_attn_loss(o, e, ws=ws)
    _, _, _, dalpha = rb.rope_attn_bwd(q, k, v, o, lse, dO, alpha, wl.base, causal, ws=ws)
    g, da_spec = rb.rope_attn_spectrum(q, k, v, o, lse, dO, alpha, wl.base, causal)
    assert rb.rope_attn_device_status(ws)[0] == 0
    want = ref.offset_signal(to64(q), to64(k), to64(v), to64(dO), to64(alpha), wl.base, causal)
    got = g.cpu().numpy().astype(np.complex128)
    # fp32: fp32 rounding only.  bf16: the diagnostic forms Delta = rowsum(dO o O) from the
    # forward's bf16 O (within its 2e-2 bound), the oracle from its exact O; that moves dS
    # by ~1e-3 of its scale.
    tol = 1e-4 if dtype == "f32" else 2e-2
    assert np.max(np.abs(got - want)) <= tol * np.max(np.abs(want))
    if causal:
        assert np.all(got[:, : wl.n - 1] == 0)
    _, th = ref.frequencies(d, wl.base, to64(alpha))
    da_ref = th * ref.dtft_derivative(want, th)
    assert np.linalg.norm(to64(da_spec) - da_ref) <= 2.5 * tol * np.linalg.norm(da_ref)
    if dtype == "f32":
        # the backward's dalpha is the same quantity reached through the band torques
        assert np.linalg.norm(to64(da_spec) - to64(dalpha)) <= 1e-4 * np.linalg.norm(to64(dalpha))
