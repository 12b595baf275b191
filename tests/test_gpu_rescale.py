"""GPU parity of the forward's lazy rescale when the two halves of a 128-key tile disagree
("RoPE attention can be trained in almost-linear time", Metodologia 1: the normalised
softmax of the scores).  Every band is fixed (no rotation), so the scores are plain dot
products and can be placed exactly: keys 192.. score about 20 log2 units above keys
0..191, and keys 448.. another 20 above those.  At the second and fourth key tiles the
lower 64 keys stay within the reference max while the upper 64 exceed it: the warpgroup
of the lower half sees no rescale in its own columns, and only the exchanged row maxima
tell it to move the reference max and rescale O with the other half."""
import numpy as np
import pytest
import torch

from helpers import TOL
from oracle import rope_attn_ref as ref
from rope_attention_fwd_b200 import binding as rb

@pytest.mark.gpu
@pytest.mark.parametrize("causal", [False, True])
def test_rescale_after_early_half_matches_oracle(causal):
    B, H, n, d = 1, 2, 512, 128
    g = torch.Generator().manual_seed(41)
    level = torch.zeros(n, dtype=torch.float64)
    level[192:] = 1.25   # q.k / sqrt(d) * log2(e) ~ 16.3 * level
    level[448:] = 2.5
    q = (1.0 + 0.1 * torch.randn((B, H, n, d), generator=g, dtype=torch.float64))
    k = level[None, None, :, None] + 0.1 * torch.randn((B, H, n, d), generator=g,
                                                        dtype=torch.float64)
    v = torch.randn((B, H, n, d), generator=g, dtype=torch.float64)
    q, k, v = (t.to(torch.bfloat16) for t in (q, k, v))
    alpha = torch.zeros(d // 2, dtype=torch.float32)
    base = 1e4
    ws = rb.workspace(rb.problem(B, H, n, d, torch.bfloat16, causal, base), "cuda")
    o, lse = rb.rope_attn_fwd(q.cuda(), k.cuda(), v.cuda(), alpha.cuda(), base, causal, ws=ws,
                              fixed_bands=d // 2)
    assert rb.rope_attn_device_status(ws)[0] == 0
    want_o, want_lse = ref.forward(q.double().numpy(), k.double().numpy(), v.double().numpy(),
                                   alpha.double().numpy(), base, causal, fixed_bands=d // 2)
    got_o = o.double().cpu().numpy()
    err_o = np.max(np.abs(got_o - want_o))
    err_lse = np.max(np.abs(lse.double().cpu().numpy() - want_lse))
    print(f"causal={causal}: max|dO| {err_o:.3e}, max|dlse| {err_lse:.3e}")
    assert err_o <= TOL["bf16"]["o"]
    assert err_lse <= TOL["bf16"]["lse"]


def test_rescale_construction_levels():
    """The score levels the test above relies on, from the same inputs on the CPU (log2
    units, scaled by 1/sqrt(d)): below 1 for keys 0..191, 19..22 for keys 192..447, above 39
    for keys 448.. ."""
    n, d = 512, 128
    g = torch.Generator().manual_seed(41)
    level = torch.zeros(n, dtype=torch.float64)
    level[192:] = 1.25
    level[448:] = 2.5
    q = (1.0 + 0.1 * torch.randn((1, 2, n, d), generator=g, dtype=torch.float64))
    k = level[None, None, :, None] + 0.1 * torch.randn((1, 2, n, d), generator=g,
                                                        dtype=torch.float64)
    q, k = (t.to(torch.bfloat16).double()[0, 0].numpy() for t in (q, k))
    s = q @ k.T / np.sqrt(d) * np.log2(np.e)
    assert s[:, :192].max() < 1 and 19 < s[:, 192:448].min() and s[:, 192:448].max() < 22
    assert s[:, 448:].min() > 39
