"""rope_attn_fwd_noalloc: the forward for callers that cannot allocate device memory.

Such callers (a fixed memory plan, a runtime that forbids allocation after start-up,
a framework that owns every device byte) cannot provide a workspace; this entry point
takes its scratch from a static array inside the library instead.  It must give the
same results as the workspace forward, on consecutive calls that share that array, and
must refuse problems larger than the array before launching anything.  This file runs
last (its name sorts last) and also passes on its own in a fresh process, where its
first call performs the once-per-device address lookup."""
import ctypes

import numpy as np
import pytest
import torch

from helpers import TOL, make, small_workload
from rope_attention_fwd_b200 import binding as rb

pytestmark = pytest.mark.gpu


def _noalloc(prob, q, k, v, alpha, o, lse):
    return rb.lib().rope_attn_fwd_noalloc(
        ctypes.byref(prob), ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()),
        ctypes.c_void_p(v.data_ptr()), ctypes.c_void_p(alpha.data_ptr()),
        ctypes.c_void_p(o.data_ptr()), ctypes.c_void_p(lse.data_ptr()),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def test_noalloc_matches_workspace_forward_on_two_calls():
    # two calls in a row with different shapes and data: stale scratch from the first
    # call must not show up in the second
    cases = [small_workload(1, 4, 300, 128, "bf16", True, seed=21),
             small_workload(2, 3, 257, 64, "bf16", False, seed=22)]
    for wl in cases:
        inp = make(wl)
        q, k, v, alpha = (getattr(inp, x).cuda() for x in ("q", "k", "v", "alpha"))
        prob = rb.problem(wl.B, wl.H, wl.n, wl.d, q.dtype, wl.causal, wl.base)
        assert rb.rope_attn_workspace_bytes(prob) <= (8 << 20)
        o_ref, lse_ref = rb.rope_attn_fwd(q, k, v, alpha, wl.base, wl.causal)
        o = torch.full_like(q, float("nan"))
        lse = torch.full((wl.B, wl.H, wl.n), float("nan"), device="cuda")
        assert _noalloc(prob, q, k, v, alpha, o, lse) == 0
        torch.cuda.synchronize()
        do = (o.double() - o_ref.double()).abs().max().item()
        dl = (lse.double() - lse_ref.double()).abs().max().item()
        assert do <= TOL["bf16"]["o"] and dl <= TOL["bf16"]["lse"], (do, dl)


def test_noalloc_rejects_problems_beyond_the_scratch():
    prob = rb.problem(2, 32, 8192, 128, torch.bfloat16, True, 1e4)
    assert rb.rope_attn_workspace_bytes(prob) > (8 << 20)
    null = ctypes.c_void_p(0)
    r = rb.lib().rope_attn_fwd_noalloc(ctypes.byref(prob), null, null, null, null, null, null,
                                       null)
    assert rb.STATUS[r] == "RA_ERR_UNSUPPORTED"
