"""rope_attn_fwd_noalloc: the forward for callers that cannot allocate device memory.

Such callers (a fixed memory plan, a runtime that forbids allocation after start-up,
a framework that owns every device byte) cannot provide a workspace; this entry point
takes its scratch from a static array inside the library instead.  It runs the same
kernels on the same inputs as the workspace forward, so its results must be bit-identical
to it (and inside the bf16 tolerances of the float64 oracle), on consecutive calls that
share that array.  It must refuse problems larger than the array before launching
anything, and the array's error word (read with rope_attn_noalloc_status) must report a
rotated entry beyond the fp16 range.  This file runs last (its name sorts last) and also
passes on its own in a fresh process, where its first call performs the once-per-device
address lookup."""
import ctypes

import pytest
import torch

from helpers import compare, make, oracle_fwd, small_workload, to64
from rope_attention_fwd_b200 import binding as rb

pytestmark = pytest.mark.gpu


def _noalloc(prob, q, k, v, alpha, o, lse):
    return rb.lib().rope_attn_fwd_noalloc(
        ctypes.byref(prob), ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()),
        ctypes.c_void_p(v.data_ptr()), ctypes.c_void_p(alpha.data_ptr()),
        ctypes.c_void_p(o.data_ptr()), ctypes.c_void_p(lse.data_ptr()),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def _status():
    info = (ctypes.c_int32 * 3)()
    code = rb.lib().rope_attn_noalloc_status(
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream), info)
    return rb.STATUS[code], list(info)


def test_noalloc_matches_workspace_forward_on_two_calls():
    # two calls in a row with different shapes and data: stale scratch from the first
    # call must not show up in the second
    cases = [small_workload(1, 4, 300, 128, "bf16", True, seed=21),
             small_workload(2, 3, 257, 64, "bf16", False, seed=22)]
    for wl in cases:
        inp = make(wl)
        q, k, v, alpha = (getattr(inp, x).cuda() for x in ("q", "k", "v", "alpha"))
        prob = rb.problem(wl.B, wl.H, wl.n, wl.d, q.dtype, wl.causal, wl.base)
        assert rb.lib().rope_attn_fwd_workspace_bytes(ctypes.byref(prob)) <= (8 << 20)
        o_ref, lse_ref = rb.rope_attn_fwd(q, k, v, alpha, wl.base, wl.causal)
        o = torch.full_like(q, float("nan"))
        lse = torch.full((wl.B, wl.H, wl.n), float("nan"), device="cuda")
        assert _noalloc(prob, q, k, v, alpha, o, lse) == 0
        assert _status()[0] == "RA_OK"
        # same kernels, same inputs: the same bits
        assert torch.equal(o, o_ref) and torch.equal(lse, lse_ref)
        errs = compare(dict(o=to64(o), lse=to64(lse)), oracle_fwd(inp), "bf16",
                       keys=("o", "lse"))
        print(wl.name, errs)


def test_noalloc_reports_range_overflow():
    """A query entry beyond the fp16 range of the score operands is clamped and reported
    in the static array's error word; the next clean call reports nothing."""
    wl = small_workload(1, 1, 64, 64, "bf16", False, seed=23)
    inp = make(wl)
    q, k, v, alpha = (getattr(inp, x).cuda() for x in ("q", "k", "v", "alpha"))
    prob = rb.problem(wl.B, wl.H, wl.n, wl.d, q.dtype, wl.causal, wl.base)
    o = torch.empty_like(q)
    lse = torch.empty((1, 1, wl.n), device="cuda")
    big = q.clone()
    big[0, 0, 0, 0] = 7.0e4  # position 0: the rotation keeps it, 7e4 > 65504
    assert _noalloc(prob, big, k, v, alpha, o, lse) == 0
    assert _status()[0] == "RA_ERR_RANGE"
    assert _noalloc(prob, q, k, v, alpha, o, lse) == 0
    assert _status()[0] == "RA_OK"


def test_noalloc_rejects_problems_beyond_the_scratch():
    prob = rb.problem(2, 32, 8192, 128, torch.bfloat16, True, 1e4)
    assert rb.lib().rope_attn_fwd_workspace_bytes(ctypes.byref(prob)) > (8 << 20)
    null = ctypes.c_void_p(0)
    r = rb.lib().rope_attn_fwd_noalloc(ctypes.byref(prob), null, null, null, null, null, null,
                                       null)
    assert rb.STATUS[r] == "RA_ERR_UNSUPPORTED"
