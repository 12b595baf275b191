"""Bounded device-side waits: a CTA whose producer never delivers must give up, record
RA_ERR_TIMEOUT in the workspace error word and leave the context usable.  The missing
arrival is made on purpose through the RA_DEBUG_STARVE_BLOCK hook (that CTA skips its
Q~ load); nothing faults, traps or hangs."""
import os

import pytest
import torch

from helpers import compare, gpu_fwd, make, oracle_fwd, small_workload
from rope_attention_fwd_b200 import binding as rb

pytestmark = pytest.mark.gpu


def test_forward_wait_expires_and_reports():
    wl = small_workload(1, 1, 128, 64, "bf16", False, seed=2)
    inp = make(wl)
    q, k, v, alpha = (getattr(inp, x).cuda() for x in ("q", "k", "v", "alpha"))
    ws = rb.workspace(rb.problem(1, 1, 128, 64, torch.bfloat16, False, wl.base), "cuda")
    os.environ["RA_WAIT_LIMIT_MS"] = "100"
    os.environ["RA_DEBUG_STARVE_BLOCK"] = "0"
    try:
        rb.rope_attn_fwd(q, k, v, alpha, wl.base, False, ws=ws)
        code, info = rb.rope_attn_device_status(ws)
    finally:
        del os.environ["RA_DEBUG_STARVE_BLOCK"]
        del os.environ["RA_WAIT_LIMIT_MS"]
    assert rb.STATUS[code] == "RA_ERR_TIMEOUT"
    assert rb.lib().rope_attn_kernel_name(info[0]) == b"fwd_sm100"
    assert info[2] == 0  # block id
    # the status was read and cleared; the context still works and gives correct results
    assert rb.rope_attn_device_status(ws)[0] == 0
    compare(gpu_fwd(inp), oracle_fwd(inp), "bf16", keys=("o", "lse"))


def test_range_overflow_is_reported():
    """A key entry beyond the fp16 range of the score operands is clamped by the rotation
    and reported as RA_ERR_RANGE through the workspace error word (nothing faults); the
    following clean call on the same workspace reports nothing."""
    wl = small_workload(1, 1, 64, 64, "bf16", False, seed=3)
    inp = make(wl)
    q, k, v, alpha = (getattr(inp, x).cuda() for x in ("q", "k", "v", "alpha"))
    ws = rb.workspace(rb.problem(1, 1, 64, 64, torch.bfloat16, False, wl.base), "cuda")
    big = k.clone()
    big[0, 0, 0, 1] = -7.0e4  # position 0: the rotation keeps it, |7e4| > 65504
    rb.rope_attn_fwd(q, big, v, alpha, wl.base, False, ws=ws)
    assert rb.STATUS[rb.rope_attn_device_status(ws)[0]] == "RA_ERR_RANGE"
    rb.rope_attn_fwd(q, k, v, alpha, wl.base, False, ws=ws)
    assert rb.rope_attn_device_status(ws)[0] == 0
