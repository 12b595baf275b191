"""GPU parity on the five workloads at full size, in the launch configuration the bench
times (rope_attn_fwd, rope_attn_loss, rope_attn_bwd_saved on the whole [B, H, n, d]
problem in one call each), against the float64 oracle on every element.

* 1x1x256x64 fp32 and 4x16x2048x64 bf16: every output against the full oracle.
* 2x32x8192x128, 1x8x32768x128, 8x16x4096x128 (bf16): every head is recomputed by the
  oracle in a spawn process pool (one head per core, see oracle_heads.py).  O and lse are
  compared on every element; dQ, dK, dV by the relative Frobenius error of the whole
  tensor; dalpha of the whole problem (summed over every head, "LeRoPE", Escolhas de
  Design Principais: alpha is shared by all heads) against the oracle's whole-problem
  dalpha.  All at the target's bounds: 2e-2 max-abs on O, 1e-2 relative Frobenius on
  dQ, dK, dV, dalpha.  Plus two exact properties of the loss: dO is the bf16 rounding of
  O - E, and L is 1/2 sum (O - E)^2 of the GPU's own O.
"""
import numpy as np
import pytest
import torch

from helpers import TOL, check_status, compare, gpu_run, oracle_run, to64
from oracle import rope_attn_ref as ref
from oracle_heads import run_heads
from rope_attention_fwd_b200 import binding as rb
from rope_attention_fwd_b200.configs import WORKLOADS
from rope_attention_fwd_b200.inputs import make_inputs

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("cfg", [1, 2])
def test_config_full_oracle(cfg):
    inp = make_inputs(WORKLOADS[cfg])
    errs = compare(gpu_run(inp), oracle_run(inp), WORKLOADS[cfg].dtype, label=f"config {cfg}")
    print(f"config {cfg}", errs)


def _gpu_step(inp, dev="cuda"):
    """One bench step through the C ABI: forward, loss, backward from the saved operands."""
    wl = inp.wl
    q, k, v, e, alpha = (getattr(inp, x).to(dev) for x in ("q", "k", "v", "e", "alpha"))
    ws = rb.workspace(rb.problem(wl.B, wl.H, wl.n, wl.d, q.dtype, wl.causal, wl.base), dev)
    o, lse = rb.rope_attn_fwd(q, k, v, alpha, wl.base, wl.causal, ws=ws)
    L, dO = rb.rope_attn_loss(o, e, ws=ws)
    dq, dk, dv, dalpha = rb.rope_attn_bwd_saved(v, o, lse, dO, alpha, wl.base, wl.causal, ws)
    check_status(ws)
    cpu = lambda t: t.cpu()
    return dict(o=cpu(o), lse=cpu(lse), L=float(L.item()), dO=cpu(dO), dq=cpu(dq), dk=cpu(dk),
                dv=cpu(dv), dalpha=cpu(dalpha))


def _bits(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


@pytest.mark.slow
@pytest.mark.parametrize("cfg", [3, 4, 5])
def test_config_every_head(cfg):
    wl = WORKLOADS[cfg]
    inp = make_inputs(wl)
    g = _gpu_step(inp)
    tol = TOL["bf16"]

    # exact properties of the loss: dO = bf16(O - E); L = 1/2 sum (O - E)^2 of the GPU's O
    diff = g["o"].float() - inp.e.float()
    assert torch.equal(g["dO"], diff.to(torch.bfloat16))
    L_host = 0.5 * float((diff.double() ** 2).sum())
    assert abs(g["L"] - L_host) <= 1e-6 * L_host

    tasks = []
    alpha = inp.alpha.double().numpy()
    for b in range(wl.B):
        for h in range(wl.H):
            t = dict(head=(b, h), n=wl.n, d=wl.d, causal=wl.causal, base=wl.base, alpha=alpha)
            for x in ("q", "k", "v", "e"):
                t[x] = _bits(getattr(inp, x)[b, h])
            for x in ("o", "dq", "dk", "dv"):
                t["g_" + x] = _bits(g[x][b, h])
            t["g_lse"] = g["lse"][b, h].numpy()
            tasks.append(t)
    res = run_heads(tasks)

    errs = {"o": max(r["o_maxabs"] for r in res), "lse": max(r["lse_maxabs"] for r in res)}
    for name in ("dq", "dk", "dv"):
        errs[name] = float(np.sqrt(sum(r[name + "_err2"] for r in res) /
                                   sum(r[name + "_norm2"] for r in res)))
        errs[name + "_worst_head"] = float(max(np.sqrt(r[name + "_err2"] / r[name + "_norm2"])
                                               for r in res))
    _, th = ref.frequencies(wl.d, wl.base, alpha)
    torque = np.zeros(wl.d // 2)
    for r in res:  # fixed head order
        torque += r["torque"]
    da_ref = th * torque
    da = g["dalpha"].double().numpy()
    errs["dalpha"] = float(np.linalg.norm(da - da_ref) / np.linalg.norm(da_ref))
    print(f"config {cfg} every head:", errs)
    assert errs["o"] <= tol["o"], errs
    assert errs["lse"] <= tol["lse"], errs
    for name in ("dq", "dk", "dv", "dalpha"):
        assert errs[name] <= tol["grad"], (name, errs)
