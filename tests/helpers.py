"""Shared helpers for the GPU parity tests: run the CUDA path through the C ABI,
run the oracle on the same seeded inputs, and compare."""
import numpy as np
import torch

from oracle import rope_attn_ref as ref
from rope_attention_fwd_b200 import binding as rb
from rope_attention_fwd_b200.configs import Workload
from rope_attention_fwd_b200.inputs import make_inputs

# Tolerances fixed by the target: fp32 -> 1e-4 max-abs on O and relative Frobenius on
# every gradient; bf16 -> 2e-2 max-abs on O, 1e-2 relative Frobenius on gradients.
# lse and L have no stated bound; the ones below follow from the same arithmetic
# (bf16 operands perturb each score by ~2^-9 relative).
TOL = {
    "f32": dict(o=1e-4, grad=1e-4, lse=1e-5, L=1e-5),
    "bf16": dict(o=2e-2, grad=1e-2, lse=2e-2, L=2e-3),
}


def rel_frob(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    den = np.linalg.norm(b.ravel())
    return np.linalg.norm((a - b).ravel()) / (den if den > 0 else 1.0)


def to64(t):
    return t.detach().to("cpu", torch.float64).numpy()


def small_workload(B, H, n, d, dtype, causal, base=1e4, seed=7, alpha_std=0.5,
                   qkve="normal"):
    return Workload(f"{B}x{H}x{n}x{d} {dtype} causal={causal}", B, H, n, d, dtype, causal, base,
                    qkve, -1.0, 1.0, "normal" if alpha_std > 0 else "zero", alpha_std, seed=seed)


def gpu_inputs(inp, device="cuda"):
    return {k: getattr(inp, k).to(device) for k in ("q", "k", "v", "e", "alpha")}


def check_status(ws):
    """The device error word of the most recent call on `ws` must be clear."""
    code, info = rb.rope_attn_device_status(ws)
    assert code == 0, (rb.STATUS.get(code, code), info)


def gpu_run(inp, device="cuda", ws=None, fixed_bands=0):
    """fwd -> loss -> bwd through the C ABI; returns float64 numpy results."""
    wl = inp.wl
    t = gpu_inputs(inp, device)
    if ws is None:
        ws = rb.workspace(rb.problem(wl.B, wl.H, wl.n, wl.d, t["q"].dtype, wl.causal, wl.base),
                          device)
    o, lse = rb.rope_attn_fwd(t["q"], t["k"], t["v"], t["alpha"], wl.base, wl.causal, ws=ws,
                              fixed_bands=fixed_bands)
    check_status(ws)
    L, dO = rb.rope_attn_loss(o, t["e"], ws=ws, causal=wl.causal, base=wl.base)
    check_status(ws)
    dq, dk, dv, dalpha = rb.rope_attn_bwd(t["q"], t["k"], t["v"], o, lse, dO, t["alpha"],
                                          wl.base, wl.causal, ws=ws, fixed_bands=fixed_bands)
    check_status(ws)
    return dict(o=to64(o), lse=to64(lse), L=float(L.item()), do=to64(dO), dq=to64(dq),
                dk=to64(dk), dv=to64(dv), dalpha=to64(dalpha))


def gpu_fwd(inp, device="cuda"):
    wl = inp.wl
    t = gpu_inputs(inp, device)
    o, lse = rb.rope_attn_fwd(t["q"], t["k"], t["v"], t["alpha"], wl.base, wl.causal)
    torch.cuda.synchronize()
    return dict(o=to64(o), lse=to64(lse))


def oracle_run(inp, fixed_bands=0):
    """Oracle results (float64) on the workload's stored inputs."""
    wl = inp.wl
    q, k, v, e, al = (inp.f64(x) for x in ("q", "k", "v", "e", "alpha"))
    o, lse = ref.forward(q, k, v, al, wl.base, wl.causal, fixed_bands=fixed_bands)
    L, do = ref.loss(o, e)
    dq, dk, dv, dalpha = ref.backward(q, k, v, do, al, wl.base, wl.causal,
                                      fixed_bands=fixed_bands)
    return dict(o=o, lse=lse, L=L, do=do, dq=dq, dk=dk, dv=dv, dalpha=dalpha)


def oracle_fwd(inp):
    wl = inp.wl
    o, lse = ref.forward(inp.f64("q"), inp.f64("k"), inp.f64("v"), inp.f64("alpha"), wl.base,
                         wl.causal)
    return dict(o=o, lse=lse)


def compare(g, r, dtype, keys=("o", "lse", "L", "dq", "dk", "dv", "dalpha"), label=""):
    """Assert every result is inside its tolerance (the target's bounds for O and the
    gradients, dalpha included, at every size); print and return the measured errors with
    their bounds."""
    tol = dict(TOL[dtype])
    errs, bounds = {}, {}
    for key in keys:
        if key == "o":
            errs[key] = float(np.max(np.abs(g["o"] - r["o"]))) if g["o"].size else 0.0
            bounds[key] = tol["o"]
        elif key == "lse":
            errs[key] = float(np.max(np.abs(g["lse"] - r["lse"]))) if g["lse"].size else 0.0
            bounds[key] = tol["lse"]
        elif key == "L":
            errs[key] = abs(g["L"] - r["L"]) / max(abs(r["L"]), 1e-30)
            bounds[key] = tol["L"]
        else:
            errs[key] = rel_frob(g[key], r[key])
            bounds[key] = tol.get(key, tol["grad"])
    print("parity", label, " ".join(f"{k}={errs[k]:.3e}/{bounds[k]:.1e}" for k in keys))
    for key in keys:
        assert errs[key] <= bounds[key], (label, key, errs[key], bounds[key])
    return errs


def make(wl):
    return make_inputs(wl)
