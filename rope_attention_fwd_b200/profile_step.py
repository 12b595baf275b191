"""Run whole fwd -> loss -> bwd steps on one synthetic problem (for profilers).

    python -m rope_attention_fwd_b200.profile_step --B 2 --H 16 --n 8192 --d 128 --causal \
        [--steps 1] [--warmup 1] [--d-model 4096]

Inputs are N(0,1) bf16 drawn on the device (profiling needs the launch sequence, not
parity).  Prints the per-kernel event times of the last step.  With --d-model > 0 each step
also runs the projections around the path (q, k, v = x W before, dW and dx after, cuBLAS)
and prints their CUDA-event times and TFLOP/s (2 B n d_model H d per product).
"""
import argparse

import torch

from . import binding as rb


def main():
    ap = argparse.ArgumentParser()
    for name, default in (("B", 2), ("H", 16), ("n", 8192), ("d", 128)):
        ap.add_argument(f"--{name}", type=int, default=default)
    ap.add_argument("--causal", action="store_true")
    ap.add_argument("--base", type=float, default=1e4)
    ap.add_argument("--steps", type=int, default=1)
    ap.add_argument("--warmup", type=int, default=1)
    ap.add_argument("--d-model", type=int, default=0)
    a = ap.parse_args()
    g = torch.Generator(device="cuda").manual_seed(0)
    shape = (a.B, a.H, a.n, a.d)
    q, k, v, e = (torch.randn(shape, device="cuda", generator=g).to(torch.bfloat16)
                  for _ in range(4))
    alpha = 0.3 * torch.randn(a.d // 2, device="cuda", generator=g)
    ws = rb.workspace(rb.problem(a.B, a.H, a.n, a.d, torch.bfloat16, a.causal, a.base), "cuda")

    proj_ms = {"proj_fwd": 0.0, "proj_bwd": 0.0}
    if a.d_model > 0:
        x = torch.randn((a.B, a.n, a.d_model), device="cuda", generator=g).to(torch.bfloat16)
        w = [(torch.randn((a.d_model, a.H * a.d), device="cuda", generator=g)
              * a.d_model ** -0.5).to(torch.bfloat16) for _ in range(3)]

    def timed(name, fn):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        out = fn()
        e1.record()
        e1.synchronize()
        proj_ms[name] = e0.elapsed_time(e1)
        return out

    def step():
        qq, kk, vv = (q, k, v) if a.d_model <= 0 else timed(
            "proj_fwd", lambda: rb.rope_attn_proj_fwd(x, *w, a.H))
        o, lse = rb.rope_attn_fwd(qq, kk, vv, alpha, a.base, a.causal, ws=ws)
        L, dO = rb.rope_attn_loss(o, e, ws=ws)
        grads = rb.rope_attn_bwd_saved(vv, o, lse, dO, alpha, a.base, a.causal, ws)
        if a.d_model > 0:
            timed("proj_bwd", lambda: rb.rope_attn_proj_bwd(x, *w, *grads[:3]))
        return grads

    for _ in range(a.warmup):
        step()
    torch.cuda.synchronize()
    rb.rope_attn_timing_read()
    rb.rope_attn_timing_enable(True)
    for _ in range(a.steps):
        step()
    torch.cuda.synchronize()
    rb.rope_attn_timing_enable(False)
    for name, (cnt, ms) in rb.rope_attn_timing_read().items():
        print(f"{name:16s} {cnt:3d} launches {ms / cnt:8.3f} ms")
    if a.d_model > 0:
        prod = 2.0 * a.B * a.n * a.d_model * a.H * a.d  # FLOPs of one x W product
        for name, nprod in (("proj_fwd", 3), ("proj_bwd", 6)):
            ms = proj_ms[name]
            print(f"{name:16s}   1 launches {ms:8.3f} ms  {nprod * prod / (ms * 1e-3) / 1e12:7.1f} TFLOP/s")
    code, info = rb.rope_attn_device_status(ws)
    if code != 0:
        raise SystemExit(f"device status {rb.STATUS.get(code, code)} {info}")


if __name__ == "__main__":
    main()
