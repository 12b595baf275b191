"""Run whole fwd -> loss -> bwd steps on one synthetic problem (for profilers).

    python -m rope_attention_fwd_b200.profile_step --B 2 --H 16 --n 8192 --d 128 --causal \
        [--steps 1] [--warmup 1]

Inputs are N(0,1) bf16 drawn on the device (profiling needs the launch sequence, not
parity).  Prints the per-kernel event times of the last step.
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
    a = ap.parse_args()
    g = torch.Generator(device="cuda").manual_seed(0)
    shape = (a.B, a.H, a.n, a.d)
    q, k, v, e = (torch.randn(shape, device="cuda", generator=g).to(torch.bfloat16)
                  for _ in range(4))
    alpha = 0.3 * torch.randn(a.d // 2, device="cuda", generator=g)
    ws = rb.workspace(rb.problem(a.B, a.H, a.n, a.d, torch.bfloat16, a.causal, a.base), "cuda")

    def step():
        o, lse = rb.rope_attn_fwd(q, k, v, alpha, a.base, a.causal, ws=ws)
        L, dO = rb.rope_attn_loss(o, e, ws=ws)
        return rb.rope_attn_bwd_saved(v, o, lse, dO, alpha, a.base, a.causal, ws)

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
    code, info = rb.rope_attn_device_status(ws)
    if code != 0:
        raise SystemExit(f"device status {rb.STATUS.get(code, code)} {info}")


if __name__ == "__main__":
    main()
