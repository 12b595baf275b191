"""The binding's argument checks, on the CPU with a stand-in for the library: every wrapper
passes well-formed tensors (the shapes the GPU tests, smoke() and bench.py use) through to
its C entry point, and refuses a non-contiguous view, a tensor of the wrong size or one on
another device before any call is made (the C ABI takes raw pointers and cannot tell)."""
import ctypes

import pytest
import torch

from rope_attention_fwd_b200 import binding as rb


class FakeLib:
    """Records each C call; the calls return RA_OK, the size queries 1024."""

    def __init__(self):
        self.calls = []

    def __getattr__(self, name):
        def call(*args):
            self.calls.append(name)
            return 1024 if name.endswith("_workspace_bytes") else 0
        return call


@pytest.fixture
def fake(monkeypatch):
    f = FakeLib()
    monkeypatch.setattr(rb, "lib", lambda: f)
    monkeypatch.setattr(rb, "_stream", lambda device: ctypes.c_void_p(0))
    return f


def _attn(B=2, H=3, n=40, d=64, dtype=torch.bfloat16):
    t = {x: torch.zeros((B, H, n, d), dtype=dtype) for x in ("q", "k", "v", "e", "o", "dO")}
    t["alpha"] = torch.zeros(d // 2)
    t["lse"] = torch.zeros((B, H, n))
    t["ws"] = torch.zeros(1024, dtype=torch.uint8)
    return t


def test_well_formed_calls_reach_the_library(fake):
    t = _attn()
    rb.rope_attn_fwd(t["q"], t["k"], t["v"], t["alpha"], 1e4, True, ws=t["ws"])
    rb.rope_attn_loss(t["o"], t["e"], ws=t["ws"])
    rb.rope_attn_bwd(t["q"], t["k"], t["v"], t["o"], t["lse"], t["dO"], t["alpha"], 1e4, True,
                     ws=t["ws"])
    rb.rope_attn_bwd_saved(t["v"], t["o"], t["lse"], t["dO"], t["alpha"], 1e4, True, t["ws"])
    rb.rope_attn_bwd(t["q"], t["k"], t["v"], t["o"], t["lse"], t["dO"], t["alpha"], 1e4, True,
                     ws=t["ws"], frozen_alpha=True)
    rb.rope_attn_spectrum(t["q"], t["k"], t["v"], t["o"], t["lse"], t["dO"], t["alpha"], 1e4,
                          True)
    x = torch.zeros((2, 40, 96), dtype=torch.bfloat16)
    w = [torch.zeros((96, 3 * 64), dtype=torch.bfloat16) for _ in range(3)]
    q, k, v = rb.rope_attn_proj_fwd(x, *w, 3)
    rb.rope_attn_proj_bwd(x, *w, q, k, v)
    m = [torch.zeros(32) for _ in range(4)]
    rb.rope_attn_alpha_adam(*m, 1, 1e-3)
    rb.rope_attn_device_status(t["ws"])
    assert fake.calls.count("rope_attn_fwd") == 1 and fake.calls.count("rope_attn_bwd") == 2
    for name in ("rope_attn_loss", "rope_attn_bwd_saved", "rope_attn_spectrum",
                 "rope_attn_proj_fwd", "rope_attn_proj_bwd", "rope_attn_alpha_adam",
                 "rope_attn_device_status"):
        assert name in fake.calls, name


def test_malformed_tensors_are_refused_before_any_call(fake):
    t = _attn()
    q, k, v, alpha, ws = t["q"], t["k"], t["v"], t["alpha"], t["ws"]
    bad_view = torch.zeros((2, 3, 64, 40), dtype=torch.bfloat16).transpose(2, 3)  # same shape
    assert bad_view.shape == k.shape and not bad_view.is_contiguous()
    cases = [
        lambda: rb.rope_attn_fwd(q, bad_view, v, alpha, 1e4, True, ws=ws),
        lambda: rb.rope_attn_fwd(q, k, v[:, :, :20], alpha, 1e4, True, ws=ws),
        lambda: rb.rope_attn_fwd(q, k, v, alpha[:8], 1e4, True, ws=ws),
        lambda: rb.rope_attn_fwd(q, k, v, alpha, 1e4, True, ws=ws,
                                 lse=torch.zeros((2, 3, 39))),
        lambda: rb.rope_attn_fwd(q, k, v.to("meta"), alpha, 1e4, True, ws=ws),
        lambda: rb.rope_attn_loss(t["o"], t["e"][:1], ws=ws),
        lambda: rb.rope_attn_bwd(q, k, v, t["o"], t["lse"], bad_view, alpha, 1e4, True, ws=ws),
        lambda: rb.rope_attn_bwd_saved(v, t["o"], t["lse"], t["dO"], alpha, 1e4, True, ws,
                                       dq=torch.zeros(7, dtype=torch.bfloat16)),
        lambda: rb.rope_attn_alpha_adam(alpha, alpha[:4], alpha.clone(), alpha.clone(), 1, 1e-3),
    ]
    for case in cases:
        with pytest.raises(ValueError):
            case()
    assert fake.calls == []
