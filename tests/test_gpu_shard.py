"""The (batch, head) sharding of the multi-GPU path, run through the C ABI on one GPU.

dist.shard_bh gives each rank a contiguous share of the B*H units; a share is the
[1, count, n, d] problem that starts at unit `start` of the [B, H, n, d] tensors.  Here two
shards are run one after the other on the same GPU and their outputs and summed dalpha are
compared with one unsharded call.  The kernels treat every (batch, head) on its own, so O,
lse and dV agree bit for bit.  dQ and dK agree to within the fp16 rounding of dS: its
power-of-two scale comes from max |dO_i| and max |v_j| over the whole call, which a shard
sees only for its own heads.  dalpha is a sum over every head, and the two shards' fp32
dalphas are summed in fp64 as dist.allreduce_sum does across ranks."""
import pytest
import torch

from helpers import make, rel_frob, small_workload, to64
from rope_attention_fwd_b200 import binding as rb
from rope_attention_fwd_b200.dist import shard_bh

pytestmark = pytest.mark.gpu


def _run(q, k, v, e, alpha, base, causal):
    o, lse = rb.rope_attn_fwd(q, k, v, alpha, base, causal)
    _, dO = rb.rope_attn_loss(o, e)
    dq, dk, dv, dalpha = rb.rope_attn_bwd(q, k, v, o, lse, dO, alpha, base, causal)
    return dict(o=o, lse=lse, dq=dq, dk=dk, dv=dv, dalpha=dalpha)


@pytest.mark.parametrize("causal", [False, True])
def test_two_shards_equal_the_whole(causal):
    wl = small_workload(2, 3, 300, 128, "bf16", causal, seed=41)
    inp = make(wl)
    t = {x: getattr(inp, x).cuda() for x in ("q", "k", "v", "e", "alpha")}
    whole = _run(t["q"], t["k"], t["v"], t["e"], t["alpha"], wl.base, causal)
    flat = {x: t[x].reshape(1, wl.B * wl.H, wl.n, wl.d) for x in ("q", "k", "v", "e")}
    parts, da = [], torch.zeros(wl.d // 2, dtype=torch.float64, device="cuda")
    for rank in range(2):
        start, count = shard_bh(wl.B, wl.H, 2, rank)
        sl = {x: flat[x][:, start:start + count].contiguous() for x in flat}
        r = _run(sl["q"], sl["k"], sl["v"], sl["e"], t["alpha"], wl.base, causal)
        parts.append(r)
        da += r["dalpha"].double()  # rank order, fp64
    joined = {x: torch.cat([p[x] for p in parts], dim=1).reshape(whole[x].shape)
              for x in ("o", "lse", "dq", "dk", "dv")}
    for x in ("o", "lse", "dv"):
        assert torch.equal(joined[x], whole[x]), x
    for x in ("dq", "dk"):
        assert rel_frob(to64(joined[x]), to64(whole[x])) <= 2e-3, x
    assert rel_frob(to64(da), to64(whole["dalpha"])) <= 2e-3
