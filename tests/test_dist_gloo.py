"""The multi-rank host path on CPU (gloo): each rank draws its own batch, computes its
dalpha and loss L (the float64 oracle stands in for the GPU kernels here), and the
deterministic all-gather reduction must give the dalpha and L of the union of every rank's
heads, bit for bit the rank-order sum, on every rank; the (batch, head) sharding covers
every unit once."""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from rope_attention_fwd_b200.configs import Workload
from rope_attention_fwd_b200.dist import allreduce_sum, rank_seed, shard_bh
from rope_attention_fwd_b200.inputs import make_inputs

WL = Workload("dist 1x2x24x8", 1, 2, 24, 8, "f32", True, 100.0, "normal", alpha="normal",
              alpha_a=0.4, seed=31)


def _oracle(seed):
    from oracle import rope_attn_ref as ref
    inp = make_inputs(WL, seed=seed)
    return ref.forward_backward(inp.f64("q"), inp.f64("k"), inp.f64("v"), inp.f64("e"),
                                inp.f64("alpha"), WL.base, WL.causal)


def _dalpha(seed):
    return _oracle(seed)["dalpha"]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        r = _oracle(rank_seed(WL.seed, rank))
        da = torch.tensor(r["dalpha"], dtype=torch.float64)
        L = torch.tensor(r["L"], dtype=torch.float64)  # a 0-d tensor, like the bench's L
        allreduce_sum(da)
        allreduce_sum(L)
        out[rank] = da.numpy().copy()
        out[("L", rank)] = float(L)
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_dalpha_allreduce_two_ranks():
    world = 2
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
        res = dict(out)
    expect = sum(_dalpha(rank_seed(WL.seed, r)) for r in range(world))
    expect_L = sum(_oracle(rank_seed(WL.seed, r))["L"] for r in range(world))
    for r in range(world):
        np.testing.assert_allclose(res[r], expect, rtol=1e-12, atol=1e-14)
        # the loss is a sum over every head of every rank too
        assert abs(res[("L", r)] - expect_L) <= 1e-12 * expect_L
    # the ranks' batches differ (independent heads), so each rank contributes
    assert not np.allclose(_dalpha(rank_seed(WL.seed, 0)), _dalpha(rank_seed(WL.seed, 1)))


def test_single_process_is_a_noop():
    da = torch.arange(4, dtype=torch.float32)
    assert torch.equal(allreduce_sum(da.clone()), da)


def _worker_f32(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        g = torch.Generator().manual_seed(1000 + rank)
        da = (torch.randn(64, generator=g) * 10 ** (rank % 3)).to(torch.float32)
        out[("in", rank)] = da.numpy().copy()
        allreduce_sum(da)
        out[("out", rank)] = da.numpy().copy()
    finally:
        dist.destroy_process_group()


def test_dalpha_reduction_is_bitwise_rank_order_sum():
    """Three ranks of fp32 partials of very different magnitudes: every rank ends with the
    same bits, the float64 rank-order sum rounded once to fp32."""
    world = 3
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker_f32, args=(world, _free_port(), out), nprocs=world, join=True)
        res = dict(out)
    acc = np.zeros(64)
    for r in range(world):
        acc += res[("in", r)].astype(np.float64)
    expect = acc.astype(np.float32)
    for r in range(world):
        assert np.array_equal(res[("out", r)], expect), r


def test_shard_bh_covers_every_unit_once():
    for B, H, world in ((2, 32, 8), (3, 5, 4), (1, 7, 8), (4, 16, 3)):
        seen = []
        counts = []
        for r in range(world):
            start, count = shard_bh(B, H, world, r)
            seen.extend(range(start, start + count))
            counts.append(count)
        assert seen == list(range(B * H)), (B, H, world)
        assert max(counts) - min(counts) <= 1
