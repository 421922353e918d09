"""Head sharding across ranks (codechina FlashAttention article, §6.3 multi-GPU scaling:
partition by attention heads): the partition, the gather of head shards and the
max-over-ranks timing reduction, with world_size-2 gloo process groups on CPU; and,
on one GPU, that the ranks' local kernel calls reproduce the whole-tensor call.
"""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp

from exact_attention_123_b200.sharding import gather_heads, head_range, max_over_ranks


@pytest.mark.parametrize("H", [1, 2, 3, 7, 16, 17, 32])
@pytest.mark.parametrize("world", [1, 2, 3, 4, 8])
def test_head_range_partitions_every_head_once(H, world):
    got, sizes = [], []
    for r in range(world):
        h0, h1 = head_range(H, world, r)
        got += list(range(h0, h1))
        sizes.append(h1 - h0)
    assert got == list(range(H))                      # contiguous, in order, each head once
    assert max(sizes) - min(sizes) <= 1               # balanced


def test_head_range_rejects_bad_requests():
    for args in ((0, 2, 0), (4, 0, 0), (4, 2, 2), (4, 2, -1)):
        with pytest.raises(ValueError):
            head_range(*args)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, H_list):
    import torch.distributed as dist
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        for H in H_list:
            full = torch.arange(2 * H * 3 * 4, dtype=torch.float32).reshape(2, H, 3, 4)
            h0, h1 = head_range(H, world, rank)
            got = gather_heads(full[:, h0:h1].contiguous(), H)
            assert torch.equal(got, full), (rank, H)
        assert max_over_ranks(1.5 + rank) == 1.5 + (world - 1)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2])
def test_gather_heads_and_max_over_ranks_gloo(world):
    mp.spawn(_worker, args=(world, _free_port(), [1, 2, 3, 5, 16]), nprocs=world, join=True)


def test_max_over_ranks_without_a_process_group():
    assert max_over_ranks(3.25) == 3.25


@pytest.mark.gpu
@pytest.mark.parametrize("world", [2, 3])
def test_sharded_ranks_reproduce_the_whole_tensor(world):
    # the ranks' local calls, run one after the other on one GPU, against one call on
    # all heads: each head's result is the same computation, so (with the
    # deterministic backward) equal bit for bit; and every shard against the oracle
    import numpy as np

    import oracle
    from exact_attention_123_b200 import build
    build.build()
    import exact_attention_123_b200 as ea
    from exact_attention_123_b200.sharding import attn_bwd_sharded, attn_fwd_sharded, head_range
    from attn_inputs import make_dense
    inp = make_dense(2, 5, 300, 128, seed=9400, causal=True, with_grad=True)
    q, k, v, do = (t.cuda() for t in (inp.q, inp.k, inp.v, inp.do))
    o, lse = ea.attn_fwd(q, k, v, scale=inp.scale, causal=True)
    dq, dk, dv = ea.attn_bwd(q, k, v, o, lse, do, scale=inp.scale, causal=True, deterministic=True)
    parts = []
    for r in range(world):
        ol, ll = attn_fwd_sharded(q, k, v, world=world, rank=r, scale=inp.scale, causal=True)
        gl = attn_bwd_sharded(q, k, v, ol, ll, do, world=world, rank=r, scale=inp.scale, causal=True,
                              deterministic=True)
        parts.append((ol, ll) + tuple(gl))
    for i, full in enumerate((o, lse, dq, dk, dv)):
        assert torch.equal(torch.cat([p_[i] for p_ in parts], dim=1), full)
    assert ea.attn_status() == ea.ATTN_OK
    # each rank's shard, as the fast backward computes it, against the float64 oracle on
    # that rank's heads (the parity tests' bands)
    ro, rl = oracle.fwd(inp.q, inp.k, inp.v, inp.scale, True)
    rg = oracle.bwd(inp.q, inp.k, inp.v, inp.do, inp.scale, True)
    for r in range(world):
        h0, h1 = head_range(5, world, r)
        ol, ll = attn_fwd_sharded(q, k, v, world=world, rank=r, scale=inp.scale, causal=True)
        gl = attn_bwd_sharded(q, k, v, ol, ll, do, world=world, rank=r, scale=inp.scale, causal=True)
        checks = [(ol, ro, 1e-2, 1e-2), (ll, rl, 1e-3, 0.0)] + [(g, x, 2e-2, 2e-2) for g, x in zip(gl, rg)]
        for got, ref, atol, rtol in checks:
            g = got.double().cpu().numpy()
            want = ref[:, h0:h1]
            assert np.all(np.isfinite(g))
            assert not (np.abs(g - want) > atol + rtol * np.abs(want)).any(), (r, h0, h1)
    assert ea.attn_status() == ea.ATTN_OK
