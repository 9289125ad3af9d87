"""Host logic of context-parallel (ring) prefill on CPU ranks (gloo).

The per-shard attention and the merge are CPU stand-ins built from the oracle
(passed in as parameters); what is checked is the zigzag sharding, the ring
schedule (which rank holds which key/value chunks at which step), the causal
pair rules and the point-to-point exchange: gathered over the ranks, the result
must equal the oracle's one-shot attention over the whole sequence.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from exact_tiled_attention_46_b200 import ring


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def cpu_attn(q, k, v, scale, causal):
    o, lse = oracle.attn_fwd(q.numpy(), k.numpy(), v.numpy(), scale, causal)
    return torch.from_numpy(o), torch.from_numpy(lse)


def cpu_merge(o_a, lse_a, o_b, lse_b):
    # oracle.merge_partials wants [S, ..., D] / [S, ...]; LSE rows are [B, H, L], O rows [B, L, H, D]
    la, lb = lse_a.permute(0, 2, 1).numpy(), lse_b.permute(0, 2, 1).numpy()
    o, lse = oracle.merge_partials(np.stack([o_a.numpy(), o_b.numpy()]), np.stack([la, lb]))
    return torch.from_numpy(o), torch.from_numpy(lse).permute(0, 2, 1).contiguous()


def full_inputs(seed, B=2, L=24, Hq=4, Hkv=2, D=8):
    g = torch.Generator().manual_seed(seed)
    return [torch.randn(B, L, h, D, dtype=torch.float64, generator=g) for h in (Hq, Hkv, Hkv)]


def test_zigzag_shard_roundtrip_and_balance():
    x = torch.arange(2 * 24 * 3).reshape(2, 24, 3, 1)
    for world in (1, 2, 3, 4):
        parts = [ring.zigzag_shard(x, r, world) for r in range(world)]
        assert torch.equal(ring.zigzag_unshard(parts), x)
        # causal work per rank (allowed chunk pairs) is the same on every rank
        work = []
        for r in range(world):
            mine = ring.zigzag_chunk_ids(r, world)
            work.append(sum(1 for i in mine for j in range(2 * world) if ring.pair_mode(i, j, True) is not None))
        assert len(set(work)) == 1


def test_pair_rules():
    assert ring.pair_mode(3, 5, True) is None
    assert ring.pair_mode(3, 3, True) is True
    assert ring.pair_mode(3, 1, True) is False
    assert ring.pair_mode(1, 3, False) is False


def test_single_rank_ring_equals_one_shot():
    q, k, v = full_inputs(5)
    ex = ring.LocalRingExchange(0, 1, [ring.zigzag_shard(k, 0, 1) + ring.zigzag_shard(v, 0, 1)])
    o, lse = ring.ring_attention_fwd(ring.zigzag_shard(q, 0, 1), ring.zigzag_shard(k, 0, 1),
                                     ring.zigzag_shard(v, 0, 1), 0, 1, 0.3, True, ex, cpu_attn, cpu_merge)
    ro, rl = oracle.attn_fwd(q.numpy(), k.numpy(), v.numpy(), 0.3, True)
    np.testing.assert_allclose(ring.zigzag_unshard([o]).numpy(), ro, atol=1e-12)
    np.testing.assert_allclose(ring.zigzag_unshard([lse], dim=2).numpy(), rl, atol=1e-12)


def _rank(rank, world, port, causal, q_out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        q, k, v = full_inputs(7)          # every rank draws the same full tensors, keeps its shards
        ex = ring.P2PExchange()
        o, lse = ring.ring_attention_fwd(ring.zigzag_shard(q, rank, world), ring.zigzag_shard(k, rank, world),
                                         ring.zigzag_shard(v, rank, world), rank, world, 0.35, causal, ex,
                                         cpu_attn, cpu_merge)
        q_out.put((rank, [t.numpy() for t in o], [t.numpy() for t in lse]))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
@pytest.mark.parametrize("causal", [True, False])
def test_ring_over_gloo_ranks_equals_one_shot(world, causal):
    ctx = mp.get_context("spawn")
    q_out = ctx.Queue()
    mp.spawn(_rank, args=(world, free_port(), causal, q_out), nprocs=world, join=True)
    got = sorted((q_out.get(timeout=60) for _ in range(world)), key=lambda t: t[0])
    o = ring.zigzag_unshard([[torch.from_numpy(a) for a in g[1]] for g in got])
    lse = ring.zigzag_unshard([[torch.from_numpy(a) for a in g[2]] for g in got], dim=2)
    q, k, v = full_inputs(7)
    ro, rl = oracle.attn_fwd(q.numpy(), k.numpy(), v.numpy(), 0.35, causal)
    np.testing.assert_allclose(o.numpy(), ro, atol=1e-12)
    np.testing.assert_allclose(lse.numpy(), rl, atol=1e-12)
