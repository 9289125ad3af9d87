"""Context-parallel (ring) prefill: one long sequence split across ranks.

"FlashAttention Explained: How AI Models Process Attention Faster and Use Less
Memory", section "Longer Context Windows": because memory grows linearly with
the sequence, long contexts become feasible; split over several GPUs, each GPU
keeps a slice of the queries and of the keys/values, and the key/value slices
travel round a ring.  Every step a rank attends its query chunks to the
key/value chunks it holds (the tiled forward kernel, fp32 partial output and
LSE), merges the partial result into its running one (the LSE merge used by
split-KV decode, "How FlashAttention Speeds Up LLM Attention": partial results
combined on a common numerical scale) and passes the key/value chunks to the
next rank while the next step's ones arrive from the previous rank.

Sharding is zigzag: the sequence is cut into 2W equal chunks and rank r holds
chunks r and 2W-1-r of Q, K and V, so that under the causal mask every rank
has the same amount of work at every step.  Chunk pairs: key chunk j is
skipped by query chunk i when j > i (causal), attended with the causal mask
when j == i (same positions, so the ordinary causal alignment), in full when
j < i.  Without the mask every pair is attended in full.

The exchange is the only collective: point-to-point sends of this rank's
current K/V chunks to rank r+1 and receives from rank r-1 (NCCL over NVLink on
GPUs), started before the step's compute and waited on after it, into
separate receive buffers.  The forward kernel only ever reads this GPU's own
memory.  ``exchange``, ``attn`` and ``merge`` are parameters so that the host
logic can be exercised with CPU ranks; the defaults are the CUDA kernels.
"""
from __future__ import annotations

from typing import Callable, List, Optional, Sequence, Tuple

import torch


def zigzag_chunk_ids(rank: int, world: int) -> Tuple[int, int]:
    """The two chunk indices (of 2 * world) that ``rank`` holds."""
    return rank, 2 * world - 1 - rank


def zigzag_shard(x: torch.Tensor, rank: int, world: int) -> List[torch.Tensor]:
    """This rank's two chunks of x [B, L, H, D] (L divisible by 2 * world), contiguous."""
    L = x.shape[1]
    if L % (2 * world):
        raise ValueError(f"sequence length {L} is not a multiple of 2 * world ({2 * world})")
    c = L // (2 * world)
    return [x[:, i * c:(i + 1) * c].contiguous() for i in zigzag_chunk_ids(rank, world)]


def zigzag_unshard(chunks_per_rank: Sequence[Sequence[torch.Tensor]], dim: int = 1) -> torch.Tensor:
    """Inverse of zigzag_shard over all ranks: the full tensor along ``dim``."""
    world = len(chunks_per_rank)
    order = [None] * (2 * world)
    for r, (a, b) in enumerate(chunks_per_rank):
        i, j = zigzag_chunk_ids(r, world)
        order[i], order[j] = a, b
    return torch.cat(order, dim=dim)


def pair_mode(i: int, j: int, causal: bool) -> Optional[bool]:
    """How query chunk i meets key chunk j: None (skipped), True (causal mask), False (full)."""
    if not causal:
        return False
    if j > i:
        return None
    return j == i


class P2PExchange:
    """Ring exchange over torch.distributed point-to-point operations.

    ``start(tensors)`` posts the sends of ``tensors`` to rank+1 and the
    receives of as many like-shaped tensors from rank-1 and returns a handle;
    ``finish(handle)`` waits and returns the received tensors.  Every rank
    posts the same operations in the same order.
    """

    def __init__(self, group=None):
        import torch.distributed as dist
        self.dist = dist
        self.group = group
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)

    def start(self, tensors: Sequence[torch.Tensor]):
        dist = self.dist
        nxt = dist.get_global_rank(self.group, (self.rank + 1) % self.world) if self.group else (self.rank + 1) % self.world
        prv = dist.get_global_rank(self.group, (self.rank - 1) % self.world) if self.group else (self.rank - 1) % self.world
        recv = [torch.empty_like(t) for t in tensors]
        ops = [dist.P2POp(dist.isend, t, nxt, self.group) for t in tensors]
        ops += [dist.P2POp(dist.irecv, t, prv, self.group) for t in recv]
        reqs = dist.batch_isend_irecv(ops)
        return reqs, recv

    def finish(self, handle):
        reqs, recv = handle
        for r in reqs:
            r.wait()
        return recv


class LocalRingExchange:
    """The exchange one rank of a W-rank ring would see, served from a list of
    every rank's chunks held in one process (for running all ranks' compute on
    one GPU, one rank after the other; nothing waits on another rank)."""

    def __init__(self, rank: int, world: int, all_kv: Sequence[Sequence[torch.Tensor]]):
        self.rank, self.world, self.all_kv = rank, world, all_kv
        self.step = 0

    def start(self, tensors):
        self.step += 1
        return [t for t in self.all_kv[(self.rank - self.step) % self.world]]

    def finish(self, handle):
        return handle


def _cuda_attn(q, k, v, scale, causal):
    from exact_tiled_attention_46_b200 import fwd
    return fwd(q, k, v, scale=scale, causal=causal, o_dtype=torch.float32)


def _cuda_merge(o_acc, lse_acc, o_new, lse_new):
    from exact_tiled_attention_46_b200 import attn_merge
    attn_merge(o_acc, lse_acc, o_new, lse_new, out=o_acc, lse_out=lse_acc)
    return o_acc, lse_acc


def ring_attention_fwd(q_chunks: Sequence[torch.Tensor], k_chunks: Sequence[torch.Tensor],
                       v_chunks: Sequence[torch.Tensor], rank: int, world: int, scale: float, causal: bool,
                       exchange, attn: Callable = _cuda_attn, merge: Callable = _cuda_merge):
    """This rank's (O, LSE) chunks of the full-sequence attention.

    q_chunks, k_chunks, v_chunks: this rank's two zigzag chunks each
    ([B, c, Hq, D] and [B, c, Hkv, D]).  Returns ([O_a, O_b] fp32 [B, c, Hq, D],
    [LSE_a, LSE_b] [B, Hq, c]).  ``attn(q, k, v, scale, causal)`` returns an
    fp32 (O, LSE) pair; ``merge(o_acc, lse_acc, o, lse)`` folds a partial
    result into the running one and returns it.
    """
    my_ids = zigzag_chunk_ids(rank, world)
    acc: List[Optional[Tuple[torch.Tensor, torch.Tensor]]] = [None, None]
    kv = list(k_chunks) + list(v_chunks)                 # [K_a, K_b, V_a, V_b] of the source rank
    for step in range(world):
        src = (rank - step) % world
        handle = exchange.start(kv) if step + 1 < world else None
        src_ids = zigzag_chunk_ids(src, world)
        for qi, i in enumerate(my_ids):
            for kj, j in enumerate(src_ids):
                mode = pair_mode(i, j, causal)
                if mode is None:
                    continue
                o, lse = attn(q_chunks[qi], kv[kj], kv[2 + kj], scale, mode)
                acc[qi] = (o, lse) if acc[qi] is None else merge(acc[qi][0], acc[qi][1], o, lse)
        if handle is not None:
            kv = list(exchange.finish(handle))
    return [a[0] for a in acc], [a[1] for a in acc]
