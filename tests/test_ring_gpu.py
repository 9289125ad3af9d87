"""Context-parallel (ring) prefill on one GPU: every rank of a W-rank ring run
one after the other (each sees exactly the key/value chunks it would receive),
with the forward kernel per chunk pair and the merge kernel; the gathered
result against the CPU fp64 oracle.  Also the merge kernel alone."""
import math

import numpy as np
import pytest
import torch

import oracle
import exact_tiled_attention_46_b200 as fa
from exact_tiled_attention_46_b200 import inputs as synth, ring

from parity import check_close, check_lse, need_gpu, f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    need_gpu()


def test_merge_kernel_matches_oracle_merge():
    rng = np.random.default_rng(4)
    B, L, H, D = 2, 37, 3, 128
    o_a, o_b = (rng.standard_normal((B, L, H, D)).astype(np.float32) for _ in range(2))
    l_a, l_b = ((rng.standard_normal((B, H, L)) * 5).astype(np.float32) for _ in range(2))
    l_a[0, 1, 3] = -np.inf                   # one side empty
    l_b[1, 2, 7] = -np.inf
    l_a[1, 0, 9] = l_b[1, 0, 9] = -np.inf    # both empty
    ro, rl = oracle.merge_partials(np.stack([o_a, o_b]), np.stack([l_a.transpose(0, 2, 1), l_b.transpose(0, 2, 1)]))
    rl = rl.transpose(0, 2, 1)
    t = lambda x: torch.from_numpy(np.ascontiguousarray(x)).cuda()
    for odt in (torch.float32, torch.bfloat16):
        o, l = fa.attn_merge(t(o_a), t(l_a), t(o_b), t(l_b), o_dtype=odt)
        torch.cuda.synchronize()
        check_close(f64(o), ro, bf16_output=(odt == torch.bfloat16), max_abs=1e-5 if odt == torch.float32 else 1e-2,
                    mean_abs=1e-6 if odt == torch.float32 else 1e-3, what=f"merge {odt}")
        check_lse(f64(l), rl)
    # in place on side a
    oa, la = t(o_a), t(l_a)
    fa.attn_merge(oa, la, t(o_b), t(l_b), out=oa, lse_out=la)
    torch.cuda.synchronize()
    check_close(f64(oa), ro, bf16_output=False, max_abs=1e-5, mean_abs=1e-6, what="merge in place")
    check_lse(f64(la), rl)


@pytest.mark.parametrize("world", [2, 4])
@pytest.mark.parametrize("causal", [True, False])
def test_ring_prefill_emulated_ranks_match_oracle(world, causal):
    B, Hq, Hkv, L, D = 1, 8, 2, 2048, 128
    x = synth.prefill_inputs(B, Hq, Hkv, L, L, D, seed=world * 10 + causal)
    scale = 1.0 / math.sqrt(D)
    q, k, v = (x[n].cuda() for n in ("q", "k", "v"))
    shards = {n: [ring.zigzag_shard(t, r, world) for r in range(world)] for n, t in (("q", q), ("k", k), ("v", v))}
    all_kv = [shards["k"][r] + shards["v"][r] for r in range(world)]
    outs, lses = [], []
    for r in range(world):
        ex = ring.LocalRingExchange(r, world, all_kv)
        o, l = ring.ring_attention_fwd(shards["q"][r], shards["k"][r], shards["v"][r], r, world, scale, causal, ex)
        outs.append(o)
        lses.append(l)
    torch.cuda.synchronize()
    o = f64(ring.zigzag_unshard(outs))
    lse = f64(ring.zigzag_unshard(lses, dim=2))
    xf = {n: synth.as_f64(x[n]) for n in ("q", "k", "v")}
    G = Hq // Hkv
    for h in (0, 5):
        ro, rl = oracle.attn_fwd(xf["q"][:, :, h:h + 1], xf["k"][:, :, h // G:h // G + 1],
                                 xf["v"][:, :, h // G:h // G + 1], scale, causal)
        check_close(o[:, :, h:h + 1], ro, bf16_output=False, what=f"ring O h{h}")
        check_lse(lse[:, h:h + 1], rl, what=f"ring LSE h{h}")
