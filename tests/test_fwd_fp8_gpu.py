"""FP8 (e4m3) forward vs the CPU fp64 oracle run on the e4m3-rounded inputs (GPU).

The oracle computes the plain definition on the dequantized inputs (e4m3 value
times the tensor's scale), so Q K^T, the softmax and the LSE must agree within
the usual tolerances; O additionally carries the rounding of P to e4m3, held
to the per-element bound derived in parity.py (fp8_o_bound).
"""
import math

import numpy as np
import pytest
import torch

import oracle
import exact_tiled_attention_46_b200 as fa
from exact_tiled_attention_46_b200 import inputs as synth

from parity import check_fp8_o, check_lse, fp8_o_bound, need_gpu, f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    need_gpu()


def deq(x):
    return {n: synth.dequant_f64(x[n], x[n + "_scale"]) for n in ("q", "k", "v")}


def run_fp8(x, scale, causal, odt):
    q, k, v = (x[n].cuda() for n in ("q", "k", "v"))
    B, Lq, Hq, D = q.shape
    out = torch.full((B, Lq, Hq, D), float("nan"), dtype=odt, device="cuda")
    lse = torch.full((B, Hq, Lq), float("nan"), dtype=torch.float32, device="cuda")
    fa.fwd_fp8(q, k, v, x["q_scale"], x["k_scale"], x["v_scale"], scale=scale, causal=causal, out=out, lse=lse)
    torch.cuda.synchronize()
    return f64(out), f64(lse)


def check_head(o_gpu, l_gpu, xf, b, h, scale, causal, bf16):
    """One (batch, head) against the oracle, O within the e4m3-P bound."""
    G = xf["q"].shape[2] // xf["k"].shape[2]
    qs, ks, vs = xf["q"][b:b + 1, :, h:h + 1], xf["k"][b:b + 1, :, h // G:h // G + 1], xf["v"][b:b + 1, :, h // G:h // G + 1]
    ro, rl = oracle.attn_fwd(qs, ks, vs, scale, causal)
    w = oracle.attn_probs(qs, ks, scale, causal)[0, 0]
    Lq, Lk = w.shape
    bound = fp8_o_bound(w, oracle.allowed_mask(Lq, Lk, causal), vs[0, :, 0], ro[0, :, 0])
    check_fp8_o(o_gpu[b, :, h], ro[0, :, 0], bound, bf16, what=f"O fp8 {'bf16' if bf16 else 'fp32'} b{b} h{h}")
    check_lse(l_gpu[b:b + 1, h:h + 1], rl, what=f"LSE fp8 b{b} h{h}")


CASES = [
    # B, Hq, Hkv, Lq, Lk, causal, boost
    (1, 2, 2, 127, 127, True, 0),
    (1, 2, 1, 129, 129, False, 0),
    (1, 3, 3, 256, 256, True, 1),
    (1, 8, 2, 1000, 1000, True, 4),
    (1, 4, 4, 300, 700, True, 0),      # Lq < Lk
    (1, 4, 4, 700, 300, True, 0),      # Lq > Lk: rows without keys
    (1, 8, 1, 512, 384, False, 0),
    (1, 2, 2, 257, 1, False, 0),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "B%dHq%dHkv%dLq%dLk%d%s_boost%d" % (*c[:5], "c" if c[5] else "n", c[6]))
def test_fwd_fp8_matches_oracle(case):
    B, Hq, Hkv, Lq, Lk, causal, boost = case
    x = synth.prefill_inputs_fp8(B, Hq, Hkv, Lq, Lk, 128, seed=sum(case[:5]) + 3, q_boost_heads=boost)
    scale = 1.0 / math.sqrt(128)
    xf = deq(x)
    for odt in (torch.float32, torch.bfloat16):
        o, l = run_fp8(x, scale, causal, odt)
        for b in range(B):
            for h in range(Hq):
                check_head(o, l, xf, b, h, scale, causal, odt == torch.bfloat16)


def test_fwd_fp8_causal_prefill_workload_sampled_heads():
    """B4 H16 L2048 D128 causal, Q x4 on heads 0-7 (the causal prefill draws,
    seed 1, quantized to e4m3): three whole heads, two of them boosted."""
    w = synth.WORKLOADS["causal_prefill"]
    x = synth.prefill_inputs_fp8(w.B, w.Hq, w.Hkv, w.Lq, w.Lk, w.D, w.seed, q_boost_heads=w.q_boost_heads)
    o, l = run_fp8(x, w.scale, True, torch.float32)
    xf = deq(x)
    for b, h in [(0, 0), (1, 7), (3, 12)]:
        check_head(o, l, xf, b, h, w.scale, True, False)


def test_fwd_fp8_rejects_other_head_dims():
    q = torch.zeros(1, 8, 1, 64, dtype=torch.float8_e4m3fn, device="cuda")
    with pytest.raises(fa.FaError) as e:
        fa.fwd_fp8(q, q, q, 1.0, 1.0, 1.0)
    assert e.value.status == fa.FA_ERR_UNSUPPORTED
