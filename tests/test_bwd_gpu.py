"""Backward kernels vs the CPU fp64 oracle gradients (GPU)."""
import math

import numpy as np
import pytest
import torch

import oracle
import exact_tiled_attention_46_b200 as fa
from exact_tiled_attention_46_b200 import inputs as synth

from parity import check_close, check_lse, need_gpu, f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    need_gpu()


def gpu_grads(x, scale, causal, grad_dtype):
    q, k, v, do = (x[n].cuda() for n in ("q", "k", "v", "do"))
    o, lse = fa.fwd(q, k, v, scale=scale, causal=causal)
    dq, dk, dv = fa.bwd(q, k, v, o, do, lse, scale=scale, causal=causal, grad_dtype=grad_dtype)
    torch.cuda.synchronize()
    return f64(dq), f64(dk), f64(dv)


CASES = [
    # B, Hq, Hkv, Lq, Lk, D, causal
    (1, 2, 2, 128, 128, 64, True),
    (1, 2, 1, 200, 200, 64, True),
    (2, 4, 2, 255, 255, 64, False),
    (1, 2, 2, 384, 384, 64, True),
    (1, 4, 1, 256, 512, 64, True),      # Lq < Lk
    (1, 2, 2, 300, 100, 64, True),      # Lq > Lk: queries without keys
    (1, 2, 2, 300, 300, 128, True),
    (1, 4, 2, 129, 257, 128, False),
    (1, 1, 1, 1, 1, 64, False),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "B%dHq%dHkv%dLq%dLk%dD%d%s" % (*c[:6], "c" if c[6] else "n"))
def test_bwd_matches_oracle(case):
    B, Hq, Hkv, Lq, Lk, D, causal = case
    x = synth.prefill_inputs(B, Hq, Hkv, Lq, Lk, D, seed=sum(case) + 7, with_do=True)
    scale = 1.0 / math.sqrt(D)
    xf = {n: synth.as_f64(x[n]) for n in x}
    rq, rk, rv, *_ = oracle.attn_bwd(xf["q"], xf["k"], xf["v"], xf["do"], scale, causal)
    for gdt in (torch.float32, torch.bfloat16):
        dq, dk, dv = gpu_grads(x, scale, causal, gdt)
        bf = gdt == torch.bfloat16
        check_close(dv, rv, bf16_output=bf, what=f"dV {gdt}")
        check_close(dk, rk, bf16_output=bf, what=f"dK {gdt}")
        check_close(dq, rq, bf16_output=bf, what=f"dQ {gdt}")


def test_bwd_power_of_two_input_scales():
    """The products run on fp16 after each input tensor is scaled by a power of
    two chosen from its largest magnitude.  Scaling the caller's q, k, v, dO by
    powers of two (o follows exactly, the LSE is unchanged) must therefore give
    the same fp16 operands and gradients scaled exactly: dV by dO's factor, dK
    by the product of dO's, V's and Q's, dQ by that of dO's, V's and K's.  dK
    and dV are bit-identical (fixed accumulation order); dQ is summed by
    reductions in any order.  dO at 2^-20 of unit scale would be subnormal in
    an unscaled fp16 copy."""
    B, Hq, Hkv, Lq, Lk, D, causal = 1, 2, 1, 200, 200, 64, True
    x = synth.prefill_inputs(B, Hq, Hkv, Lq, Lk, D, seed=11, with_do=True)
    scale = 1.0 / math.sqrt(D)
    eq, ek, ev, edo = -10, 10, 12, -20
    q, k, v, do = (x[n].cuda() for n in ("q", "k", "v", "do"))
    o, lse = fa.fwd(q, k, v, scale=scale, causal=causal)
    dq, dk, dv = fa.bwd(q, k, v, o, do, lse, scale=scale, causal=causal, grad_dtype=torch.float32)
    qs, ks, vs, dos, os_ = q * 2.0 ** eq, k * 2.0 ** ek, v * 2.0 ** ev, do * 2.0 ** edo, o * 2.0 ** ev
    for a, b_, e in ((qs, q, eq), (ks, k, ek), (vs, v, ev), (dos, do, edo), (os_, o, ev)):
        assert a.dtype == torch.bfloat16 and torch.equal(a.float(), b_.float() * 2.0 ** e)   # exact in bf16
    dq2, dk2, dv2 = fa.bwd(qs, ks, vs, os_, dos, lse, scale=scale, causal=causal, grad_dtype=torch.float32)
    torch.cuda.synchronize()
    assert torch.equal(dv2, dv * 2.0 ** edo)
    assert torch.equal(dk2, dk * 2.0 ** (edo + ev + eq))
    torch.testing.assert_close(dq2, dq * 2.0 ** (edo + ev + ek), rtol=1e-5, atol=0.0)
    # and against the oracle on the scaled inputs, errors measured at unit scale
    xf = {n: synth.as_f64(x[n]) for n in x}
    xf["q"] = xf["q"] * 2.0 ** eq; xf["k"] = xf["k"] * 2.0 ** ek
    xf["v"] = xf["v"] * 2.0 ** ev; xf["do"] = xf["do"] * 2.0 ** edo
    rq, rk, rv, *_ = oracle.attn_bwd(xf["q"], xf["k"], xf["v"], xf["do"], scale, causal)
    check_close(f64(dv2) / 2.0 ** edo, rv / 2.0 ** edo, bf16_output=False, what="dV scaled inputs")
    check_close(f64(dk2) / 2.0 ** (edo + ev + eq), rk / 2.0 ** (edo + ev + eq), bf16_output=False, what="dK scaled inputs")
    check_close(f64(dq2) / 2.0 ** (edo + ev + ek), rq / 2.0 ** (edo + ev + ek), bf16_output=False, what="dQ scaled inputs")


def test_bwd_zero_and_nan_gradients():
    """Input scales come from each tensor's largest magnitude: an all-zero dO
    (largest magnitude 0, no scaling) gives exactly zero gradients, and a NaN
    in dO gives non-finite gradients of its head, with the call itself fine."""
    B, Hq, Hkv, Lq, Lk, D = 1, 2, 1, 130, 130, 64
    x = synth.prefill_inputs(B, Hq, Hkv, Lq, Lk, D, seed=5, with_do=True)
    q, k, v, do = (x[n].cuda() for n in ("q", "k", "v", "do"))
    o, lse = fa.fwd(q, k, v, causal=True)
    dq, dk, dv = fa.bwd(q, k, v, o, torch.zeros_like(do), lse, causal=True, grad_dtype=torch.float32)
    torch.cuda.synchronize()
    assert torch.count_nonzero(dq) == 0 and torch.count_nonzero(dk) == 0 and torch.count_nonzero(dv) == 0
    bad = do.clone()
    bad[0, 7, 1, 3] = float("nan")
    dq, dk, dv = fa.bwd(q, k, v, o, bad, lse, causal=True, grad_dtype=torch.float32)
    torch.cuda.synchronize()
    assert not torch.isfinite(dv).all() and not torch.isfinite(dq).all()


def test_bwd_empty_queries():
    k = torch.randn(1, 64, 2, 64, device="cuda").to(torch.bfloat16)
    q = torch.empty(1, 0, 2, 64, device="cuda", dtype=torch.bfloat16)
    lse = torch.empty(1, 2, 0, device="cuda")
    dq, dk, dv = fa.bwd(q, k, k, q, q, lse, causal=False)
    torch.cuda.synchronize()
    assert torch.all(dk == 0) and torch.all(dv == 0) and dq.numel() == 0


def test_bwd_training_workload_sampled_heads():
    """B8 H16 L4096 D64 causal fwd+bwd (seed 3): on three whole heads, the
    forward's O and LSE and the fp32 and bf16 gradients against the oracle."""
    w = synth.WORKLOADS["train_fwd_bwd"]
    x = synth.workload_inputs(w)
    q, k, v, do = (x[n].cuda() for n in ("q", "k", "v", "do"))
    o, lse = fa.fwd(q, k, v, scale=w.scale, causal=w.causal)
    o32, _ = fa.fwd(q, k, v, scale=w.scale, causal=w.causal, o_dtype=torch.float32)
    grads = {}
    for gdt in (torch.float32, torch.bfloat16):
        grads[gdt] = [f64(t) for t in fa.bwd(q, k, v, o, do, lse, scale=w.scale, causal=w.causal, grad_dtype=gdt)]
    torch.cuda.synchronize()
    o, o32, lse = f64(o), f64(o32), f64(lse)
    xf = {n: synth.as_f64(x[n]) for n in x}
    for b, h in [(0, 0), (3, 9), (7, 15)]:
        sl = lambda t: t[b:b + 1, :, h:h + 1]
        rq, rk, rv, ro, rl, _ = oracle.attn_bwd(sl(xf["q"]), sl(xf["k"]), sl(xf["v"]), sl(xf["do"]), w.scale,
                                                w.causal)
        check_close(sl(o32), ro, bf16_output=False, what=f"O fp32 b{b} h{h}")
        check_close(sl(o), ro, bf16_output=True, what=f"O bf16 b{b} h{h}")
        check_lse(lse[b:b + 1, h:h + 1], rl, what=f"LSE b{b} h{h}")
        for gdt, (dq, dk, dv) in grads.items():
            bf = gdt == torch.bfloat16
            check_close(sl(dv), rv, bf16_output=bf, what=f"dV {gdt} b{b} h{h}")
            check_close(sl(dk), rk, bf16_output=bf, what=f"dK {gdt} b{b} h{h}")
            check_close(sl(dq), rq, bf16_output=bf, what=f"dQ {gdt} b{b} h{h}")
