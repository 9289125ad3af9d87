"""Forward kernel vs the CPU fp64 oracle, element by element (GPU)."""
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


def run_case(B, Hq, Hkv, Lq, Lk, D, causal, seed, scale=None, boost=0):
    x = synth.prefill_inputs(B, Hq, Hkv, Lq, Lk, D, seed, q_boost_heads=boost)
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    q, k, v = (x[n].cuda() for n in ("q", "k", "v"))
    res = {}
    for odt in (torch.float32, torch.bfloat16):
        out = torch.full((B, Lq, Hq, D), float("nan"), dtype=odt, device="cuda")     # canary
        lse = torch.full((B, Hq, Lq), float("nan"), dtype=torch.float32, device="cuda")
        fa.fwd(q, k, v, scale=scale, causal=causal, out=out, lse=lse)
        torch.cuda.synchronize()
        res[odt] = (f64(out), f64(lse))
    ro, rl = oracle.attn_fwd(synth.as_f64(x["q"]), synth.as_f64(x["k"]), synth.as_f64(x["v"]), scale, causal)
    return res, ro, rl


CASES = [
    # B, Hq, Hkv, Lq, Lk, D, causal
    (2, 4, 4, 1, 1, 64, True),
    (1, 2, 2, 127, 127, 128, True),
    (1, 2, 1, 129, 129, 128, False),
    (2, 4, 2, 255, 255, 64, True),
    (1, 3, 3, 256, 256, 128, True),
    (1, 8, 2, 1000, 1000, 128, True),
    (1, 4, 4, 300, 700, 128, True),    # Lq < Lk: bottom-right alignment
    (1, 4, 4, 700, 300, 64, True),     # Lq > Lk: the first 400 rows see no key
    (1, 8, 1, 512, 384, 128, False),   # G = 8
    (1, 2, 2, 257, 1, 64, False),      # one key
    (1, 4, 2, 640, 1536, 64, False),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "B%dHq%dHkv%dLq%dLk%dD%d%s" % (*c[:6], "c" if c[6] else "n"))
def test_fwd_matches_oracle(case):
    B, Hq, Hkv, Lq, Lk, D, causal = case
    res, ro, rl = run_case(B, Hq, Hkv, Lq, Lk, D, causal, seed=sum(case))
    for odt, (o, l) in res.items():
        check_close(o, ro, bf16_output=(odt == torch.bfloat16), what=f"O {odt}")
        check_lse(l, rl)


@pytest.mark.parametrize("D", [64, 128])
def test_fwd_output_only_16_byte_aligned(D):
    """O at a 16-byte (not 32-byte) offset: rows go out in 16-byte stores; the
    guard elements around the output stay untouched."""
    B, Hq, Hkv, Lq, Lk, causal = 1, 4, 2, 300, 300, True
    x = synth.prefill_inputs(B, Hq, Hkv, Lq, Lk, D, seed=77)
    q, k, v = (x[n].cuda() for n in ("q", "k", "v"))
    scale = 1.0 / math.sqrt(D)
    ro, rl = oracle.attn_fwd(synth.as_f64(x["q"]), synth.as_f64(x["k"]), synth.as_f64(x["v"]), scale, causal)
    n = B * Lq * Hq * D
    for odt, off in ((torch.bfloat16, 8), (torch.float32, 4)):       # 16 bytes either way
        buf = torch.full((n + 2 * off + 64,), 7.0, dtype=odt, device="cuda")
        base = buf.data_ptr() % 32
        start = off + ((32 - base) % 32) // buf.element_size()        # 32-byte aligned + 16 bytes
        out = buf[start:start + n].view(B, Lq, Hq, D)
        assert out.data_ptr() % 32 == 16
        out.fill_(float("nan"))
        _, lse = fa.fwd(q, k, v, scale=scale, causal=causal, out=out)
        torch.cuda.synchronize()
        check_close(f64(out), ro, bf16_output=(odt == torch.bfloat16), what=f"O {odt}")
        check_lse(f64(lse), rl)
        assert torch.all(buf[:start] == 7.0) and torch.all(buf[start + n:] == 7.0)


def test_fwd_tiny_workload():
    """B1 H1 L128 D64 non-causal, scale 1/8, seed 0."""
    w = synth.WORKLOADS["tiny_fwd"]
    res, ro, rl = run_case(w.B, w.Hq, w.Hkv, w.Lq, w.Lk, w.D, w.causal, w.seed, scale=w.scale)
    for odt, (o, l) in res.items():
        check_close(o, ro, bf16_output=(odt == torch.bfloat16))
        check_lse(l, rl)


def test_fwd_empty_keys():
    q = torch.randn(1, 64, 2, 64, device="cuda").to(torch.bfloat16)
    k = torch.empty(1, 0, 2, 64, device="cuda", dtype=torch.bfloat16)
    o, l = fa.fwd(q, k, k, causal=True)
    torch.cuda.synchronize()
    assert torch.all(o == 0) and torch.all(torch.isneginf(l))


def _sampled_rows(w, x, rows, o, l):
    ro, rl = oracle.attn_rows(x["q"], x["k"], x["v"], w.scale, w.causal, rows)
    got_o = np.stack([o[b, i, h] for b, h, i in rows])
    got_l = np.array([l[b, h, i] for b, h, i in rows])
    return got_o, ro, got_l, rl


def _full_size(name, rows, full_heads):
    w = synth.WORKLOADS[name]
    x = synth.workload_inputs(w)
    q, k, v = (x[n].cuda() for n in ("q", "k", "v"))
    o32, l = fa.fwd(q, k, v, scale=w.scale, causal=w.causal, o_dtype=torch.float32)
    o16, _ = fa.fwd(q, k, v, scale=w.scale, causal=w.causal)
    torch.cuda.synchronize()
    o32, o16, l = f64(o32), f64(o16), f64(l)
    xf = {n: synth.as_f64(x[n]) for n in ("q", "k", "v")}
    go, ro, gl, rl = _sampled_rows(w, xf, rows, o32, l)
    check_close(go, ro, bf16_output=False, what="sampled O fp32")
    check_lse(gl, rl)
    go16 = np.stack([o16[b, i, h] for b, h, i in rows])
    check_close(go16, ro, bf16_output=True, what="sampled O bf16")
    G = w.Hq // w.Hkv
    for b, h in full_heads:      # every row of a few whole heads
        fo, fl = oracle.attn_fwd(xf["q"][b:b + 1, :, h:h + 1], xf["k"][b:b + 1, :, h // G:h // G + 1],
                                 xf["v"][b:b + 1, :, h // G:h // G + 1], w.scale, w.causal)
        check_close(o32[b:b + 1, :, h:h + 1], fo, bf16_output=False, what=f"O b{b} h{h}")
        check_close(o16[b:b + 1, :, h:h + 1], fo, bf16_output=True, what=f"O16 b{b} h{h}")
        check_lse(l[b:b + 1, h:h + 1], fl)


def test_fwd_causal_prefill_full_size():
    """B4 H16 L2048 D128 causal, Q x4 on heads 0-7."""
    idx = [0, 1, 127, 128, 255, 256, 1023, 1500, 2046, 2047]
    rows = [(b, h, i) for b in (0, 3) for h in (0, 7, 8, 15) for i in idx]
    _full_size("causal_prefill", rows, full_heads=[(1, 3), (2, 12)])


def test_fwd_long_gqa_full_size():
    """B1 Hq32 Hkv8 L16384 D128 causal."""
    idx = [0, 129, 4095, 8191, 12000, 16256, 16383]
    rows = [(0, h, i) for h in (0, 5, 31) for i in idx]
    _full_size("long_gqa_prefill", rows, full_heads=[(0, 9)])


def test_wait_timeout_is_reported_and_context_survives():
    fa.device_status(reset=True)
    fa.selftest_wait_timeout(20_000_000)          # 20 ms; nothing ever arrives
    code, where = fa.device_status(reset=True)
    assert code == fa.FA_ERR_TIMEOUT and where == 0x9001
    assert fa.device_status() == (0, 0)
    res, ro, rl = run_case(1, 2, 2, 200, 200, 64, True, seed=5)
    check_close(res[torch.float32][0], ro, bf16_output=False)
    assert fa.device_status() == (0, 0)
