"""Split-KV decode and the combine kernel vs the CPU fp64 oracle (GPU)."""
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


def run_decode(B, Hq, Hkv, Lmax, D, lens, seed, pad):
    x = synth.decode_inputs(B, Hq, Hkv, Lmax, D, seed, 1, Lmax, lens=lens, pad_value=pad)
    scale = 1.0 / math.sqrt(D)
    q, kc, vc, sl = x["q"].cuda(), x["k_cache"].cuda(), x["v_cache"].cuda(), x["seqlens"].cuda()
    out = {}
    for odt in (torch.float32, torch.bfloat16):
        o = torch.full((B, Hq, D), float("nan"), dtype=odt, device="cuda")
        l = torch.full((B, Hq), float("nan"), dtype=torch.float32, device="cuda")
        fa.decode(q, kc, vc, sl, scale=scale, out=o, lse=l)
        torch.cuda.synchronize()
        out[odt] = (f64(o), f64(l))
    ro, rl = oracle.attn_decode(synth.as_f64(x["q"]), synth.as_f64(x["k_cache"]), synth.as_f64(x["v_cache"]),
                                x["seqlens"].numpy(), scale)
    return out, ro, rl


@pytest.mark.parametrize("Hq,Hkv,D", [(4, 1, 128), (8, 2, 128), (32, 8, 128), (16, 2, 64), (6, 3, 64), (4, 4, 128)])
def test_decode_matches_oracle(Hq, Hkv, D):
    C = fa.decode_chunk()
    lens = [0, 1, 31, 33, C - 1, C, C + 1, 3000]
    out, ro, rl = run_decode(len(lens), Hq, Hkv, 3100, D, lens, seed=Hq + D, pad=float("nan"))
    for odt, (o, l) in out.items():
        check_close(o, ro, bf16_output=(odt == torch.bfloat16), what=f"O {odt}")
        check_lse(l, rl)
    assert np.all(out[torch.float32][0][0] == 0)         # empty sequence: O = 0
    assert np.all(np.isneginf(out[torch.float32][1][0]))  # and LSE = -inf


def test_decode_full_size_sampled():
    """B64 Hq32 Hkv8 D128, cache [64,32768,8,128], lengths U[1024,32768] (seed 4)."""
    w = synth.WORKLOADS["splitkv_decode"]
    x = synth.decode_inputs(w.B, w.Hq, w.Hkv, w.Lk, w.D, w.seed, w.len_lo, w.len_hi, device="cuda")
    q, sl = x["q"].cuda(), x["seqlens"].cuda()
    o, l = fa.decode(q, x["k_cache"], x["v_cache"], sl, scale=w.scale, o_dtype=torch.float32)
    o16, _ = fa.decode(q, x["k_cache"], x["v_cache"], sl, scale=w.scale)
    torch.cuda.synchronize()
    o, o16, l = f64(o), f64(o16), f64(l)
    lens = x["seqlens"].numpy()
    qf = synth.as_f64(x["q"])
    rng = np.random.default_rng(0)
    bs = sorted(set([int(np.argmax(lens)), int(np.argmin(lens))] + list(rng.choice(w.B, 6, replace=False))))
    for b in bs:
        kb, vb = synth.decode_sequence_kv(b, int(lens[b]), w.Hkv, w.D, w.seed)
        kf, vf = synth.as_f64(kb)[None], synth.as_f64(vb)[None]
        ro, rl = oracle.attn_decode(qf[b:b + 1], kf, vf, lens[b:b + 1], w.scale)
        check_close(o[b:b + 1], ro, bf16_output=False, what=f"seq {b}")
        check_close(o16[b:b + 1], ro, bf16_output=True, what=f"seq {b} bf16")
        check_lse(l[b:b + 1], rl)


def test_combine_matches_oracle_merge():
    rng = np.random.default_rng(3)
    B, Hq, S, D = 3, 5, 7, 128
    o_part = rng.standard_normal((B, Hq, S, D)).astype(np.float32)
    lse_part = (rng.standard_normal((B, Hq, S)) * 4).astype(np.float32)
    lse_part[0, :, 2] = -np.inf                  # an empty part
    lse_part[1, 3, :] = -np.inf                  # a head with no keys at all
    nsplit = np.array([S, 4, 1], dtype=np.int32)
    o, l = fa.decode_combine(torch.from_numpy(o_part).cuda(), torch.from_numpy(lse_part).cuda(),
                             torch.from_numpy(nsplit).cuda(), o_dtype=torch.float32)
    torch.cuda.synchronize()
    o, l = f64(o), f64(l)
    for b in range(B):
        n = nsplit[b]
        ro, rl = oracle.merge_partials(o_part[b, :, :n].transpose(1, 0, 2), lse_part[b, :, :n].T)
        check_close(o[b], ro, bf16_output=False, max_abs=1e-5, mean_abs=1e-6)
        check_lse(l[b], rl)
