"""Decode with the new token's K/V appended, and decode from a paged cache,
against the CPU fp64 oracle (GPU)."""
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


def bits(t):
    return t.view(torch.int16).cpu()


def reset_status():
    fa.device_status(reset=True)


# ------------------------------------------------------------- KV append --
@pytest.mark.parametrize("Hq,Hkv,D", [(32, 8, 128), (8, 2, 128), (16, 2, 64), (6, 3, 64), (4, 4, 128)])
def test_decode_append_matches_oracle(Hq, Hkv, D):
    reset_status()
    C, Lmax = fa.decode_chunk(), 3100
    lens = [0, 1, 31, 33, C - 1, C, C + 1, 3000, Lmax - 1]
    B = len(lens)
    seed = Hq + D + 100
    x = synth.decode_inputs(B, Hq, Hkv, Lmax, D, seed, 1, Lmax, lens=lens, pad_value=float("nan"))
    kn, vn = synth.decode_new_rows(B, Hkv, D, seed)
    scale = 1.0 / math.sqrt(D)
    ro, rl, rk, rv = oracle.attn_decode_append(synth.as_f64(x["q"]), synth.as_f64(kn), synth.as_f64(vn),
                                               synth.as_f64(x["k_cache"]), synth.as_f64(x["v_cache"]),
                                               x["seqlens"].numpy(), scale)
    for odt in (torch.float32, torch.bfloat16):
        kc, vc = x["k_cache"].cuda(), x["v_cache"].cuda()
        o = torch.full((B, Hq, D), float("nan"), dtype=odt, device="cuda")
        lse = torch.full((B, Hq), float("nan"), dtype=torch.float32, device="cuda")
        fa.decode_append(x["q"].cuda(), kn.cuda(), vn.cuda(), kc, vc, x["seqlens"].cuda(), scale=scale, out=o,
                         lse=lse)
        torch.cuda.synchronize()
        check_close(f64(o), ro, bf16_output=(odt == torch.bfloat16), what=f"O {odt}")
        check_lse(f64(lse), rl)
        # the new rows land at row seqlens[b]; every other row (NaN canaries included) is untouched
        exp_k, exp_v = bits(x["k_cache"]).clone(), bits(x["v_cache"]).clone()
        for b, n in enumerate(lens):
            exp_k[b, n] = bits(kn)[b]
            exp_v[b, n] = bits(vn)[b]
        assert torch.equal(bits(kc), exp_k) and torch.equal(bits(vc), exp_v)
        np.testing.assert_array_equal(f64(kc), rk)        # the oracle's cache, NaN canaries included
    assert fa.device_status() == (0, 0)


def test_decode_append_full_cache_has_no_room():
    """A sequence whose cache is full attends nothing, writes nothing, and the
    device status says so; the other sequences are unaffected."""
    reset_status()
    B, Hq, Hkv, D, Lmax = 3, 8, 2, 128, 300
    lens = [300, 5, 299]
    x = synth.decode_inputs(B, Hq, Hkv, Lmax, D, 7, 1, Lmax, lens=lens)
    kn, vn = synth.decode_new_rows(B, Hkv, D, 7)
    kc, vc = x["k_cache"].cuda(), x["v_cache"].cuda()
    o, lse = fa.decode_append(x["q"].cuda(), kn.cuda(), vn.cuda(), kc, vc, x["seqlens"].cuda(),
                              o_dtype=torch.float32)
    code, where = fa.device_status(reset=True)
    assert code == fa.FA_ERR_INVALID_ARG and where != 0
    assert torch.all(o[0] == 0) and torch.all(torch.isneginf(lse[0]))
    assert torch.equal(bits(kc[0]), bits(x["k_cache"][0]))
    ro, rl, _, _ = oracle.attn_decode_append(synth.as_f64(x["q"]), synth.as_f64(kn), synth.as_f64(vn),
                                             synth.as_f64(x["k_cache"]), synth.as_f64(x["v_cache"]), lens,
                                             1.0 / math.sqrt(D))
    check_close(f64(o), ro, bf16_output=False, what="O")
    check_lse(f64(lse), rl)


# ------------------------------------------------------------ paged cache --
def paged_case(B, Hq, Hkv, D, page, lens, seed, append):
    rows = [n + 1 for n in lens] if append else None
    x = synth.paged_decode_inputs(B, Hq, Hkv, D, page, seed, 1, max(lens) + 1, lens=lens, rows_per_seq=rows,
                                  pad_value=float("nan"))
    return x


@pytest.mark.parametrize("page", [16, 32, 48, 64, 256])
@pytest.mark.parametrize("Hq,Hkv,D", [(32, 8, 128), (16, 2, 64), (6, 3, 64)])
def test_decode_paged_matches_oracle_and_contiguous(page, Hq, Hkv, D):
    reset_status()
    C = fa.decode_chunk()
    lens = [0, 1, 17, 31, 33, C - 1, C, C + 1, 2500]
    B = len(lens)
    seed = page + Hq + D
    x = paged_case(B, Hq, Hkv, D, page, lens, seed, append=False)
    scale = 1.0 / math.sqrt(D)
    q, kp, vp, tab, sl = (x[n].cuda() for n in ("q", "k_pages", "v_pages", "page_table", "seqlens"))
    ro, rl = oracle.attn_decode_paged(synth.as_f64(x["q"]), synth.as_f64(x["k_pages"]), synth.as_f64(x["v_pages"]),
                                      x["page_table"].numpy(), x["seqlens"].numpy(), scale)
    # the same rows in a contiguous cache (same streams)
    c = synth.decode_inputs(B, Hq, Hkv, max(lens), D, seed, 1, max(lens) + 1, lens=lens)
    for odt in (torch.float32, torch.bfloat16):
        o, lse = fa.decode_paged(q, kp, vp, tab, sl, scale=scale, o_dtype=odt)
        oc, lc = fa.decode(q, c["k_cache"].cuda(), c["v_cache"].cuda(), sl, scale=scale, o_dtype=odt)
        torch.cuda.synchronize()
        check_close(f64(o), ro, bf16_output=(odt == torch.bfloat16), what=f"O {odt}")
        check_lse(f64(lse), rl)
        # same keys in the same tiles: the paged result is the contiguous one, bit for bit
        assert torch.equal(o, oc) and torch.equal(lse, lc)
    assert fa.device_status() == (0, 0)


@pytest.mark.parametrize("page", [16, 64])
def test_decode_paged_append(page):
    reset_status()
    Hq, Hkv, D = 32, 8, 128
    C = fa.decode_chunk()
    lens = [0, 15, 16, 63, 64, C - 1, C, 1500]
    B = len(lens)
    x = paged_case(B, Hq, Hkv, D, page, lens, 55 + page, append=True)
    kn, vn = synth.decode_new_rows(B, Hkv, D, 55 + page)
    scale = 1.0 / math.sqrt(D)
    kp, vp = x["k_pages"].cuda(), x["v_pages"].cuda()
    o, lse = fa.decode_paged(x["q"].cuda(), kp, vp, x["page_table"].cuda(), x["seqlens"].cuda(), k_new=kn.cuda(),
                             v_new=vn.cuda(), scale=scale, o_dtype=torch.float32)
    torch.cuda.synchronize()
    # oracle: the appended step on the de-paged cache
    table = x["page_table"].numpy()
    Lc = table.shape[1] * page
    kc = np.full((B, Lc, Hkv, D), np.nan)
    vc = np.full((B, Lc, Hkv, D), np.nan)
    for b, n in enumerate(lens):
        kc[b, :n] = oracle.paged_rows(synth.as_f64(x["k_pages"]), table[b], n)
        vc[b, :n] = oracle.paged_rows(synth.as_f64(x["v_pages"]), table[b], n)
    ro, rl, _, _ = oracle.attn_decode_append(synth.as_f64(x["q"]), synth.as_f64(kn), synth.as_f64(vn), kc, vc,
                                             np.array(lens), scale)
    check_close(f64(o), ro, bf16_output=False, what="O")
    check_lse(f64(lse), rl)
    # the new rows are in their pages; the rest of the pool is untouched
    exp_k, exp_v = bits(x["k_pages"]).clone(), bits(x["v_pages"]).clone()
    for b, n in enumerate(lens):
        pg, r = int(table[b, n // page]), n % page
        exp_k[pg, r] = bits(kn)[b]
        exp_v[pg, r] = bits(vn)[b]
    assert torch.equal(bits(kp), exp_k) and torch.equal(bits(vp), exp_v)
    assert fa.device_status() == (0, 0)


def test_decode_paged_page_index_outside_pool_is_flagged():
    """A table entry outside the pool is never dereferenced: its rows are
    skipped and the device status reports it (the call itself succeeds)."""
    reset_status()
    B, Hq, Hkv, D, page = 2, 8, 2, 128, 32
    x = paged_case(B, Hq, Hkv, D, page, [100, 200], 9, append=False)
    tab = x["page_table"].clone()
    tab[1, 2] = x["k_pages"].shape[0] + 5
    o, lse = fa.decode_paged(x["q"].cuda(), x["k_pages"].cuda(), x["v_pages"].cuda(), tab.cuda(),
                             x["seqlens"].cuda(), o_dtype=torch.float32)
    code, where = fa.device_status(reset=True)
    assert code == fa.FA_ERR_INVALID_ARG and where != 0
    ro, rl = oracle.attn_decode_paged(synth.as_f64(x["q"])[:1], synth.as_f64(x["k_pages"]),
                                      synth.as_f64(x["v_pages"]), x["page_table"].numpy()[:1],
                                      x["seqlens"].numpy()[:1], 1.0 / math.sqrt(D))
    check_close(f64(o)[:1], ro, bf16_output=False, what="O of the intact sequence")


# --------------------------------------------------------- full-size cases --
def test_decode_paged_full_size_sampled():
    """The decode workload (B64 Hq32 Hkv8 D128, lengths U[1024,32768], seed 4)
    in a pool of 16-row pages: sampled sequences against the oracle, and the
    whole output equal to the contiguous-cache decode."""
    w = synth.WORKLOADS["splitkv_decode"]
    x = synth.paged_decode_inputs(w.B, w.Hq, w.Hkv, w.D, 16, w.seed, w.len_lo, w.len_hi, device="cuda")
    q, tab, sl = x["q"].cuda(), x["page_table"].cuda(), x["seqlens"].cuda()
    o, l = fa.decode_paged(q, x["k_pages"], x["v_pages"], tab, sl, scale=w.scale, o_dtype=torch.float32)
    torch.cuda.synchronize()
    del x["k_pages"], x["v_pages"]
    c = synth.decode_inputs(w.B, w.Hq, w.Hkv, w.Lk, w.D, w.seed, w.len_lo, w.len_hi, device="cuda")
    oc, lc = fa.decode(q, c["k_cache"], c["v_cache"], sl, scale=w.scale, o_dtype=torch.float32)
    torch.cuda.synchronize()
    assert torch.equal(o, oc) and torch.equal(l, lc)
    del c
    o, l = f64(o), f64(l)
    lens = x["seqlens"].numpy()
    qf = synth.as_f64(x["q"])
    rng = np.random.default_rng(1)
    for b in sorted(set([int(np.argmax(lens)), int(np.argmin(lens))] + list(rng.choice(w.B, 3, replace=False)))):
        kb, vb = synth.decode_sequence_kv(b, int(lens[b]), w.Hkv, w.D, w.seed)
        ro, rl = oracle.attn_decode(qf[b:b + 1], synth.as_f64(kb)[None], synth.as_f64(vb)[None], lens[b:b + 1],
                                    w.scale)
        check_close(o[b:b + 1], ro, bf16_output=False, what=f"seq {b}")
        check_lse(l[b:b + 1], rl)


def test_decode_append_full_size_sampled():
    """The decode workload's contiguous cache with one appended token per
    sequence: sampled sequences against the oracle, new rows written."""
    w = synth.WORKLOADS["splitkv_decode"]
    x = synth.decode_inputs(w.B, w.Hq, w.Hkv, w.Lk, w.D, w.seed, w.len_lo, w.len_hi, device="cuda")
    kn, vn = synth.decode_new_rows(w.B, w.Hkv, w.D, w.seed)
    q, sl = x["q"].cuda(), x["seqlens"].cuda()
    lens = x["seqlens"].numpy()
    assert lens.max() < w.Lk
    o, l = fa.decode_append(q, kn.cuda(), vn.cuda(), x["k_cache"], x["v_cache"], sl, scale=w.scale,
                            o_dtype=torch.float32)
    torch.cuda.synchronize()
    for b in range(w.B):
        assert torch.equal(bits(x["k_cache"][b, int(lens[b])]), bits(kn[b]))
    o, l = f64(o), f64(l)
    qf = synth.as_f64(x["q"])
    for b in sorted(set([int(np.argmax(lens)), int(np.argmin(lens)), 5, 40])):
        kb, vb = synth.decode_sequence_kv(b, int(lens[b]), w.Hkv, w.D, w.seed)
        kx = np.concatenate([synth.as_f64(kb), synth.as_f64(kn)[b][None]])[None]
        vx = np.concatenate([synth.as_f64(vb), synth.as_f64(vn)[b][None]])[None]
        ro, rl = oracle.attn_decode(qf[b:b + 1], kx, vx, lens[b:b + 1] + 1, w.scale)
        check_close(o[b:b + 1], ro, bf16_output=False, what=f"seq {b}")
        check_lse(l[b:b + 1], rl)
