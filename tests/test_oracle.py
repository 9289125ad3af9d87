"""Pins for the CPU fp64 oracle, each tied to something other than the oracle.

P1  rows of P sum to one (softmax gives normalised weights).
P2  uniform logits: O is the mean of the allowed V rows, LSE = ln(#allowed).
P3  one dominant logit selects its value row; LSE -> that logit.
P4  non-causal outputs do not change under a joint permutation of K/V rows.
P5  the tile-by-tile running max / running sum recurrence, written here as a
    plain loop over key tiles, equals the one-shot oracle; any partition of the
    keys merged with ``merge_partials`` equals the one-shot result.
P6  torch's CPU fp64 scaled_dot_product_attention (and its autograd) agrees.
P7  gradient invariants and central finite differences.
P8  decode equals the last row of causal prefill.
P9  a pure-Python loop (math.exp only) equals the NumPy oracle.
P10 the element counts the pages print reproduce.
Plus: fully masked rows, input-generator determinism, and planted mistakes
that the pins must catch.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import attn as oattn
from exact_tiled_attention_46_b200 import inputs as synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rnd(rng, *shape):
    return rng.standard_normal(shape)


# ---------------------------------------------------------------- P1 -----
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("Lq,Lk", [(7, 7), (5, 9), (9, 5)])
def test_p1_rows_sum_to_one(causal, Lq, Lk):
    rng = np.random.default_rng(1)
    q, k = rnd(rng, 2, Lq, 4, 8), rnd(rng, 2, Lk, 2, 8)
    P = oracle.attn_probs(q, k, 0.5, causal)
    sums = P.sum(-1)
    allowed = oracle.allowed_mask(Lq, Lk, causal).any(-1)
    assert np.all(P >= 0)
    np.testing.assert_allclose(sums[..., allowed], 1.0, atol=1e-14)
    assert np.all(sums[..., ~allowed] == 0)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("Lq,Lk", [(7, 7), (5, 9), (9, 5)])
def test_p1_probs_match_torch_softmax(causal, Lq, Lk):
    """attn_probs against torch's fp64 softmax of the scaled logits (an
    independent library routine): catches a wrong scale, a wrong kv-head
    mapping, a transposed product or a mis-aligned causal mask."""
    rng = np.random.default_rng(11)
    scale = 0.37
    q, k = rnd(rng, 2, Lq, 4, 8), rnd(rng, 2, Lk, 2, 8)
    P = oracle.attn_probs(q, k, scale, causal)
    qt = torch.from_numpy(q).permute(0, 2, 1, 3)                     # [B, Hq, Lq, D]
    kt = torch.from_numpy(k).permute(0, 2, 1, 3).repeat_interleave(2, dim=1)   # head h -> kv head h // 2
    logits = scale * qt @ kt.transpose(-1, -2)
    i = torch.arange(Lq)[:, None]
    j = torch.arange(Lk)[None, :]
    allowed = (j <= i + (Lk - Lq)) if causal else torch.ones(Lq, Lk, dtype=torch.bool)
    ref = torch.softmax(logits.masked_fill(~allowed, float("-inf")), dim=-1)
    rows = allowed.any(-1)
    np.testing.assert_allclose(P[:, :, rows.numpy()], ref[:, :, rows].numpy(), rtol=0, atol=1e-14)
    assert np.all(P[:, :, ~rows.numpy()] == 0)


# ---------------------------------------------------------------- P2 -----
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("Lq,Lk", [(6, 6), (4, 10), (10, 4), (33, 33)])
def test_p2_uniform_logits_closed_form(causal, Lq, Lk):
    rng = np.random.default_rng(2)
    D = 8
    q = np.zeros((1, Lq, 2, D))
    k, v = rnd(rng, 1, Lk, 1, D), rnd(rng, 1, Lk, 1, D)
    o, lse = oracle.attn_fwd(q, k, v, 0.3, causal)
    for i in range(Lq):
        n = Lk if not causal else max(0, min(Lk, i + (Lk - Lq) + 1))
        for h in range(2):
            if n == 0:
                assert lse[0, h, i] == -np.inf
                assert np.all(o[0, i, h] == 0)
            else:
                np.testing.assert_allclose(o[0, i, h], v[0, :n, 0].mean(0), atol=1e-13)
                np.testing.assert_allclose(lse[0, h, i], math.log(n), atol=1e-13)


# ---------------------------------------------------------------- P3 -----
def test_p3_dominant_logit_selects_value():
    rng = np.random.default_rng(3)
    Lk, D = 12, 16
    k = rnd(rng, 1, Lk, 1, D)
    v = rnd(rng, 1, Lk, 1, D)
    # orthogonalise keys so that q picks one key with logit alpha*scale and 0 for the rest
    Qm, _ = np.linalg.qr(rng.standard_normal((D, D)))
    k[0, :, 0, :] = Qm[:Lk] * 3.0
    j, alpha, scale = 5, 400.0, 0.25
    q = np.zeros((1, 1, 1, D))
    q[0, 0, 0] = alpha * k[0, j, 0] / np.dot(k[0, j, 0], k[0, j, 0])
    o, lse = oracle.attn_fwd(q, k, v, scale, False)
    np.testing.assert_allclose(o[0, 0, 0], v[0, j, 0], atol=1e-12)
    # other logits are exactly 0, so LSE = ln(exp(alpha*scale) + Lk - 1)
    np.testing.assert_allclose(lse[0, 0, 0], scale * alpha + math.log1p((Lk - 1) * math.exp(-scale * alpha)),
                               rtol=1e-14)


# ---------------------------------------------------------------- P4 -----
def test_p4_permutation_invariance():
    rng = np.random.default_rng(4)
    q, k, v = rnd(rng, 2, 9, 4, 8), rnd(rng, 2, 13, 2, 8), rnd(rng, 2, 13, 2, 8)
    perm = rng.permutation(13)
    o1, l1 = oracle.attn_fwd(q, k, v, 0.35, False)
    o2, l2 = oracle.attn_fwd(q, k[:, perm], v[:, perm], 0.35, False)
    np.testing.assert_allclose(o1, o2, atol=1e-12)
    np.testing.assert_allclose(l1, l2, atol=1e-12)


# ---------------------------------------------------------------- P5 -----
def online_recurrence_row(q_row, K, V, scale, allowed, tile):
    """Running max / running sum / rescaled accumulator over key tiles.

    Written from the pages' description ("How FlashAttention Speeds Up LLM
    Attention": one query consumes score tiles with a running state; "Flash
    Attention Explained: Same Maths, Far Less Memory", "The idea": carry a
    running maximum and a running sum and rescale the accumulated result when a
    new block reveals a larger value).  Plain Python floats, one key at a time
    inside each tile.
    """
    m, l = -math.inf, 0.0
    acc = [0.0] * len(V[0])
    for t0 in range(0, len(K), tile):
        scores = []
        for j in range(t0, min(len(K), t0 + tile)):
            if allowed[j]:
                scores.append((j, scale * sum(a * b for a, b in zip(q_row, K[j]))))
        if not scores:
            continue
        m_new = max(m, max(s for _, s in scores))
        corr = math.exp(m - m_new) if m > -math.inf else 0.0
        l *= corr
        acc = [a * corr for a in acc]
        for j, s in scores:
            p = math.exp(s - m_new)
            l += p
            acc = [a + p * vv for a, vv in zip(acc, V[j])]
        m = m_new
    if l == 0.0:
        return [0.0] * len(acc), -math.inf
    return [a / l for a in acc], m + math.log(l)


@pytest.mark.parametrize("tile", [1, 2, 3, 4])
def test_p5_two_tile_recurrence_equals_one_shot(tile):
    # the pages' example: one query, four scores, consumed as two tiles of two
    rng = np.random.default_rng(5)
    D = 3
    q, k, v = rnd(rng, 1, 1, 1, D), rnd(rng, 1, 4, 1, D), rnd(rng, 1, 4, 1, D)
    o, lse = oracle.attn_fwd(q, k, v, 1.3, False)
    orow, l = online_recurrence_row(list(q[0, 0, 0]), k[0, :, 0].tolist(), v[0, :, 0].tolist(),
                                    1.3, [True] * 4, tile)
    np.testing.assert_allclose(o[0, 0, 0], orow, rtol=1e-15, atol=1e-15)
    np.testing.assert_allclose(lse[0, 0, 0], l, rtol=1e-15)


@pytest.mark.parametrize("causal", [False, True])
def test_p5_recurrence_random_tiles(causal):
    rng = np.random.default_rng(55)
    Lq, Lk, D = 6, 11, 5
    q, k, v = rnd(rng, 1, Lq, 1, D) * 3, rnd(rng, 1, Lk, 1, D), rnd(rng, 1, Lk, 1, D)
    o, lse = oracle.attn_fwd(q, k, v, 0.9, causal)
    mask = oracle.allowed_mask(Lq, Lk, causal)
    for tile in (2, 3, 5):
        for i in range(Lq):
            orow, l = online_recurrence_row(list(q[0, i, 0]), k[0, :, 0].tolist(), v[0, :, 0].tolist(),
                                            0.9, list(mask[i]), tile)
            np.testing.assert_allclose(o[0, i, 0], orow, rtol=1e-13, atol=1e-14)
            np.testing.assert_allclose(lse[0, 0, i], l, rtol=1e-14)


def test_p5_merge_of_any_partition_equals_one_shot():
    rng = np.random.default_rng(6)
    Lk, D = 40, 8
    q, k, v = rnd(rng, 1, 3, 2, D), rnd(rng, 1, Lk, 2, D), rnd(rng, 1, Lk, 2, D)
    o_full, lse_full = oracle.attn_fwd(q, k, v, 0.4, False)
    for trial in range(5):
        labels = rng.integers(0, 4, size=Lk)       # part 3 may be empty
        labels[labels == 3] = 2 if trial % 2 else 3
        o_parts, l_parts = [], []
        for s in range(4):
            idx = np.nonzero(labels == s)[0]
            if len(idx) == 0:
                o_parts.append(np.zeros_like(o_full))
                l_parts.append(np.full_like(lse_full, -np.inf))
            else:
                op, lp = oracle.attn_fwd(q, k[:, idx], v[:, idx], 0.4, False)
                o_parts.append(op)
                l_parts.append(lp)
        # o_parts are [B,L,H,D], lse [B,H,L]; align lse to o's layout
        o_m, l_m = oracle.merge_partials(np.stack(o_parts), np.stack([lp.transpose(0, 2, 1) for lp in l_parts]))
        np.testing.assert_allclose(o_m, o_full, atol=1e-13)
        np.testing.assert_allclose(l_m, lse_full.transpose(0, 2, 1), atol=1e-13)


def test_merge_all_empty():
    o, l = oracle.merge_partials(np.zeros((3, 2, 4)), np.full((3, 2), -np.inf))
    assert np.all(o == 0) and np.all(l == -np.inf)


# ---------------------------------------------------------------- P6 -----
def _torch_ref(q, k, v, scale, causal, do=None):
    from torch.nn.attention.bias import causal_lower_right
    tq = torch.tensor(q).permute(0, 2, 1, 3).contiguous().requires_grad_(True)
    tk = torch.tensor(k).permute(0, 2, 1, 3).contiguous().requires_grad_(True)
    tv = torch.tensor(v).permute(0, 2, 1, 3).contiguous().requires_grad_(True)
    Lq, Lk = q.shape[1], k.shape[1]
    mask = causal_lower_right(Lq, Lk) if causal else None
    G = q.shape[2] // k.shape[2]
    kk = tk.repeat_interleave(G, dim=1)
    vv = tv.repeat_interleave(G, dim=1)
    out = torch.nn.functional.scaled_dot_product_attention(tq, kk, vv, attn_mask=mask, scale=scale)
    res = {"o": out.detach().permute(0, 2, 1, 3).numpy()}
    if do is not None:
        out.backward(torch.tensor(do).permute(0, 2, 1, 3))
        res["dq"] = tq.grad.permute(0, 2, 1, 3).numpy()
        res["dk"] = tk.grad.permute(0, 2, 1, 3).numpy()
        res["dv"] = tv.grad.permute(0, 2, 1, 3).numpy()
    return res


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("Hq,Hkv,Lq,Lk", [(4, 4, 37, 37), (8, 2, 50, 50), (4, 1, 20, 45)])
def test_p6_matches_torch_cpu_fp64(causal, Hq, Hkv, Lq, Lk):
    rng = np.random.default_rng(7)
    D = 16
    q, k, v = rnd(rng, 2, Lq, Hq, D), rnd(rng, 2, Lk, Hkv, D), rnd(rng, 2, Lk, Hkv, D)
    do = rnd(rng, 2, Lq, Hq, D)
    ref = _torch_ref(q, k, v, 0.25, causal, do)
    o, _ = oracle.attn_fwd(q, k, v, 0.25, causal)
    dq, dk, dv, o2, _, _ = oracle.attn_bwd(q, k, v, do, 0.25, causal)
    np.testing.assert_allclose(o, ref["o"], atol=1e-12)
    np.testing.assert_allclose(o2, ref["o"], atol=1e-12)
    np.testing.assert_allclose(dq, ref["dq"], atol=1e-11)
    np.testing.assert_allclose(dk, ref["dk"], atol=1e-11)
    np.testing.assert_allclose(dv, ref["dv"], atol=1e-11)


# ---------------------------------------------------------------- P7 -----
@pytest.mark.parametrize("causal", [False, True])
def test_p7_gradient_invariants(causal):
    rng = np.random.default_rng(8)
    q, k, v, do = (rnd(rng, 1, 9, 2, 6), rnd(rng, 1, 9, 2, 6), rnd(rng, 1, 9, 2, 6), rnd(rng, 1, 9, 2, 6))
    dq, dk, dv, o, lse, delta = oracle.attn_bwd(q, k, v, do, 0.5, causal)
    # logits are shift invariant per query row => sum_j dS_ij = 0 => sum_j dK_j = 0
    np.testing.assert_allclose(dk.sum(axis=1), 0.0, atol=1e-12)
    # rows of P sum to one => sum_j dV_j = sum_i dO_i (G = 1)
    np.testing.assert_allclose(dv.sum(axis=1), do.sum(axis=1), atol=1e-12)
    np.testing.assert_allclose(delta, np.einsum("blhd,blhd->bhl", do, o), atol=1e-13)


@pytest.mark.parametrize("causal", [False, True])
def test_p7_finite_differences(causal):
    rng = np.random.default_rng(9)
    B, H, L, D = 1, 1, 6, 4
    q, k, v, do = (rnd(rng, B, L, H, D) for _ in range(4))
    scale = 0.7
    dq, dk, dv, *_ = oracle.attn_bwd(q, k, v, do, scale, causal)

    def loss(qq, kk, vv):
        o, _ = oracle.attn_fwd(qq, kk, vv, scale, causal)
        return float(np.sum(o * do))

    eps = 1e-5
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        num = np.zeros_like(x)
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            xp, xm = x.copy(), x.copy()
            xp[idx] += eps
            xm[idx] -= eps
            args_p = {"q": q, "k": k, "v": v}
            args_m = dict(args_p)
            args_p[name], args_m[name] = xp, xm
            num[idx] = (loss(**{"qq": args_p["q"], "kk": args_p["k"], "vv": args_p["v"]})
                        - loss(**{"qq": args_m["q"], "kk": args_m["k"], "vv": args_m["v"]})) / (2 * eps)
        np.testing.assert_allclose(g, num, atol=1e-7, err_msg=name)


# ---------------------------------------------------------------- P8 -----
def test_p8_decode_equals_last_causal_row():
    rng = np.random.default_rng(10)
    Hq, Hkv, D, n = 8, 2, 16, 23
    q, k, v = rnd(rng, 1, n, Hq, D), rnd(rng, 1, n, Hkv, D), rnd(rng, 1, n, Hkv, D)
    o, lse = oracle.attn_fwd(q, k, v, 0.25, True)
    for i in (0, 5, n - 1):
        od, ld = oracle.attn_decode(q[:, i], k, v, np.array([i + 1]), 0.25)
        np.testing.assert_allclose(od[0], o[0, i], atol=1e-13)
        np.testing.assert_allclose(ld[0], lse[0, :, i], atol=1e-13)


def test_decode_zero_length_and_padding_ignored():
    rng = np.random.default_rng(11)
    q, kc, vc = rnd(rng, 3, 4, 8), rnd(rng, 3, 10, 2, 8), rnd(rng, 3, 10, 2, 8)
    lens = np.array([0, 10, 4])
    o1, l1 = oracle.attn_decode(q, kc, vc, lens, 0.3)
    kc2, vc2 = kc.copy(), vc.copy()
    kc2[2, 4:] = np.nan
    vc2[2, 4:] = np.nan
    o2, l2 = oracle.attn_decode(q, kc2, vc2, lens, 0.3)
    assert np.all(o1[0] == 0) and np.all(l1[0] == -np.inf)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(l1, l2)


# ------------------------------------------------ paged rows, appended KV --
def test_paged_rows_hand_example():
    """Pool of 4 pages of 2 rows; the sequence's pages are 3, 0, 2: its rows
    0..4 are (page 3, row 0), (3, 1), (0, 0), (0, 1), (2, 0)."""
    pool = np.arange(4 * 2).reshape(4, 2, 1, 1).astype(np.float64)      # value = 2 * page + row
    rows = oracle.paged_rows(pool, [3, 0, 2], 5)
    assert rows[:, 0, 0].tolist() == [6.0, 7.0, 0.0, 1.0, 4.0]


@pytest.mark.parametrize("P", [1, 3, 4, 16])
def test_paged_decode_equals_contiguous_decode(P):
    """Any page size and any page order give the contiguous result exactly:
    scatter a contiguous cache into a shuffled pool, read it back paged."""
    rng = np.random.default_rng(20 + P)
    B, Hq, Hkv, D, Lmax = 3, 4, 2, 8, 13
    q, kc, vc = rnd(rng, B, Hq, D), rnd(rng, B, Lmax, Hkv, D), rnd(rng, B, Lmax, Hkv, D)
    lens = np.array([13, 0, 6])
    pps = -(-Lmax // P)
    order = rng.permutation(B * pps + 2)                  # 2 spare pages never referenced
    kp = np.full((B * pps + 2, P, Hkv, D), np.nan)
    vp = np.full_like(kp, np.nan)
    table = np.full((B, pps), -1)
    for b in range(B):
        for j in range(pps):
            pg = order[b * pps + j]
            table[b, j] = pg
            r = np.arange(j * P, min(Lmax, (j + 1) * P))
            kp[pg, :len(r)], vp[pg, :len(r)] = kc[b, r], vc[b, r]
    for b in range(B):
        np.testing.assert_array_equal(oracle.paged_rows(kp, table[b], lens[b]), kc[b, :lens[b]])
    o1, l1 = oracle.attn_decode(q, kc, vc, lens, 0.3)
    o2, l2 = oracle.attn_decode_paged(q, kp, vp, table, lens, 0.3)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(l1, l2)


def test_decode_append_equals_last_row_of_extended_causal_prefill():
    """One step with the new token appended equals the last causal prefill row
    of the sequence extended by that token (P8 for the appended cache), the
    new rows land at row seqlens[b], nothing else in the cache changes, and a
    full cache has no room."""
    rng = np.random.default_rng(31)
    B, Hq, Hkv, D, Lmax = 4, 4, 2, 8, 9
    kc, vc = rnd(rng, B, Lmax, Hkv, D), rnd(rng, B, Lmax, Hkv, D)
    q, kn, vn = rnd(rng, B, Hq, D), rnd(rng, B, Hkv, D), rnd(rng, B, Hkv, D)
    lens = np.array([0, 5, 8, 9])                         # the last one is full
    o, lse, kc2, vc2 = oracle.attn_decode_append(q, kn, vn, kc, vc, lens, 0.35)
    for b in range(B):
        n = lens[b]
        if n >= Lmax:
            assert np.all(o[b] == 0) and np.all(np.isneginf(lse[b]))
            np.testing.assert_array_equal(kc2[b], kc[b])
            continue
        np.testing.assert_array_equal(kc2[b, n], kn[b])
        np.testing.assert_array_equal(vc2[b, n], vn[b])
        keep = np.arange(Lmax) != n
        np.testing.assert_array_equal(kc2[b, keep], kc[b, keep])
        kx = np.concatenate([kc[b, :n], kn[b][None]])[None]          # [1, n+1, Hkv, D]
        vx = np.concatenate([vc[b, :n], vn[b][None]])[None]
        qx = np.zeros((1, n + 1, Hq, D))
        qx[0, n] = q[b]
        of, lf = oracle.attn_fwd(qx, kx, vx, 0.35, True)
        np.testing.assert_allclose(o[b], of[0, n], atol=1e-13)
        np.testing.assert_allclose(lse[b], lf[0, :, n], atol=1e-13)


# ---------------------------------------------------------------- P9 -----
def brute_force(q, k, v, scale, causal):
    B, Lq, Hq, D = q.shape
    _, Lk, Hkv, _ = k.shape
    G = Hq // Hkv
    o = np.zeros(q.shape)
    lse = np.zeros((B, Hq, Lq))
    for b in range(B):
        for h in range(Hq):
            for i in range(Lq):
                ws, tot = [], 0.0
                for j in range(Lk):
                    if causal and j > i + Lk - Lq:
                        continue
                    s = scale * sum(float(q[b, i, h, d]) * float(k[b, j, h // G, d]) for d in range(D))
                    ws.append((j, s))
                if not ws:
                    lse[b, h, i] = -math.inf
                    continue
                m = max(s for _, s in ws)
                tot = sum(math.exp(s - m) for _, s in ws)
                for j, s in ws:
                    p = math.exp(s - m) / tot
                    for d in range(D):
                        o[b, i, h, d] += p * float(v[b, j, h // G, d])
                lse[b, h, i] = m + math.log(tot)
    return o, lse


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("Lq,Lk", [(5, 5), (3, 7), (7, 3)])
def test_p9_pure_python_loop(causal, Lq, Lk):
    rng = np.random.default_rng(12)
    q, k, v = rnd(rng, 2, Lq, 4, 5), rnd(rng, 2, Lk, 2, 5), rnd(rng, 2, Lk, 2, 5)
    o, lse = oracle.attn_fwd(q, k, v, 0.6, causal)
    ob, lb = brute_force(q, k, v, 0.6, causal)
    np.testing.assert_allclose(o, ob, atol=1e-13)
    np.testing.assert_allclose(lse, lb, atol=1e-13)
    ro, rl = oracle.attn_rows(q, k, v, 0.6, causal, [(1, 3, Lq - 1), (0, 0, 0)])
    np.testing.assert_allclose(ro[0], ob[1, Lq - 1, 3], atol=1e-13)
    np.testing.assert_allclose(rl[1], lb[0, 0, 0], atol=1e-13)


def test_fully_masked_rows():
    # causal with Lq > Lk: the first Lq - Lk queries see no key at all
    rng = np.random.default_rng(13)
    q, k, v = rnd(rng, 1, 6, 1, 4), rnd(rng, 1, 2, 1, 4), rnd(rng, 1, 2, 1, 4)
    o, lse = oracle.attn_fwd(q, k, v, 1.0, True)
    assert np.all(o[0, :4] == 0) and np.all(lse[0, 0, :4] == -np.inf)
    assert np.all(np.isfinite(lse[0, 0, 4:]))


# ---------------------------------------------------------------- P10 ----
def test_p10_printed_element_counts():
    rows = [ln.split() for ln in open(os.path.join(GOLDEN, "score_matrix_elements.txt"))
            if ln.strip() and not ln.startswith("#")]
    assert len(rows) == 7
    for kind, n, e in rows:
        got = oracle.score_matrix_elements(int(n))
        if kind == "exact":
            assert got == int(e)
        else:
            assert abs(got - int(e)) <= 0.05 * int(e)


def test_flop_accounting():
    # causal pairs counted once: L(L+1)/2 when Lq = Lk
    assert oracle.allowed_pairs(2048, 2048, True) == 2048 * 2049 // 2
    assert oracle.allowed_pairs(5, 3, True) == int(oracle.allowed_mask(5, 3, True).sum())
    assert oracle.allowed_pairs(3, 8, True) == int(oracle.allowed_mask(3, 8, True).sum())
    assert oracle.fwd_flops(4, 16, 2048, 2048, 128, True) == 4 * 4 * 16 * 128 * (2048 * 2049 // 2)


# ------------------------------------------------- planted mistakes ------
def test_planted_mistakes_are_caught(monkeypatch):
    """Each mutant of the oracle's arithmetic must fail at least one pin."""
    rng = np.random.default_rng(14)
    q, k, v = rnd(rng, 1, 6, 2, 4), rnd(rng, 1, 6, 1, 4), rnd(rng, 1, 6, 1, 4)
    ref = _torch_ref(q, k, v, 0.5, True)["o"]
    good = oattn._softmax_rows

    def no_mask(S, mask):                 # dropped mask
        return good(S, np.ones_like(mask))

    def no_norm(S, mask):                 # dropped denominator
        P, l = good(S, mask)
        return P * np.exp(l)[..., None] * 0 + np.where(mask, np.exp(S), 0), l

    def transposed(S, mask):              # transposed probabilities
        P, l = good(S.T, mask.T)
        return P.T, l[: S.shape[0]] if l.shape[0] >= S.shape[0] else np.resize(l, S.shape[0])

    for mutant in (no_mask, no_norm, transposed):
        monkeypatch.setattr(oattn, "_softmax_rows", mutant)
        o, _ = oracle.attn_fwd(q, k, v, 0.5, True)
        assert not np.allclose(o, ref, atol=1e-6), mutant.__name__
    monkeypatch.setattr(oattn, "_softmax_rows", good)
    o, _ = oracle.attn_fwd(q, k, v, 0.5, True)
    np.testing.assert_allclose(o, ref, atol=1e-12)


# ------------------------------------------------- input generator -------
def test_inputs_deterministic_and_bf16():
    a = synth.prefill_inputs(1, 4, 2, 16, 16, 8, seed=3, q_boost_heads=2, with_do=True)
    b = synth.prefill_inputs(1, 4, 2, 16, 16, 8, seed=3, q_boost_heads=2, with_do=True)
    for key in a:
        assert a[key].dtype == torch.bfloat16
        assert torch.equal(a[key], b[key])
    rng = np.random.default_rng(3)
    q = rng.standard_normal((1, 16, 4, 8), dtype=np.float32)
    q[:, :, :2] *= 4
    assert torch.equal(a["q"], torch.from_numpy(q).to(torch.bfloat16))


def test_decode_inputs_per_sequence_streams():
    d = synth.decode_inputs(3, 4, 2, 40, 8, seed=4, len_lo=5, len_hi=40)
    lens = d["seqlens"].numpy()
    assert np.all((lens >= 5) & (lens <= 40))
    kb, vb = synth.decode_sequence_kv(1, int(lens[1]), 2, 8, seed=4)
    assert torch.equal(d["k_cache"][1, :lens[1]], kb)
    assert torch.equal(d["v_cache"][1, :lens[1]], vb)
    assert torch.all(d["k_cache"][1, lens[1]:] == 0)
