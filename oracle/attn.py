"""CPU fp64 oracle for exact scaled dot-product attention.

TEST INFRASTRUCTURE ONLY.  Only the test-suite, the package smoke check and the
benchmark's CPU-baseline leg may import this module; the library itself never
does, and it shares no code with the CUDA path.

What it computes is the plain definition the pages give, written out with full
score matrices (the naive three-stage form: scores, softmax, weighted sum of
values), in float64 on the host:

* "FlashAttention Explained: How AI Models Process Attention Faster and Use
  Less Memory", section "Understanding Attention in Transformer Models": the
  scaled dot-product attention equation softmax(Q K^T / sqrt(d_k)) V.
* same page, section "Why Traditional Attention Can Be Inefficient": the
  three stages S = Q K^T, P = softmax(S / sqrt(d_k)), O = P V.
* same page, "FlashAttention vs. Approximate Attention Methods", and "Flash
  Attention Explained: Same Maths, Far Less Memory", section "Why it is not a
  trade-off": tiled attention is exact, so this one-shot definition is the
  result the tiled kernels must reach up to rounding.

Readings where the pages are silent (each one is listed in the design notes):

* layout: q/o [B, Lq, Hq, D], k/v [B, Lk, Hkv, D]; decode q/o [B, Hq, D],
  cache [B, Lmax, Hkv, D];
* ``scale`` is passed in (1/sqrt(D) is the pages' choice; any value is
  accepted);
* grouped-query attention ("Flash Attention Explained: Same Maths, Far Less
  Memory", "What it does not solve"): query head h reads kv head h // G with
  G = Hq / Hkv;
* causal masking ("How FlashAttention Speeds Up LLM Attention": each query
  compares with keys from other *allowed* positions): key j is allowed for
  query i when j <= i + (Lk - Lq) (bottom-right alignment, the KV-cache
  reading);
* LSE_i = ln sum_{allowed j} exp(S_ij), natural log; a query with no allowed
  key gets O = 0 and LSE = -inf;
* backward: the standard analytic gradient of the definition above; dK/dV of
  a kv head sum over its G query heads;
* decode: one query per (sequence, head) against cache rows 0..len_b-1, all
  allowed (the cache already holds the current token).

Pinned by tests/test_oracle.py (closed forms, invariants, brute-force loops,
finite differences, torch's CPU fp64 attention, and the element counts the
pages print).
"""
from __future__ import annotations

import numpy as np

NEG_INF = -np.inf


def allowed_mask(Lq: int, Lk: int, causal: bool) -> np.ndarray:
    """Boolean [Lq, Lk]: True where key j may be attended by query i."""
    if not causal:
        return np.ones((Lq, Lk), dtype=bool)
    i = np.arange(Lq)[:, None]
    j = np.arange(Lk)[None, :]
    return j <= i + (Lk - Lq)


def _softmax_rows(S: np.ndarray, mask: np.ndarray):
    """Row softmax of S over the allowed entries.

    Returns (P, lse).  Rows with no allowed entry give P = 0 and lse = -inf.
    The shift by the row maximum is only for range; softmax does not depend
    on it (page "FlashAttention Explained ...", section "3. Online Softmax":
    a running maximum is tracked for numerical stability).
    """
    Sm = np.where(mask, S, NEG_INF)
    m = Sm.max(axis=-1, keepdims=True, initial=NEG_INF)
    empty = ~np.isfinite(m)
    m_safe = np.where(empty, 0.0, m)
    E = np.exp(Sm - m_safe)                 # exp(-inf) = 0 on masked entries
    l = E.sum(axis=-1, keepdims=True)
    P = np.where(empty, 0.0, E / np.where(empty, 1.0, l))
    lse = np.where(empty, NEG_INF, m_safe + np.log(np.where(empty, 1.0, l)))
    return P, lse[..., 0]


def _group(Hq: int, Hkv: int) -> int:
    if Hkv <= 0 or Hq % Hkv:
        raise ValueError("Hq must be a positive multiple of Hkv")
    return Hq // Hkv


def attn_probs(q, k, scale, causal):
    """Full probability matrix P [B, Hq, Lq, Lk] (small inputs only)."""
    B, Lq, Hq, D = q.shape
    _, Lk, Hkv, _ = k.shape
    G = _group(Hq, Hkv)
    mask = allowed_mask(Lq, Lk, causal)
    P = np.zeros((B, Hq, Lq, Lk))
    for b in range(B):
        for h in range(Hq):
            S = scale * (q[b, :, h, :] @ k[b, :, h // G, :].T)
            P[b, h], _ = _softmax_rows(S, mask)
    return P


def attn_fwd(q, k, v, scale, causal, row_chunk: int = 2048):
    """Forward: (O [B,Lq,Hq,D], LSE [B,Hq,Lq]) in float64.

    Per (batch, head) and per block of query rows it forms the full score rows
    S = scale * Q K^T over every key, the row softmax P and O = P V.  The row
    blocking only bounds host memory; each row is still computed in one shot.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    B, Lq, Hq, D = q.shape
    _, Lk, Hkv, Dv = v.shape
    G = _group(Hq, Hkv)
    o = np.zeros((B, Lq, Hq, Dv))
    lse = np.zeros((B, Hq, Lq))
    for b in range(B):
        for h in range(Hq):
            K = k[b, :, h // G, :]
            V = v[b, :, h // G, :]
            for r0 in range(0, Lq, row_chunk):
                r1 = min(Lq, r0 + row_chunk)
                S = scale * (q[b, r0:r1, h, :] @ K.T)
                i = np.arange(r0, r1)[:, None]
                j = np.arange(Lk)[None, :]
                mask = (j <= i + (Lk - Lq)) if causal else np.ones_like(S, dtype=bool)
                P, l = _softmax_rows(S, mask)
                o[b, r0:r1, h, :] = P @ V
                lse[b, h, r0:r1] = l
    return o, lse


def attn_rows(q, k, v, scale, causal, rows):
    """O and LSE of selected query rows only: ``rows`` is a list of (b, h, i).

    Used to check full-size outputs one row at a time.  Each row is the same
    definition as ``attn_fwd`` (full score row, softmax, weighted sum).
    """
    B, Lq, Hq, D = q.shape
    _, Lk, Hkv, Dv = v.shape
    G = _group(Hq, Hkv)
    o = np.zeros((len(rows), Dv))
    lse = np.zeros(len(rows))
    for n, (b, h, i) in enumerate(rows):
        K = np.asarray(k[b, :, h // G, :], dtype=np.float64)
        V = np.asarray(v[b, :, h // G, :], dtype=np.float64)
        s = scale * (K @ np.asarray(q[b, i, h, :], dtype=np.float64))
        mask = (np.arange(Lk) <= i + (Lk - Lq)) if causal else np.ones(Lk, dtype=bool)
        P, l = _softmax_rows(s[None, :], mask[None, :])
        o[n] = P[0] @ V
        lse[n] = l[0]
    return o, lse


def attn_bwd(q, k, v, do, scale, causal):
    """Backward of the definition: (dQ, dK, dV, O, LSE, Delta) in float64.

    The page "FlashAttention Explained ...", section "More Efficient
    Backpropagation", says the gradients are obtained without keeping the
    probability matrix around; the oracle does keep it (per batch and head)
    and applies the textbook softmax-attention gradient:

        dV   = P^T dO                      (summed over the G heads of a kv head)
        dP   = dO V^T
        Delta_i = sum_d dO_id O_id
        dS   = P * (dP - Delta)            (row-broadcast Delta)
        dQ   = scale * dS K
        dK   = scale * dS^T Q              (summed over the G heads)
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    do = np.asarray(do, dtype=np.float64)
    B, Lq, Hq, D = q.shape
    _, Lk, Hkv, Dv = v.shape
    G = _group(Hq, Hkv)
    mask = allowed_mask(Lq, Lk, causal)
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    o = np.zeros((B, Lq, Hq, Dv))
    lse = np.zeros((B, Hq, Lq))
    delta = np.zeros((B, Hq, Lq))
    for b in range(B):
        for h in range(Hq):
            kv = h // G
            Q, K, V, dO = q[b, :, h, :], k[b, :, kv, :], v[b, :, kv, :], do[b, :, h, :]
            P, l = _softmax_rows(scale * (Q @ K.T), mask)
            O = P @ V
            dv[b, :, kv, :] += P.T @ dO
            dP = dO @ V.T
            Delta = np.sum(dO * O, axis=-1)
            dS = P * (dP - Delta[:, None])
            dq[b, :, h, :] = scale * (dS @ K)
            dk[b, :, kv, :] += scale * (dS.T @ Q)
            o[b, :, h, :] = O
            lse[b, h, :] = l
            delta[b, h, :] = Delta
    return dq, dk, dv, o, lse, delta


def attn_decode(q, k_cache, v_cache, seqlens, scale, pairs=None):
    """Single-query attention against a KV cache: (O [B,Hq,D], LSE [B,Hq]).

    Page "Flash Attention Explained: Same Maths, Far Less Memory", section
    "Where you actually feel it": in decode one new query attends over the
    cached keys and values, so the score matrix is a single row.  Sequence b
    attends to cache rows 0..seqlens[b]-1.  ``pairs`` restricts the work to a
    list of (b, h); other entries stay 0.
    """
    B, Hq, D = q.shape
    _, Lmax, Hkv, Dv = v_cache.shape
    G = _group(Hq, Hkv)
    o = np.zeros((B, Hq, Dv))
    lse = np.full((B, Hq), NEG_INF)
    todo = pairs if pairs is not None else [(b, h) for b in range(B) for h in range(Hq)]
    for b, h in todo:
        n = int(seqlens[b])
        K = np.asarray(k_cache[b, :n, h // G, :], dtype=np.float64)
        V = np.asarray(v_cache[b, :n, h // G, :], dtype=np.float64)
        s = scale * (K @ np.asarray(q[b, h], dtype=np.float64))
        P, l = _softmax_rows(s[None, :], np.ones((1, n), dtype=bool))
        o[b, h] = P[0] @ V if n else 0.0
        lse[b, h] = l[0] if n else NEG_INF
    return o, lse


def paged_rows(pages, table_row, n):
    """Rows 0..n-1 of one sequence kept in a pool of fixed-size pages.

    Page "Flash Attention Explained: Speed From Memory Movement", section "What
    changed in 2026" and its linked note on paged KV caches: a sequence's cache
    is a list of pages from a shared pool.  ``pages`` is [num_pages, P, ...];
    ``table_row`` lists the sequence's pages in order, so row r is row r % P of
    page table_row[r // P].
    """
    P = pages.shape[1]
    r = np.arange(int(n))
    return pages[np.asarray(table_row)[r // P], r % P]


def attn_decode_paged(q, k_pages, v_pages, page_table, seqlens, scale, pairs=None):
    """Single-query attention against a paged KV cache: (O [B,Hq,D], LSE [B,Hq]).

    The same definition as ``attn_decode``; only where the rows are stored
    differs (``paged_rows``).  ``pairs`` restricts the work to a list of (b, h).
    """
    B, Hq, D = q.shape
    Dv = v_pages.shape[-1]
    o = np.zeros((B, Hq, Dv))
    lse = np.full((B, Hq), NEG_INF)
    for b in range(B):
        hs = [h for (bb, h) in pairs if bb == b] if pairs is not None else list(range(Hq))
        if not hs:
            continue
        n = int(seqlens[b])
        kb = paged_rows(k_pages, page_table[b], n)[None]
        vb = paged_rows(v_pages, page_table[b], n)[None]
        ob, lb = attn_decode(q[b:b + 1], kb, vb, np.array([n]), scale, pairs=[(0, h) for h in hs])
        o[b, hs], lse[b, hs] = ob[0, hs], lb[0, hs]
    return o, lse


def attn_decode_append(q, k_new, v_new, k_cache, v_cache, seqlens, scale):
    """One generation step with a KV cache: (O, LSE, K cache, V cache).

    Page "FlashAttention Explained: How AI Models Process Attention Faster and
    Use Less Memory", section "FlashAttention vs. KV Cache": the cache keeps
    the keys and values of earlier tokens and each new token adds its own.
    Sequence b holds seqlens[b] rows; the new token's rows k_new[b], v_new[b]
    ([B, Hkv, D]) are stored at row seqlens[b] and its query attends over all
    seqlens[b] + 1 rows.  A sequence whose cache is full (seqlens[b] >= Lmax)
    has no room: its cache is left as it is and it attends nothing (O = 0,
    LSE = -inf).  Returns new cache arrays; the inputs are not modified.
    """
    kc = np.array(k_cache, dtype=np.float64, copy=True)
    vc = np.array(v_cache, dtype=np.float64, copy=True)
    Lmax = kc.shape[1]
    lens = np.maximum(np.asarray(seqlens, dtype=np.int64), 0)
    n = np.zeros_like(lens)
    for b in range(kc.shape[0]):
        if lens[b] < Lmax:
            kc[b, lens[b]] = k_new[b]
            vc[b, lens[b]] = v_new[b]
            n[b] = lens[b] + 1
    o, lse = attn_decode(q, kc, vc, n, scale)
    return o, lse, kc, vc


def merge_partials(o_parts, lse_parts):
    """Merge attention results over disjoint key sets.

    ``o_parts`` [S, ..., D] are the normalised outputs of S disjoint key
    subsets, ``lse_parts`` [S, ...] their log-sum-exps (-inf for an empty
    subset).  The merged result is the attention over the union:
    lse = ln sum_s exp(lse_s), o = sum_s exp(lse_s - lse) o_s; all-empty gives
    o = 0, lse = -inf.  This is the "combine pieces that sit on different
    scales" step the page "How FlashAttention Speeds Up LLM Attention" names.
    """
    o_parts = np.asarray(o_parts, dtype=np.float64)
    lse_parts = np.asarray(lse_parts, dtype=np.float64)
    m = lse_parts.max(axis=0)
    empty = ~np.isfinite(m)
    m_safe = np.where(empty, 0.0, m)
    w = np.exp(lse_parts - m_safe[None])          # 0 for empty parts
    tot = w.sum(axis=0)
    lse = np.where(empty, NEG_INF, m_safe + np.log(np.where(empty, 1.0, tot)))
    o = (w[..., None] * o_parts).sum(axis=0) / np.where(empty, 1.0, tot)[..., None]
    o = np.where(empty[..., None], 0.0, o)
    return o, lse


def fwd_flops(B, Hq, Lq, Lk, D, causal) -> float:
    """Two matmuls (Q K^T and P V) over the allowed (query, key) pairs."""
    return 4.0 * B * Hq * D * allowed_pairs(Lq, Lk, causal)


def allowed_pairs(Lq, Lk, causal) -> int:
    if not causal:
        return Lq * Lk
    off = Lk - Lq
    # sum over i of clamp(i + off + 1, 0, Lk)
    return int(sum(max(0, min(Lk, i + off + 1)) for i in range(Lq)))


def score_matrix_elements(n_tokens: int) -> int:
    """Entries of one head's full score matrix (what naive attention stores)."""
    return n_tokens * n_tokens
