"""Seeded synthetic inputs for the attention workloads.

This module only draws random numbers and rounds them to bf16; it holds none
of the attention arithmetic, so both the CPU oracle and the CUDA path can be
fed from it without sharing any part of the method.

Draw recipe (one NumPy PCG64 generator per workload, float32 standard normals,
then round-to-nearest-even to bf16 through torch):

* prefill / training workloads draw Q, K, V (and dO for training) in that
  order from ``default_rng(seed)``, each with the full tensor shape;
* the causal-prefill workload multiplies Q of the first half of the query
  heads by 4 before rounding (x4 is exact in bf16), which makes the running
  maximum jump often;
* the decode workload draws the per-sequence lengths (uniform integers on
  [1024, 32768], both ends included) and then Q from ``default_rng(seed)``;
  the cache rows of sequence b come from their own stream
  ``default_rng([seed, b + 1])`` (K then V, only the first ``len_b`` rows), so
  that any one sequence can be regenerated alone.  Rows at or past ``len_b``
  are zero (or a caller-chosen fill).

* paged decode inputs hold the same rows (same streams) in a pool of
  fixed-size pages: the pages a sequence needs are drawn, in a seeded random
  order, from ``default_rng([seed, 0, 2])``; unused table entries are -1 and
  spare pool pages hold a fill value;
* e4m3 (FP8) prefill inputs are the same float32 draws as the bf16 ones,
  divided by a per-tensor scale (max |x| / 448, e4m3's largest finite value)
  and rounded to e4m3 (nearest even) through torch; the value of an element is
  its e4m3 value times the scale;
* the new token's rows of a decode step with KV append come from
  ``default_rng([seed, 0, 1])`` (K then V, [B, Hkv, D]).

Tensors are laid out [B, L, H, D] (queries, keys, values, outputs) and
[B, Lmax, Hkv, D] for the KV cache; decode queries are [B, Hq, D].
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np
import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    kind: str            # "fwd", "train" or "decode"
    B: int
    Hq: int
    Hkv: int
    Lq: int
    Lk: int
    D: int
    causal: bool
    scale: float
    seed: int
    q_boost_heads: int = 0      # first heads whose Q is multiplied by 4
    len_lo: int = 0             # decode: per-sequence length range
    len_hi: int = 0


WORKLOADS = {
    "tiny_fwd": Workload("tiny_fwd", "fwd", 1, 1, 1, 128, 128, 64, False, 1.0 / 8.0, 0),
    "causal_prefill": Workload("causal_prefill", "fwd", 4, 16, 16, 2048, 2048, 128, True,
                               1.0 / math.sqrt(128.0), 1, q_boost_heads=8),
    "long_gqa_prefill": Workload("long_gqa_prefill", "fwd", 1, 32, 8, 16384, 16384, 128, True,
                                 1.0 / math.sqrt(128.0), 2),
    "train_fwd_bwd": Workload("train_fwd_bwd", "train", 8, 16, 16, 4096, 4096, 64, True,
                              1.0 / math.sqrt(64.0), 3),
    "splitkv_decode": Workload("splitkv_decode", "decode", 64, 32, 8, 1, 32768, 128, False,
                               1.0 / math.sqrt(128.0), 4, len_lo=1024, len_hi=32768),
}


def to_bf16(x: np.ndarray) -> torch.Tensor:
    """Round a float32 array to bf16 (round to nearest even) as a CPU tensor."""
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)


def as_f64(t: torch.Tensor) -> np.ndarray:
    """Exact widening of a (bf16 or fp32) tensor to a float64 NumPy array."""
    return t.detach().to("cpu").to(torch.float64).numpy()


def prefill_inputs(B, Hq, Hkv, Lq, Lk, D, seed, q_boost_heads=0, with_do=False):
    """Q [B,Lq,Hq,D], K/V [B,Lk,Hkv,D] (and dO like Q) as bf16 CPU tensors."""
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, Lq, Hq, D), dtype=np.float32)
    if q_boost_heads:
        q[:, :, :q_boost_heads, :] *= 4.0
    k = rng.standard_normal((B, Lk, Hkv, D), dtype=np.float32)
    v = rng.standard_normal((B, Lk, Hkv, D), dtype=np.float32)
    out = {"q": to_bf16(q), "k": to_bf16(k), "v": to_bf16(v)}
    del q, k, v
    if with_do:
        out["do"] = to_bf16(rng.standard_normal((B, Lq, Hq, D), dtype=np.float32))
    return out


def workload_inputs(w: Workload):
    if w.kind == "decode":
        raise ValueError("use decode_inputs for decode workloads")
    return prefill_inputs(w.B, w.Hq, w.Hkv, w.Lq, w.Lk, w.D, w.seed,
                          q_boost_heads=w.q_boost_heads, with_do=(w.kind == "train"))


def decode_lengths_and_q(B, Hq, D, seed, len_lo, len_hi):
    rng = np.random.default_rng(seed)
    lens = rng.integers(len_lo, len_hi, size=B, endpoint=True).astype(np.int32)
    q = rng.standard_normal((B, Hq, D), dtype=np.float32)
    return lens, to_bf16(q)


def decode_sequence_kv(b, n, Hkv, D, seed):
    """K and V rows [n, Hkv, D] of sequence b, as bf16 CPU tensors."""
    rng = np.random.default_rng([seed, b + 1])
    k = rng.standard_normal((n, Hkv, D), dtype=np.float32)
    v = rng.standard_normal((n, Hkv, D), dtype=np.float32)
    return to_bf16(k), to_bf16(v)


def decode_inputs(B, Hq, Hkv, Lmax, D, seed, len_lo, len_hi, lens=None,
                  pad_value: Optional[float] = 0.0, device=None):
    """Decode inputs: q [B,Hq,D], k/v cache [B,Lmax,Hkv,D], seqlens int32 [B].

    ``lens`` overrides the drawn lengths (Q is still drawn from the same
    stream).  Cache rows past each length hold ``pad_value`` (NaN works as a
    canary).  With ``device`` set, the cache is filled there sequence by
    sequence, so the host never holds the whole cache.
    """
    drawn, q = decode_lengths_and_q(B, Hq, D, seed, len_lo, len_hi)
    lens = drawn if lens is None else np.asarray(lens, dtype=np.int32)
    assert lens.shape == (B,) and int(lens.max(initial=0)) <= Lmax
    dev = device if device is not None else "cpu"
    kc = torch.full((B, Lmax, Hkv, D), float(pad_value), dtype=torch.bfloat16, device=dev)
    vc = torch.full((B, Lmax, Hkv, D), float(pad_value), dtype=torch.bfloat16, device=dev)
    for b in range(B):
        n = int(lens[b])
        if n == 0:
            continue
        kb, vb = decode_sequence_kv(b, n, Hkv, D, seed)
        kc[b, :n].copy_(kb)
        vc[b, :n].copy_(vb)
    return {"q": q, "k_cache": kc, "v_cache": vc, "seqlens": torch.from_numpy(lens.copy())}


def decode_new_rows(B, Hkv, D, seed):
    """The new token's K and V rows [B, Hkv, D] (bf16) for a decode step with append."""
    rng = np.random.default_rng([seed, 0, 1])
    k = rng.standard_normal((B, Hkv, D), dtype=np.float32)
    v = rng.standard_normal((B, Hkv, D), dtype=np.float32)
    return to_bf16(k), to_bf16(v)


def paged_decode_inputs(B, Hq, Hkv, D, page_size, seed, len_lo, len_hi, lens=None, rows_per_seq=None,
                        spare_pages=3, pad_value: Optional[float] = 0.0, device=None):
    """Decode inputs in a paged cache.

    Returns q [B,Hq,D], k_pages / v_pages [num_pages, page_size, Hkv, D],
    page_table int32 [B, pages_per_seq] and seqlens int32 [B].  Sequence b's
    rows are those of ``decode_inputs`` (same streams).  Each sequence owns
    ceil(rows_per_seq_b / page_size) pages, where rows_per_seq_b is its length,
    or ``rows_per_seq`` (a capacity, e.g. length + 1 to leave room for an
    appended row); the pages are a seeded random permutation of the pool, which
    also holds ``spare_pages`` pages no table entry names.  Table entries past a
    sequence's pages are -1.  Pool rows that hold no cache row are
    ``pad_value``.
    """
    drawn, q = decode_lengths_and_q(B, Hq, D, seed, len_lo, len_hi)
    lens = drawn if lens is None else np.asarray(lens, dtype=np.int32)
    need = [max(int(lens[b]), 0) if rows_per_seq is None else int(rows_per_seq[b]) for b in range(B)]
    npg = [-(-n // page_size) for n in need]
    pps = max(1, max(npg))
    total = sum(npg) + spare_pages
    order = np.random.default_rng([seed, 0, 2]).permutation(total)
    dev = device if device is not None else "cpu"
    kp = torch.full((total, page_size, Hkv, D), float(pad_value), dtype=torch.bfloat16, device=dev)
    vp = torch.full((total, page_size, Hkv, D), float(pad_value), dtype=torch.bfloat16, device=dev)
    table = np.full((B, pps), -1, dtype=np.int32)
    nxt = 0
    for b in range(B):
        table[b, :npg[b]] = order[nxt:nxt + npg[b]]
        nxt += npg[b]
        n = int(lens[b])
        if n <= 0:
            continue
        kb, vb = decode_sequence_kv(b, n, Hkv, D, seed)
        m = -(-n // page_size)
        idx = torch.from_numpy(table[b, :m].astype(np.int64)).to(dev)
        for src, dst in ((kb, kp), (vb, vp)):
            full = torch.full((m * page_size, Hkv, D), float(pad_value), dtype=torch.bfloat16)
            full[:n] = src
            dst.index_copy_(0, idx, full.view(m, page_size, Hkv, D).to(dev))
    return {"q": q, "k_pages": kp, "v_pages": vp, "page_table": torch.from_numpy(table),
            "seqlens": torch.from_numpy(lens.copy())}


E4M3_MAX = 448.0


def to_e4m3(x: np.ndarray):
    """(e4m3 tensor, scale) with x ~= e4m3 * scale; scale = max|x| / 448 (1 for all-zero x)."""
    amax = float(np.max(np.abs(x))) if x.size else 0.0
    scale = amax / E4M3_MAX if amax > 0 else 1.0
    t = torch.from_numpy(np.ascontiguousarray(x / np.float32(scale), dtype=np.float32)).to(torch.float8_e4m3fn)
    return t, scale


def dequant_f64(t: torch.Tensor, scale: float) -> np.ndarray:
    """Exact float64 value of an e4m3 tensor times its scale."""
    return t.to(torch.float64).numpy() * float(scale)


def prefill_inputs_fp8(B, Hq, Hkv, Lq, Lk, D, seed, q_boost_heads=0):
    """e4m3 Q [B,Lq,Hq,D], K/V [B,Lk,Hkv,D] (CPU tensors) and their scales,
    from the same draws as ``prefill_inputs``."""
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, Lq, Hq, D), dtype=np.float32)
    if q_boost_heads:
        q[:, :, :q_boost_heads, :] *= 4.0
    k = rng.standard_normal((B, Lk, Hkv, D), dtype=np.float32)
    v = rng.standard_normal((B, Lk, Hkv, D), dtype=np.float32)
    out = {}
    for name, x in (("q", q), ("k", k), ("v", v)):
        out[name], out[name + "_scale"] = to_e4m3(x)
    return out
