// Split-KV decode: one new query per (sequence, head) against a KV cache
// ("Flash Attention Explained: Same Maths, Far Less Memory", section "Where
// you actually feel it": in decode the score matrix is one row and the cost is
// reading the cache; "Flash Attention Explained: Speed From Memory Movement",
// "What changed in 2026": decode-phase variants, with its linked note on paged
// KV caches; "FlashAttention Explained: How AI Models Process Attention Faster
// and Use Less Memory", "FlashAttention vs. KV Cache": the cache stores the
// past keys and values and each step adds the new token's).
//
// The cache of one sequence is cut into fixed chunks of keys.  A work item is
// one (sequence, kv head, group of GP query heads, chunk); the GP heads share
// every K/V byte read for them.  The grid is persistent and the items are
// handed out dynamically: the producer warp of a CTA takes the next item
// number from a device counter (zeroed before the launch), maps it to its
// rows through the device-side sequence lengths (items exist only for chunks
// that hold keys) and passes it to the consumer warps through a small
// shared-memory queue.  The grid carries no empty CTAs, CTAs that run faster
// take more items, and one CTA's K/V ring runs on from item to item.
//
// Warp NW (the producer) streams K and V tiles of T keys by TMA through an
// NS-slot mbarrier ring; the rows come from a contiguous cache [B, Lmax, Hkv,
// D] or, in the PAGED variant, from a page pool [num_pages, page_size, Hkv, D]
// through a per-sequence page table (one TMA box per page-aligned run of
// sub_rows rows).  Warps 0..NW-1 split every tile's keys, LPK = D/8 lanes per
// key, each lane owning 8 consecutive dimensions (one 16-byte chunk of a row).
// Each key group keeps its own running max / running sum / accumulator (log2
// units); at the end of the item the groups and warps are merged and the
// item's normalised partial output and LSE are written.  In the APPEND variant
// the new token's K and V rows (k_new, v_new) are attended as key seqlens[b]
// straight from their input rows and written into the cache at row
// seqlens[b] by one CTA, in the same launch.  The combine kernel merges the
// chunks of a sequence:
//   lse = ln sum_s exp(lse_s),  o = sum_s exp(lse_s - lse) o_s.
#pragma once
#include "sm100.cuh"

namespace fa {

struct DecParams {
  const int* seqlens;      // [B] rows already in the cache (device)
  const uint16_t* q;       // [B, Hq, D] bf16
  const uint16_t* k_new;   // APPEND: [B, Hkv, D] bf16, the new token's rows
  const uint16_t* v_new;
  uint16_t* k_cache;       // APPEND: cache (contiguous) or page pool (PAGED), written at row seqlens[b]
  uint16_t* v_cache;
  const int* page_table;   // PAGED: [B, pages_per_seq] int32 page indices
  float* o_part;           // [B, Hq, max_splits, D]
  float* lse_part;         // [B, Hq, max_splits] (natural log)
  int* work_counter;       // next item number; 0 when the launch starts
  int B, Hq, Hkv, max_splits, chunk;
  int cap;                 // rows one sequence can hold (Lmax, or pages_per_seq * page_size)
  int page_size, pages_per_seq, num_pages;   // PAGED
  int sub_rows;            // rows per TMA box: 32, or 16 (pages of an odd multiple of 16 rows)
  float scale_log2;
  uint64_t wait_limit_ns;
};

template <int D, int GP>
struct DecCfg {
  static constexpr int T = 32;                  // keys per ring slot
  static constexpr int NS = 4;                  // ring slots (K and V tile each)
  static constexpr int NW = 4;                  // consumer warps
  static constexpr int LPK = D / 8;             // lanes per key (8 dimensions each)
  static constexpr int KPW = 32 / LPK;          // keys per warp step
  static constexpr int TILE_BYTES = T * D * 2;
  static constexpr int STAGE_BYTES = 2 * TILE_BYTES;
  static constexpr int MRG_FLOATS = NW * GP * (D + 2);
  static constexpr int NI = 2;                  // item queue entries (producer -> consumers)
  static constexpr int ITEM_OFF = NS * STAGE_BYTES + MRG_FLOATS * 4;
  static constexpr int BAR_OFF = ITEM_OFF + 16;
  static constexpr int SMEM_BYTES = BAR_OFF + (2 * NS + 2 * NI) * 8 + 128;
  static constexpr int THREADS = (NW + 1) * 32;
  static constexpr int CTAS_PER_SM = 3;
  static_assert((T / NW) % KPW == 0, "keys per warp must be a multiple of keys per step");
};

constexpr float DEC_TAU = 8.0f;

enum : uint32_t {
  W_DEC_FULL = 0x201, W_DEC_EMPTY = 0x202, W_DEC_DRAIN = 0x203, W_DEC_PAGE = 0x204, W_DEC_APPEND_ROOM = 0x205,
  W_DEC_APPEND_PAGE = 0x206, W_DEC_ITEM = 0x207, W_DEC_ITEM_EMPTY = 0x208
};

__device__ __forceinline__ void bf16x8_to_f32(const uint4 u, float* f) {
  f[0] = __uint_as_float(u.x << 16); f[1] = __uint_as_float(u.x & 0xffff0000u);
  f[2] = __uint_as_float(u.y << 16); f[3] = __uint_as_float(u.y & 0xffff0000u);
  f[4] = __uint_as_float(u.z << 16); f[5] = __uint_as_float(u.z & 0xffff0000u);
  f[6] = __uint_as_float(u.w << 16); f[7] = __uint_as_float(u.w & 0xffff0000u);
}

// Keys attended for sequence b, and how many of them come from the cache.
// Without APPEND: the first min(max(seqlens[b], 0), cap) cache rows.  With
// APPEND: those rows plus the new one, when the cache has room for it (a full
// sequence attends nothing; the combine kernel flags it).
template <bool APPEND>
__device__ __forceinline__ int dec_keys(const DecParams& p, int b, int& cached) {
  const int len = max(p.seqlens[b], 0);
  if (APPEND) {
    if (len >= p.cap) { cached = 0; return 0; }
    cached = len;
    return len + 1;
  }
  cached = min(len, p.cap);
  return cached;
}

// Work-list cursor.  Items are numbered sequence by sequence; sequence b owns
// ceil(keys_b / chunk) * HG consecutive numbers (HG head groups per chunk).
// dec_find maps item number w (non-decreasing from call to call: a CTA's
// numbers come from a counter that only grows) to its sequence and its offset
// u inside that sequence, scanning the lengths 32 sequences at a time from
// where the previous call stopped.  All lanes of the
// warp call it together and get the same answer; false once w is past the
// last item.
struct DecCursor {
  int b;       // first sequence not yet passed
  int base;    // items of the sequences before b
};
template <bool APPEND>
__device__ __forceinline__ bool dec_find(const DecParams& p, int HG, int w, DecCursor& cur, int& b, int& u) {
  const int lane = threadIdx.x & 31;
  while (cur.b < p.B) {
    const int bb = cur.b + lane;
    int cached;
    const int n = bb < p.B ? dec_keys<APPEND>(p, bb, cached) : 0;
    const int c = ((n + p.chunk - 1) / p.chunk) * HG;
    int incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += t;
    }
    const unsigned hit = __ballot_sync(0xffffffffu, bb < p.B && cur.base + incl > w);
    if (hit) {
      const int L = __ffs(hit) - 1;
      cur.base += __shfl_sync(0xffffffffu, incl - c, L);
      cur.b += L;
      b = cur.b;
      u = w - cur.base;
      return true;
    }
    cur.base += __shfl_sync(0xffffffffu, incl, 31);
    cur.b += 32;
  }
  return false;
}

// The rows of one work item.
struct DecItem {
  int b, hkv, hg, split;
  int cached;     // cache rows of the sequence attended
  int k_begin;    // first key of the chunk
  int k_end;      // one past its last key (the new key counts)
  int c_end;      // one past its last cache row
  int ntiles;     // ring slots it takes
};
template <int T, bool APPEND>
__device__ __forceinline__ DecItem dec_item(const DecParams& p, int HG, int GPK, int b, int u) {
  DecItem I;
  I.b = b;
  I.hg = u % HG;
  I.split = u / HG;
  I.hkv = I.hg / GPK;
  const int n = dec_keys<APPEND>(p, b, I.cached);
  I.k_begin = I.split * p.chunk;
  I.k_end = min(n, I.k_begin + p.chunk);
  I.c_end = min(I.k_end, I.cached);
  I.ntiles = I.c_end > I.k_begin ? (I.c_end - I.k_begin + T - 1) / T : 0;
  return I;
}

// Sums each of the GP partial dot products over the LPK lanes of a key group
// and leaves every lane with all GP totals.  For GP = 4 and LPK = 8 the sums
// are transposed while they are reduced (lane bits 2 and 1 pick which heads a
// lane keeps), so that 4 shuffles + 4 adds give each lane one head's total and
// 3 more shuffles collect the other three.
template <int GP, int LPK>
__device__ __forceinline__ void reduce_scores(float (&sc)[GP], int lane) {
  if constexpr (GP == 4 && (LPK == 8 || LPK == 16)) {
    // the two highest lane bits of the group (H = LPK/2, H/2) choose the kept head
    constexpr int H = LPK / 2;
    const bool bh = lane & H, bl = lane & (H / 2);
    float k0 = bh ? sc[2] : sc[0], k1 = bh ? sc[3] : sc[1];
    const float s0 = bh ? sc[0] : sc[2], s1 = bh ? sc[1] : sc[3];
    k0 += __shfl_xor_sync(0xffffffffu, s0, H);
    k1 += __shfl_xor_sync(0xffffffffu, s1, H);
    float kept = bl ? k1 : k0;
    kept += __shfl_xor_sync(0xffffffffu, bl ? k0 : k1, H / 2);
#pragma unroll
    for (int o = H / 4; o >= 1; o >>= 1) kept += __shfl_xor_sync(0xffffffffu, kept, o);
    // lane holds head (bh, bl) summed over the group; collect all four
    const int base = lane & ~(LPK - 1);
#pragma unroll
    for (int g = 0; g < 4; ++g) sc[g] = __shfl_sync(0xffffffffu, kept, base + g * (H / 2));
  } else {
#pragma unroll
    for (int o = 1; o < LPK; o <<= 1)
#pragma unroll
      for (int g = 0; g < GP; ++g) sc[g] += __shfl_xor_sync(0xffffffffu, sc[g], o);
  }
}

template <int D, int GP, bool PAGED, bool APPEND>
__global__ void __launch_bounds__(DecCfg<D, GP>::THREADS, DecCfg<D, GP>::CTAS_PER_SM)
decode_split_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                    const DecParams p) {
  using C = DecCfg<D, GP>;
  constexpr int NS = C::NS, T = C::T, LPK = C::LPK, KPW = C::KPW, NW = C::NW;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
  float* mrg = reinterpret_cast<float*>(smem + NS * C::STAGE_BYTES);
  volatile int* item_w = reinterpret_cast<volatile int*>(smem + C::ITEM_OFF);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);
  uint64_t* empty = full + NS;
  uint64_t* item_full = empty + NS;             // [NI] an item number was posted
  uint64_t* item_empty = item_full + C::NI;     // [NI] every consumer warp has read it

  const int G = p.Hq / p.Hkv;
  const int GPK = G / GP;                       // head groups per kv head
  const int HG = p.Hkv * GPK;                   // head groups per chunk
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint64_t lim = p.wait_limit_ns;

  if (threadIdx.x == 0) {
    for (int i = 0; i < NS; ++i) { mbar_init(&full[i], 1); mbar_init(&empty[i], NW); }
    for (int i = 0; i < C::NI; ++i) { mbar_init(&item_full[i], 1); mbar_init(&item_empty[i], NW); }
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == NW) {
    // ------------------------------------------------------------ producer --
    // The whole warp walks the work list (page indices are spread over its
    // lanes); lane 0 issues the copies.
    if (lane == 0) { tma_prefetch_desc(&tm_k); tma_prefetch_desc(&tm_v); }
    DecCursor cur{0, 0};
    int it = 0;                                 // ring slots filled so far
    int ni = 0;                                 // items posted to the consumers
    bool ok = true;
    while (ok) {
      int w = 0;
      if (lane == 0) w = atomicAdd(p.work_counter, 1);
      w = __shfl_sync(0xffffffffu, w, 0);
      int b = 0, u = 0;
      const bool more = dec_find<APPEND>(p, HG, w, cur, b, u);
      // post the item number (-1: no more items) to the consumers
      const int qs = ni % C::NI;
      if (ni >= C::NI && !(ok = mbar_wait_warp(&item_empty[qs], ((ni / C::NI) + 1) & 1, lim, W_DEC_ITEM_EMPTY)))
        break;
      if (lane == 0) {
        item_w[qs] = more ? w : -1;
        mbar_arrive(&item_full[qs]);            // release: the consumers' wait sees the number
      }
      ++ni;
      if (!more) break;
      const DecItem I = dec_item<T, APPEND>(p, HG, GPK, b, u);
      int pg0 = 0, pg1 = 0, first_pg = 0;
      if (PAGED && I.ntiles > 0) {
        // a chunk spans at most 64 pages (pages hold >= 16 rows, chunks 1024)
        first_pg = I.k_begin / p.page_size;
        const int last_pg = (I.c_end - 1) / p.page_size;
        const int* row = p.page_table + static_cast<size_t>(b) * p.pages_per_seq;
        if (first_pg + lane <= last_pg) pg0 = row[first_pg + lane];
        if (first_pg + 32 + lane <= last_pg) pg1 = row[first_pg + 32 + lane];
      }
      for (int i = 0; i < I.ntiles; ++i) {
        const int slot = it % NS;
        if (it >= NS && !(ok = mbar_wait_warp(&empty[slot], ((it / NS) + 1) & 1, lim, W_DEC_EMPTY))) break;
        const int key0 = I.k_begin + i * T;
        // boxes of sub_rows rows that hold at least one cache row of the item
        int pages[2], rows[2];
        uint32_t bytes = 0, use = 0;
#pragma unroll
        for (int s = 0; s < 2; ++s) {
          const int pos = key0 + s * p.sub_rows;
          pages[s] = b;
          rows[s] = pos;
          if (s * p.sub_rows >= T || pos >= I.c_end) continue;
          if (PAGED) {
            const int idx = pos / p.page_size - first_pg;
            pages[s] = __shfl_sync(0xffffffffu, idx < 32 ? pg0 : pg1, idx & 31);
            rows[s] = pos % p.page_size;
            if (pages[s] < 0 || pages[s] >= p.num_pages) {   // not in the pool: skipped and flagged
              if (lane == 0) record_status(FA_DEV_BAD_INPUT, W_DEC_PAGE);
              continue;
            }
          }
          use |= 1u << s;
          bytes += 2u * p.sub_rows * D * 2;
        }
        if (lane == 0) {
          mbar_arrive_expect_tx(&full[slot], bytes);
          uint8_t* dst = smem + slot * C::STAGE_BYTES;
#pragma unroll
          for (int s = 0; s < 2; ++s) {
            if (!((use >> s) & 1u)) continue;
            tma_load_4d(dst + s * p.sub_rows * D * 2, &tm_k, &full[slot], 0, I.hkv, rows[s], pages[s]);
            tma_load_4d(dst + C::TILE_BYTES + s * p.sub_rows * D * 2, &tm_v, &full[slot], 0, I.hkv, rows[s],
                        pages[s]);
          }
        }
        ++it;
      }
    }
    // the CTA may not exit with copies in flight: wait for the last loads
    if (lane == 0)
      for (int i = max(0, it - NS); i < it; ++i) mbar_wait(&full[i % NS], (i / NS) & 1, lim, W_DEC_DRAIN);
    return;
  }

  // -------------------------------------------------------------- consumers --
  const int kg = lane / LPK;                    // key slot within a warp step
  const int ds = lane % LPK;                    // 16-byte chunk: dimensions 8*ds .. 8*ds+7
  constexpr int KS = (T / NW) / KPW;            // keys per lane group per tile
  DecCursor cur{0, 0};
  int it = 0;                                   // ring slots consumed so far
  int ni = 0;                                   // items taken from the queue
  bool ok = true;
  for (;;) {
    const int qs = ni % C::NI;
    ok = mbar_wait_warp(&item_full[qs], (ni / C::NI) & 1, lim, W_DEC_ITEM);
    const int w = ok ? item_w[qs] : -1;
    __syncwarp();
    if (ok && lane == 0) mbar_arrive(&item_empty[qs]);
    ++ni;
    // every consumer warp leaves together, at the end of the list or if any of
    // them gave up waiting (the barriers below need all of them)
    if (!bar_sync_and(1, NW * 32, ok && w >= 0)) break;
    int b, u;
    dec_find<APPEND>(p, HG, w, cur, b, u);
    const DecItem I = dec_item<T, APPEND>(p, HG, GPK, b, u);
    const int hq0 = I.hkv * G + (I.hg % GPK) * GP;

    float qf[GP][8];
#pragma unroll
    for (int g = 0; g < GP; ++g) {
      const uint4* qrow = reinterpret_cast<const uint4*>(p.q + (static_cast<size_t>(b) * p.Hq + hq0 + g) * D);
      bf16x8_to_f32(qrow[ds], qf[g]);
#pragma unroll
      for (int e = 0; e < 8; ++e) qf[g][e] *= p.scale_log2;
    }
    float m[GP], l[GP], acc[GP][8];
#pragma unroll
    for (int g = 0; g < GP; ++g) {
      m[g] = -INFINITY; l[g] = 0.f;
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[g][e] = 0.f;
    }

    // Per tile, a lane group owns KS keys (kt = warp*T/NW + st*KPW + kg).  Their
    // scores are formed first (independent, so their reductions overlap), then
    // one tile max per head decides a (rare) rescale, then p and the P.V update.
    for (int i = 0; ok && i < I.ntiles; ++i) {
      const int s = it % NS;
      if (!(ok = mbar_wait_warp(&full[s], (it / NS) & 1, lim, W_DEC_FULL))) break;
      const uint8_t* ks = smem + s * C::STAGE_BYTES;
      const uint8_t* vs = ks + C::TILE_BYTES;
      const int key0 = I.k_begin + i * T;
      const bool full_tile = key0 + T <= I.c_end;
      float sc[KS][GP];
#pragma unroll
      for (int st = 0; st < KS; ++st) {
        const int kt = warp * (T / NW) + st * KPW + kg;
        float kf[8];
        bf16x8_to_f32(*reinterpret_cast<const uint4*>(ks + kt * D * 2 + ds * 16), kf);
#pragma unroll
        for (int g = 0; g < GP; ++g) {
          float a0 = 0.f, a1 = 0.f;
#pragma unroll
          for (int e = 0; e < 8; e += 2) ffma2(a0, a1, qf[g][e], qf[g][e + 1], kf[e], kf[e + 1], a0, a1);
          sc[st][g] = a0 + a1;
        }
      }
#pragma unroll
      for (int st = 0; st < KS; ++st) reduce_scores<GP, LPK>(sc[st], lane);
      if (!full_tile) {                           // rows past the item's cache rows do not count
#pragma unroll
        for (int st = 0; st < KS; ++st) {
          const int kt = warp * (T / NW) + st * KPW + kg;
          if (key0 + kt >= I.c_end) {
#pragma unroll
            for (int g = 0; g < GP; ++g) sc[st][g] = -INFINITY;
          }
        }
      }
#pragma unroll
      for (int g = 0; g < GP; ++g) {
        float mt = sc[0][g];
#pragma unroll
        for (int st = 1; st < KS; ++st) mt = fmaxf(mt, sc[st][g]);
        if (mt > m[g] + DEC_TAU) {                // false while both are -inf
          const float a = ex2_approx(m[g] - mt);
          l[g] *= a;
#pragma unroll
          for (int e = 0; e < 8; ++e) acc[g][e] *= a;
          m[g] = mt;
        }
      }
#pragma unroll
      for (int st = 0; st < KS; ++st) {
        const int kt = warp * (T / NW) + st * KPW + kg;
        if (!full_tile && key0 + kt >= I.c_end) continue;   // never read V rows past the item's cache rows
        float vf[8];
        bf16x8_to_f32(*reinterpret_cast<const uint4*>(vs + kt * D * 2 + ds * 16), vf);
#pragma unroll
        for (int g = 0; g < GP; ++g) {
          const float pr = ex2_approx(sc[st][g] - m[g]);
          l[g] += pr;
#pragma unroll
          for (int e = 0; e < 8; e += 2) ffma2(acc[g][e], acc[g][e + 1], pr, pr, vf[e], vf[e + 1], acc[g][e], acc[g][e + 1]);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
      ++it;
    }

    // the new token's key (APPEND): read from its input rows by warp 0, taken
    // by key group 0 of that warp
    const bool has_new = APPEND && I.cached >= I.k_begin && I.cached < I.k_end;
    if (has_new && warp == 0 && ok) {
      const size_t nrow = (static_cast<size_t>(b) * p.Hkv + I.hkv) * D;
      float kf[8], vf[8], sc[GP];
      bf16x8_to_f32(reinterpret_cast<const uint4*>(p.k_new + nrow)[ds], kf);
      bf16x8_to_f32(reinterpret_cast<const uint4*>(p.v_new + nrow)[ds], vf);
#pragma unroll
      for (int g = 0; g < GP; ++g) {
        float a0 = 0.f, a1 = 0.f;
#pragma unroll
        for (int e = 0; e < 8; e += 2) ffma2(a0, a1, qf[g][e], qf[g][e + 1], kf[e], kf[e + 1], a0, a1);
        sc[g] = a0 + a1;
      }
      reduce_scores<GP, LPK>(sc, lane);
      if (kg == 0) {
#pragma unroll
        for (int g = 0; g < GP; ++g) {
          if (sc[g] > m[g] + DEC_TAU) {
            const float a = ex2_approx(m[g] - sc[g]);
            l[g] *= a;
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[g][e] *= a;
            m[g] = sc[g];
          }
          const float pr = ex2_approx(sc[g] - m[g]);
          l[g] += pr;
#pragma unroll
          for (int e = 0; e < 8; e += 2) ffma2(acc[g][e], acc[g][e + 1], pr, pr, vf[e], vf[e + 1], acc[g][e], acc[g][e + 1]);
        }
      }
    }

    // merge the key groups of this warp (lanes ds, ds+LPK, ...)
#pragma unroll
    for (int o = LPK; o < 32; o <<= 1) {
#pragma unroll
      for (int g = 0; g < GP; ++g) {
        const float mo = __shfl_xor_sync(0xffffffffu, m[g], o);
        const float lo = __shfl_xor_sync(0xffffffffu, l[g], o);
        const float mn = fmaxf(m[g], mo);
        const float a = (m[g] == -INFINITY) ? 0.f : ex2_approx(m[g] - mn);
        const float c = (mo == -INFINITY) ? 0.f : ex2_approx(mo - mn);
        l[g] = l[g] * a + lo * c;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float ao = __shfl_xor_sync(0xffffffffu, acc[g][e], o);
          acc[g][e] = acc[g][e] * a + ao * c;
        }
        m[g] = mn;
      }
    }
    // the previous item's readers of the merge area are done
    asm volatile("bar.sync 1, %0;" :: "r"(NW * 32) : "memory");
    // per-warp state to shared memory: [w][g] -> m, l, acc[D]
    if (kg == 0) {
#pragma unroll
      for (int g = 0; g < GP; ++g) {
        float* dst = mrg + (warp * GP + g) * (D + 2);
        if (ds == 0) { dst[0] = m[g]; dst[1] = l[g]; }
#pragma unroll
        for (int e = 0; e < 8; ++e) dst[2 + ds * 8 + e] = acc[g][e];
      }
    }
    // every consumer warp leaves together if any of them gave up waiting
    if (!bar_sync_and(1, NW * 32, ok)) break;
    for (int idx = threadIdx.x; idx < GP * D; idx += NW * 32) {
      const int g = idx / D, d = idx % D;
      float mw[NW], mx = -INFINITY;
#pragma unroll
      for (int w2 = 0; w2 < NW; ++w2) { mw[w2] = mrg[(w2 * GP + g) * (D + 2)]; mx = fmaxf(mx, mw[w2]); }
      float L = 0.f, O = 0.f;
#pragma unroll
      for (int w2 = 0; w2 < NW; ++w2) {
        const float* src = mrg + (w2 * GP + g) * (D + 2);
        const float a = (mw[w2] == -INFINITY) ? 0.f : ex2_approx(mw[w2] - mx);
        L = fmaf(src[1], a, L);
        O = fmaf(src[2 + d], a, O);
      }
      const size_t prow = (static_cast<size_t>(b) * p.Hq + hq0 + g) * p.max_splits + I.split;
      if (!index_ok(prow, 1, static_cast<size_t>(p.B) * p.Hq * p.max_splits, W_IDX_DEC_PART)) continue;
      p.o_part[prow * D + d] = L > 0.f ? O / L : 0.f;
      if (d == 0) p.lse_part[prow] = L > 0.f ? (mx + log2f(L)) * LN2 : -INFINITY;
    }

    // APPEND: the first head group of each kv head writes the new rows into the
    // cache at row `cached` (nothing of this launch reads that row from the cache)
    if (has_new && warp == 1 && (I.hg % GPK) == 0 && lane < 2 * (D / 8)) {
      size_t rowaddr;
      bool room = true;
      if (PAGED) {
        const int pg = p.page_table[static_cast<size_t>(b) * p.pages_per_seq + I.cached / p.page_size];
        room = pg >= 0 && pg < p.num_pages;
        rowaddr = ((static_cast<size_t>(pg) * p.page_size + I.cached % p.page_size) * p.Hkv + I.hkv) * D;
        if (!room && lane == 0) record_status(FA_DEV_BAD_INPUT, W_DEC_APPEND_PAGE);
      } else {
        rowaddr = ((static_cast<size_t>(b) * p.cap + I.cached) * p.Hkv + I.hkv) * D;
      }
      const size_t cache_elems = PAGED ? static_cast<size_t>(p.num_pages) * p.page_size * p.Hkv * D
                                       : static_cast<size_t>(p.B) * p.cap * p.Hkv * D;
      if (room && index_ok(rowaddr, D, cache_elems, W_IDX_DEC_APPEND)) {
        const int half = lane / (D / 8), c = lane % (D / 8);
        const size_t nrow = (static_cast<size_t>(b) * p.Hkv + I.hkv) * D;
        const uint4 val = reinterpret_cast<const uint4*>((half ? p.v_new : p.k_new) + nrow)[c];
        reinterpret_cast<uint4*>((half ? p.v_cache : p.k_cache) + rowaddr)[c] = val;
      }
    }
  }
}

struct CombineParams {
  const float* o_part;     // [B, Hq, max_splits, D]
  const float* lse_part;   // [B, Hq, max_splits]
  const int* counts;       // [B]: number of valid parts, or cache lengths when chunk > 0; may be null
  void* o;                 // [B, Hq, D] bf16 or fp32
  float* lse;              // [B, Hq] or null
  int B, Hq, D, max_splits, chunk, o_fp32;
  int cap, append;         // chunk > 0: rows a sequence can hold; 1 if a new row is attended
};

// One block per (sequence, head); thread d owns output column d.
__global__ void __launch_bounds__(128) decode_combine_kernel(const CombineParams p) {
  const int bh = blockIdx.x;
  const int b = bh / p.Hq;
  int ns = p.max_splits;
  if (p.counts != nullptr) {
    const int c = max(p.counts[b], 0);
    if (p.chunk > 0) {
      int n;
      if (p.append) {
        n = c >= p.cap ? 0 : c + 1;
        if (c >= p.cap && bh % p.Hq == 0 && threadIdx.x == 0) record_status(FA_DEV_BAD_INPUT, W_DEC_APPEND_ROOM);
      } else {
        n = min(c, p.cap);
      }
      ns = (n + p.chunk - 1) / p.chunk;
    } else {
      ns = c;
    }
    ns = min(ns, p.max_splits);
  }
  const float* lp = p.lse_part + static_cast<size_t>(bh) * p.max_splits;
  float mx = -INFINITY;
  for (int s = 0; s < ns; ++s) mx = fmaxf(mx, lp[s]);
  float wsum = 0.f;
  for (int s = 0; s < ns; ++s) wsum += (lp[s] == -INFINITY) ? 0.f : expf(lp[s] - mx);
  const bool has = wsum > 0.f;
  for (int d = threadIdx.x; d < p.D; d += blockDim.x) {
    float acc = 0.f;
    for (int s = 0; s < ns; ++s) {
      const float w = (lp[s] == -INFINITY) ? 0.f : expf(lp[s] - mx);
      acc = fmaf(w, p.o_part[(static_cast<size_t>(bh) * p.max_splits + s) * p.D + d], acc);
    }
    const float v = has ? acc / wsum : 0.f;
    if (!index_ok(static_cast<size_t>(bh) * p.D + d, 1, static_cast<size_t>(p.B) * p.Hq * p.D, W_IDX_DEC_OUT)) continue;
    if (p.o_fp32) static_cast<float*>(p.o)[static_cast<size_t>(bh) * p.D + d] = v;
    else static_cast<__nv_bfloat16*>(p.o)[static_cast<size_t>(bh) * p.D + d] = __float2bfloat16_rn(v);
  }
  if (threadIdx.x == 0 && p.lse != nullptr) p.lse[bh] = has ? mx + logf(wsum) : -INFINITY;
}

// Merge of two attention results over disjoint key sets, row by row, in the
// prefill layout (the merge step of context-parallel prefill: each rank's
// queries meet the key blocks one at a time):
//   lse = ln(e^lse_a + e^lse_b),  o = e^(lse_a - lse) o_a + e^(lse_b - lse) o_b,
// an empty side having lse = -inf.  o_* [B, L, H, D] fp32, lse_* [B, H, L].
// One warp per (b, l, h) row; o_out / lse_out may be o_a / lse_a.
struct MergeParams {
  const float* o_a; const float* lse_a;
  const float* o_b; const float* lse_b;
  void* o_out; float* lse_out;
  int B, H, L, D, o_fp32;
};
__global__ void __launch_bounds__(256) attn_merge_kernel(const MergeParams p) {
  const int lane = threadIdx.x & 31;
  const size_t rows = static_cast<size_t>(p.B) * p.L * p.H;
  for (size_t row = (static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x) / 32; row < rows;
       row += static_cast<size_t>(gridDim.x) * blockDim.x / 32) {
    const int h = static_cast<int>(row % p.H);
    const size_t bl = row / p.H;
    const int l = static_cast<int>(bl % p.L);
    const int b = static_cast<int>(bl / p.L);
    const size_t li = (static_cast<size_t>(b) * p.H + h) * p.L + l;
    const float la = p.lse_a[li], lb = p.lse_b[li];
    const float mx = fmaxf(la, lb);
    const bool empty = mx == -INFINITY;
    const float wa = (la == -INFINITY) ? 0.f : expf(la - mx);
    const float wb = (lb == -INFINITY) ? 0.f : expf(lb - mx);
    const float inv = empty ? 0.f : 1.f / (wa + wb);
    const float ca = wa * inv, cb = wb * inv;
    if (!index_ok(row * p.D, p.D, rows * p.D, W_IDX_MERGE)) continue;
    const float* oa = p.o_a + row * p.D;
    const float* ob = p.o_b + row * p.D;
    for (int d = lane * 4; d < p.D; d += 128) {
      const float4 x = *reinterpret_cast<const float4*>(oa + d);
      const float4 y = *reinterpret_cast<const float4*>(ob + d);
      const float4 r = make_float4(ca * x.x + cb * y.x, ca * x.y + cb * y.y, ca * x.z + cb * y.z, ca * x.w + cb * y.w);
      if (p.o_fp32) {
        *reinterpret_cast<float4*>(static_cast<float*>(p.o_out) + row * p.D + d) = r;
      } else {
        uint2 w;
        w.x = pack_bf16x2(r.x, r.y);
        w.y = pack_bf16x2(r.z, r.w);
        *reinterpret_cast<uint2*>(static_cast<uint16_t*>(p.o_out) + row * p.D + d) = w;
      }
    }
    __syncwarp();
    if (lane == 0 && p.lse_out != nullptr) p.lse_out[li] = empty ? -INFINITY : mx + logf(wa + wb);
  }
}

}  // namespace fa
