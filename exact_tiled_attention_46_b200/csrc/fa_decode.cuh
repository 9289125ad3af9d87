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
// through a per-sequence page table (TMA boxes of 64 dimensions by sub_rows
// rows, 128-byte swizzled).  Each consumer warp takes 8 of every tile's 32
// keys: the scores of the GP query heads (padded to 16 rows) come from
// mma.sync m16n8k16 with K read by ldmatrix, the softmax runs on the score
// fragments, and P.V is mma.sync m16n8k8 with P straight from the score
// fragment and V read by ldmatrix.trans, into a 16 x D fp32 accumulator
// fragment.  Each warp keeps its own running max / sums (log2 units); at the
// end of the item the warps are merged and the item's normalised partial
// output and LSE are written.  In the APPEND variant
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
  static constexpr int NW = 4;                  // consumer warps, 8 keys of each tile apiece
  static constexpr int TILE_BYTES = T * D * 2;  // D / 64 blocks of T rows x 128 bytes (128B swizzle)
  static constexpr int BLOCK_BYTES = T * 128;
  static constexpr int STAGE_BYTES = 2 * TILE_BYTES;
  static constexpr int MRG_STRIDE = D + 4;      // per (warp, head): m, l, l of the rounded p, pad, O[D]
  static constexpr int MRG_FLOATS = NW * GP * MRG_STRIDE;
  static constexpr int NI = 2;                  // item queue entries (producer -> consumers)
  static constexpr int ITEM_OFF = NS * STAGE_BYTES + MRG_FLOATS * 4;
  static constexpr int BAR_OFF = ITEM_OFF + 16;
  static constexpr int SMEM_BYTES = BAR_OFF + (2 * NS + 2 * NI) * 8 + 1024;
  static constexpr int THREADS = (NW + 1) * 32;
  static constexpr int CTAS_PER_SM = 3;
  static_assert(T == 8 * NW && GP <= 8 && D % 64 == 0, "8 keys per consumer warp; heads fit the 16-row fragment");
};

constexpr float DEC_TAU = 8.0f;

enum : uint32_t {
  W_DEC_FULL = 0x201, W_DEC_EMPTY = 0x202, W_DEC_DRAIN = 0x203, W_DEC_PAGE = 0x204, W_DEC_APPEND_ROOM = 0x205,
  W_DEC_APPEND_PAGE = 0x206, W_DEC_ITEM = 0x207, W_DEC_ITEM_EMPTY = 0x208
};

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

template <int D, int GP, bool PAGED, bool APPEND>
__global__ void __launch_bounds__(DecCfg<D, GP>::THREADS, DecCfg<D, GP>::CTAS_PER_SM)
decode_split_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                    const DecParams p) {
  using C = DecCfg<D, GP>;
  constexpr int NS = C::NS, T = C::T, NW = C::NW;
  extern __shared__ uint8_t smem_raw[];
  // the 128-byte swizzle repeats every 1024 bytes: tiles start on such a boundary
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
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
#pragma unroll
            for (int db = 0; db < D / 64; ++db) {   // 64 dimensions (128 bytes) per box
              const int off = db * C::BLOCK_BYTES + s * p.sub_rows * 128;
              tma_load_4d(dst + off, &tm_k, &full[slot], db * 64, I.hkv, rows[s], pages[s]);
              tma_load_4d(dst + C::TILE_BYTES + off, &tm_v, &full[slot], db * 64, I.hkv, rows[s], pages[s]);
            }
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
  // Fragment coordinates (mma.sync m16n8): row g = query head of the group
  // (rows >= GP are padding), columns 2 t4, 2 t4 + 1 = keys (scores) or
  // dimensions (output).
  const int g = lane >> 2, t4 = lane & 3;
  constexpr int KSTEPS = D / 16, NT = D / 8;
  const bool row_real = g < GP;
  const uint32_t ring_base = smem_u32(smem);
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

    // Q of head g as the A fragment: per 16-dimension step, dims 2 t4.. and 2 t4 + 8..
    uint32_t qa[KSTEPS][2];
    {
      const uint32_t* qrow = reinterpret_cast<const uint32_t*>(
          p.q + (static_cast<size_t>(b) * p.Hq + hq0 + (row_real ? g : 0)) * D);
#pragma unroll
      for (int ks = 0; ks < KSTEPS; ++ks) {
        qa[ks][0] = row_real ? qrow[ks * 8 + t4] : 0u;
        qa[ks][1] = row_real ? qrow[ks * 8 + 4 + t4] : 0u;
      }
    }
    float m_run = -INFINITY, l = 0.f, lr = 0.f;   // l, lr: this lane's share of the row sums
    float o[NT][4];
#pragma unroll
    for (int n = 0; n < NT; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;

    for (int i = 0; ok && i < I.ntiles; ++i) {
      const int s = it % NS;
      if (!(ok = mbar_wait_warp(&full[s], (it / NS) & 1, lim, W_DEC_FULL))) break;
      const uint32_t kt = ring_base + s * C::STAGE_BYTES;
      const uint32_t vt = kt + C::TILE_BYTES;
      const int key0 = I.k_begin + i * T;
      // V rows of this warp's keys at or past the item's last cache row hold
      // stale or never-written data; their p is 0, but 0 * NaN is not, so they
      // are cleared before the products read them
      const bool partial = key0 + warp * 8 + 8 > I.c_end;
      if (partial) {
        const int kr = warp * 8 + (lane >> 2);      // 4 lanes per row, 32 bytes each per block
        if (key0 + (kr - warp * 8) + warp * 8 >= I.c_end) {
#pragma unroll
          for (int db = 0; db < D / 64; ++db) {
            uint4* row = reinterpret_cast<uint4*>(smem + s * C::STAGE_BYTES + C::TILE_BYTES + db * C::BLOCK_BYTES + kr * 128);
            row[(lane & 3) * 2] = make_uint4(0u, 0u, 0u, 0u);
            row[(lane & 3) * 2 + 1] = make_uint4(0u, 0u, 0u, 0u);
          }
        }
        __syncwarp();
      }
      // S = Q K^T for this warp's keys 8 warp .. 8 warp + 7, two 16-dimension steps per ldmatrix
      float sc[4] = {0.f, 0.f, 0.f, 0.f};
      {
        const int kr = warp * 8 + (lane & 7);       // key row this lane addresses
        const int mi = lane >> 3;                   // which of the four 8x8 matrices
#pragma unroll
        for (int ks = 0; ks < KSTEPS; ks += 2) {
          const int ksm = ks + (mi >> 1);
          const int cc = (ksm & 3) * 2 + (mi & 1);  // 16-byte chunk (8 dimensions) in the 128-byte row
          uint32_t b0, b1, b2, b3;
          ldsm_x4(kt + (ksm >> 2) * C::BLOCK_BYTES + kr * 128 + ((cc ^ (kr & 7)) << 4), b0, b1, b2, b3);
          mma_16816(sc, qa[ks][0], 0u, qa[ks][1], 0u, b0, b1);
          mma_16816(sc, qa[ks + 1][0], 0u, qa[ks + 1][1], 0u, b2, b3);
        }
      }
      const int kc = key0 + warp * 8 + 2 * t4;      // keys of this lane's two scores
      float s0 = (kc < I.c_end) ? sc[0] * p.scale_log2 : -INFINITY;
      float s1 = (kc + 1 < I.c_end) ? sc[1] * p.scale_log2 : -INFINITY;
      float mt = fmaxf(s0, s1);
      mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 1));
      mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 2));
      const bool resc = mt > m_run + DEC_TAU;       // false while both are -inf
      if (__any_sync(0xffffffffu, resc)) {
        const float a = resc ? ex2_approx(m_run - mt) : 1.f;
        l *= a; lr *= a;
#pragma unroll
        for (int n = 0; n < NT; ++n) { o[n][0] *= a; o[n][1] *= a; }
        if (resc) m_run = mt;
      }
      const float msub = (m_run == -INFINITY) ? 0.f : m_run;
      const float p0 = ex2_approx(s0 - msub), p1 = ex2_approx(s1 - msub);
      const uint32_t pa = pack_bf16x2(p0, p1);
      l += p0 + p1;
      lr += __uint_as_float(pa << 16) + __uint_as_float(pa & 0xffff0000u);   // the rounded p, exactly
      // O += P V: this warp's 8 keys x 8 dimensions per n-tile, four n-tiles per ldmatrix.trans
      {
        const int kr = warp * 8 + (lane & 7);
        const int mi = lane >> 3;
#pragma unroll
        for (int n0 = 0; n0 < NT; n0 += 4) {
          const int n = n0 + mi;                    // n-tile this lane addresses: dims 8n .. 8n + 7
          uint32_t v0, v1, v2, v3;
          ldsm_x4_trans(vt + (n >> 3) * C::BLOCK_BYTES + kr * 128 + (((n & 7) ^ (kr & 7)) << 4), v0, v1, v2, v3);
          mma_1688(o[n0 + 0], pa, 0u, v0);
          mma_1688(o[n0 + 1], pa, 0u, v1);
          mma_1688(o[n0 + 2], pa, 0u, v2);
          mma_1688(o[n0 + 3], pa, 0u, v3);
        }
      }
      // generic writes to the slot (the cleared rows) come before the next TMA into it
      if (partial) fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
      ++it;
    }

    // the new token's key (APPEND), in warp 0: scores from its input rows
    const bool has_new = APPEND && I.cached >= I.k_begin && I.cached < I.k_end;
    if (has_new && warp == 0 && ok) {
      const size_t nrow = (static_cast<size_t>(b) * p.Hkv + I.hkv) * D;
      constexpr int DL = D / 32;                    // dimensions per lane in the dot products
      float kf[DL];
#pragma unroll
      for (int e = 0; e < DL; ++e) kf[e] = __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(p.k_new)[nrow + lane * DL + e]);
      float snew = -INFINITY;
#pragma unroll
      for (int h2 = 0; h2 < GP; ++h2) {
        const __nv_bfloat16* qh = reinterpret_cast<const __nv_bfloat16*>(p.q) + (static_cast<size_t>(b) * p.Hq + hq0 + h2) * D;
        float d = 0.f;
#pragma unroll
        for (int e = 0; e < DL; ++e) d = fmaf(__bfloat162float(qh[lane * DL + e]), kf[e], d);
#pragma unroll
        for (int o2 = 16; o2 >= 1; o2 >>= 1) d += __shfl_xor_sync(0xffffffffu, d, o2);
        if (h2 == g) snew = d * p.scale_log2;
      }
      // one more key for row g: the same online update as above
      const bool rs = row_real && snew > m_run + DEC_TAU;
      if (__any_sync(0xffffffffu, rs)) {
        const float a = rs ? ex2_approx(m_run - snew) : 1.f;
        l *= a; lr *= a;
#pragma unroll
        for (int n = 0; n < NT; ++n) { o[n][0] *= a; o[n][1] *= a; }
        if (rs) m_run = snew;
      }
      const float msub = (m_run == -INFINITY) ? 0.f : m_run;
      const float pn = row_real ? ex2_approx(snew - msub) : 0.f;
      const float pnr = __bfloat162float(__float2bfloat16_rn(pn));   // the rounded p, as in the products
      if (t4 == 0) { l += pn; lr += pnr; }          // counted once per row (the quad's shares are summed)
      const __nv_bfloat16* vn = reinterpret_cast<const __nv_bfloat16*>(p.v_new) + nrow;
#pragma unroll
      for (int n = 0; n < NT; ++n) {
        o[n][0] = fmaf(pnr, __bfloat162float(vn[n * 8 + 2 * t4]), o[n][0]);
        o[n][1] = fmaf(pnr, __bfloat162float(vn[n * 8 + 2 * t4 + 1]), o[n][1]);
      }
    }

    // this warp's row sums: the four lanes of a row hold shares
    l += __shfl_xor_sync(0xffffffffu, l, 1);
    l += __shfl_xor_sync(0xffffffffu, l, 2);
    lr += __shfl_xor_sync(0xffffffffu, lr, 1);
    lr += __shfl_xor_sync(0xffffffffu, lr, 2);
    // the previous item's readers of the merge area are done
    asm volatile("bar.sync 1, %0;" :: "r"(NW * 32) : "memory");
    // per-warp state to shared memory: [w][g] -> m, l, lr, pad, O[D]
    if (row_real) {
      float* dst = mrg + (warp * GP + g) * C::MRG_STRIDE;
      if (t4 == 0) { dst[0] = m_run; dst[1] = l; dst[2] = lr; }
#pragma unroll
      for (int n = 0; n < NT; ++n) { dst[4 + n * 8 + 2 * t4] = o[n][0]; dst[4 + n * 8 + 2 * t4 + 1] = o[n][1]; }
    }
    // every consumer warp leaves together if any of them gave up waiting
    if (!bar_sync_and(1, NW * 32, ok)) break;
    for (int idx = threadIdx.x; idx < GP * D; idx += NW * 32) {
      const int h2 = idx / D, d = idx % D;
      float mw[NW], mx = -INFINITY;
#pragma unroll
      for (int w2 = 0; w2 < NW; ++w2) { mw[w2] = mrg[(w2 * GP + h2) * C::MRG_STRIDE]; mx = fmaxf(mx, mw[w2]); }
      float L = 0.f, LR = 0.f, O = 0.f;
#pragma unroll
      for (int w2 = 0; w2 < NW; ++w2) {
        const float* src = mrg + (w2 * GP + h2) * C::MRG_STRIDE;
        const float a = (mw[w2] == -INFINITY) ? 0.f : ex2_approx(mw[w2] - mx);
        L = fmaf(src[1], a, L);
        LR = fmaf(src[2], a, LR);
        O = fmaf(src[4 + d], a, O);
      }
      const size_t prow = (static_cast<size_t>(b) * p.Hq + hq0 + h2) * p.max_splits + I.split;
      if (!index_ok(prow, 1, static_cast<size_t>(p.B) * p.Hq * p.max_splits, W_IDX_DEC_PART)) continue;
      // O is normalised by the sum of the rounded p that the products used, the
      // LSE by the exact sum
      p.o_part[prow * D + d] = LR > 0.f ? O / LR : 0.f;
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
