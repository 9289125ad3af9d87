// Split-KV decode: one new query per (sequence, head) against a contiguous KV
// cache ("Flash Attention Explained: Same Maths, Far Less Memory", section
// "Where you actually feel it": in decode the score matrix is one row and the
// cost is reading the cache; "Flash Attention Explained: Speed From Memory
// Movement", "What changed in 2026": decode-phase variants).
//
// The cache of one sequence is cut into fixed chunks of keys.  A CTA owns one
// (sequence, kv head, chunk) and the GP query heads of that kv head that it
// packs, so each K/V byte is read from HBM once for GP heads.  Warp 4 streams
// K and V tiles of T keys with TMA through an NS-slot mbarrier ring; warps 0-3
// split every tile's keys, LPK = D/8 lanes per key, each lane owning 8
// consecutive dimensions (one 16-byte chunk of a row).  Each key group keeps its own running max / running sum /
// accumulator (log2 units); at the end of the chunk the groups and warps are
// merged and the chunk's normalised partial output and LSE are written.  The
// combine kernel merges the chunks of a sequence:
//   lse = ln sum_s exp(lse_s),  o = sum_s exp(lse_s - lse) o_s.
#pragma once
#include "sm100.cuh"

namespace fa {

struct DecParams {
  const int* seqlens;      // [B] keys per sequence (device)
  const uint16_t* q;       // [B, Hq, D] bf16
  float* o_part;           // [B, Hq, max_splits, D]
  float* lse_part;         // [B, Hq, max_splits] (natural log)
  int B, Hq, Hkv, Lmax, max_splits, chunk;
  float scale_log2;
  uint64_t wait_limit_ns;
};

template <int D, int GP>
struct DecCfg {
  static constexpr int T = 32;                  // keys per TMA box
  static constexpr int NS = 4;                  // ring slots (K and V tile each)
  static constexpr int NW = 4;                  // consumer warps
  static constexpr int LPK = D / 8;             // lanes per key (8 dimensions each)
  static constexpr int KPW = 32 / LPK;          // keys per warp step
  static constexpr int TILE_BYTES = T * D * 2;
  static constexpr int STAGE_BYTES = 2 * TILE_BYTES;
  static constexpr int MRG_FLOATS = NW * GP * (D + 2);
  static constexpr int BAR_OFF = NS * STAGE_BYTES + MRG_FLOATS * 4;
  static constexpr int SMEM_BYTES = BAR_OFF + 2 * NS * 8 + 128;
  static constexpr int THREADS = (NW + 1) * 32;
  static_assert((T / NW) % KPW == 0, "keys per warp must be a multiple of keys per step");
};

constexpr float DEC_TAU = 8.0f;

enum : uint32_t { W_DEC_FULL = 0x201, W_DEC_EMPTY = 0x202, W_DEC_DRAIN = 0x203 };

__device__ __forceinline__ void bf16x8_to_f32(const uint4 u, float* f) {
  f[0] = __uint_as_float(u.x << 16); f[1] = __uint_as_float(u.x & 0xffff0000u);
  f[2] = __uint_as_float(u.y << 16); f[3] = __uint_as_float(u.y & 0xffff0000u);
  f[4] = __uint_as_float(u.z << 16); f[5] = __uint_as_float(u.z & 0xffff0000u);
  f[6] = __uint_as_float(u.w << 16); f[7] = __uint_as_float(u.w & 0xffff0000u);
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

template <int D, int GP>
__global__ void __launch_bounds__(DecCfg<D, GP>::THREADS, 3)
decode_split_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                    const DecParams p) {
  using C = DecCfg<D, GP>;
  constexpr int NS = C::NS, T = C::T, LPK = C::LPK, KPW = C::KPW, NW = C::NW;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
  float* mrg = reinterpret_cast<float*>(smem + NS * C::STAGE_BYTES);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);
  uint64_t* empty = full + NS;

  const int split = blockIdx.x;
  const int groups_per_kv = (p.Hq / p.Hkv) / GP;
  const int hkv = blockIdx.y / groups_per_kv;
  const int hq0 = hkv * (p.Hq / p.Hkv) + (blockIdx.y % groups_per_kv) * GP;
  const int b = blockIdx.z;
  const int len = min(max(p.seqlens[b], 0), p.Lmax);
  const int k_begin = split * p.chunk;
  if (k_begin >= len) return;                   // this chunk is past the sequence: nothing to write
  const int k_end = min(len, k_begin + p.chunk);
  const int ntiles = (k_end - k_begin + T - 1) / T;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint64_t lim = p.wait_limit_ns;

  if (threadIdx.x == 0) {
    for (int i = 0; i < NS; ++i) { mbar_init(&full[i], 1); mbar_init(&empty[i], NW); }
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == NW) {
    // ------------------------------------------------------------ producer --
    if (lane == 0) {
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      int issued = 0;
      for (int i = 0; i < ntiles; ++i) {
        const int s = i % NS;
        if (i >= NS && !mbar_wait(&empty[s], ((i / NS) + 1) & 1, lim, W_DEC_EMPTY)) break;
        mbar_arrive_expect_tx(&full[s], C::STAGE_BYTES);
        uint8_t* dst = smem + s * C::STAGE_BYTES;
        tma_load_4d(dst, &tm_k, &full[s], 0, hkv, k_begin + i * T, b);
        tma_load_4d(dst + C::TILE_BYTES, &tm_v, &full[s], 0, hkv, k_begin + i * T, b);
        issued = i + 1;
      }
      for (int i = max(0, issued - NS); i < issued; ++i) mbar_wait(&full[i % NS], (i / NS) & 1, lim, W_DEC_DRAIN);
    }
    return;
  }

  // -------------------------------------------------------------- consumers --
  const int kg = lane / LPK;                    // key slot within a warp step
  const int ds = lane % LPK;                    // 16-byte chunk: dimensions 8*ds .. 8*ds+7
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
  constexpr int KS = (T / NW) / KPW;
  bool ok = true;
  for (int i = 0; i < ntiles; ++i) {
    const int s = i % NS;
    if (!(ok = mbar_wait(&full[s], (i / NS) & 1, lim, W_DEC_FULL))) break;
    const uint8_t* ks = smem + s * C::STAGE_BYTES;
    const uint8_t* vs = ks + C::TILE_BYTES;
    const int key0 = k_begin + i * T;
    const bool full_tile = key0 + T <= k_end;
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
    if (!full_tile) {                             // keys past the chunk end do not count
#pragma unroll
      for (int st = 0; st < KS; ++st) {
        const int kt = warp * (T / NW) + st * KPW + kg;
        if (key0 + kt >= k_end) {
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
      if (mt > m[g] + DEC_TAU) {                  // false while both are -inf
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
      if (!full_tile && key0 + kt >= k_end) continue;   // never read V rows past the chunk end
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
  asm volatile("bar.sync 1, %0;" :: "r"(NW * 32) : "memory");
  if (!ok) return;
  for (int idx = threadIdx.x; idx < GP * D; idx += NW * 32) {
    const int g = idx / D, d = idx % D;
    float mw[NW], mx = -INFINITY;
#pragma unroll
    for (int w = 0; w < NW; ++w) { mw[w] = mrg[(w * GP + g) * (D + 2)]; mx = fmaxf(mx, mw[w]); }
    float L = 0.f, O = 0.f;
#pragma unroll
    for (int w = 0; w < NW; ++w) {
      const float* src = mrg + (w * GP + g) * (D + 2);
      const float a = (mw[w] == -INFINITY) ? 0.f : ex2_approx(mw[w] - mx);
      L = fmaf(src[1], a, L);
      O = fmaf(src[2 + d], a, O);
    }
    const size_t prow = (static_cast<size_t>(b) * p.Hq + hq0 + g) * p.max_splits + split;
    p.o_part[prow * D + d] = L > 0.f ? O / L : 0.f;
    if (d == 0) p.lse_part[prow] = L > 0.f ? (mx + log2f(L)) * LN2 : -INFINITY;
  }
}

struct CombineParams {
  const float* o_part;     // [B, Hq, max_splits, D]
  const float* lse_part;   // [B, Hq, max_splits]
  const int* counts;       // [B]: number of valid parts, or key counts when chunk > 0; may be null
  void* o;                 // [B, Hq, D] bf16 or fp32
  float* lse;              // [B, Hq] or null
  int B, Hq, D, max_splits, chunk, o_fp32;
};

// One block per (sequence, head); thread d owns output column d.
__global__ void __launch_bounds__(128) decode_combine_kernel(const CombineParams p) {
  const int bh = blockIdx.x;
  const int b = bh / p.Hq;
  int ns = p.max_splits;
  if (p.counts != nullptr) {
    const int c = max(p.counts[b], 0);
    ns = p.chunk > 0 ? (c + p.chunk - 1) / p.chunk : c;
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
    if (p.o_fp32) static_cast<float*>(p.o)[static_cast<size_t>(bh) * p.D + d] = v;
    else static_cast<__nv_bfloat16*>(p.o)[static_cast<size_t>(bh) * p.D + d] = __float2bfloat16_rn(v);
  }
  if (threadIdx.x == 0 && p.lse != nullptr) p.lse[bh] = has ? mx + logf(wsum) : -INFINITY;
}

}  // namespace fa
