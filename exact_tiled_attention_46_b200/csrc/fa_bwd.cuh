// Backward pass with the probabilities recomputed from the saved LSE instead
// of being stored ("FlashAttention Explained: How AI Models Process Attention
// Faster and Use Less Memory", section "More Efficient Backpropagation"; "How
// FlashAttention Speeds Up LLM Attention", "Recompute probabilities for
// training").  With S = scale Q K^T and P = exp(S - LSE):
//     dV = P^T dO,   dP = dO V^T,   Delta_i = sum_d dO_id O_id,
//     dS = P * (dP - Delta),   dQ = scale dS K,   dK = scale dS^T Q.
//
// The products run on fp16 operands.  Every bf16 input value is an fp16 value
// once scaled by a power of two into fp16's range, so each input tensor is
// scaled by 2^k (from its largest magnitude) and converted exactly: Q, K, V to
// a largest magnitude in [2^7, 2^8), dO so that |dP|, |Delta| and |dS| stay
// below 2^15.  P^T and dS^T enter the products as single fp16 values (10
// fraction bits); the scales come out exactly at the end.
//
// Four launches on the caller's stream (plus memsets of the dQ accumulator and
// of the four maxima):
//   bwd_amax_kernel  the largest |q|, |k|, |v|, |dO|.
//   bwd_pre_kernel   Delta, the LSE in log2 units (+inf for rows without a key,
//                    so that their P is 0), both padded to 128-row tiles; the
//                    scaled fp16 copies of q and dO.
//   bwd_main_kernel  persistent (at most one CTA per SM); a work item is one
//                    (batch, kv head, 128-key tile), numbered head-major and
//                    taken from a launch-wide counter through a two-entry item
//                    queue in shared memory; per item it loops over the (query
//                    tile, query head of the group) pairs:
//        warp 12    takes items and posts them; TMA: the item's K, V (bf16,
//                   converted to scaled fp16 in place by warps 0-7; two
//                   buffers at D = 64, so the next item's tile loads during
//                   this one); Q, dO (fp16 copies), LSE, Delta per pair (NQ
//                   stages, running on from item to item)
//        warp 13    tcgen05: S^T = K Q^T and dP^T = V dO^T into TMEM,
//                   dV += P^T dO, dK += dS^T Q, dQ = dS K
//        P^T (fp16) goes to TMEM over S^T columns already read, dS^T (fp16)
//        to swizzled shared memory.
//        warps 0-7  one thread per key row; warps w and w + 4 share a TMEM lane
//                   quadrant and take 64 of the 128 query columns each (no row
//                   reduction is needed: P = 2^(s - LSE)); causal / ragged mask
//                   on the tiles that need it; P^T is published first (the dV
//                   product, then the next pair's S^T, run while dS^T is
//                   formed from P kept in registers)
//        warps 8-11 one thread per query row: dQ tile from TMEM (two buffers at
//                   D = 64) into a swizzled shared-memory box per warp, added to
//                   the fp32 accumulator by TMA reduce-add (32 rows x 32
//                   columns per operation); after an item's last pair its dK,
//                   dV out of TMEM, while the next item's first pairs start
//                   (their first dV / dK products wait for this read-out)
//        warp 14    TMEM allocation; warp 15 idles.  The control warpgroup
//                   (12-15) lends registers to the other three.
//   bwd_post_kernel  dQ = scale * accumulator (with the input scales taken
//                    out), converted to the output dtype.
#pragma once
#include "sm100.cuh"
#include "fa.h"

namespace fa {

// Instruction descriptor, kind::f16 with A and B fp16 (format 0), D fp32;
// bits as for idesc_bf16_f32.
__host__ __device__ constexpr uint32_t idesc_f16_f32(int M, int N, bool a_mn_major, bool b_mn_major) {
  return (1u << 4) | (uint32_t(a_mn_major) << 15) | (uint32_t(b_mn_major) << 16) | (uint32_t(N >> 3) << 17) |
         (uint32_t(M >> 4) << 24);
}
// Two floats rounded (nearest even) to fp16, packed with lo in the low half.
__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

template <int D>
struct BwdCfg {
  static constexpr int TILE = 128 * D * 2;            // 128 rows of bf16
  static constexpr int NQ = (D == 64) ? 2 : 1;        // Q/dO stages (two do not fit at D = 128)
  static constexpr bool DQ_IN_DP = (D == 128);        // dQ reuses the dP^T columns
  static constexpr int DQ_BUFS = DQ_IN_DP ? 1 : 2;    // dQ TMEM buffers
  static constexpr int KVB = (D == 64) ? 2 : 1;       // K/V buffers (the next key tile loads during this one)
  static constexpr int K_OFF = 0;                     // buffer u: K at +u*2*TILE, V after it
  static constexpr int V_OFF = TILE;
  static constexpr int Q_OFF = KVB * 2 * TILE;        // stage s: Q at +s*2*TILE, dO after it
  static constexpr int DS_OFF = Q_OFF + NQ * 2 * TILE;
  static constexpr int DS_BYTES = 128 * 128 * 2;     // one 128 x 128 fp16 operand (128B swizzle)
  static constexpr int DS_BUFS = 1;                   // dS^T buffers (two measured slower at D = 64)
  static constexpr int ROW_OFF = DS_OFF + DS_BUFS * DS_BYTES;   // stage s: lse2[128], delta[128]
  // dQ staging: per read-out warp two 4 KB boxes (32 rows x 32 fp32, 128-byte swizzle)
  static constexpr int DQS_OFF = ROW_OFF + NQ * 1024;
  static constexpr int BAR_OFF = DQS_OFF + 4 * 8192;
  static constexpr int NBARS = 3 * KVB + 2 * NQ + 6 + 4 + 2 + 4 + 1;
  static constexpr int SMEM_BYTES = BAR_OFF + NBARS * 8 + 32 + 1024;   // + TMEM address, item queue
  // TMEM columns
  static constexpr uint32_t T_S = 0, T_DP = 128, T_DV = 256, T_DK = 256 + D;
  static constexpr uint32_t T_DQ = DQ_IN_DP ? T_DP : 256 + 2 * D;   // buffer b at T_DQ + b * D
  static constexpr int THREADS = 512;
};

struct BwdParams {
  const float* lse2;     // [B*Hq, Lq_pad]  LSE * log2(e), +inf on rows without keys / padding
  const float* delta;    // [B*Hq, Lq_pad]  Delta times the dO and V scales
  const uint32_t* amax;  // largest |q|, |k|, |v|, |dO| (float bits)
  void* dk;              // [B, Lk, Hkv, D]
  void* dv;
  int B, Hq, Hkv, Lq, Lk, Lq_pad;
  int num_items;         // key tiles: B * Hkv * ceil(Lk / 128)
  int* work_counter;     // next key tile to take; 0 when the launch starts
  float scale, scale_log2;
  int g_fp32;
  uint64_t wait_limit_ns;
};

constexpr int BWD_LAUNCH_REGS = 128, BWD_WORK_REGS = 136, BWD_CTRL_REGS = 104;
static_assert(3 * BWD_WORK_REGS + BWD_CTRL_REGS == 4 * BWD_LAUNCH_REGS, "register split must match the launch");

enum : uint32_t {
  W_BWD_KV = 0x301, W_BWD_QF = 0x302, W_BWD_QE = 0x303, W_BWD_SDP = 0x304, W_BWD_P = 0x305,
  W_BWD_DS = 0x306, W_BWD_DSF = 0x307, W_BWD_DQF = 0x308, W_BWD_DQ = 0x309, W_BWD_DKV = 0x30a,
  W_BWD_DONE = 0x30b, W_BWD_DRAIN = 0x30c, W_BWD_ITEM = 0x30d, W_BWD_ITEM_EMPTY = 0x30e, W_BWD_KVF = 0x30f
};

// A work item is one (batch, kv head, 128-key tile), numbered head-major: the
// key tiles of one (b, kv head) are adjacent, heaviest (j = 0) first, so the
// items running at the same time touch a few heads' Q, dO and fp32 dQ
// accumulator, which then stay in L2 (all heads together do not).
struct BwdItem {
  int b, hkv, j, i0, npairs;
};
template <bool CAUSAL>
__device__ __forceinline__ BwdItem bwd_item(const BwdParams& p, int w) {
  BwdItem I;
  const int nk = (p.Lk + 127) >> 7, nq = (p.Lq + 127) >> 7;
  I.j = w % nk;
  const int bh = w / nk;
  I.b = bh / p.Hkv;
  I.hkv = bh % p.Hkv;
  I.i0 = 0;
  if (CAUSAL) {
    const int first_q = I.j * 128 - (p.Lk - p.Lq);        // lowest query that sees a key of this tile
    I.i0 = first_q <= 0 ? 0 : (first_q >> 7);
  }
  I.npairs = (I.i0 < nq) ? (nq - I.i0) * (p.Hq / p.Hkv) : 0;
  return I;
}

__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
               :: "r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar)) : "memory");
}

// Power-of-two input scales.  k maps the largest magnitude into [2^t, 2^(t+1))
// (0 for an all-zero, subnormal-only, inf or NaN tensor), clamped to [-60, 60]
// so that every factor and its products stay finite in fp32.
__device__ __forceinline__ int bwd_pow2_exp(uint32_t amax_bits, int t) {
  const int e = static_cast<int>((amax_bits >> 23) & 0xffu);
  if (e == 0 || e == 255) return 0;
  return max(-60, min(60, t - (e - 127)));
}
__device__ __forceinline__ float bwd_pow2(int k) { return __int_as_float((127 + k) << 23); }
struct BwdScales {
  int kq, kk, kv, kdo;
};
// Q, K, V to [2^7, 2^8); dO to [2^(5-log2 D), 2^(6-log2 D)), so that
// |dP^T|, |Delta| <= D * |dO| * |V| < 2^14 and |dS^T| < 2^15 (fp16: 65504).
__device__ __forceinline__ BwdScales bwd_scales(const uint32_t* amax, int D) {
  BwdScales sc;
  sc.kq = bwd_pow2_exp(amax[0], 7);
  sc.kk = bwd_pow2_exp(amax[1], 7);
  sc.kv = bwd_pow2_exp(amax[2], 7);
  sc.kdo = bwd_pow2_exp(amax[3], D == 128 ? -2 : -1);
  return sc;
}

// Largest |x| of q, k, v, dO (bf16) into amax[0..3] (float bits; zeroed
// before).  blockIdx.y picks the tensor; one atomic per block.
__global__ void __launch_bounds__(256) bwd_amax_kernel(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                                                       const uint16_t* dO, size_t nq, size_t nk, uint32_t* amax) {
  __shared__ uint32_t wmax[8];
  const int t = static_cast<int>(blockIdx.y);
  const uint16_t* src = t == 0 ? q : t == 1 ? k : t == 2 ? v : dO;
  const uint4* p4 = reinterpret_cast<const uint4*>(src);
  const size_t n8 = ((t == 1 || t == 2) ? nk : nq) / 8;   // element counts are multiples of D (64 or 128)
  const size_t stride = size_t(gridDim.x) * blockDim.x;
  uint32_t m = 0;
  for (size_t i = blockIdx.x * size_t(blockDim.x) + threadIdx.x; i < n8; i += 4 * stride) {
    uint4 w[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) w[u] = (i + u * stride < n8) ? p4[i + u * stride] : make_uint4(0, 0, 0, 0);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const uint32_t ws[4] = {w[u].x, w[u].y, w[u].z, w[u].w};
#pragma unroll
      for (int e = 0; e < 4; ++e) m = max(m, max(ws[e] & 0x7fffu, (ws[e] >> 16) & 0x7fffu));
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int w = 1; w < static_cast<int>(blockDim.x >> 5); ++w) m = max(m, wmax[w]);
    if (m != 0) atomicMax(&amax[t], m << 16);      // |x| as float bits
  }
}

// Delta = rowsum(dO * O) and the log2-scaled LSE, both padded to Lq_pad rows;
// also the scaled fp16 copies of q and dO.  Delta carries the dO and V scales
// of the dP^T products.  One thread per 8-element chunk of a (b, i, h) row,
// h fastest, so that a warp reads and writes contiguous memory; the D / 8
// threads of a row sum Delta with shuffles.
__global__ void __launch_bounds__(256) bwd_pre_kernel(const uint16_t* o, const uint16_t* dO, const uint16_t* q,
                                                      const float* lse, const uint32_t* amax, float* lse2,
                                                      float* delta, uint16_t* q16, uint16_t* do16, int B, int Hq,
                                                      int Lq, int Lq_pad, int D) {
  const BwdScales sc = bwd_scales(amax, D);
  const float fq = bwd_pow2(sc.kq), fdo = bwd_pow2(sc.kdo), fdelta = bwd_pow2(sc.kdo + sc.kv);
  const int cpr = D / 8;                           // chunks per row: 8 or 16, a power of two dividing 32
  const size_t n = size_t(B) * Lq_pad * Hq * cpr;  // a multiple of 32: Lq_pad is a multiple of 128
  for (size_t t = blockIdx.x * size_t(blockDim.x) + threadIdx.x; t < n; t += size_t(gridDim.x) * blockDim.x) {
    const int c = static_cast<int>(t % cpr);
    const size_t rr = t / cpr;
    const int h = static_cast<int>(rr % Hq);
    const size_t bi = rr / Hq;
    const int i = static_cast<int>(bi % Lq_pad);
    const int b = static_cast<int>(bi / Lq_pad);
    float acc = 0.f;
    if (i < Lq) {
      const size_t off = ((size_t(b) * Lq + i) * Hq + h) * D / 8 + c;     // in 16-byte chunks
      const uint4 a = reinterpret_cast<const uint4*>(o)[off];
      const uint4 g = reinterpret_cast<const uint4*>(dO)[off];
      const uint4 x = reinterpret_cast<const uint4*>(q)[off];
      const uint32_t av[4] = {a.x, a.y, a.z, a.w}, gv[4] = {g.x, g.y, g.z, g.w}, xv[4] = {x.x, x.y, x.z, x.w};
      uint32_t hq[4], hd[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float g0 = __uint_as_float(gv[e] << 16), g1 = __uint_as_float(gv[e] & 0xffff0000u);
        acc = fmaf(__uint_as_float(av[e] << 16), g0, acc);
        acc = fmaf(__uint_as_float(av[e] & 0xffff0000u), g1, acc);
        hd[e] = pack_f16x2(g0 * fdo, g1 * fdo);
        hq[e] = pack_f16x2(__uint_as_float(xv[e] << 16) * fq, __uint_as_float(xv[e] & 0xffff0000u) * fq);
      }
      reinterpret_cast<uint4*>(q16)[off] = make_uint4(hq[0], hq[1], hq[2], hq[3]);
      reinterpret_cast<uint4*>(do16)[off] = make_uint4(hd[0], hd[1], hd[2], hd[3]);
    }
    // the row's chunks are cpr consecutive lanes of one warp (every lane of the
    // warp takes part: the loop bound is a multiple of 32)
    for (int m = 1; m < cpr; m <<= 1) acc += __shfl_xor_sync(0xffffffffu, acc, m);
    if (c == 0) {
      const size_t dst = (size_t(b) * Hq + h) * Lq_pad + i;
      if (i >= Lq) {
        lse2[dst] = INFINITY;
        delta[dst] = 0.f;
      } else {
        const float l = lse[(size_t(b) * Hq + h) * Lq + i];
        lse2[dst] = (l == -INFINITY) ? INFINITY : l * 1.4426950408889634f;
        delta[dst] = acc * fdelta;
      }
    }
  }
}

__global__ void __launch_bounds__(256) bwd_post_kernel(const float* acc, void* dq, size_t n, float scale_in,
                                                       const uint32_t* amax, int D, int g_fp32) {
  const BwdScales sc = bwd_scales(amax, D);
  const float scale = scale_in * bwd_pow2(-(sc.kdo + sc.kv + sc.kk));   // dS^T carries dO, V scales; K its own
  for (size_t t = blockIdx.x * size_t(blockDim.x) + threadIdx.x; t < n / 4; t += size_t(gridDim.x) * blockDim.x) {
    const float4 v = reinterpret_cast<const float4*>(acc)[t];
    if (g_fp32) {
      reinterpret_cast<float4*>(dq)[t] = make_float4(v.x * scale, v.y * scale, v.z * scale, v.w * scale);
    } else {
      uint2 w;
      w.x = pack_bf16x2(v.x * scale, v.y * scale);
      w.y = pack_bf16x2(v.z * scale, v.w * scale);
      reinterpret_cast<uint2*>(dq)[t] = w;
    }
  }
}

template <int D, bool CAUSAL>
__global__ void __launch_bounds__(512, 1)
bwd_main_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                const __grid_constant__ CUtensorMap tm_dq, const BwdParams p) {
  using C = BwdCfg<D>;
  constexpr int NQ = C::NQ, KB = D / 64, NB = C::DQ_BUFS;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);
  uint64_t* kv_full = bars;                       // [KVB] K and V landed
  uint64_t* kv_conv = kv_full + C::KVB;           // [KVB] K and V converted to fp16 in shared memory
  uint64_t* kv_free = kv_conv + C::KVB;           // [KVB] the item's last product read them
  uint64_t* q_full = kv_free + C::KVB;
  uint64_t* q_empty = q_full + NQ;
  uint64_t* s_full = q_empty + NQ;                // S^T of the pair is in TMEM
  uint64_t* dp_full = s_full + 1;                 // dP^T of the pair is in TMEM
  uint64_t* p_ready = dp_full + 1;
  uint64_t* ds_ready = p_ready + 1;
  uint64_t* ds_free = ds_ready + 1;      // [2] per dS^T buffer
  uint64_t* dq_full = ds_free + 2;       // [2]
  uint64_t* dq_free = dq_full + 2;       // [2]
  uint64_t* dkv_done = dq_free + 2;               // the item's dK, dV are in TMEM
  uint64_t* dkv_free = dkv_done + 1;              // and have been read out
  uint64_t* item_full = dkv_free + 1;             // [2] an item number was posted
  uint64_t* item_empty = item_full + 2;           // [2] every role has read it
  uint64_t* mma_done = item_empty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + C::NBARS);
  volatile int* item_w = reinterpret_cast<volatile int*>(tmem_holder + 4);   // [2] item numbers (-1: none left)

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint64_t lim = p.wait_limit_ns;
  const int G = p.Hq / p.Hkv;
  const int off = p.Lk - p.Lq;

  if (threadIdx.x == 0) {
    for (int u = 0; u < C::KVB; ++u) { mbar_init(&kv_full[u], 1); mbar_init(&kv_conv[u], 256); mbar_init(&kv_free[u], 1); }
    for (int s = 0; s < NQ; ++s) { mbar_init(&q_full[s], 1); mbar_init(&q_empty[s], 1); }
    mbar_init(s_full, 1);
    mbar_init(dp_full, 1);
    mbar_init(p_ready, 256);
    mbar_init(ds_ready, 256);
    mbar_init(&ds_free[0], 1);
    mbar_init(&ds_free[1], 1);
    for (int u = 0; u < 2; ++u) { mbar_init(&dq_full[u], 1); mbar_init(&dq_free[u], 128); }
    mbar_init(dkv_done, 1);
    mbar_init(dkv_free, 128);
    // item queue readers: the MMA thread, lane 0 of the eight compute and four dQ warps
    for (int u = 0; u < 2; ++u) { mbar_init(&item_full[u], 1); mbar_init(&item_empty[u], 13); }
    mbar_init(mma_done, 1);
    fence_mbar_init();
  }
  if (warp == 14) { tmem_alloc(tmem_holder, 512); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp >= 12) {
  setmaxnreg_dec<BWD_CTRL_REGS>();
  if (warp == 12) {
    // ------------------------------------------------------------ producer --
    // Takes key tiles from the launch-wide counter, posts each to the item
    // queue, loads its K and V (into the buffer its previous user released)
    // and then Q, dO, LSE, Delta pair by pair through the NQ stages.
    if (lane == 0) {
      tma_prefetch_desc(&tm_q); tma_prefetch_desc(&tm_do);
      bool ok = true;
      int it = 0, gp = 0;                          // items with pairs, pairs issued so far
      for (int ni = 0; ok; ++ni) {
        const int qs = ni & 1;
        if (ni >= 2 && !(ok = mbar_wait(&item_empty[qs], ((ni >> 1) + 1) & 1, lim, W_BWD_ITEM_EMPTY))) break;
        const int w0 = atomicAdd(p.work_counter, 1);
        const int w = w0 < p.num_items ? w0 : -1;
        item_w[qs] = w;
        mbar_arrive(&item_full[qs]);               // release: the readers' wait sees the number
        if (w < 0) break;
        const BwdItem I = bwd_item<CAUSAL>(p, w);
        if (I.npairs == 0) continue;
        const int u = it % C::KVB;
        if (it >= C::KVB && !(ok = mbar_wait(&kv_free[u], ((it / C::KVB) + 1) & 1, lim, W_BWD_KVF))) break;
        mbar_arrive_expect_tx(&kv_full[u], 2 * C::TILE);
        uint8_t* kvd = smem + u * 2 * C::TILE;
        for (int kb = 0; kb < KB; ++kb) {
          tma_load_4d(kvd + C::K_OFF + kb * 16384, &tm_k, &kv_full[u], kb * 64, I.hkv, I.j * 128, I.b);
          tma_load_4d(kvd + C::V_OFF + kb * 16384, &tm_v, &kv_full[u], kb * 64, I.hkv, I.j * 128, I.b);
        }
        ++it;
        for (int n = 0; ok && n < I.npairs; ++n) {
          const int g = gp + n, s = g % NQ;
          if (g >= NQ && !(ok = mbar_wait(&q_empty[s], ((g / NQ) + 1) & 1, lim, W_BWD_QE))) break;
          const int i = I.i0 + n / G, hq = I.hkv * G + n % G;
          mbar_arrive_expect_tx(&q_full[s], 2 * C::TILE + 1024);
          uint8_t* qdst = smem + C::Q_OFF + s * 2 * C::TILE;
          for (int kb = 0; kb < KB; ++kb) {
            tma_load_4d(qdst + kb * 16384, &tm_q, &q_full[s], kb * 64, hq, i * 128, I.b);
            tma_load_4d(qdst + C::TILE + kb * 16384, &tm_do, &q_full[s], kb * 64, hq, i * 128, I.b);
          }
          const size_t rowbase = (size_t(I.b) * p.Hq + hq) * p.Lq_pad + size_t(i) * 128;
          float* rdst = reinterpret_cast<float*>(smem + C::ROW_OFF + s * 1024);
          bulk_load(rdst, p.lse2 + rowbase, 512, &q_full[s]);
          bulk_load(rdst + 128, p.delta + rowbase, 512, &q_full[s]);
        }
        gp += I.npairs;
      }
      // the CTA may not exit with copies in flight: wait for the last loads
      for (int k = max(0, it - C::KVB); k < it; ++k)
        mbar_wait(&kv_full[k % C::KVB], (k / C::KVB) & 1, lim, W_BWD_DRAIN);
      for (int g = max(0, gp - NQ); g < gp; ++g) mbar_wait(&q_full[g % NQ], (g / NQ) & 1, lim, W_BWD_DRAIN);
    }
  } else if (warp == 13) {
    // ----------------------------------------------------------------- MMA --
    if (lane == 0) {
      constexpr uint32_t ID_SS = idesc_f16_f32(128, 128, false, false);    // S^T, dP^T
      constexpr uint32_t ID_DVK = idesc_f16_f32(128, D, false, true);      // dV, dK: B = dO / Q (MN-major)
      constexpr uint32_t ID_DQ = idesc_f16_f32(128, D, true, true);        // dQ: A = dS (MN-major), B = K (MN-major)
      const uint32_t q_base = smem_u32(smem + C::Q_OFF), ds_base = smem_u32(smem + C::DS_OFF);
      // P^T of queries 16kk..16kk+15 in TMEM: 8 columns (fp16 pairs) at the start
      // of the S^T columns of query half kk / 4 that the compute warp has read
      auto p_col = [](int kk) { return C::T_S + (kk >> 2) * 64 + (kk & 3) * 8; };
      auto kmaj = [](uint32_t base, int kk) { return sdesc_sw128(base + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024); };
      auto mnmaj = [](uint32_t base, int kk) { return sdesc_sw128(base + kk * 2048, 16384, 1024); };
      uint32_t k_base = 0, v_base = 0;             // this item's K / V buffer
      auto issue_s = [&](int g) {                  // g: pair index over the CTA's items
        const uint32_t qa = q_base + (g % NQ) * 2 * C::TILE;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) umma_ss(tmem + C::T_S, kmaj(k_base, kk), kmaj(qa, kk), ID_SS, kk > 0);
        umma_commit(s_full);
      };
      auto issue_dp = [&](int g) {
        const uint32_t da = q_base + (g % NQ) * 2 * C::TILE + C::TILE;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) umma_ss(tmem + C::T_DP, kmaj(v_base, kk), kmaj(da, kk), ID_SS, kk > 0);
        umma_commit(dp_full);
      };
      bool ok = true;
      int it = 0, gp = 0;
      for (int ni = 0; ok; ++ni) {
        const int qs = ni & 1;
        if (!(ok = mbar_wait(&item_full[qs], (ni >> 1) & 1, lim, W_BWD_ITEM))) break;
        const int w = item_w[qs];
        mbar_arrive(&item_empty[qs]);
        if (w < 0) break;
        const BwdItem I = bwd_item<CAUSAL>(p, w);
        if (I.npairs == 0) continue;
        const int u = it % C::KVB;
        k_base = smem_u32(smem + u * 2 * C::TILE + C::K_OFF);
        v_base = smem_u32(smem + u * 2 * C::TILE + C::V_OFF);
        if (!(ok = mbar_wait(&kv_conv[u], (it / C::KVB) & 1, lim, W_BWD_KV) &&
                   mbar_wait(&q_full[gp % NQ], (gp / NQ) & 1, lim, W_BWD_QF)))
          break;
        // with dQ in the dP^T columns, the previous item's last dQ must be read out first
        if (C::DQ_IN_DP && gp > 0 && !(ok = mbar_wait(&dq_free[0], (gp - 1) & 1, lim, W_BWD_DQF))) break;
        tc_fence_after();
        issue_s(gp);
        issue_dp(gp);
        for (int n = 0; ok && n < I.npairs; ++n) {
          const int g = gp + n, s = g % NQ, bq = g % NB;
          const uint32_t qa = q_base + s * 2 * C::TILE, da = qa + C::TILE;
          const bool more = n + 1 < I.npairs;
          const int db = g % C::DS_BUFS;
          const uint32_t dsa = ds_base + db * C::DS_BYTES;   // this pair's dS^T buffer
          if (!(ok = mbar_wait(p_ready, g & 1, lim, W_BWD_P))) break;
          // the first dV / dK products overwrite the accumulators: the previous
          // item's dK, dV must have been read out
          if (n == 0 && it > 0 && !(ok = mbar_wait(dkv_free, (it - 1) & 1, lim, W_BWD_DKV))) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)      // dV += P^T dO  (K = 128 queries)
            umma_ts(tmem + C::T_DV, tmem + p_col(kk), mnmaj(da, kk), ID_DVK, (n > 0 || kk > 0) ? 1u : 0u);
          // the next pair's S^T goes over P^T as soon as the dV products are issued
          // (the pipe runs them in order; the compute warps keep P in registers),
          // when its Q has a stage of its own (with one stage, Q(n+1) replaces
          // Q(n) only after this pair's last product)
          if (more && NQ > 1) {
            if (!(ok = mbar_wait(&q_full[(g + 1) % NQ], ((g + 1) / NQ) & 1, lim, W_BWD_QF))) break;
            tc_fence_after();
            issue_s(g + 1);
          }
          if (!(ok = mbar_wait(ds_ready, g & 1, lim, W_BWD_DS))) break;
          tc_fence_after();
          if (!C::DQ_IN_DP && more) issue_dp(g + 1);   // dP^T was read by the dS^T phase
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)      // dK += dS^T Q  (K = 128 queries)
            umma_ss(tmem + C::T_DK, kmaj(dsa, kk), mnmaj(qa, kk), ID_DVK, (n > 0 || kk > 0) ? 1u : 0u);
          if (!C::DQ_IN_DP && g >= NB) {      // this dQ buffer must have been read out (pair g - NB)
            if (!(ok = mbar_wait(&dq_free[bq], ((g / NB) - 1) & 1, lim, W_BWD_DQF))) break;
            tc_fence_after();
          }
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)      // dQ = dS K  (K = 128 keys)
            umma_ss(tmem + C::T_DQ + bq * D, mnmaj(dsa, kk), mnmaj(k_base, kk), ID_DQ, kk > 0 ? 1u : 0u);
          umma_commit(&dq_full[bq]);
          umma_commit(&ds_free[db]);
          umma_commit(&q_empty[s]);
          if (C::DQ_IN_DP && more) {          // dP^T(g+1) overwrites dQ(g): wait for its read-out
            if (!(ok = mbar_wait(&dq_free[0], g & 1, lim, W_BWD_DQF))) break;
            tc_fence_after();
          }
          if (more && NQ == 1) {
            if (!(ok = mbar_wait(&q_full[(g + 1) % NQ], ((g + 1) / NQ) & 1, lim, W_BWD_QF))) break;
            tc_fence_after();
            issue_s(g + 1);
          }
          if (C::DQ_IN_DP && more) issue_dp(g + 1);
        }
        if (!ok) break;
        umma_commit(dkv_done);                     // dK, dV complete for the read-out
        umma_commit(&kv_free[u]);                  // the item's K and V are no longer read
        ++it;
        gp += I.npairs;
      }
      // nothing may be in flight on the tensor pipe when the CTA tears down
      umma_commit(mma_done);
      mbar_wait(mma_done, 0, lim, W_BWD_DONE);
    }
  }
  // take the launch budget back only after the other warpgroups returned theirs
  asm volatile("bar.sync 2, %0;" :: "n"(C::THREADS) : "memory");
  setmaxnreg_inc<BWD_LAUNCH_REGS>();
  } else if (warp < 8) {
    setmaxnreg_inc<BWD_WORK_REGS>();
    // --------------------------------------------- P^T and dS^T (key rows) --
    const int wq = warp & 3, hh = warp >> 2;          // lane quadrant, which 64 query columns
    const int r = wq * 32 + lane;
    const uint32_t lane_bits = static_cast<uint32_t>(wq * 32) << 16;
    const BwdScales sc_in = bwd_scales(p.amax, D);
    const float sl2 = p.scale_log2 * bwd_pow2(-(sc_in.kq + sc_in.kk));   // S^T carries the Q and K scales
    bool npairs_ok = true;
    int it = 0, gp = 0;
    for (int ni = 0; npairs_ok; ++ni) {
      const int qs = ni & 1;
      if (!mbar_wait_warp(&item_full[qs], (ni >> 1) & 1, lim, W_BWD_ITEM)) break;
      const int w = item_w[qs];
      __syncwarp();
      if (lane == 0) mbar_arrive(&item_empty[qs]);
      if (w < 0) break;
      const BwdItem I = bwd_item<CAUSAL>(p, w);
      if (I.npairs == 0) continue;
      const int u = it % C::KVB;
      const int key = I.j * 128 + r;
      // this item's K and V (bf16) to scaled fp16 in place, before its first product
      if (!mbar_wait_warp(&kv_full[u], (it / C::KVB) & 1, lim, W_BWD_KV)) {
        npairs_ok = false;
      } else {
        const float fk = bwd_pow2(sc_in.kk), fv = bwd_pow2(sc_in.kv);
        uint4* kv4 = reinterpret_cast<uint4*>(smem + u * 2 * C::TILE + C::K_OFF);   // K then V, contiguous
        constexpr int N16 = 2 * C::TILE / 16;
#pragma unroll 4
        for (int c = threadIdx.x; c < N16; c += 256) {
          const float f = (c < C::TILE / 16) ? fk : fv;
          const uint4 w = kv4[c];
          const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
          uint32_t hs[4];
#pragma unroll
          for (int e = 0; e < 4; ++e)
            hs[e] = pack_f16x2(__uint_as_float(ws[e] << 16) * f, __uint_as_float(ws[e] & 0xffff0000u) * f);
          kv4[c] = make_uint4(hs[0], hs[1], hs[2], hs[3]);
        }
        fence_proxy_async_smem();
        mbar_arrive(&kv_conv[u]);
      }
      for (int n = 0; npairs_ok && n < I.npairs; ++n) {
        const int g = gp + n, s = g % NQ;
        const int i = I.i0 + n / G;
        const float* lse2 = reinterpret_cast<const float*>(smem + C::ROW_OFF + s * 1024);
        const float* dlt = lse2 + 128;
        if (!(npairs_ok = mbar_wait_warp(s_full, g & 1, lim, W_BWD_SDP))) break;
        tc_fence_after();
        // allowed when key <= query + off, i.e. column c >= cmin (nothing for keys past Lk)
        const int cmin = key < p.Lk ? (CAUSAL ? key - off - i * 128 : -1) : (1 << 30);
        const int rowoff = r * 128;
        bool ok = true;
        // Phase 1: P^T = 2^(S^T * scale - LSE) (masked) for this warp's 64 query
        // columns, 16 at a time: kept in registers (fp32) for phase 2 and stored
        // as fp16 over S^T columns already read (8 columns per 16 queries, at the
        // start of this half's region), the A operand of the dV products;
        // published at once.
        float pv[64];
#pragma unroll
        for (int sc = 0; sc < 4; ++sc) {
          const int c0 = hh * 64 + sc * 16;              // first query column of this sub-chunk
          uint32_t sv[16];
          tmem_ld_32x32b_x16(tmem + lane_bits + C::T_S + c0, sv);
          // the mask only matters where some key row of the warp starts after c0
          // (the causal diagonal, keys past Lk); elsewhere every column is allowed
          const bool masked = __any_sync(0xffffffffu, cmin > c0);
          uint32_t ph[8];
#pragma unroll
          for (int t4 = 0; t4 < 4; ++t4) {
            const float4 l4 = *reinterpret_cast<const float4*>(lse2 + c0 + 4 * t4);
#pragma unroll
            for (int u = 0; u < 2; ++u) {
              const int t = 2 * t4 + u;
              const int c = c0 + 2 * t;
              float x0, x1;
              ffma2(x0, x1, __uint_as_float(sv[2 * t]), __uint_as_float(sv[2 * t + 1]), sl2, sl2,
                    -(u ? l4.z : l4.x), -(u ? l4.w : l4.y));
              float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
              if (masked) {
                p0 = (c >= cmin) ? p0 : 0.f;
                p1 = (c + 1 >= cmin) ? p1 : 0.f;
              }
              pv[sc * 16 + 2 * t] = p0;
              pv[sc * 16 + 2 * t + 1] = p1;
              ph[t] = pack_f16x2(p0, p1);
            }
          }
          tmem_st_32x32b_x8(tmem + lane_bits + C::T_S + hh * 64 + sc * 8, ph);
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(p_ready);
        // Phase 2: dS^T = P^T * (dP^T - Delta) into swizzled shared memory as
        // fp16, 16 query columns at a time.
        if (!(npairs_ok = mbar_wait_warp(dp_full, g & 1, lim, W_BWD_SDP))) break;
        tc_fence_after();
#pragma unroll
        for (int sc = 0; sc < 4; ++sc) {
          const int c0 = hh * 64 + sc * 16;
          uint32_t dp[16];
          tmem_ld_32x32b_x16(tmem + lane_bits + C::T_DP + c0, dp);
          uint32_t dh[8];
#pragma unroll
          for (int t4 = 0; t4 < 4; ++t4) {
            const float4 d4 = *reinterpret_cast<const float4*>(dlt + c0 + 4 * t4);
#pragma unroll
            for (int u = 0; u < 2; ++u) {
              const int t = 2 * t4 + u;
              float e0, e1, s0, s1;
              fadd2(e0, e1, __uint_as_float(dp[2 * t]), __uint_as_float(dp[2 * t + 1]), -(u ? d4.z : d4.x),
                    -(u ? d4.w : d4.y));
              ffma2(s0, s1, pv[sc * 16 + 2 * t], pv[sc * 16 + 2 * t + 1], e0, e1, 0.f, 0.f);
              dh[t] = pack_f16x2(s0, s1);
            }
          }
          // the dS^T buffer's previous pair (g - DS_BUFS) must have been consumed
          if (sc == 0 && g >= C::DS_BUFS &&
              !(ok = mbar_wait_warp(&ds_free[g % C::DS_BUFS], ((g / C::DS_BUFS) - 1) & 1, lim, W_BWD_DSF)))
            break;
          // query columns c0..c0+15: two 16-byte chunks of the 128-byte row of block hh (128B swizzle)
          const int blk = hh * 16384 + rowoff;
#pragma unroll
          for (int t = 0; t < 2; ++t) {
            const int o16 = blk + (((sc * 2 + t) ^ (r & 7)) << 4);
            *reinterpret_cast<uint4*>(smem + C::DS_OFF + (g % C::DS_BUFS) * C::DS_BYTES + o16) =
                make_uint4(dh[4 * t], dh[4 * t + 1], dh[4 * t + 2], dh[4 * t + 3]);
          }
        }
        if (!(npairs_ok = ok)) break;
        fence_proxy_async_smem();
        tc_fence_before();                               // the phase-2 reads of dP^T come first
        mbar_arrive(ds_ready);
      }
      ++it;
      gp += I.npairs;
    }
    setmaxnreg_dec<BWD_LAUNCH_REGS>();
    asm volatile("bar.arrive 2, %0;" :: "n"(C::THREADS) : "memory");
  } else {
    setmaxnreg_inc<BWD_WORK_REGS>();
    // ------------------------------------- dQ read-out, then dK/dV epilogue --
    const int wq = warp & 3;
    const int r = wq * 32 + lane;
    const uint32_t lane_bits = static_cast<uint32_t>(wq * 32) << 16;
    bool ok = true;
    uint8_t* stg = smem + C::DQS_OFF + wq * 8192;
    // the input scales come out here: dV carries dO's, dK^T = dS^T Q carries
    // those of dO, V and Q
    const BwdScales sc_out = bwd_scales(p.amax, D);
    const float mul_dv = bwd_pow2(-sc_out.kdo), mul_dk = p.scale * bwd_pow2(-(sc_out.kdo + sc_out.kv + sc_out.kq));
    int it = 0, gp = 0;
    for (int ni = 0; ok; ++ni) {
      const int qs = ni & 1;
      if (!(ok = mbar_wait_warp(&item_full[qs], (ni >> 1) & 1, lim, W_BWD_ITEM))) break;
      const int w = item_w[qs];
      __syncwarp();
      if (lane == 0) mbar_arrive(&item_empty[qs]);
      if (w < 0) break;
      const BwdItem I = bwd_item<CAUSAL>(p, w);
      for (int n = 0; n < I.npairs; ++n) {
        const int g = gp + n, bq = g % NB;
        if (!(ok = mbar_wait_warp(&dq_full[bq], (g / NB) & 1, lim, W_BWD_DQ))) break;
        tc_fence_after();
        const int i = I.i0 + n / G, hq = I.hkv * G + n % G;
        const int row0 = i * 128 + wq * 32;         // first query row of this warp's box
        // D / 32 pieces of 32 columns, two per round (the two staging boxes)
#pragma unroll
        for (int rd = 0; rd < D / 64; ++rd) {
          if (lane == 0) bulk_wait_read_all();      // the boxes of the previous round are read
          __syncwarp();
#pragma unroll
          for (int pc = 0; pc < 2; ++pc) {
            uint32_t v[32];
            tmem_ld_32x32b_x32(tmem + lane_bits + C::T_DQ + bq * D + (rd * 2 + pc) * 32, v);
            uint4* my_row = reinterpret_cast<uint4*>(stg + pc * 4096 + lane * 128);
#pragma unroll
            for (int c = 0; c < 8; ++c)            // 16-byte chunk c of row lane at c ^ (lane % 8)
              my_row[c ^ (lane & 7)] = make_uint4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0 && row0 < p.Lq) {
#pragma unroll
            for (int pc = 0; pc < 2; ++pc)
              tma_reduce_add_4d(&tm_dq, stg + pc * 4096, (rd * 2 + pc) * 32, hq, row0, I.b);
            bulk_commit_group();
          }
        }
        tc_fence_before();
        mbar_arrive(&dq_free[bq]);
      }
      if (!ok) break;
      gp += I.npairs;
      // dK, dV of this key tile (zero when no query sees it) out of TMEM; the
      // next item's first products wait for this read-out
      const bool have = I.npairs > 0 && (ok = mbar_wait_warp(dkv_done, it & 1, lim, W_BWD_DKV));
      if (I.npairs > 0 && !ok) break;
      if (have) tc_fence_after();
      const int key = I.j * 128 + r;
      const size_t krow = ((size_t(I.b) * p.Lk + key) * p.Hkv + I.hkv) * D;
#pragma unroll
      for (int which = 0; which < 2; ++which) {       // 0: dV, 1: dK (scaled)
        const float mul = which ? mul_dk : mul_dv;
        void* out = which ? p.dk : p.dv;
#pragma unroll
        for (int c0 = 0; c0 < D; c0 += 32) {
          uint32_t v[32];
          if (have) {
            tmem_ld_32x32b_x32(tmem + lane_bits + (which ? C::T_DK : C::T_DV) + c0, v);
          } else {
#pragma unroll
            for (int t = 0; t < 32; ++t) v[t] = 0u;
          }
          if (key >= p.Lk) continue;
          if (!index_ok(krow + c0, 32, static_cast<size_t>(p.B) * p.Lk * p.Hkv * D, W_IDX_BWD_DKV)) continue;
          if (p.g_fp32) {
            float4* d4 = reinterpret_cast<float4*>(static_cast<float*>(out) + krow + c0);
#pragma unroll
            for (int t = 0; t < 8; ++t)
              d4[t] = make_float4(__uint_as_float(v[4 * t]) * mul, __uint_as_float(v[4 * t + 1]) * mul,
                                  __uint_as_float(v[4 * t + 2]) * mul, __uint_as_float(v[4 * t + 3]) * mul);
          } else {
            uint4* d4 = reinterpret_cast<uint4*>(static_cast<uint16_t*>(out) + krow + c0);
#pragma unroll
            for (int t = 0; t < 4; ++t)
              d4[t] = make_uint4(pack_bf16x2(__uint_as_float(v[8 * t]) * mul, __uint_as_float(v[8 * t + 1]) * mul),
                                 pack_bf16x2(__uint_as_float(v[8 * t + 2]) * mul, __uint_as_float(v[8 * t + 3]) * mul),
                                 pack_bf16x2(__uint_as_float(v[8 * t + 4]) * mul, __uint_as_float(v[8 * t + 5]) * mul),
                                 pack_bf16x2(__uint_as_float(v[8 * t + 6]) * mul, __uint_as_float(v[8 * t + 7]) * mul));
          }
        }
      }
      if (have) {
        tc_fence_before();                         // the TMEM reads come first
        mbar_arrive(dkv_free);
        ++it;
      }
    }
    // the CTA may not exit while a reduction still reads its staging boxes
    if (lane == 0) bulk_wait_all();
    __syncwarp();
    setmaxnreg_dec<BWD_LAUNCH_REGS>();
    asm volatile("bar.arrive 2, %0;" :: "n"(C::THREADS) : "memory");
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 14) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace fa
