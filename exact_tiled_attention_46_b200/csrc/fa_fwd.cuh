// Prefill forward: exact softmax(Q K^T * scale) V, tile by tile with an online
// softmax ("FlashAttention Explained: How AI Models Process Attention Faster
// and Use Less Memory", sections "1. Tiling", "3. Online Softmax" and "Fused
// Computation"; "Flash Attention Explained: Same Maths, Far Less Memory",
// section "The idea: never materialise the matrix").  The score matrix lives
// only in tensor memory; Q is read and O/LSE written once, K and V once per
// work item (the re-reads of a head's K and V by its other items hit L2).
//
// The grid is persistent (at most one CTA per SM).  A work item is a pair of
// 128-row query tiles of one (batch, head); a CTA takes its items one after the
// other and, for each, walks the key tiles of the kv head:
//   warp 8      TMA producer: the item's Q tiles (each slot refilled once the
//               previous item's last S on it is done), then K_j, V_j into a
//               slot ring that runs on from item to item
//   warp 9      MMA issuer:   S_t = Q_t K_j^T into TMEM, O_t += P_t V_j
//   warps 0-3   softmax for query tile 0, warps 4-7 for query tile 1: one
//               thread per query row; causal / ragged mask; running max m and
//               running sum l in log2 units; P (bf16) written over S in TMEM;
//               O rescaled in TMEM only when the max grows by more than TAU;
//               epilogue O / l and LSE.
//   warp 10     allocates / frees the 512 TMEM columns; warp 11 idles.
// Registers: the block is launched with FWD_LAUNCH_REGS per thread (3 warps per
// SM sub-partition); the control warpgroup (warps 8-11) gives registers back
// (setmaxnreg.dec to FWD_CTRL_REGS) and the two softmax warpgroups take them
// (setmaxnreg.inc to FWD_SOFTMAX_REGS).  The split sums to exactly the launch
// allocation: 2 * 224 + 56 = 3 * 168 registers per lane slot.
// TMEM columns: S_0 [0,128), S_1 [128,256), O_0 [256,256+D), O_1 after it.
#pragma once
#include "sm100.cuh"
#include "exp2_poly.cuh"

namespace fa {

struct FwdParams {
  void* o;                 // [B, Lq, Hq, D] bf16 or fp32
  float* lse;              // [B, Hq, Lq] or nullptr
  int B, Hq, Hkv, Lq, Lk;
  int num_pairs;           // ceil(Lq / 256)
  float scale_log2;        // scale * log2(e) (e4m3 inputs: times the Q and K scales)
  float o_scale;           // multiplies O (e4m3 inputs: the V scale; else 1)
  int o_fp32;
  uint64_t wait_limit_ns;
};

// FP8: Q, K, V are e4m3 (one byte per element) and both products run as
// kind::f8f6f4 (D = 128 only: one 128-byte swizzle column per row).
template <int D, bool FP8 = false>
struct FwdCfg {
  static constexpr int ES = FP8 ? 1 : 2;               // bytes per input element
  static constexpr int TILE_BYTES = 128 * D * ES;      // one 128-row tile
  static constexpr int KB = D * ES / 128;              // 128-byte column blocks per row (one TMA box each)
  static constexpr int NS = (TILE_BYTES == 32768) ? 4 : 8;   // K/V slots
  static constexpr int Q_OFF = 0;
  static constexpr int KV_OFF = 2 * TILE_BYTES;
  static constexpr int BAR_OFF = KV_OFF + NS * TILE_BYTES;
  static constexpr int NBARS = 2 + 2 + 2 * NS + 2 + 2 + 2 + 1;
  static constexpr int SMEM_BYTES = BAR_OFF + NBARS * 8 + 16 + 1024;
  static constexpr int THREADS = 384;
};

// The running max m is a reference only: any m gives the same exact result.
// A tile is first exponentiated against the current m; if no lane's tile sum
// exceeds 2^FWD_FAST_LOG2 (so every p <= 2^16, a range bf16 and the fp32
// accumulators hold with unchanged relative precision), that is the tile's P.
// Otherwise (and on a row's first tile) the tile max is taken, m moves to it
// when it grows by more than FWD_TAU, O and the sums are rescaled in place, and
// P is recomputed.
constexpr float FWD_TAU = 8.0f;
constexpr int FWD_LAUNCH_REGS = 168, FWD_SOFTMAX_REGS = 224, FWD_CTRL_REGS = 56;
static_assert(2 * FWD_SOFTMAX_REGS + FWD_CTRL_REGS == 3 * FWD_LAUNCH_REGS, "register split must match the launch");
constexpr float FWD_FAST_LIMIT = 65536.0f;
// Every FWD_POLY_PERIOD-th pair of an unmasked tile can be exponentiated on the
// FMA pipe (exp2_poly2) instead of the MUFU unit; 0 turns this off.  Measured
// against a share of 1/3 on the causal prefill (B4 H16 L2048 D128) and long GQA
// (B1 Hq32 Hkv8 L16384 D128) workloads: 1/2 gave -4% / -1%, 1/4 +2% / +3.5%,
// 1/8 +3% / +5%, none +3% / +7%.  The softmax warps here are bound by their
// issue slots rather than by the MUFU rate, so the longer polynomial sequence
// does not pay.
constexpr int FWD_POLY_PERIOD = 0;
__host__ __device__ constexpr bool fwd_poly_pair(int i) {
  return FWD_POLY_PERIOD > 0 && (i % (FWD_POLY_PERIOD > 0 ? FWD_POLY_PERIOD : 1)) == FWD_POLY_PERIOD - 1;
}

// 2^x for two lanes on the FMA pipe: x = j + f with j = round(x), f in
// [-1/2, 1/2]; 2^f by the fitted polynomial (exp2_poly.cuh, Horner on packed
// fp32); 2^j added into the exponent field.  x is clamped to [-126, 127]:
// below, the result is a tiny positive number (not 0) far below 2^-126, so
// callers use it only where no entry is masked; above, it stays the finite
// 2^127 (never a wrapped exponent), which still trips the fast path's sum
// limit.  Relative error <= FA_EXP2_MAX_REL_ERR + fp32 rounding in the range.
__device__ __forceinline__ void exp2_poly2(float x0, float x1, float& p0, float& p1) {
  x0 = fminf(fmaxf(x0, -126.f), 127.f);
  x1 = fminf(fmaxf(x1, -126.f), 127.f);
  constexpr float RND = 12582912.f;                  // 1.5 * 2^23: x + RND rounds x to an integer
  float t0, t1, r0, r1, f0, f1, q0, q1;
  fadd2(t0, t1, x0, x1, RND, RND);
  fadd2(r0, r1, t0, t1, -RND, -RND);                 // round(x) as a float
  ffma2(f0, f1, r0, r1, -1.f, -1.f, x0, x1);         // f = x - round(x)
  ffma2(q0, q1, f0, f1, FA_EXP2_C3, FA_EXP2_C3, FA_EXP2_C2, FA_EXP2_C2);
  ffma2(q0, q1, q0, q1, f0, f1, FA_EXP2_C1, FA_EXP2_C1);
  ffma2(q0, q1, q0, q1, f0, f1, FA_EXP2_C0, FA_EXP2_C0);
  // the low mantissa bits of t hold round(x) (two's complement); << 23 moves it to the exponent
  p0 = __uint_as_float(__float_as_uint(q0) + (__float_as_uint(t0) << 23));
  p1 = __uint_as_float(__float_as_uint(q1) + (__float_as_uint(t1) << 23));
}

// The e4m3 path stores P scaled by 2^FWD_F8_P_LOG2 against the reference max
// and moves the reference whenever a tile max exceeds it by more than
// FWD_F8_TAU, so every stored value is at most 2^(8 + 0.75) = 431 (e4m3's
// largest finite value is 448) and values down to 2^-17 of the row's largest
// stay representable.
constexpr float FWD_F8_P_LOG2 = 8.0f, FWD_F8_TAU = 0.75f;

enum : uint32_t {
  W_FWD_Q = 0x101, W_FWD_KV_EMPTY = 0x102, W_FWD_KV_FULL = 0x103, W_FWD_P = 0x104,
  W_FWD_S = 0x105, W_FWD_O = 0x106, W_FWD_DONE = 0x107, W_FWD_DRAIN = 0x108, W_FWD_Q_EMPTY = 0x109
};

// One work item is a pair of 128-row query tiles of one (batch, head).  Items
// are numbered heaviest first (causal work grows with the pair index); the grid
// is persistent (at most one CTA per SM) and CTA c takes, in round r, item
// r * G + c (r even) or r * G + G - 1 - c (r odd), a boustrophedon order that
// evens out the causal work across CTAs.
struct FwdItem {
  int b, h, hkv, q0, n_t0, n_t1, n;
};
template <bool CAUSAL>
__device__ __forceinline__ FwdItem fwd_item(const FwdParams& p, int w) {
  FwdItem I;
  const int bh_count = p.B * p.Hq;
  const int pair = p.num_pairs - 1 - w / bh_count;
  const int bh = w % bh_count;
  I.b = bh / p.Hq;
  I.h = bh % p.Hq;
  I.hkv = I.h / (p.Hq / p.Hkv);
  I.q0 = pair * 256;
  const int off = p.Lk - p.Lq;
  const int nk_all = (p.Lk + 127) >> 7;
  int nt[2];
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    const int r0 = I.q0 + t * 128;
    if (r0 >= p.Lq) {
      nt[t] = 0;
    } else if (!CAUSAL) {
      nt[t] = nk_all;
    } else {
      const int lim_keys = min(r0 + 127, p.Lq - 1) + off + 1;   // keys < lim_keys for the last row
      nt[t] = lim_keys <= 0 ? 0 : min(nk_all, (lim_keys + 127) >> 7);
    }
  }
  I.n_t0 = nt[0];
  I.n_t1 = nt[1];
  I.n = max(nt[0], nt[1]);
  return I;
}
__device__ __forceinline__ int fwd_item_index(int r) {
  const int G = static_cast<int>(gridDim.x);
  return r * G + ((r & 1) ? (G - 1 - static_cast<int>(blockIdx.x)) : static_cast<int>(blockIdx.x));
}

template <int D, bool CAUSAL, bool FP8 = false>
__global__ void __launch_bounds__(384, 1)
fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
           const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
  static_assert(!FP8 || D == 128, "the e4m3 path is built for D = 128");
  using C = FwdCfg<D, FP8>;
  constexpr int NS = C::NS;
  constexpr int KB = C::KB;                        // 128-byte column blocks per row
  constexpr int BOX_COLS = 128 / C::ES;            // elements per 128-byte block
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);
  uint64_t* q_full = bars;                         // [2] Q tile t landed
  uint64_t* q_empty = q_full + 2;                  // [2] last S of Q tile t done
  uint64_t* kv_full = q_empty + 2;                 // [NS]
  uint64_t* kv_empty = kv_full + NS;               // [NS]
  uint64_t* s_full = kv_empty + NS;                // [2]
  uint64_t* p_full = s_full + 2;                   // [2]
  uint64_t* o_full = p_full + 2;                   // [2]
  uint64_t* mma_done = o_full + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + C::NBARS);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint64_t lim = p.wait_limit_ns;
  const int G = static_cast<int>(gridDim.x);
  const int num_items = p.num_pairs * p.B * p.Hq;
  const int off = p.Lk - p.Lq;                     // bottom-right causal alignment

  if (threadIdx.x == 0) {
    for (int t = 0; t < 2; ++t) {
      mbar_init(&q_full[t], 1); mbar_init(&q_empty[t], 1);
      mbar_init(&s_full[t], 1); mbar_init(&p_full[t], 128); mbar_init(&o_full[t], 1);
    }
    for (int i = 0; i < NS; ++i) { mbar_init(&kv_full[i], 1); mbar_init(&kv_empty[i], 1); }
    mbar_init(mma_done, 1);
    fence_mbar_init();
  }
  if (warp == 10) { tmem_alloc(tmem_holder, 512); tmem_relinquish(); }
  if (warp == 8 && lane == 0) { tma_prefetch_desc(&tm_q); tma_prefetch_desc(&tm_k); tma_prefetch_desc(&tm_v); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp >= 8) {
  setmaxnreg_dec<FWD_CTRL_REGS>();
  if (warp == 8) {
    // ------------------------------------------------------------ producer --
    if (lane == 0) {
      int it = 0;                                  // K/V ring loads issued
      uint32_t q_loaded = 0, q_par = 0;            // bit t: Q slot t loaded before / parity of its loads
      bool ok = true;
      for (int r = 0; ok && r * G < num_items; ++r) {
        const int w = fwd_item_index(r);
        if (w >= num_items) continue;
        const FwdItem I = fwd_item<CAUSAL>(p, w);
        if (I.n == 0) continue;
#pragma unroll 1
        for (int t = 0; t < 2; ++t) {
          if ((t ? I.n_t1 : I.n_t0) == 0) continue;
          // wait for the previous item's last S on this slot (phase = loads so far - 1)
          if (((q_loaded >> t) & 1u) && !(ok = mbar_wait(&q_empty[t], ((q_par >> t) & 1u) ^ 1u, lim, W_FWD_Q_EMPTY))) break;
          mbar_arrive_expect_tx(&q_full[t], C::TILE_BYTES);
          for (int kb = 0; kb < KB; ++kb)
            tma_load_4d(smem + C::Q_OFF + t * C::TILE_BYTES + kb * 16384, &tm_q, &q_full[t], kb * BOX_COLS, I.h,
                        I.q0 + t * 128, I.b);
          q_loaded |= 1u << t;
          q_par ^= 1u << t;
        }
        for (int i = 0; ok && i < 2 * I.n; ++i) {
          const int slot = it % NS;
          if (it >= NS && !(ok = mbar_wait(&kv_empty[slot], ((it / NS) + 1) & 1, lim, W_FWD_KV_EMPTY))) break;
          mbar_arrive_expect_tx(&kv_full[slot], C::TILE_BYTES);
          const CUtensorMap* m = (i & 1) ? &tm_v : &tm_k;
          uint8_t* dst = smem + C::KV_OFF + slot * C::TILE_BYTES;
          for (int kb = 0; kb < KB; ++kb)
            tma_load_4d(dst + kb * 16384, m, &kv_full[slot], kb * BOX_COLS, I.hkv, (i >> 1) * 128, I.b);
          ++it;
        }
      }
      // the CTA may not exit with copies in flight: wait for the last loads
      for (int t = 0; t < 2; ++t)
        if ((q_loaded >> t) & 1u) mbar_wait(&q_full[t], ((q_par >> t) & 1u) ^ 1u, lim, W_FWD_DRAIN);
      for (int i = max(0, it - NS); i < it; ++i) mbar_wait(&kv_full[i % NS], (i / NS) & 1, lim, W_FWD_DRAIN);
    }
  } else if (warp == 9) {
    // ----------------------------------------------------------------- MMA --
    if (lane == 0) {
      constexpr uint32_t IDESC_S = FP8 ? idesc_e4m3_f32(128, 128, false, false) : idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t IDESC_O = FP8 ? idesc_e4m3_f32(128, D, false, true) : idesc_bf16_f32(128, D, false, true);
      // every instruction consumes 32 bytes of K: 16 bf16 or 32 e4m3 elements
      constexpr int KS_S = D * C::ES / 32, KS_PV = 128 * C::ES / 32;
      const uint32_t q_base = smem_u32(smem + C::Q_OFF);
      const uint32_t kv_base = smem_u32(smem + C::KV_OFF);
      auto issue_s = [&](int t, int slot) {
        const uint32_t qa = q_base + t * C::TILE_BYTES, ka = kv_base + slot * C::TILE_BYTES;
#pragma unroll
        for (int kk = 0; kk < KS_S; ++kk) {
          const uint32_t o = (kk >> 2) * 16384 + (kk & 3) * 32;
          if constexpr (FP8)
            umma_ss_f8(tmem + t * 128, sdesc_sw128(qa + o, 16, 1024), sdesc_sw128(ka + o, 16, 1024), IDESC_S, kk > 0);
          else
            umma_ss(tmem + t * 128, sdesc_sw128(qa + o, 16, 1024), sdesc_sw128(ka + o, 16, 1024), IDESC_S, kk > 0);
        }
      };
      auto issue_pv = [&](int t, int slot, bool acc) {
        const uint32_t va = kv_base + slot * C::TILE_BYTES;
        // P (K = 128 keys) from TMEM, 8 columns per instruction; V MN-major,
        // 32 bytes of keys (16 or 32 rows of 128 bytes) per instruction
#pragma unroll
        for (int kk = 0; kk < KS_PV; ++kk) {
          if constexpr (FP8)
            umma_ts_f8(tmem + 256 + t * D, tmem + t * 128 + kk * 8, sdesc_sw128(va + kk * 4096, 16384, 1024), IDESC_O,
                       (acc || kk > 0) ? 1u : 0u);
          else
            umma_ts(tmem + 256 + t * D, tmem + t * 128 + kk * 8, sdesc_sw128(va + kk * 2048, 16384, 1024), IDESC_O,
                    (acc || kk > 0) ? 1u : 0u);
        }
      };
      auto wait_item = [&](int i) { return mbar_wait(&kv_full[i % NS], (i / NS) & 1, lim, W_FWD_KV_FULL); };

      int it = 0;                                  // K/V ring loads consumed
      uint32_t q_par = 0, p_par = 0;               // bit t: parity of the next q_full / p_full phase
      bool ok = true;
      for (int r = 0; ok && r * G < num_items; ++r) {
        const int w = fwd_item_index(r);
        if (w >= num_items) continue;
        const FwdItem I = fwd_item<CAUSAL>(p, w);
        if (I.n == 0) continue;
        const int it0 = it;                        // K_j at it0 + 2j, V_j at it0 + 2j + 1
        if (!(ok = wait_item(it0))) break;
#pragma unroll 1
        for (int t = 0; t < 2; ++t) {
          const int ntt = t ? I.n_t1 : I.n_t0;
          if (ntt == 0) continue;
          if (!(ok = mbar_wait(&q_full[t], (q_par >> t) & 1u, lim, W_FWD_Q))) break;
          q_par ^= 1u << t;
          tc_fence_after();
          issue_s(t, it0 % NS);
          umma_commit(&s_full[t]);
          if (ntt == 1) umma_commit(&q_empty[t]);
        }
        if (!ok) break;
        umma_commit(&kv_empty[it0 % NS]);
        for (int j = 0; ok && j < I.n; ++j) {
          const int it_v = it0 + 2 * j + 1, it_k = it0 + 2 * j + 2;
          if (!(ok = wait_item(it_v))) break;
          tc_fence_after();
          bool k_ready = false;
#pragma unroll 1
          for (int t = 0; t < 2 && ok; ++t) {
            const int ntt = t ? I.n_t1 : I.n_t0;
            if (j >= ntt) continue;
            if (!(ok = mbar_wait(&p_full[t], (p_par >> t) & 1u, lim, W_FWD_P))) break;
            p_par ^= 1u << t;
            tc_fence_after();
            issue_pv(t, it_v % NS, j > 0);
            if (j + 1 < ntt) {
              if (!k_ready) {
                if (!(ok = wait_item(it_k))) break;
                tc_fence_after();
                k_ready = true;
              }
              issue_s(t, it_k % NS);
              umma_commit(&s_full[t]);
              if (j + 2 == ntt) umma_commit(&q_empty[t]);   // the last S of this Q tile
            } else {
              umma_commit(&o_full[t]);
            }
          }
          if (!ok) break;
          umma_commit(&kv_empty[it_v % NS]);
          if (k_ready) umma_commit(&kv_empty[it_k % NS]);
        }
        it = it0 + 2 * I.n;
      }
      // nothing may be in flight on the tensor pipe when the CTA tears down
      umma_commit(mma_done);
      mbar_wait(mma_done, 0, lim, W_FWD_DONE);
    }
  }
  // Take the launch budget back only after the softmax warps have returned
  // theirs (named barrier 2): re-acquiring earlier could starve a softmax warp
  // that has not yet grown, and both would wait forever.
  asm volatile("bar.sync 2, %0;" :: "n"(C::THREADS) : "memory");
  setmaxnreg_inc<FWD_LAUNCH_REGS>();
  } else {
    setmaxnreg_inc<FWD_SOFTMAX_REGS>();
    // ------------------------------------------------------------- softmax --
    const int t = warp >> 2;
    const int wq = warp & 3;                       // TMEM lane quadrant of this warp
    const uint32_t lane_bits = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t t_s = tmem + lane_bits + t * 128;
    const uint32_t t_o = tmem + lane_bits + 256 + t * D;
    const float sl2 = p.scale_log2;
    int s_cnt = 0, o_cnt = 0;                      // phases consumed on s_full[t], o_full[t]
    bool ok = true;
    for (int r = 0; ok && r * G < num_items; ++r) {
      const int w = fwd_item_index(r);
      if (w >= num_items) continue;
      const FwdItem I = fwd_item<CAUSAL>(p, w);
      const int b = I.b, h = I.h;
      const int row_tile0 = I.q0 + t * 128;
      const int row = row_tile0 + wq * 32 + lane;    // global query row of this thread
      const int nt = t ? I.n_t1 : I.n_t0;
      // l: exact fp32 sum of p (for LSE); lr: sum of the bf16-rounded p that the
      // P.V product uses (the normaliser of O)
      float m_used = -INFINITY, l = 0.f, lr = 0.f;

      for (int j = 0; j < nt; ++j) {
        if (!(ok = mbar_wait_warp(&s_full[t], s_cnt & 1, lim, W_FWD_S))) break;
        ++s_cnt;
        tc_fence_after();
        uint32_t sr[128];
        tmem_ld_32x32b_x128(t_s, sr);
        float* s = reinterpret_cast<float*>(sr);
        const int kbase = j * 128;
        const bool need_mask = (kbase + 128 > p.Lk) || (CAUSAL && kbase + 127 > row_tile0 + off);
        if (need_mask) {
          int lim_c = p.Lk - kbase;
          if (CAUSAL) lim_c = min(lim_c, row + off + 1 - kbase);
  #pragma unroll
          for (int c = 0; c < 128; ++c) s[c] = (c < lim_c) ? s[c] : -INFINITY;
        }
        float ls0 = 0.f, ls1 = 0.f, lr0 = 0.f, lr1 = 0.f;
        // P = 2^(s*scale*log2e - m), packed to bf16 and stored over the first 64
        // columns of S; ls = exact sum, lr = sum of the bf16 values (O's normaliser)
        auto exp_tile = [&](float msub, bool use_poly) {
          ls0 = ls1 = lr0 = lr1 = 0.f;
  #pragma unroll
          for (int half = 0; half < 2; ++half) {
            uint32_t pk[32];
  #pragma unroll
            for (int i = 0; i < 32; ++i) {
              const int c = half * 64 + 2 * i;
              float x0, x1, p0, p1;
              ffma2(x0, x1, s[c], s[c + 1], sl2, sl2, -msub, -msub);
              if (use_poly && fwd_poly_pair(i)) {
                exp2_poly2(x0, x1, p0, p1);
              } else {
                p0 = ex2_approx(x0);
                p1 = ex2_approx(x1);
              }
              pk[i] = pack_bf16x2(p0, p1);
              fadd2(ls0, ls1, ls0, ls1, p0, p1);
              add_bf16x2_f32(lr0, lr1, pk[i]);
            }
            tmem_st_32x32b_x32(t_s + half * 32, pk);
          }
        };
        if constexpr (FP8) {
          // tile max first, then P = 2^(s - m + FWD_F8_P_LOG2) as e4m3, four per column
          float mx0 = s[0], mx1 = s[1], mx2 = s[2], mx3 = s[3];
  #pragma unroll
          for (int c = 4; c < 128; c += 4) {
            mx0 = fmaxf(mx0, s[c]); mx1 = fmaxf(mx1, s[c + 1]); mx2 = fmaxf(mx2, s[c + 2]); mx3 = fmaxf(mx3, s[c + 3]);
          }
          const float m_tile = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3)) * sl2;
          const bool resc = m_tile > m_used + FWD_F8_TAU;   // false while both are -inf
          float alpha = 1.f;
          if (resc) { alpha = ex2_approx(m_used - m_tile); l *= alpha; lr *= alpha; m_used = m_tile; }
          if (j > 0 && __any_sync(0xffffffffu, resc)) {
  #pragma unroll
            for (int c0 = 0; c0 < D; c0 += 32) {
              uint32_t ov[32];
              tmem_ld_32x32b_x32(t_o + c0, ov);
  #pragma unroll
              for (int i = 0; i < 32; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * alpha);
              tmem_st_32x32b_x32(t_o + c0, ov);
            }
          }
          const float msub = (m_used == -INFINITY) ? 0.f : m_used - FWD_F8_P_LOG2;
  #pragma unroll
          for (int half = 0; half < 2; ++half) {
            uint32_t pk[16];
  #pragma unroll
            for (int i = 0; i < 16; ++i) {
              const int c = half * 64 + 4 * i;
              float x0, x1, x2, x3;
              ffma2(x0, x1, s[c], s[c + 1], sl2, sl2, -msub, -msub);
              ffma2(x2, x3, s[c + 2], s[c + 3], sl2, sl2, -msub, -msub);
              const float p0 = ex2_approx(x0), p1 = ex2_approx(x1), p2 = ex2_approx(x2), p3 = ex2_approx(x3);
              pk[i] = pack_e4m3x4(p0, p1, p2, p3);
              fadd2(ls0, ls1, ls0, ls1, p0, p1);
              fadd2(ls0, ls1, ls0, ls1, p2, p3);
              add_e4m3x4_f32(lr0, lr1, pk[i]);
            }
            tmem_st_32x32b_x16(t_s + half * 16, pk);
          }
        } else {
        bool slow = __any_sync(0xffffffffu, m_used == -INFINITY);
        if (!slow) {
          // the branch keeps the polynomial loop and the all-MUFU loop apart, so
          // that the compiler cannot evaluate both and select
          if (need_mask) exp_tile(m_used, false);
          else exp_tile(m_used, true);
          slow = __any_sync(0xffffffffu, !(ls0 + ls1 <= FWD_FAST_LIMIT));
        }
        if (slow) {
          float mx0 = s[0], mx1 = s[1], mx2 = s[2], mx3 = s[3];
  #pragma unroll
          for (int c = 4; c < 128; c += 4) {
            mx0 = fmaxf(mx0, s[c]); mx1 = fmaxf(mx1, s[c + 1]); mx2 = fmaxf(mx2, s[c + 2]); mx3 = fmaxf(mx3, s[c + 3]);
          }
          const float m_tile = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3)) * sl2;
          const bool resc = m_tile > m_used + FWD_TAU;   // false while both are -inf
          float alpha = 1.f;
          if (resc) { alpha = ex2_approx(m_used - m_tile); l *= alpha; lr *= alpha; m_used = m_tile; }
          if (j > 0 && __any_sync(0xffffffffu, resc)) {
  #pragma unroll
            for (int c0 = 0; c0 < D; c0 += 32) {
              uint32_t ov[32];
              tmem_ld_32x32b_x32(t_o + c0, ov);
  #pragma unroll
              for (int i = 0; i < 32; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * alpha);
              tmem_st_32x32b_x32(t_o + c0, ov);
            }
          }
          exp_tile((m_used == -INFINITY) ? 0.f : m_used, false);
        }
        }
        l += ls0 + ls1;
        lr += lr0 + lr1;
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&p_full[t]);
      }

      // ------------------------------------------------------------ epilogue --
      const bool have_o = ok && nt > 0 && mbar_wait_warp(&o_full[t], o_cnt & 1, lim, W_FWD_O);
      if (nt > 0) ++o_cnt;
      if (have_o) tc_fence_after();
      const bool has = l > 0.f;
      const float inv_l = (lr > 0.f) ? p.o_scale / lr : 0.f;
      const float m_lse = FP8 ? m_used - FWD_F8_P_LOG2 : m_used;   // the reference l is counted against
      if (row < p.Lq && p.lse != nullptr) {
        const size_t li = (static_cast<size_t>(b) * p.Hq + h) * p.Lq + row;
        if (index_ok(li, 1, static_cast<size_t>(p.B) * p.Hq * p.Lq, W_IDX_FWD_LSE))
          p.lse[li] = has ? (m_lse + log2f(l)) * LN2 : -INFINITY;
      }
      const size_t orow = (static_cast<size_t>(b) * p.Lq + row) * p.Hq + h;
#pragma unroll
      for (int c0 = 0; c0 < D; c0 += 32) {
        uint32_t ov[32];
        if (have_o) {
          tmem_ld_32x32b_x32(t_o + c0, ov);
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) ov[i] = 0u;
        }
        if (row >= p.Lq) continue;
        if (!index_ok(orow * D + c0, 32, static_cast<size_t>(p.B) * p.Lq * p.Hq * D, W_IDX_FWD_O)) continue;
        if (p.o_fp32) {
          float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.o) + orow * D + c0);
#pragma unroll
          for (int i = 0; i < 8; ++i)
            dst[i] = make_float4(__uint_as_float(ov[4 * i]) * inv_l, __uint_as_float(ov[4 * i + 1]) * inv_l,
                                 __uint_as_float(ov[4 * i + 2]) * inv_l, __uint_as_float(ov[4 * i + 3]) * inv_l);
        } else {
          uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.o) + orow * D + c0);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            uint4 wv;
            wv.x = pack_bf16x2(__uint_as_float(ov[8 * i + 0]) * inv_l, __uint_as_float(ov[8 * i + 1]) * inv_l);
            wv.y = pack_bf16x2(__uint_as_float(ov[8 * i + 2]) * inv_l, __uint_as_float(ov[8 * i + 3]) * inv_l);
            wv.z = pack_bf16x2(__uint_as_float(ov[8 * i + 4]) * inv_l, __uint_as_float(ov[8 * i + 5]) * inv_l);
            wv.w = pack_bf16x2(__uint_as_float(ov[8 * i + 6]) * inv_l, __uint_as_float(ov[8 * i + 7]) * inv_l);
            dst[i] = wv;
          }
        }
      }
    }
    setmaxnreg_dec<FWD_LAUNCH_REGS>();    // give the extra registers back first
    asm volatile("bar.arrive 2, %0;" :: "n"(C::THREADS) : "memory");
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 10) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace fa
