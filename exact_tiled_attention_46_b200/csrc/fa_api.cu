// Host side of the C ABI declared in include/fa.h: argument checks, tensor-map
// encoding, kernel selection and launches.  Nothing here allocates device
// memory or synchronises (except fa_device_status, which says so).
#include <atomic>
#include <climits>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <algorithm>
#include <mutex>

#include <cuda.h>
#include <cuda_runtime.h>

#include "fa.h"
#include "sm100.cuh"
#include "fa_fwd.cuh"
#include "fa_decode.cuh"
#include "fa_bwd.cuh"

namespace {

constexpr int kAbiVersion = 1;
constexpr int kDecodeChunk = 1024;
std::atomic<unsigned long long> g_wait_limit_ns{2000000000ull};

// ---------------------------------------------------------- tensor maps ----
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

// 4-D map over a [B, L, H, D] tensor (bf16; fp32 or single bytes when asked):
// dims (D, H, L, B), box (box_d, 1, box_rows, 1).
bool map_bshd(CUtensorMap* m, const void* base, int B, int L, int H, int D, int box_d, int box_rows, bool sw128,
              bool fp32 = false, bool bytes = false) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) return false;
  const cuuint64_t es_bytes = fp32 ? 4 : bytes ? 1 : 2;
  cuuint64_t dims[4] = {cuuint64_t(D), cuuint64_t(H), cuuint64_t(L), cuuint64_t(B)};
  cuuint64_t strides[3] = {cuuint64_t(D) * es_bytes, cuuint64_t(H) * D * es_bytes, cuuint64_t(L) * H * D * es_bytes};
  cuuint32_t box[4] = {cuuint32_t(box_d), 1, cuuint32_t(box_rows), 1};
  cuuint32_t es[4] = {1, 1, 1, 1};
  const CUtensorMapDataType dt = fp32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                                : bytes ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  return enc(m, dt, 4, const_cast<void*>(base),
             dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, sw128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ------------------------------------------------------------- helpers -----
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned256(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 255u) == 0; }
size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
bool scale_ok(float s) { return std::isfinite(s) && s > 0.f; }
bool fits_int(long long x) { return x >= 0 && x <= INT_MAX; }

// Sets the dynamic shared-memory limit of `func` once per device.
template <typename F>
bool ensure_smem_attr(F* func, int bytes, std::atomic<uint64_t>& done_mask) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
  const uint64_t bit = uint64_t(1) << dev;
  if (done_mask.load(std::memory_order_acquire) & bit) return true;
  if (cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess) return false;
  done_mask.fetch_or(bit, std::memory_order_acq_rel);
  return true;
}

fa_status launch_status() { return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA; }

// Number of SMs of the current device (cached per device); 0 on failure.
int sm_count() {
  static std::atomic<int> cached[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  int n = cached[dev].load(std::memory_order_relaxed);
  if (n > 0) return n;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 0;
  cached[dev].store(n, std::memory_order_relaxed);
  return n;
}

__global__ void fill_empty_rows_kernel(void* o, float* lse, size_t n_o, size_t n_lse, int o_fp32) {
  const size_t i = blockIdx.x * size_t(blockDim.x) + threadIdx.x;
  const size_t stride = size_t(gridDim.x) * blockDim.x;
  for (size_t k = i; k < n_o; k += stride) {
    if (o_fp32) static_cast<float*>(o)[k] = 0.f;
    else static_cast<uint16_t*>(o)[k] = 0;
  }
  if (lse != nullptr)
    for (size_t k = i; k < n_lse; k += stride) lse[k] = -INFINITY;
}

__global__ void selftest_wait_kernel(unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) { fa::mbar_init(&bar, 1); fa::fence_mbar_init(); }
  __syncthreads();
  fa::mbar_wait(&bar, 0, limit_ns, 0x9001);   // no thread ever arrives
}

__global__ void selftest_exp2_poly_kernel(const float* x, float* y, int n) {
  const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
  if (i + 1 < n) {
    fa::exp2_poly2(x[i], x[i + 1], y[i], y[i + 1]);
  } else if (i < n) {
    float unused;
    fa::exp2_poly2(x[i], x[i], y[i], unused);
  }
}

// The forward and backward kernels move registers between warpgroups
// (setmaxnreg); that is only safe when the launch allocation per thread is
// exactly the one the split was computed for.  A build that allocates
// differently is refused, never run.  The result is kept per kernel
// instantiation (each launch_* template instance owns its `state`), because
// all instantiations of one kernel template share a function type.
enum : int { REGS_UNKNOWN = 0, REGS_MATCH = 1, REGS_MISMATCH = 2 };
template <typename F>
bool launch_regs_match(F* func, int expected, std::atomic<int>& state) {
  int s = state.load();
  if (s == REGS_UNKNOWN) {
    cudaFuncAttributes a;
    if (cudaFuncGetAttributes(&a, func) != cudaSuccess) return false;
    s = (a.numRegs == expected) ? REGS_MATCH : REGS_MISMATCH;
    state.store(s);
  }
  return s == REGS_MATCH;
}
// Per-instantiation guard states, indexed by kernel_slot().
std::atomic<int> g_regs_state[10];
constexpr int kernel_slot(bool bwd, int D, bool causal, bool fp8 = false) {
  return fp8 ? 8 + (causal ? 1 : 0) : (bwd ? 4 : 0) + (D == 128 ? 2 : 0) + (causal ? 1 : 0);
}

template <int D, bool CAUSAL, bool FP8 = false>
fa_status launch_fwd(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, const fa::FwdParams& p,
                     long long grid, cudaStream_t st) {
  static std::atomic<uint64_t> attr_done{0};
  constexpr int smem = fa::FwdCfg<D, FP8>::SMEM_BYTES;
  if (!launch_regs_match(fa::fwd_kernel<D, CAUSAL, FP8>, fa::FWD_LAUNCH_REGS,
                         g_regs_state[kernel_slot(false, D, CAUSAL, FP8)]))
    return FA_ERR_UNSUPPORTED;
  if (!ensure_smem_attr(fa::fwd_kernel<D, CAUSAL, FP8>, smem, attr_done)) return FA_ERR_CUDA;
  fa::fwd_kernel<D, CAUSAL, FP8><<<static_cast<unsigned>(grid), fa::FwdCfg<D, FP8>::THREADS, smem, st>>>(mq, mk, mv, p);
  return launch_status();
}

template <int D, int GP, bool PAGED, bool APPEND>
fa_status launch_decode(const CUtensorMap& mk, const CUtensorMap& mv, const fa::DecParams& p, unsigned grid,
                        cudaStream_t st) {
  static std::atomic<uint64_t> attr_done{0};
  using C = fa::DecCfg<D, GP>;
  if (!ensure_smem_attr(fa::decode_split_kernel<D, GP, PAGED, APPEND>, C::SMEM_BYTES, attr_done)) return FA_ERR_CUDA;
  fa::decode_split_kernel<D, GP, PAGED, APPEND><<<grid, C::THREADS, C::SMEM_BYTES, st>>>(mk, mv, p);
  return launch_status();
}

template <bool PAGED, bool APPEND>
fa_status dispatch_decode(int D, int GP, const CUtensorMap& mk, const CUtensorMap& mv, const fa::DecParams& p,
                          unsigned grid, cudaStream_t st) {
  if (D == 128)
    return GP == 4 ? launch_decode<128, 4, PAGED, APPEND>(mk, mv, p, grid, st)
         : GP == 2 ? launch_decode<128, 2, PAGED, APPEND>(mk, mv, p, grid, st)
                   : launch_decode<128, 1, PAGED, APPEND>(mk, mv, p, grid, st);
  return GP == 4 ? launch_decode<64, 4, PAGED, APPEND>(mk, mv, p, grid, st)
       : GP == 2 ? launch_decode<64, 2, PAGED, APPEND>(mk, mv, p, grid, st)
                 : launch_decode<64, 1, PAGED, APPEND>(mk, mv, p, grid, st);
}

// One split-KV decode call, every variant: cache rows from a contiguous cache
// (page_table == nullptr: "pages" are the sequences, page_size = Lmax) or a
// page pool, and, when k_new != nullptr, the new token's rows attended and
// appended.  Checks every argument before anything is launched.
fa_status run_decode(const void* q, const void* k_new, const void* v_new, const void* k_cache, const void* v_cache,
                     const int* page_table, const int* seqlens, void* o, float* lse, int B, int Hq, int Hkv,
                     int num_pages, int page_size, int pages_per_seq, int D, float scale, int o_dtype,
                     void* workspace, size_t workspace_bytes, cudaStream_t st) {
  const bool paged = page_table != nullptr, append = k_new != nullptr || v_new != nullptr;
  if (!q || !k_cache || !v_cache || !seqlens || !o || !workspace) return FA_ERR_INVALID_ARG;
  if (append && (!k_new || !v_new)) return FA_ERR_INVALID_ARG;
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0) return FA_ERR_INVALID_ARG;
  if (num_pages <= 0 || page_size <= 0 || pages_per_seq <= 0) return FA_ERR_INVALID_ARG;
  if (paged && page_size % 16 != 0) return FA_ERR_UNSUPPORTED;
  if (!scale_ok(scale)) return FA_ERR_INVALID_ARG;
  if (o_dtype != FA_BF16 && o_dtype != FA_FP32) return FA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(o) || !aligned256(workspace) ||
      !aligned16(k_new) || !aligned16(v_new))
    return FA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(seqlens) & 3u) != 0 || (reinterpret_cast<uintptr_t>(lse) & 3u) != 0 ||
      (reinterpret_cast<uintptr_t>(page_table) & 3u) != 0)
    return FA_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return FA_ERR_UNSUPPORTED;
  const long long cap = static_cast<long long>(page_size) * pages_per_seq;
  if (cap + 1 > INT_MAX) return FA_ERR_UNSUPPORTED;
  const int G = Hq / Hkv;
  const int GP = (G % 4 == 0) ? 4 : (G % 2 == 0) ? 2 : 1;
  const int HG = Hkv * (G / GP);
  const long long keys = cap + (append ? 1 : 0);
  const long long max_splits = (keys + kDecodeChunk - 1) / kDecodeChunk;
  if (!fits_int(static_cast<long long>(B) * max_splits * HG) || !fits_int(static_cast<long long>(B) * Hq))
    return FA_ERR_UNSUPPORTED;
  if (workspace_bytes < fa_decode_workspace_size(B, Hq, static_cast<int>(keys), D)) return FA_ERR_INVALID_ARG;
  const int sub_rows = (page_size % 32 == 0 || !paged) ? 32 : 16;
  CUtensorMap mk, mv;
  // boxes of 64 dimensions (128 bytes, 128-byte swizzle) by sub_rows rows
  if (!map_bshd(&mk, k_cache, num_pages, page_size, Hkv, D, 64, sub_rows, true) ||
      !map_bshd(&mv, v_cache, num_pages, page_size, Hkv, D, 64, sub_rows, true))
    return FA_ERR_CUDA;
  float* o_part = static_cast<float*>(workspace);
  const size_t lse_off = align_up(size_t(B) * Hq * max_splits * D * 4, 256);
  float* lse_part = reinterpret_cast<float*>(static_cast<char*>(workspace) + lse_off);
  int* counter = reinterpret_cast<int*>(static_cast<char*>(workspace) + lse_off +
                                        align_up(size_t(B) * Hq * max_splits * 4, 256));
  if (cudaMemsetAsync(counter, 0, sizeof(int), st) != cudaSuccess) return FA_ERR_CUDA;
  fa::DecParams p;
  p.seqlens = seqlens; p.q = static_cast<const uint16_t*>(q);
  p.k_new = static_cast<const uint16_t*>(k_new); p.v_new = static_cast<const uint16_t*>(v_new);
  p.k_cache = static_cast<uint16_t*>(const_cast<void*>(k_cache));
  p.v_cache = static_cast<uint16_t*>(const_cast<void*>(v_cache));
  p.page_table = page_table;
  p.o_part = o_part; p.lse_part = lse_part; p.work_counter = counter;
  p.B = B; p.Hq = Hq; p.Hkv = Hkv; p.max_splits = static_cast<int>(max_splits); p.chunk = kDecodeChunk;
  p.cap = static_cast<int>(cap); p.page_size = page_size; p.pages_per_seq = pages_per_seq; p.num_pages = num_pages;
  p.sub_rows = sub_rows;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.wait_limit_ns = g_wait_limit_ns.load();
  // persistent grid: as many CTAs as fit (3 per SM), never more than there can be items
  const int sms = sm_count();
  if (sms <= 0) return FA_ERR_CUDA;
  const long long items = static_cast<long long>(B) * max_splits * HG;
  const unsigned grid = static_cast<unsigned>(std::min<long long>(items, 3LL * sms));
  fa_status s;
  if (paged) s = append ? dispatch_decode<true, true>(D, GP, mk, mv, p, grid, st)
                        : dispatch_decode<true, false>(D, GP, mk, mv, p, grid, st);
  else s = append ? dispatch_decode<false, true>(D, GP, mk, mv, p, grid, st)
                  : dispatch_decode<false, false>(D, GP, mk, mv, p, grid, st);
  if (s != FA_OK) return s;
  fa::CombineParams c;
  c.o_part = o_part; c.lse_part = lse_part; c.counts = seqlens; c.o = o; c.lse = lse;
  c.B = B; c.Hq = Hq; c.D = D; c.max_splits = static_cast<int>(max_splits); c.chunk = kDecodeChunk;
  c.o_fp32 = (o_dtype == FA_FP32); c.cap = static_cast<int>(cap); c.append = append ? 1 : 0;
  fa::decode_combine_kernel<<<B * Hq, 128, 0, st>>>(c);
  return launch_status();
}

template <int D, bool CAUSAL>
fa_status launch_bwd(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, const CUtensorMap& mdo,
                     const CUtensorMap& mdq, const fa::BwdParams& p, unsigned grid, cudaStream_t st) {
  static std::atomic<uint64_t> attr_done{0};
  constexpr int smem = fa::BwdCfg<D>::SMEM_BYTES;
  if (!launch_regs_match(fa::bwd_main_kernel<D, CAUSAL>, fa::BWD_LAUNCH_REGS, g_regs_state[kernel_slot(true, D, CAUSAL)]))
    return FA_ERR_UNSUPPORTED;
  if (!ensure_smem_attr(fa::bwd_main_kernel<D, CAUSAL>, smem, attr_done)) return FA_ERR_CUDA;
  fa::bwd_main_kernel<D, CAUSAL><<<grid, fa::BwdCfg<D>::THREADS, smem, st>>>(mq, mk, mv, mdo, mdq, p);
  return launch_status();
}

// Scratch of fa_decode_splitkv_static: the split-KV partial results of the
// most recent call.  In host code this name is only a stand-in for the device
// array; its device address is looked up per device with cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_decode_static_scratch[FA_DECODE_STATIC_SCRATCH_BYTES];
std::mutex g_static_mu;
void* g_static_scratch_ptr[64] = {};

}  // namespace

extern "C" {

int fa_abi_version(void) { return kAbiVersion; }

int fa_debug_build(void) {
#ifdef FA_DEBUG
  return 1;
#else
  return 0;
#endif
}

const char* fa_status_string(int s) {
  switch (s) {
    case FA_OK: return "ok";
    case FA_ERR_INVALID_ARG: return "invalid argument";
    case FA_ERR_UNSUPPORTED: return "unsupported configuration";
    case FA_ERR_CUDA: return "CUDA call failed";
    case FA_ERR_TIMEOUT: return "kernel wait timed out";
    case FA_ERR_DEVICE_INDEX: return "device index check failed (debug build)";
    default: return "unknown status";
  }
}

void fa_set_wait_limit_ns(unsigned long long ns) { g_wait_limit_ns.store(ns > 0 ? ns : 1); }

fa_status fa_fwd_ex(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv,
                    int Lq, int Lk, int D, float scale, int causal, int o_dtype, fa_stream_t stream) {
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || Lq < 0 || Lk < 0 || Hq % Hkv != 0) return FA_ERR_INVALID_ARG;
  // empty tensors may come with null pointers: q/o only matter when Lq > 0, k/v when Lk > 0
  if (Lq > 0 && (!q || !o)) return FA_ERR_INVALID_ARG;
  if (Lq > 0 && Lk > 0 && (!k || !v)) return FA_ERR_INVALID_ARG;
  if (!scale_ok(scale)) return FA_ERR_INVALID_ARG;
  if (o_dtype != FA_BF16 && o_dtype != FA_FP32) return FA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return FA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(lse) & 3u) != 0) return FA_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return FA_ERR_UNSUPPORTED;
  const long long pairs = (static_cast<long long>(Lq) + 255) / 256;
  const long long items = pairs * B * Hq;          // work items of the persistent grid
  if (!fits_int(items) || !fits_int(static_cast<long long>(B) * Hq)) return FA_ERR_UNSUPPORTED;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (Lq == 0) return FA_OK;
  if (Lk == 0) {
    const size_t n_o = size_t(B) * Lq * Hq * D, n_l = size_t(B) * Hq * Lq;
    fill_empty_rows_kernel<<<296, 256, 0, st>>>(o, lse, n_o, n_l, o_dtype == FA_FP32);
    return launch_status();
  }
  CUtensorMap mq, mk, mv;
  if (!map_bshd(&mq, q, B, Lq, Hq, D, 64, 128, true) || !map_bshd(&mk, k, B, Lk, Hkv, D, 64, 128, true) ||
      !map_bshd(&mv, v, B, Lk, Hkv, D, 64, 128, true))
    return FA_ERR_CUDA;
  fa::FwdParams p;
  p.o = o; p.lse = lse; p.B = B; p.Hq = Hq; p.Hkv = Hkv; p.Lq = Lq; p.Lk = Lk;
  p.num_pairs = static_cast<int>(pairs);
  p.scale_log2 = scale * 1.4426950408889634f;
  p.o_scale = 1.f;
  p.o_fp32 = (o_dtype == FA_FP32);
  p.wait_limit_ns = g_wait_limit_ns.load();
  const int sms = sm_count();
  if (sms <= 0) return FA_ERR_CUDA;
  const long long grid = items < sms ? items : sms;
  if (D == 128) return causal ? launch_fwd<128, true>(mq, mk, mv, p, grid, st) : launch_fwd<128, false>(mq, mk, mv, p, grid, st);
  return causal ? launch_fwd<64, true>(mq, mk, mv, p, grid, st) : launch_fwd<64, false>(mq, mk, mv, p, grid, st);
}

fa_status fa_fwd_fp8(const void* q, const void* k, const void* v, float q_scale, float k_scale, float v_scale,
                     void* o, float* lse, int B, int Hq, int Hkv, int Lq, int Lk, int D, float scale, int causal,
                     int o_dtype, fa_stream_t stream) {
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || Lq < 0 || Lk < 0 || Hq % Hkv != 0) return FA_ERR_INVALID_ARG;
  if (Lq > 0 && (!q || !o)) return FA_ERR_INVALID_ARG;
  if (Lq > 0 && Lk > 0 && (!k || !v)) return FA_ERR_INVALID_ARG;
  if (!scale_ok(scale) || !scale_ok(q_scale) || !scale_ok(k_scale) || !scale_ok(v_scale)) return FA_ERR_INVALID_ARG;
  if (o_dtype != FA_BF16 && o_dtype != FA_FP32) return FA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return FA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(lse) & 3u) != 0) return FA_ERR_INVALID_ARG;
  if (D != 128) return FA_ERR_UNSUPPORTED;
  const long long pairs = (static_cast<long long>(Lq) + 255) / 256;
  const long long items = pairs * B * Hq;
  if (!fits_int(items) || !fits_int(static_cast<long long>(B) * Hq)) return FA_ERR_UNSUPPORTED;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (Lq == 0) return FA_OK;
  if (Lk == 0) {
    const size_t n_o = size_t(B) * Lq * Hq * D, n_l = size_t(B) * Hq * Lq;
    fill_empty_rows_kernel<<<296, 256, 0, st>>>(o, lse, n_o, n_l, o_dtype == FA_FP32);
    return launch_status();
  }
  CUtensorMap mq, mk, mv;
  if (!map_bshd(&mq, q, B, Lq, Hq, D, 128, 128, true, false, true) ||
      !map_bshd(&mk, k, B, Lk, Hkv, D, 128, 128, true, false, true) ||
      !map_bshd(&mv, v, B, Lk, Hkv, D, 128, 128, true, false, true))
    return FA_ERR_CUDA;
  fa::FwdParams p;
  p.o = o; p.lse = lse; p.B = B; p.Hq = Hq; p.Hkv = Hkv; p.Lq = Lq; p.Lk = Lk;
  p.num_pairs = static_cast<int>(pairs);
  p.scale_log2 = scale * q_scale * k_scale * 1.4426950408889634f;
  p.o_scale = v_scale;
  p.o_fp32 = (o_dtype == FA_FP32);
  p.wait_limit_ns = g_wait_limit_ns.load();
  const int sms = sm_count();
  if (sms <= 0) return FA_ERR_CUDA;
  const long long grid = items < sms ? items : sms;
  return causal ? launch_fwd<128, true, true>(mq, mk, mv, p, grid, st)
                : launch_fwd<128, false, true>(mq, mk, mv, p, grid, st);
}

fa_status fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv, int Lq,
                 int Lk, int D, float scale, int causal, fa_stream_t stream) {
  return fa_fwd_ex(q, k, v, o, lse, B, Hq, Hkv, Lq, Lk, D, scale, causal, FA_BF16, stream);
}

int fa_decode_chunk(void) { return kDecodeChunk; }

size_t fa_decode_workspace_size(int B, int Hq, int Lmax, int D) {
  if (B <= 0 || Hq <= 0 || Lmax < 0 || D <= 0) return 0;
  const size_t ms = std::max<size_t>(1, (size_t(Lmax) + kDecodeChunk - 1) / kDecodeChunk);
  // partial outputs, partial LSEs, the work counter of the split kernel
  return align_up(size_t(B) * Hq * ms * D * 4, 256) + align_up(size_t(B) * Hq * ms * 4, 256) + 256;
}

fa_status fa_decode_combine(const float* o_part, const float* lse_part, const int* num_splits, void* o, float* lse,
                            int B, int Hq, int D, int max_splits, int o_dtype, fa_stream_t stream) {
  if (!o_part || !lse_part || !o) return FA_ERR_INVALID_ARG;
  if (B <= 0 || Hq <= 0 || D <= 0 || D > 4096 || max_splits <= 0) return FA_ERR_INVALID_ARG;
  if (o_dtype != FA_BF16 && o_dtype != FA_FP32) return FA_ERR_INVALID_ARG;
  if (!fits_int(static_cast<long long>(B) * Hq)) return FA_ERR_UNSUPPORTED;
  fa::CombineParams c;
  c.o_part = o_part; c.lse_part = lse_part; c.counts = num_splits; c.o = o; c.lse = lse;
  c.B = B; c.Hq = Hq; c.D = D; c.max_splits = max_splits; c.chunk = 0; c.o_fp32 = (o_dtype == FA_FP32);
  c.cap = 0; c.append = 0;
  fa::decode_combine_kernel<<<B * Hq, 128, 0, reinterpret_cast<cudaStream_t>(stream)>>>(c);
  return launch_status();
}

fa_status fa_decode_splitkv(const void* q, const void* k_cache, const void* v_cache, const int* seqlens, void* o,
                            float* lse, int B, int Hq, int Hkv, int Lmax, int D, float scale, int o_dtype,
                            void* workspace, size_t workspace_bytes, fa_stream_t stream) {
  if (B <= 0 || Lmax <= 0) return FA_ERR_INVALID_ARG;
  return run_decode(q, nullptr, nullptr, k_cache, v_cache, nullptr, seqlens, o, lse, B, Hq, Hkv, B, Lmax, 1, D,
                    scale, o_dtype, workspace, workspace_bytes, reinterpret_cast<cudaStream_t>(stream));
}

fa_status fa_decode_append_splitkv(const void* q, const void* k_new, const void* v_new, void* k_cache,
                                   void* v_cache, const int* seqlens, void* o, float* lse, int B, int Hq, int Hkv,
                                   int Lmax, int D, float scale, int o_dtype, void* workspace,
                                   size_t workspace_bytes, fa_stream_t stream) {
  if (B <= 0 || Lmax <= 0 || !k_new || !v_new) return FA_ERR_INVALID_ARG;
  return run_decode(q, k_new, v_new, k_cache, v_cache, nullptr, seqlens, o, lse, B, Hq, Hkv, B, Lmax, 1, D, scale,
                    o_dtype, workspace, workspace_bytes, reinterpret_cast<cudaStream_t>(stream));
}

fa_status fa_decode_paged_splitkv(const void* q, const void* k_new, const void* v_new, void* k_pages,
                                  void* v_pages, const int* page_table, const int* seqlens, void* o, float* lse,
                                  int B, int Hq, int Hkv, int num_pages, int page_size, int pages_per_seq, int D,
                                  float scale, int o_dtype, void* workspace, size_t workspace_bytes,
                                  fa_stream_t stream) {
  if (!page_table) return FA_ERR_INVALID_ARG;
  return run_decode(q, k_new, v_new, k_pages, v_pages, page_table, seqlens, o, lse, B, Hq, Hkv, num_pages,
                    page_size, pages_per_seq, D, scale, o_dtype, workspace, workspace_bytes,
                    reinterpret_cast<cudaStream_t>(stream));
}

fa_status fa_attn_merge(const float* o_a, const float* lse_a, const float* o_b, const float* lse_b, void* o_out,
                        float* lse_out, int B, int H, int L, int D, int o_dtype, fa_stream_t stream) {
  if (B <= 0 || H <= 0 || L < 0 || D <= 0 || D % 4 != 0) return FA_ERR_INVALID_ARG;
  if (o_dtype != FA_BF16 && o_dtype != FA_FP32) return FA_ERR_INVALID_ARG;
  if (L == 0) return FA_OK;
  if (!o_a || !lse_a || !o_b || !lse_b || !o_out) return FA_ERR_INVALID_ARG;
  if (!aligned16(o_a) || !aligned16(o_b) || !aligned16(o_out)) return FA_ERR_INVALID_ARG;
  if (((reinterpret_cast<uintptr_t>(lse_a) | reinterpret_cast<uintptr_t>(lse_b) |
        reinterpret_cast<uintptr_t>(lse_out)) & 3u) != 0)
    return FA_ERR_INVALID_ARG;
  // the output may be either input: every element is read by the thread that writes it, before it writes
  fa::MergeParams p;
  p.o_a = o_a; p.lse_a = lse_a; p.o_b = o_b; p.lse_b = lse_b; p.o_out = o_out; p.lse_out = lse_out;
  p.B = B; p.H = H; p.L = L; p.D = D; p.o_fp32 = (o_dtype == FA_FP32);
  const size_t rows = size_t(B) * L * H;
  const int sms = sm_count();
  if (sms <= 0) return FA_ERR_CUDA;
  const unsigned blocks = static_cast<unsigned>(std::min<size_t>((rows + 7) / 8, size_t(sms) * 16));
  fa::attn_merge_kernel<<<blocks, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(p);
  return launch_status();
}

fa_status fa_decode_splitkv_static(const void* q, const void* k_cache, const void* v_cache, const int* seqlens,
                                   void* o, float* lse, int B, int Hq, int Hkv, int Lmax, int D, float scale,
                                   int o_dtype, fa_stream_t stream) {
  if (fa_decode_workspace_size(B, Hq, Lmax, D) > FA_DECODE_STATIC_SCRATCH_BYTES) return FA_ERR_UNSUPPORTED;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return FA_ERR_CUDA;
  void* scratch = nullptr;
  {
    // set-up, once per device, with that device current
    std::lock_guard<std::mutex> lock(g_static_mu);
    if (g_static_scratch_ptr[dev] == nullptr) {
      void* ptr = nullptr;
      if (cudaGetSymbolAddress(&ptr, g_decode_static_scratch) != cudaSuccess || ptr == nullptr) return FA_ERR_CUDA;
      g_static_scratch_ptr[dev] = ptr;
    }
    scratch = g_static_scratch_ptr[dev];
  }
  return fa_decode_splitkv(q, k_cache, v_cache, seqlens, o, lse, B, Hq, Hkv, Lmax, D, scale, o_dtype, scratch,
                           FA_DECODE_STATIC_SCRATCH_BYTES, stream);
}

size_t fa_bwd_workspace_size(int B, int Hq, int Lq, int D) {
  if (B <= 0 || Hq <= 0 || Lq < 0 || D <= 0) return 0;
  const size_t lq_pad = align_up(size_t(Lq), 128);
  // fp32 dQ accumulator, the padded log2 LSE and Delta rows, the scaled fp16
  // copies of q and dO, the four input maxima
  return align_up(size_t(B) * Lq * Hq * D * 4, 256) + 2 * align_up(size_t(B) * Hq * lq_pad * 4, 256) +
         2 * align_up(size_t(B) * Lq * Hq * D * 2, 256) + 256;
}

fa_status fa_bwd(const void* q, const void* k, const void* v, const void* o, const void* dO, const float* lse,
                 void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int Lq, int Lk, int D, float scale, int causal,
                 int grad_dtype, void* workspace, size_t workspace_bytes, fa_stream_t stream) {
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || Lq < 0 || Lk < 0 || Hq % Hkv != 0) return FA_ERR_INVALID_ARG;
  // empty tensors may come with null pointers
  if (Lq > 0 && (!q || !o || !dO || !lse || !dq)) return FA_ERR_INVALID_ARG;
  if (Lk > 0 && (!k || !v || !dk || !dv)) return FA_ERR_INVALID_ARG;
  if (Lq > 0 && Lk > 0 && !workspace) return FA_ERR_INVALID_ARG;
  if (!scale_ok(scale)) return FA_ERR_INVALID_ARG;
  if (grad_dtype != FA_BF16 && grad_dtype != FA_FP32) return FA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(dO) || !aligned16(dq) ||
      !aligned16(dk) || !aligned16(dv) || !aligned256(workspace) || (reinterpret_cast<uintptr_t>(lse) & 3u))
    return FA_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return FA_ERR_UNSUPPORTED;
  if (workspace_bytes < fa_bwd_workspace_size(B, Hq, Lq, D)) return FA_ERR_INVALID_ARG;
  if (!fits_int(static_cast<long long>((Lk + 127) / 128) * B * Hkv)) return FA_ERR_UNSUPPORTED;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const size_t g_elt = grad_dtype == FA_FP32 ? 4 : 2;
  if (Lq == 0 || Lk == 0) {   // no (query, key) pair: the gradients that exist are zero
    const size_t nk = size_t(B) * Lk * Hkv * D * g_elt, nq = size_t(B) * Lq * Hq * D * g_elt;
    if ((nk && (cudaMemsetAsync(dk, 0, nk, st) != cudaSuccess || cudaMemsetAsync(dv, 0, nk, st) != cudaSuccess)) ||
        (nq && cudaMemsetAsync(dq, 0, nq, st) != cudaSuccess))
      return FA_ERR_CUDA;
    return FA_OK;
  }
  const int lq_pad = static_cast<int>(align_up(size_t(Lq), 128));
  const size_t acc_bytes = size_t(B) * Lq * Hq * D * 4;
  const size_t row_bytes = align_up(size_t(B) * Hq * lq_pad * 4, 256);
  const size_t h_bytes = align_up(size_t(B) * Lq * Hq * D * 2, 256);
  char* ws = static_cast<char*>(workspace);
  float* dq_acc = reinterpret_cast<float*>(ws);
  float* lse2 = reinterpret_cast<float*>(ws + align_up(acc_bytes, 256));
  float* delta = reinterpret_cast<float*>(reinterpret_cast<char*>(lse2) + row_bytes);
  uint16_t* q16 = reinterpret_cast<uint16_t*>(reinterpret_cast<char*>(delta) + row_bytes);
  uint16_t* do16 = reinterpret_cast<uint16_t*>(reinterpret_cast<char*>(q16) + h_bytes);
  uint32_t* amax = reinterpret_cast<uint32_t*>(reinterpret_cast<char*>(do16) + h_bytes);
  int* counter = reinterpret_cast<int*>(amax + 4);                 // the main kernel's work counter
  if (cudaMemsetAsync(dq_acc, 0, acc_bytes, st) != cudaSuccess || cudaMemsetAsync(amax, 0, 32, st) != cudaSuccess)
    return FA_ERR_CUDA;
  {
    const size_t nq = size_t(B) * Lq * Hq * D, nk = size_t(B) * Lk * Hkv * D;
    const unsigned blocks = static_cast<unsigned>(std::min<size_t>((std::max(nq, nk) / 8 + 1023) / 1024, 148 * 4));
    fa::bwd_amax_kernel<<<dim3(blocks, 4), 256, 0, st>>>(static_cast<const uint16_t*>(q), static_cast<const uint16_t*>(k),
                                                static_cast<const uint16_t*>(v), static_cast<const uint16_t*>(dO),
                                                nq, nk, amax);
    if (launch_status() != FA_OK) return FA_ERR_CUDA;
  }
  {
    const size_t chunks = size_t(B) * lq_pad * Hq * (D / 8);         // one thread per 16-byte chunk of a row
    const unsigned blocks = static_cast<unsigned>(std::min<size_t>((chunks + 255) / 256, 148 * 16));
    fa::bwd_pre_kernel<<<blocks, 256, 0, st>>>(static_cast<const uint16_t*>(o), static_cast<const uint16_t*>(dO),
                                               static_cast<const uint16_t*>(q), lse, amax, lse2, delta, q16, do16, B,
                                               Hq, Lq, lq_pad, D);
    if (launch_status() != FA_OK) return FA_ERR_CUDA;
  }
  CUtensorMap mq, mk, mv, mdo, mdq;
  // q and dO are read from their fp16 copies (2-byte elements: the bf16 map
  // type only sets the element size here), k and v as given; the fp32 dQ
  // accumulator takes reductions of 32-row x 32-column boxes
  if (!map_bshd(&mq, q16, B, Lq, Hq, D, 64, 128, true) || !map_bshd(&mk, k, B, Lk, Hkv, D, 64, 128, true) ||
      !map_bshd(&mv, v, B, Lk, Hkv, D, 64, 128, true) || !map_bshd(&mdo, do16, B, Lq, Hq, D, 64, 128, true) ||
      !map_bshd(&mdq, dq_acc, B, Lq, Hq, D, 32, 32, true, true))
    return FA_ERR_CUDA;
  fa::BwdParams p;
  p.lse2 = lse2; p.delta = delta; p.amax = amax; p.dk = dk; p.dv = dv;
  p.B = B; p.Hq = Hq; p.Hkv = Hkv; p.Lq = Lq; p.Lk = Lk; p.Lq_pad = lq_pad;
  p.scale = scale; p.scale_log2 = scale * 1.4426950408889634f; p.g_fp32 = (grad_dtype == FA_FP32);
  p.wait_limit_ns = g_wait_limit_ns.load();
  // persistent: at most one CTA per SM, taking key tiles from the counter
  p.num_items = static_cast<int>(((Lk + 127) / 128) * B * Hkv);
  p.work_counter = counter;
  const int sms = sm_count();
  if (sms <= 0) return FA_ERR_CUDA;
  const unsigned grid = static_cast<unsigned>(std::min(p.num_items, sms));
  fa_status s;
  if (D == 128) s = causal ? launch_bwd<128, true>(mq, mk, mv, mdo, mdq, p, grid, st) : launch_bwd<128, false>(mq, mk, mv, mdo, mdq, p, grid, st);
  else s = causal ? launch_bwd<64, true>(mq, mk, mv, mdo, mdq, p, grid, st) : launch_bwd<64, false>(mq, mk, mv, mdo, mdq, p, grid, st);
  if (s != FA_OK) return s;
  const size_t n = size_t(B) * Lq * Hq * D;
  const unsigned blocks = static_cast<unsigned>(std::min<size_t>((n / 4 + 255) / 256, 148 * 16));
  fa::bwd_post_kernel<<<blocks, 256, 0, st>>>(dq_acc, dq, n, scale, amax, D, grad_dtype == FA_FP32);
  return launch_status();
}

fa_status fa_device_status(int* code, int* where, int reset, fa_stream_t stream) {
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint32_t s = 0, w = 0;
  if (cudaMemcpyFromSymbolAsync(&s, fa::g_fa_dev_status, 4, 0, cudaMemcpyDeviceToHost, st) != cudaSuccess ||
      cudaMemcpyFromSymbolAsync(&w, fa::g_fa_dev_where, 4, 0, cudaMemcpyDeviceToHost, st) != cudaSuccess ||
      cudaStreamSynchronize(st) != cudaSuccess)
    return FA_ERR_CUDA;
  if (code)
    *code = (s == fa::FA_DEV_TIMEOUT)     ? FA_ERR_TIMEOUT
            : (s == fa::FA_DEV_BAD_INPUT) ? FA_ERR_INVALID_ARG
            : (s == fa::FA_DEV_BAD_INDEX) ? FA_ERR_DEVICE_INDEX
                                          : FA_OK;
  if (where) *where = static_cast<int>(w);
  if (reset) {
    const uint32_t zero = 0;
    if (cudaMemcpyToSymbolAsync(fa::g_fa_dev_status, &zero, 4, 0, cudaMemcpyHostToDevice, st) != cudaSuccess ||
        cudaMemcpyToSymbolAsync(fa::g_fa_dev_where, &zero, 4, 0, cudaMemcpyHostToDevice, st) != cudaSuccess ||
        cudaStreamSynchronize(st) != cudaSuccess)
      return FA_ERR_CUDA;
  }
  return FA_OK;
}

fa_status fa_launch_guard(int bwd, int D, int causal, int* num_regs, int* expected_regs, int* state) {
  // D = -128 names the e4m3 forward
  const bool fp8 = (D == -128 && !bwd);
  if (D != 64 && D != 128 && !fp8) return FA_ERR_INVALID_ARG;
  const int slot = kernel_slot(bwd != 0, D, causal != 0, fp8);
  if (state) *state = g_regs_state[slot].load();
  if (expected_regs) *expected_regs = bwd ? fa::BWD_LAUNCH_REGS : fa::FWD_LAUNCH_REGS;
  if (num_regs) {
    cudaFuncAttributes a;
    cudaError_t e;
    if (fp8) {
      e = causal ? cudaFuncGetAttributes(&a, fa::fwd_kernel<128, true, true>)
                 : cudaFuncGetAttributes(&a, fa::fwd_kernel<128, false, true>);
    } else if (bwd) {
      e = D == 128 ? (causal ? cudaFuncGetAttributes(&a, fa::bwd_main_kernel<128, true>)
                             : cudaFuncGetAttributes(&a, fa::bwd_main_kernel<128, false>))
                   : (causal ? cudaFuncGetAttributes(&a, fa::bwd_main_kernel<64, true>)
                             : cudaFuncGetAttributes(&a, fa::bwd_main_kernel<64, false>));
    } else {
      e = D == 128 ? (causal ? cudaFuncGetAttributes(&a, fa::fwd_kernel<128, true>)
                             : cudaFuncGetAttributes(&a, fa::fwd_kernel<128, false>))
                   : (causal ? cudaFuncGetAttributes(&a, fa::fwd_kernel<64, true>)
                             : cudaFuncGetAttributes(&a, fa::fwd_kernel<64, false>));
    }
    if (e != cudaSuccess) return FA_ERR_CUDA;
    *num_regs = a.numRegs;
  }
  return FA_OK;
}

fa_status fa_selftest_exp2_poly(const float* x, float* y, int n, fa_stream_t stream) {
  if (!x || !y || n < 0) return FA_ERR_INVALID_ARG;
  if (n == 0) return FA_OK;
  const int threads = 256, pairs = (n + 1) / 2;
  selftest_exp2_poly_kernel<<<(pairs + threads - 1) / threads, threads, 0, reinterpret_cast<cudaStream_t>(stream)>>>(x, y, n);
  return launch_status();
}

fa_status fa_selftest_wait_timeout(unsigned long long wait_ns, fa_stream_t stream) {
  if (wait_ns == 0 || wait_ns > 10000000000ull) return FA_ERR_INVALID_ARG;
  selftest_wait_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(wait_ns);
  return launch_status();
}

}  // extern "C"
