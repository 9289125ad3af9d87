// Backward pass (placeholder until the tcgen05 backward kernels land).
#pragma once
#include "sm100.cuh"
#include "fa.h"

namespace fa {
inline fa_status bwd_dispatch(const void*, const void*, const void*, const void*, const void*, const float*, void*,
                              void*, void*, int, int, int, int, int, int, float, int, bool, void*, cudaStream_t,
                              uint64_t) {
  return FA_ERR_UNSUPPORTED;
}
}  // namespace fa
