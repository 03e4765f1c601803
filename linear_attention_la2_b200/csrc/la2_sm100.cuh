// Tensor-core (tcgen05 / TMEM / TMA) kernels for sm_100a.
#pragma once

#include "la2_common.cuh"
#include "la2.h"

namespace la2 {

inline bool sm100_supports(int64_t d, int64_t dv, int block, bool is_bwd) { return false; }

inline la2_status sm100_forward(const void*, const void*, const void*, void*, int64_t, int64_t, int,
                                int, int, int, float*, int64_t, int64_t, int64_t, cudaStream_t) {
  return LA2_ERR_UNSUPPORTED;
}
inline la2_status sm100_backward(const void*, const void*, const void*, const void*, void*, void*,
                                 void*, int64_t, int64_t, int, int, int, int, float*, float*,
                                 int64_t, int64_t, int64_t, cudaStream_t) {
  return LA2_ERR_UNSUPPORTED;
}

}  // namespace la2
