// prefill.cuh -- paged causal prefill (placeholder until the tensor-core kernel lands).
#pragma once
#include "pa_common.cuh"

namespace pa {
inline int launch_prefill(void *, const void *, const int32_t *, int, const void *, const void *, const int32_t *,
                          int, const int32_t *, int, int, int, int64_t, float, int, int, cudaStream_t) {
  return -2;
}
}  // namespace pa
