// fwd_tc.cuh -- tensor-core (tcgen05 / TMEM / TMA) prefill kernel.  (placeholder)
#pragma once
#include "common.cuh"

namespace pia {
inline bool tc_supported(bool bf16, int d, int n) { (void)bf16; (void)d; (void)n; return false; }
inline cudaError_t launch_fwd_tc(const void*, const void*, const void*, const float*, const float*, void*, float*, int,
                                 int, int, int, int, int, int, cudaStream_t, const char** why) {
  *why = "tensor-core path not built";
  return cudaErrorNotSupported;
}
}  // namespace pia
