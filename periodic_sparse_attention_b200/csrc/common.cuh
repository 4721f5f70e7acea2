// common.cuh -- pieces every pi-attention kernel shares: element access, the index rule, the
// gate's log-priors, warp reductions, the device error word and bounded waits.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace pia {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// ---- device error word ------------------------------------------------------------------------
// One word per device for this library.  Kernels OR flags into it; pi_attn_check reads and clears.
enum : unsigned {
  kErrWaitTimeout = 1u,  // a bounded wait of the tensor-core kernel gave up (pipeline stalled)
  kErrCacheLen = 2u,     // decode: cache_len[b] outside [1, n_cache]
  kErrInternal = 4u,     // an internal consistency check failed (e.g. tile list overflow)
};
__device__ unsigned int g_error_word = 0u;

__device__ __forceinline__ void raise_error(unsigned flag) { atomicOr(&g_error_word, flag); }

// ---- element access ---------------------------------------------------------------------------
__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

// Widen 8 packed bf16 (one 16-byte load) to fp32.
__device__ __forceinline__ void bf16x8_to_f32(const uint4& u, float* f) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int t = 0; t < 4; ++t) {
    f[2 * t] = __uint_as_float(w[t] << 16);
    f[2 * t + 1] = __uint_as_float(w[t] & 0xFFFF0000u);
  }
}

// ---- the index rule ---------------------------------------------------------------------------
// Window  L(i) = [max(0, i - k), i];  skips P(i) = { i - m*pi : m0 <= m <= S, i - m*pi >= 0 }
// with m0 = floor(k / pi) + 1 the first m whose skip lands outside the window (m*pi > k).
__host__ __device__ __forceinline__ int first_skip_m(int k, int pi) { return k / pi + 1; }

// log(sigmoid(x)) = min(x, 0) - log1p(exp(-|x|)), free of overflow for any x.
__device__ __forceinline__ float log_sigmoid(float x) { return fminf(x, 0.f) - log1pf(expf(-fabsf(x))); }

// ---- packed fp32 pairs (Blackwell f32x2 arithmetic: two lanes of work per instruction) ----------
__device__ __forceinline__ unsigned long long f2pack(float a, float b) {
  unsigned long long r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ void f2unpack(unsigned long long r, float& a, float& b) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(r));
}
__device__ __forceinline__ unsigned long long f2fma(unsigned long long a, unsigned long long b, unsigned long long c) {
  unsigned long long d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ unsigned long long f2add(unsigned long long a, unsigned long long b) {
  unsigned long long d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ unsigned long long f2mul(unsigned long long a, unsigned long long b) {
  unsigned long long d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

// 2^x (the hardware approximation, flushing subnormals; relative error about 2^-22)
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// ---- warp reductions ---------------------------------------------------------------------------
__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}
__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}

// ---- time ---------------------------------------------------------------------------------------
__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
// Upper bound for any wait inside a kernel, in SM clock cycles (about 2 s at the B200's 1.965 GHz
// boost clock, longer at lower clocks).  A healthy pipeline waits microseconds.
constexpr long long kWaitLimitCycles = 4000000000ll;

}  // namespace pia
