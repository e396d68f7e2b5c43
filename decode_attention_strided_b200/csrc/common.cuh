// common.cuh -- small device helpers shared by the kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cstdint>

#include "internal.h"

namespace dkv {

template <typename T> __device__ __forceinline__ float to_f(T v);
template <> __device__ __forceinline__ float to_f<float>(float v) { return v; }
template <> __device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 v) {
  return __bfloat162float(v);
}

template <typename T> __device__ __forceinline__ T from_f(float v);
template <> __device__ __forceinline__ float from_f<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float v) {
  return __float2bfloat16_rn(v);
}

// Record the first device-side error of a call; later ones are dropped.
__device__ __forceinline__ void latch_error(uint32_t* err, uint32_t code, uint32_t detail) {
  if (atomicCAS(err, 0u, code) == 0u) err[1] = detail;
}

// The codec nonlinearity.  GELU_ERF is x * Phi(x) evaluated with CUDA's erff;
// GELU_TANH is the tanh approximation; NONE is the identity.
__device__ __forceinline__ float act_eval(int act, float z) {
  if (act == DELTAKV_ACT_GELU_ERF) return 0.5f * z * (1.0f + erff(z * 0.70710678118654752f));
  if (act == DELTAKV_ACT_GELU_TANH)
    return 0.5f * z * (1.0f + tanhf(0.79788456080286536f * (z + 0.044715f * z * z * z)));
  return z;
}

// Keep the KC smallest (distance, slot) pairs in ascending order; ties go to
// the lower slot.  The arrays live in registers: every index is static after
// unrolling, so the insertion is a compare-and-swap chain.
template <int KC>
__device__ __forceinline__ void topk_insert(float (&bd)[KC], int (&bi)[KC], float d, int j) {
  if (!(d < bd[KC - 1] || (d == bd[KC - 1] && j < bi[KC - 1]))) return;
  bd[KC - 1] = d;
  bi[KC - 1] = j;
#pragma unroll
  for (int i = KC - 1; i > 0; --i) {
    bool sw = bd[i] < bd[i - 1] || (bd[i] == bd[i - 1] && bi[i] < bi[i - 1]);
    if (sw) {
      float td = bd[i]; bd[i] = bd[i - 1]; bd[i - 1] = td;
      int ti = bi[i]; bi[i] = bi[i - 1]; bi[i - 1] = ti;
    }
  }
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Code row of non-reference token t.
__device__ __forceinline__ int64_t code_row_of(int64_t t, int s) { return t - t / s - 1; }
// Token of code row n (inverse of code_row_of).
__device__ __forceinline__ int64_t token_of_code_row(int64_t n, int s) {
  return (n / (s - 1)) * s + (n % (s - 1)) + 1;
}

}  // namespace dkv
