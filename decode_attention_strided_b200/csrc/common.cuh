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

// Exact GELU x Phi(x) as relu(x) - g(|x|) with g(a) = a Phi(-a), a smooth bump
// that is below 1.5e-6 beyond a = 5.  g is approximated on [0, 5] by a
// degree-11 polynomial in t = 0.4 a - 1 (least-squares fit on Chebyshev
// nodes, evaluated by Horner in fp32); |gelu_fast - GELU| <= 1.1e-5 for all
// finite x.  About 15 fp32 instructions, no special-function unit.
__device__ __forceinline__ float gelu_fast(float x) {
  const float a = fminf(fabsf(x), 5.0f);
  const float t = fmaf(a, 0.4f, -1.0f);
  float p = 4.889592901e-02f;
  p = fmaf(p, t, -7.081953436e-02f);
  p = fmaf(p, t, -1.480407715e-01f);
  p = fmaf(p, t, 3.208711743e-01f);
  p = fmaf(p, t, 1.524367370e-02f);
  p = fmaf(p, t, -4.781557322e-01f);
  p = fmaf(p, t, 4.370784760e-01f);
  p = fmaf(p, t, -2.034248412e-02f);
  p = fmaf(p, t, -2.592293620e-01f);
  p = fmaf(p, t, 2.329209447e-01f);
  p = fmaf(p, t, -9.394139796e-02f);
  p = fmaf(p, t, 1.552190445e-02f);
  return fmaxf(x, 0.0f) - p;
}

// gelu_fast on two values at once: the same operations, with the polynomial
// evaluated by packed fp32x2 FMAs (each lane rounds exactly as fmaf does, so
// the results equal two gelu_fast calls bit for bit).
__device__ __forceinline__ float2 gelu_fast2(float x0, float x1) {
  unsigned long long t, p, c;
  const float a0 = fminf(fabsf(x0), 5.0f), a1 = fminf(fabsf(x1), 5.0f);
  asm("{\n\t.reg .b64 a, s, o;\n\t"
      "mov.b64 a, {%1, %2};\n\t"
      "mov.b64 s, {%3, %3};\n\t"
      "mov.b64 o, {%4, %4};\n\t"
      "fma.rn.f32x2 %0, a, s, o;\n\t}"
      : "=l"(t)
      : "f"(a0), "f"(a1), "f"(0.4f), "f"(-1.0f));
  const float k[12] = {4.889592901e-02f,  -7.081953436e-02f, -1.480407715e-01f, 3.208711743e-01f,
                       1.524367370e-02f,  -4.781557322e-01f, 4.370784760e-01f,  -2.034248412e-02f,
                       -2.592293620e-01f, 2.329209447e-01f,  -9.394139796e-02f, 1.552190445e-02f};
  asm("mov.b64 %0, {%1, %1};" : "=l"(p) : "f"(k[0]));
#pragma unroll
  for (int i = 1; i < 12; ++i) {
    asm("mov.b64 %0, {%1, %1};" : "=l"(c) : "f"(k[i]));
    asm("fma.rn.f32x2 %0, %0, %1, %2;" : "+l"(p) : "l"(t), "l"(c));
  }
  float p0, p1;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(p0), "=f"(p1) : "l"(p));
  return make_float2(fmaxf(x0, 0.0f) - p0, fmaxf(x1, 0.0f) - p1);
}

// Exact GELU for the decode token loop, where the activation count sets the
// pace: x Phi(x) ~= x/2 (1 + tanh(y)) with y = xc (c1 + c3 xc^2 + c5 xc^4)
// and xc = clamp(x, -8, 8) (one min.xorsign.abs).  (c1, c3, c5) is the
// builder's own minimax fit of this form to exact GELU on [-8, 8] (the
// argument rises monotonically there; beyond it tanh is saturated and the
// form returns x or 0): |form - GELU| <= 2.6e-5 with an exact tanh.  tanh
// itself comes from the special-function unit (tanh.approx.f32, whose
// relative error the tests measure), the rest runs as packed fp32x2
// arithmetic; so one activation costs one MUFU operation and about five
// issue slots, against about fifteen for gelu_fast.
__device__ __forceinline__ float2 gelu_tanhfit2(float x0, float x1) {
  float a0, a1;
  asm("min.xorsign.abs.f32 %0, %1, %2;" : "=f"(a0) : "f"(x0), "f"(8.0f));
  asm("min.xorsign.abs.f32 %0, %1, %2;" : "=f"(a1) : "f"(x1), "f"(8.0f));
  unsigned long long xc, xx, s, p, y, u;
  asm("mov.b64 %0, {%1, %2};" : "=l"(xc) : "f"(a0), "f"(a1));
  asm("mov.b64 %0, {%1, %2};" : "=l"(xx) : "f"(x0), "f"(x1));
  asm("mul.rn.f32x2 %0, %1, %1;" : "=l"(s) : "l"(xc));
  asm("{\n\t.reg .b64 c5, c3, c1;\n\t"
      "mov.b64 c5, {%2, %2};\n\tmov.b64 c3, {%3, %3};\n\tmov.b64 c1, {%4, %4};\n\t"
      "fma.rn.f32x2 %0, c5, %1, c3;\n\t"
      "fma.rn.f32x2 %0, %0, %1, c1;\n\t}"
      : "=l"(p)
      : "l"(s), "f"(-3.515167919e-04f), "f"(3.700564429e-02f), "f"(7.975078821e-01f));
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(y) : "l"(p), "l"(xc));
  float y0, y1, t0, t1;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(y0), "=f"(y1) : "l"(y));
  asm("tanh.approx.f32 %0, %1;" : "=f"(t0) : "f"(y0));
  asm("tanh.approx.f32 %0, %1;" : "=f"(t1) : "f"(y1));
  asm("{\n\t.reg .b64 hf, t, h;\n\t"
      "mov.b64 hf, {%2, %2};\n\tmov.b64 t, {%3, %4};\n\t"
      "mul.rn.f32x2 h, %1, hf;\n\t"
      "fma.rn.f32x2 %0, h, t, h;\n\t}"
      : "=l"(u)
      : "l"(xx), "f"(0.5f), "f"(t0), "f"(t1));
  float u0, u1;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(u0), "=f"(u1) : "l"(u));
  return make_float2(u0, u1);
}

// The activation inside the tensor-core kernels: exact GELU through
// gelu_fast, the other forms as in act_eval.
__device__ __forceinline__ float act_fast(int act, float z) {
  return act == DELTAKV_ACT_GELU_ERF ? gelu_fast(z) : act_eval(act, z);
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

// Insert (d, j) into a list kept in ascending order, for a caller that offers
// slots in increasing order (so an equal distance ranks after every entry
// already held).  Each new entry is computed from the old list directly --
// eight comparisons and selects with no chain between positions -- so the
// insertion has a short dependency depth.  No-op when d is not below the
// last entry.
template <int KC>
__device__ __forceinline__ void topk_insert_inorder(float (&bd)[KC], int (&bi)[KC], float d, int j) {
  bool lt[KC];
#pragma unroll
  for (int i = 0; i < KC; ++i) lt[i] = d < bd[i];
#pragma unroll
  for (int i = KC - 1; i > 0; --i) {
    bd[i] = lt[i - 1] ? bd[i - 1] : (lt[i] ? d : bd[i]);
    bi[i] = lt[i - 1] ? bi[i - 1] : (lt[i] ? j : bi[i]);
  }
  bd[0] = lt[0] ? d : bd[0];
  bi[0] = lt[0] ? j : bi[0];
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

// Element e of code row `row` (a row index of the whole plane).  With 4-bit
// codes (cscale non-null) the plane holds d_c / 2 bytes per row, element 2i in
// the low nibble of byte i and 2i + 1 in its high nibble, two's complement,
// and the value is q * scale[row] (exact in fp32: |q| <= 7 times a bf16).
template <typename E>
__device__ __forceinline__ float code_at(const E* code, const __nv_bfloat16* cscale, int64_t row, int d_c, int e) {
  if (cscale != nullptr) {
    const int b = reinterpret_cast<const int8_t*>(code)[row * (d_c >> 1) + (e >> 1)];
    const int qv = (e & 1) ? (b >> 4) : ((int)(int8_t)(b << 4) >> 4);
    return (float)qv * __bfloat162float(cscale[row]);
  }
  return to_f(code[row * d_c + e]);
}

// Quantise one code row to 4 bits: scale = bf16(max |c| / 7), q =
// clamp(rne(c / scale), -7, 7), packed two per byte (low nibble first) into
// `out` (n / 2 bytes).  Returns the scale.
template <int N>
__device__ __forceinline__ __nv_bfloat16 quantize_row4(const float (&c)[N], uint8_t (&out)[N / 2]) {
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < N; ++i) amax = fmaxf(amax, fabsf(c[i]));
  const __nv_bfloat16 sb = __float2bfloat16_rn(amax / 7.0f);
  const float sc = __bfloat162float(sb);
#pragma unroll
  for (int i = 0; i < N; i += 2) {
    int q0 = 0, q1 = 0;
    if (sc > 0.f) {
      q0 = (int)fminf(fmaxf(rintf(__fdiv_rn(c[i], sc)), -7.f), 7.f);
      q1 = (int)fminf(fmaxf(rintf(__fdiv_rn(c[i + 1], sc)), -7.f), 7.f);
    }
    out[i / 2] = (uint8_t)((q0 & 0xF) | ((q1 & 0xF) << 4));
  }
  return sb;
}

// Code row of non-reference token t.
__device__ __forceinline__ int64_t code_row_of(int64_t t, int s) { return t - t / s - 1; }
// Token of code row n (inverse of code_row_of).
__device__ __forceinline__ int64_t token_of_code_row(int64_t n, int s) {
  return (n / (s - 1)) * s + (n % (s - 1)) + 1;
}

}  // namespace dkv
