// common.cuh -- device status word, activations and small helpers shared by
// the kernels of this library.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "tpl.h"

namespace tpl {

// Per-device status word: a kernel that gives up on a pipeline wait records
// TPL_ERR_TIMEOUT here; tpl_get_device_status reads and clears it.
__device__ int g_status_word;

__device__ __forceinline__ void record_timeout() {
  atomicExch(&g_status_word, static_cast<int>(TPL_ERR_TIMEOUT));
}

__device__ __forceinline__ float gelu_erf(float v) {
  return 0.5f * v * (1.0f + erff(v * 0.70710678118654752f));
}

__device__ __forceinline__ float gelu_tanh(float v) {
  const float u = 0.79788456080286536f * (v + 0.044715f * v * v * v);
  return 0.5f * v * (1.0f + tanhf(u));
}

__device__ __forceinline__ float apply_act(float v, int act) {
  if (act == TPL_ACT_GELU_ERF) return gelu_erf(v);
  if (act == TPL_ACT_GELU_TANH) return gelu_tanh(v);
  return v;
}

// Exact-form GELU y * Phi(y) for the bf16 epilogues, with the complementary
// error function from Abramowitz & Stegun, Handbook of Mathematical Functions,
// formula 7.1.26 (Hastings' rational approximation):
//   erfc(u) = (a1 t + a2 t^2 + a3 t^3 + a4 t^4 + a5 t^5) exp(-u^2),
//   t = 1 / (1 + p u),  u >= 0,  |error| <= 1.5e-7.
// With u = |y| / sqrt 2: Phi(y) = 1 - erfc(u) / 2 for y >= 0 and erfc(u) / 2
// for y < 0 (no cancellation on the negative side).  The reciprocal and the
// exponential use the hardware approximations; the total error stays below
// 1e-6, far under the bf16 rounding of the stored result.
__device__ __forceinline__ float gelu_erf_fast(float y) {
  const float u = fabsf(y) * 0.70710678118654752f;
  const float t = __fdividef(1.0f, fmaf(0.3275911f, u, 1.0f));
  float poly = fmaf(1.061405429f, t, -1.453152027f);
  poly = fmaf(poly, t, 1.421413741f);
  poly = fmaf(poly, t, -0.284496736f);
  poly = fmaf(poly, t, 0.254829592f);
  poly *= t;
  const float half_erfc = 0.5f * poly * __expf(-u * u);
  const float phi = (y >= 0.0f) ? (1.0f - half_erfc) : half_erfc;
  return y * phi;
}

__device__ __forceinline__ float apply_act_fast(float v, int act) {
  if (act == TPL_ACT_GELU_ERF) return gelu_erf_fast(v);
  if (act == TPL_ACT_GELU_TANH) return gelu_tanh(v);
  return v;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&p);
}

__device__ __forceinline__ float bf16_lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t u) { return __uint_as_float(u & 0xFFFF0000u); }

__device__ __forceinline__ float bf16_to_f(__nv_bfloat16 b) { return __bfloat162float(b); }

}  // namespace tpl
