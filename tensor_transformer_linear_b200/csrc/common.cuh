// common.cuh -- device status word, activations and small helpers shared by
// the kernels of this library.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "../../include/tpl.h"

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

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&p);
}

__device__ __forceinline__ float bf16_lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t u) { return __uint_as_float(u & 0xFFFF0000u); }

__device__ __forceinline__ float bf16_to_f(__nv_bfloat16 b) { return __bfloat162float(b); }

}  // namespace tpl
