// norm_fold.cuh -- folds an RMSNorm scale into the weight that follows it.
//
// google-research allgather_layernorm: y = x * rsqrt(mean(x^2) + eps) * g with
// g = 1 + scale (centred) or scale.  Ahead of a column-parallel linear,
// RMSNorm(x) W^T = diag(rsqrt(mean(x^2) + eps)) x (W diag(g))^T, so g can be
// multiplied into the weight's columns once, at load time, and the per-row
// factor applied in the GEMM epilogue (tpl_column_linear_rmsnorm).
#pragma once

#include "common.cuh"

namespace tpl {

// w_out[n][k] = bf16(w[n][k] * g[k]), one 8-element vector per thread step.
__global__ void fold_norm_scale_kernel(const __nv_bfloat16* __restrict__ w, int64_t rows,
                                       int64_t K, const float* __restrict__ scale, int centered,
                                       __nv_bfloat16* __restrict__ out) {
  const int64_t vpr = K / 8;  // vectors per row
  const int64_t n = rows * vpr;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t k0 = (i % vpr) * 8;
    const uint4 q = __ldg(reinterpret_cast<const uint4*>(w) + i);
    const float4 s0 = __ldg(reinterpret_cast<const float4*>(scale + k0));
    const float4 s1 = __ldg(reinterpret_cast<const float4*>(scale + k0 + 4));
    const float c = centered ? 1.0f : 0.0f;
    uint4 r;
    r.x = pack_bf16x2(bf16_lo(q.x) * (s0.x + c), bf16_hi(q.x) * (s0.y + c));
    r.y = pack_bf16x2(bf16_lo(q.y) * (s0.z + c), bf16_hi(q.y) * (s0.w + c));
    r.z = pack_bf16x2(bf16_lo(q.z) * (s1.x + c), bf16_hi(q.z) * (s1.y + c));
    r.w = pack_bf16x2(bf16_lo(q.w) * (s1.z + c), bf16_hi(q.w) * (s1.w + c));
    reinterpret_cast<uint4*>(out)[i] = r;
  }
}

}  // namespace tpl
