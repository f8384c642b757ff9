// rmsnorm.cuh -- RMSNorm (google-research allgather_layernorm: mean of squares
// in fp32, epsilon inside the rsqrt, optional centred scale 1 + s).
//
// HBM-bound: one read and one write of the row.  A warp owns a row, keeps it in
// registers (16-byte vector loads, lane-interleaved so every load instruction
// is a fully coalesced 512-byte segment), reduces the sum of squares with
// shuffles and writes the scaled row back, so y may alias x.  Rows wider than
// the register budget, or rows not 16-byte aligned, go through a two-pass
// kernel whose second read hits L2.
#pragma once

#include "common.cuh"
#include "ptx.cuh"

namespace tpl {

constexpr int kNormWarps = 8;

template <typename T>
struct VecTraits;
template <>
struct VecTraits<__nv_bfloat16> {
  static constexpr int kPer = 8;  // elements per 16-byte vector
  __device__ static void unpack(const uint4& q, float (&f)[8]) {
    f[0] = bf16_lo(q.x); f[1] = bf16_hi(q.x); f[2] = bf16_lo(q.y); f[3] = bf16_hi(q.y);
    f[4] = bf16_lo(q.z); f[5] = bf16_hi(q.z); f[6] = bf16_lo(q.w); f[7] = bf16_hi(q.w);
  }
  __device__ static uint4 pack(const float (&f)[8]) {
    uint4 q;
    q.x = pack_bf16x2(f[0], f[1]); q.y = pack_bf16x2(f[2], f[3]);
    q.z = pack_bf16x2(f[4], f[5]); q.w = pack_bf16x2(f[6], f[7]);
    return q;
  }
  __device__ static float load1(const __nv_bfloat16* p) { return __bfloat162float(*p); }
  __device__ static void store1(__nv_bfloat16* p, float v) { *p = __float2bfloat16_rn(v); }
};
template <>
struct VecTraits<float> {
  static constexpr int kPer = 4;
  __device__ static void unpack(const uint4& q, float (&f)[4]) {
    f[0] = __uint_as_float(q.x); f[1] = __uint_as_float(q.y);
    f[2] = __uint_as_float(q.z); f[3] = __uint_as_float(q.w);
  }
  __device__ static uint4 pack(const float (&f)[4]) {
    return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]),
                      __float_as_uint(f[3]));
  }
  __device__ static float load1(const float* p) { return *p; }
  __device__ static void store1(float* p, float v) { *p = v; }
};

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// VPL = 16-byte vectors per lane (row width <= 32 * VPL * kPer).
template <typename T, int VPL>
__global__ void __launch_bounds__(kNormWarps * 32)
    rmsnorm_reg(const T* x, T* y, const float* __restrict__ scale, int centered, float eps,
                int64_t M, int H) {
  ptx::griddep_wait();
  ptx::griddep_launch_dependents();
  using VT = VecTraits<T>;
  constexpr int P = VT::kPer;
  const int lane = threadIdx.x & 31;
  const int nvec = H / P;
  const float inv_h = 1.0f / static_cast<float>(H);
  for (int64_t row = static_cast<int64_t>(blockIdx.x) * kNormWarps + (threadIdx.x >> 5); row < M;
       row += static_cast<int64_t>(gridDim.x) * kNormWarps) {
    const uint4* xr = reinterpret_cast<const uint4*>(x + row * H);
    uint4 q[VPL];
    float ss = 0.f;
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      const int v = lane + 32 * i;
      if (v < nvec) {
        q[i] = __ldcs(xr + v);
        float f[P];
        VT::unpack(q[i], f);
#pragma unroll
        for (int e = 0; e < P; ++e) ss = fmaf(f[e], f[e], ss);
      }
    }
    ss = warp_sum(ss);
    const float rinv = rsqrtf(ss * inv_h + eps);
    uint4* yr = reinterpret_cast<uint4*>(y + row * H);
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      const int v = lane + 32 * i;
      if (v < nvec) {
        float f[P];
        VT::unpack(q[i], f);
        if (scale != nullptr) {
          const float4* s4 = reinterpret_cast<const float4*>(scale + v * P);
#pragma unroll
          for (int e4 = 0; e4 < P / 4; ++e4) {
            float4 s = __ldg(s4 + e4);
            if (centered) {
              s.x += 1.f; s.y += 1.f; s.z += 1.f; s.w += 1.f;
            }
            f[4 * e4 + 0] = f[4 * e4 + 0] * rinv * s.x;
            f[4 * e4 + 1] = f[4 * e4 + 1] * rinv * s.y;
            f[4 * e4 + 2] = f[4 * e4 + 2] * rinv * s.z;
            f[4 * e4 + 3] = f[4 * e4 + 3] * rinv * s.w;
          }
        } else {
#pragma unroll
          for (int e = 0; e < P; ++e) f[e] *= rinv;
        }
        __stcs(yr + v, VT::pack(f));
      }
    }
  }
}

constexpr int kNormCtaThreads = 128;

// Wide rows: one 128-thread CTA per row, VPT 16-byte vectors per thread held in
// registers (about 40 registers), so an SM keeps 16 CTAs -- 64 warps of loads --
// in flight.  Sum of squares: shuffles within each warp, then 4 partials through
// shared memory.  y may alias x (each thread rewrites only what it read).
template <typename T, int VPT>
__global__ void __launch_bounds__(kNormCtaThreads)
    rmsnorm_cta(const T* x, T* y, const float* __restrict__ scale, int centered, float eps,
                int64_t M, int H) {
  ptx::griddep_wait();
  ptx::griddep_launch_dependents();
  using VT = VecTraits<T>;
  constexpr int P = VT::kPer;
  __shared__ float part[kNormCtaThreads / 32];
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  const int nvec = H / P;
  const float inv_h = 1.0f / static_cast<float>(H);
  for (int64_t row = blockIdx.x; row < M; row += gridDim.x) {
    const uint4* xr = reinterpret_cast<const uint4*>(x + row * H);
    uint4 q[VPT];
    float ss = 0.f;
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
      const int v = tid + kNormCtaThreads * i;
      if (v < nvec) {
        q[i] = __ldcs(xr + v);
        float f[P];
        VT::unpack(q[i], f);
#pragma unroll
        for (int e = 0; e < P; ++e) ss = fmaf(f[e], f[e], ss);
      }
    }
    ss = warp_sum(ss);
    if (lane == 0) part[w] = ss;
    __syncthreads();
    float tot = 0.f;
#pragma unroll
    for (int i = 0; i < kNormCtaThreads / 32; ++i) tot += part[i];
    __syncthreads();  // part[] is rewritten by the next row
    const float rinv = rsqrtf(tot * inv_h + eps);
    uint4* yr = reinterpret_cast<uint4*>(y + row * H);
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
      const int v = tid + kNormCtaThreads * i;
      if (v < nvec) {
        float f[P];
        VT::unpack(q[i], f);
        if (scale != nullptr) {
          const float4* s4 = reinterpret_cast<const float4*>(scale + v * P);
#pragma unroll
          for (int e4 = 0; e4 < P / 4; ++e4) {
            float4 s = __ldg(s4 + e4);
            if (centered) {
              s.x += 1.f; s.y += 1.f; s.z += 1.f; s.w += 1.f;
            }
            f[4 * e4 + 0] = f[4 * e4 + 0] * rinv * s.x;
            f[4 * e4 + 1] = f[4 * e4 + 1] * rinv * s.y;
            f[4 * e4 + 2] = f[4 * e4 + 2] * rinv * s.z;
            f[4 * e4 + 3] = f[4 * e4 + 3] * rinv * s.w;
          }
        } else {
#pragma unroll
          for (int e = 0; e < P; ++e) f[e] *= rinv;
        }
        __stcs(yr + v, VT::pack(f));
      }
    }
  }
}

// Any width and alignment: pass 1 sums squares, pass 2 rescales (re-read from L2).
template <typename T>
__global__ void __launch_bounds__(kNormWarps * 32)
    rmsnorm_generic(const T* x, T* y, const float* __restrict__ scale, int centered, float eps,
                    int64_t M, int64_t H) {
  ptx::griddep_wait();
  ptx::griddep_launch_dependents();
  using VT = VecTraits<T>;
  const int lane = threadIdx.x & 31;
  for (int64_t row = static_cast<int64_t>(blockIdx.x) * kNormWarps + (threadIdx.x >> 5); row < M;
       row += static_cast<int64_t>(gridDim.x) * kNormWarps) {
    const T* xr = x + row * H;
    float ss = 0.f;
    for (int64_t i = lane; i < H; i += 32) {
      const float f = VT::load1(xr + i);
      ss = fmaf(f, f, ss);
    }
    ss = warp_sum(ss);
    const float rinv = rsqrtf(ss / static_cast<float>(H) + eps);
    T* yr = y + row * H;
    for (int64_t i = lane; i < H; i += 32) {
      float f = VT::load1(xr + i) * rinv;
      if (scale != nullptr) f *= centered ? (1.f + scale[i]) : scale[i];
      VT::store1(yr + i, f);
    }
  }
}

}  // namespace tpl
