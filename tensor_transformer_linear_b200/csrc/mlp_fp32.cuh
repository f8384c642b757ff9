// mlp_fp32.cuh -- the whole fp32 TP MLP block in one launch, for latency
// (nanotron "MLP Module": c_fc column-parallel -> activation -> c_proj
// row-parallel with the partial-sum reduction; google-research residual
// section).
//
//   y = act(x W1^T + b1) W2^T (+ b2) (+ residual)
//
// is computed the way its TP shards are.  The intermediate dimension I is cut
// into kMlpSlices slices, each inside one rank's shard.  A thread-block
// cluster of kMlpSlices CTAs takes one kMlpRows-row token tile; CTA s owns
// slice s:
//   1. its slice of h = act(x W1^T + b1), into shared memory (h never reaches
//      global memory);
//   2. that slice's partial product h_s W2_s^T, into shared memory;
//   3. after a cluster barrier, its 1/kMlpSlices of the output columns: the
//      partials of all CTAs summed in slice order (= rank order) through
//      distributed shared memory, then b2 and the residual.
// Weights are copied with cp.async before the wait on the previous kernel
// (they do not depend on it); x after it.  fp32 FMA on the CUDA cores: the
// 1e-5 relative error of the fp32 path rules out TF32 tensor-core inputs.
#pragma once

#include <cooperative_groups.h>

#include "common.cuh"
#include "ptx.cuh"

namespace tpl {

constexpr int kMlpSlices = 16;  // CTAs of one cluster (a non-portable cluster size)
constexpr int kMlpRows = 8;     // token rows of one tile
constexpr int kMlpThreads = 256;
constexpr int kMlpRows1 = 2;  // token rows per thread item in phase 1
constexpr int kMlpRows2 = 8;  // token rows per thread item in phase 2

struct MlpArgs {
  const float* x;         // [M][H]
  const float* w1;        // [I][H]
  const float* b1;        // [I] or null
  const float* w2;        // rank r's block [H][kr] at element H * r * kr
  const float* b2;        // [H] or null
  const float* residual;  // [M][H] or null; may alias y
  float* y;               // [M][H]
  int64_t M;
  int32_t H, I, kr, hc;   // hc = I / kMlpSlices columns of h per CTA
  int32_t act;
};

// Shared-memory layout (floats): x tile [kMlpRows][H], W1 slice [hc][H + 4],
// W2 slice [H][hc + 4], h slice [kMlpRows][hc + 4].  The partial product
// [kMlpRows][H] reuses the x tile and W1 slice once h is complete.  The +4
// row padding keeps each quarter-warp's 16-byte loads on distinct banks.
__host__ __device__ constexpr int64_t mlp_smem_floats(int H, int hc) {
  return static_cast<int64_t>(kMlpRows) * H + static_cast<int64_t>(hc) * (H + 4) +
         static_cast<int64_t>(H) * (hc + 4) + static_cast<int64_t>(kMlpRows) * (hc + 4);
}

__device__ __forceinline__ void cp_async16(float* dst, const float* src, bool valid) {
  const uint32_t d = ptx::smem_u32(dst);
  const int n = valid ? 16 : 0;  // 0 source bytes: the 16 bytes are zero-filled
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(d), "l"(src), "r"(n)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ float dot4(float acc, const float4& a, const float4& b) {
  acc = fmaf(a.x, b.x, acc);
  acc = fmaf(a.y, b.y, acc);
  acc = fmaf(a.z, b.z, acc);
  return fmaf(a.w, b.w, acc);
}

__global__ void __launch_bounds__(kMlpThreads, 1) mlp_fp32_fused(const __grid_constant__ MlpArgs a) {
  extern __shared__ float4 smem_v4[];
  float* smem = reinterpret_cast<float*>(smem_v4);
  const int H = a.H, hc = a.hc;
  const int ldw1 = H + 4, ldw2 = hc + 4, ldh = hc + 4;
  float* xs = smem;                                           // [kMlpRows][H]
  float* w1s = xs + kMlpRows * H;                             // [hc][ldw1]
  float* w2s = w1s + static_cast<int64_t>(hc) * ldw1;         // [H][ldw2]
  float* hs = w2s + static_cast<int64_t>(H) * ldw2;           // [kMlpRows][ldh]
  float* part = smem;                                         // [kMlpRows][H], after phase 1

  const int tid = threadIdx.x;
  const int s = blockIdx.x;                  // slice = rank of this CTA in its cluster
  const int64_t m0 = static_cast<int64_t>(blockIdx.y) * kMlpRows;
  const int c0 = s * hc;                     // first column of h of this slice
  const int r = c0 / a.kr, k0 = c0 - r * a.kr;  // its rank and offset inside the rank's shard
  const int hv = H / 4, cv = hc / 4;

  // W1 slice: hc contiguous rows of W1.
  for (int i = tid; i < hc * hv; i += kMlpThreads) {
    const int row = i / hv, v = i - row * hv;
    cp_async16(w1s + row * ldw1 + 4 * v, a.w1 + static_cast<int64_t>(c0 + row) * H + 4 * v, true);
  }
  cp_async_commit();
  // the previous kernel may still be writing x; weights are never written by it
  ptx::griddep_wait();
  ptx::griddep_launch_dependents();
  for (int i = tid; i < kMlpRows * hv; i += kMlpThreads) {
    const int row = i / hv, v = i - row * hv;
    const bool ok = m0 + row < a.M;
    const float* src = a.x + (ok ? (m0 + row) * H + 4 * v : 0);
    cp_async16(xs + row * H + 4 * v, src, ok);
  }
  cp_async_commit();
  // W2 slice: row n holds columns k0 .. k0 + hc of row n of rank r's block.
  const float* w2r = a.w2 + static_cast<int64_t>(H) * r * a.kr + k0;
  for (int i = tid; i < H * cv; i += kMlpThreads) {
    const int n = i / cv, v = i - n * cv;
    cp_async16(w2s + n * ldw2 + 4 * v, w2r + static_cast<int64_t>(n) * a.kr + 4 * v, true);
  }
  cp_async_commit();
  cp_async_wait<1>();  // W1 and x have landed; W2 may still be in flight
  __syncthreads();

  // ---- phase 1: h[i][c] = act(x[i] . W1[c0 + c] + b1), kMlpRows1 rows per item
  for (int o = tid; o < (kMlpRows / kMlpRows1) * hc; o += kMlpThreads) {
    const int c = o % hc, rg = o / hc;
    const float* wr = w1s + c * ldw1;
    const float* xr = xs + kMlpRows1 * rg * H;
    // two accumulators per row (K blocks of 4 alternating): half the length of
    // the dependent FMA chain; H % 8 == 0
    float acc[kMlpRows1][2];
#pragma unroll
    for (int j = 0; j < kMlpRows1; ++j) acc[j][0] = acc[j][1] = 0.f;
#pragma unroll 2
    for (int k = 0; k < H; k += 8) {
      const float4 w0 = *reinterpret_cast<const float4*>(wr + k);
      const float4 w1 = *reinterpret_cast<const float4*>(wr + k + 4);
#pragma unroll
      for (int j = 0; j < kMlpRows1; ++j) {
        acc[j][0] = dot4(acc[j][0], *reinterpret_cast<const float4*>(xr + j * H + k), w0);
        acc[j][1] = dot4(acc[j][1], *reinterpret_cast<const float4*>(xr + j * H + k + 4), w1);
      }
    }
    const float bias = a.b1 != nullptr ? a.b1[c0 + c] : 0.f;
#pragma unroll
    for (int j = 0; j < kMlpRows1; ++j)
      hs[(kMlpRows1 * rg + j) * ldh + c] = apply_act(acc[j][0] + acc[j][1] + bias, a.act);
  }
  cp_async_wait<0>();
  __syncthreads();  // h complete, W2 landed; x tile and W1 slice free for the partial

  // ---- phase 2: part[i][n] = h[i] . W2_slice[n], kMlpRows2 rows per item
  for (int o = tid; o < (kMlpRows / kMlpRows2) * H; o += kMlpThreads) {
    const int n = o % H, rg = o / H;
    const float* wr = w2s + n * ldw2;
    const float* hr = hs + kMlpRows2 * rg * ldh;
    float acc[kMlpRows2];
#pragma unroll
    for (int i = 0; i < kMlpRows2; ++i) acc[i] = 0.f;
#pragma unroll 2
    for (int k = 0; k < hc; k += 4) {
      const float4 w = *reinterpret_cast<const float4*>(wr + k);
#pragma unroll
      for (int i = 0; i < kMlpRows2; ++i)
        acc[i] = dot4(acc[i], *reinterpret_cast<const float4*>(hr + i * ldh + k), w);
    }
#pragma unroll
    for (int i = 0; i < kMlpRows2; ++i) part[(kMlpRows2 * rg + i) * H + n] = acc[i];
  }

  // ---- the partials summed across the cluster in slice order
  namespace cg = cooperative_groups;
  cg::cluster_group cl = cg::this_cluster();
  cl.sync();
  const int per = H / kMlpSlices;  // output columns reduced by this CTA
  for (int e = tid; e < kMlpRows * per; e += kMlpThreads) {
    const int i = e / per, n = s * per + (e - i * per);
    const int64_t m = m0 + i;
    float p[kMlpSlices];  // every CTA's value loaded before the sum: one round trip
#pragma unroll
    for (int q = 0; q < kMlpSlices; ++q) p[q] = cl.map_shared_rank(part, q)[i * H + n];
    float v = 0.f;
#pragma unroll
    for (int q = 0; q < kMlpSlices; ++q) v += p[q];
    if (m < a.M) {
      if (a.b2 != nullptr) v += a.b2[n];
      if (a.residual != nullptr) v += a.residual[m * H + n];
      a.y[m * H + n] = v;
    }
  }
  cl.sync();  // every CTA's partial has been read before any CTA leaves
}

}  // namespace tpl
