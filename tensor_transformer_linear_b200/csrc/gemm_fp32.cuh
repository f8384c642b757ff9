// gemm_fp32.cuh -- fp32 column- and row-parallel linears on the CUDA cores.
//
// fp32 in / fp32 out must meet a 1e-5 relative error, which rules out TF32 or
// bf16 tensor-core inputs; these shapes are small (the tiny TP MLP), so a
// shared-memory-tiled SIMT GEMM with fp32 FMA is the right tool.  Same
// semantics as the bf16 kernel: column mode maps output columns through the
// partition pieces and fuses bias + activation; row mode accumulates the ranks'
// partial products into one register accumulator in rank order and fuses bias
// + residual.
#pragma once

#include "common.cuh"

namespace tpl {

constexpr int kF32BM = 64, kF32BN = 64, kF32BK = 16, kF32Threads = 256;
constexpr int kF32MaxPieces = 64;

struct F32Piece {
  int64_t out_off;
  int32_t src_row;
  int32_t width;
  int32_t ld;
  int32_t nt_begin;  // first 64-column tile of this piece
};

struct F32Args {
  int32_t mode;  // 0 column, 1 row
  int32_t act;
  int64_t M;
  int32_t K;       // column mode contraction width
  int32_t n_tiles;
  // column
  int32_t n_pieces;
  F32Piece pieces[kF32MaxPieces];
  const float* x;
  const float* w;
  const float* bias;
  float* y;
  // row
  int32_t N;
  int32_t r0, r1;
  int64_t koff[TPL_MAX_TP + 1];
  const float* h;
  const float* residual;
  float* partials;  // when set: write this launch's fp32 sum here (no bias/residual)
  // Sequence parallelism, as in GemmArgs: rank-major rows for A (a_remap) or for
  // the output and residual (out_remap).
  int32_t sp_batch, sp_seq, sp_seg;
  int32_t a_remap, out_remap;
};

__device__ __forceinline__ int64_t seq_row_f32(const F32Args& a, int64_t m) {
  const int64_t b = m / a.sp_seq, t = m - b * a.sp_seq;
  const int64_t r = t / a.sp_seg, tl = t - r * a.sp_seg;
  return (r * a.sp_batch + b) * a.sp_seg + tl;
}

__global__ void __launch_bounds__(kF32Threads) gemm_fp32_simt(const __grid_constant__ F32Args a) {
  __shared__ float As[kF32BK][kF32BM + 4];
  __shared__ float Bs[kF32BK][kF32BN + 4];
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  const int nt = blockIdx.x;
  const int64_t m0 = static_cast<int64_t>(blockIdx.y) * kF32BM;

  // Output column mapping of this tile.
  int32_t wrow0, valid, ld, bias0;
  int64_t out0;
  if (a.mode == 0) {
    int p = 0;
    while (p + 1 < a.n_pieces && a.pieces[p + 1].nt_begin <= nt) ++p;
    const F32Piece& pc = a.pieces[p];
    const int local = (nt - pc.nt_begin) * kF32BN;
    wrow0 = pc.src_row + local;
    valid = min(kF32BN, pc.width - local);
    ld = pc.ld;
    out0 = pc.out_off + local;
    bias0 = wrow0;
  } else {
    wrow0 = nt * kF32BN;
    valid = min(kF32BN, a.N - wrow0);
    ld = a.N;
    out0 = wrow0;
    bias0 = wrow0;
  }

  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;

  const int nr = (a.mode == 0) ? 1 : (a.r1 - a.r0);
  for (int rr = 0; rr < nr; ++rr) {
    const float* A;
    const float* B;
    int64_t lda, ldb;
    int Kr;
    if (a.mode == 0) {
      A = a.x;
      B = a.w + static_cast<int64_t>(wrow0) * a.K;
      lda = ldb = a.K;
      Kr = a.K;
    } else {
      const int r = a.r0 + rr;
      Kr = static_cast<int>(a.koff[r + 1] - a.koff[r]);
      A = a.h + a.M * a.koff[r];
      B = a.w + static_cast<int64_t>(a.N) * a.koff[r] + static_cast<int64_t>(wrow0) * Kr;
      lda = ldb = Kr;
    }
    for (int k0 = 0; k0 < Kr; k0 += kF32BK) {
      for (int i = threadIdx.x; i < kF32BM * kF32BK; i += kF32Threads) {
        const int mm = i / kF32BK, kk = i % kF32BK;
        const int64_t gm = m0 + mm;
        const int64_t am = (a.a_remap && gm < a.M) ? seq_row_f32(a, gm) : gm;
        As[kk][mm] = (gm < a.M && k0 + kk < Kr) ? A[am * lda + k0 + kk] : 0.f;
      }
      for (int i = threadIdx.x; i < kF32BN * kF32BK; i += kF32Threads) {
        const int nn = i / kF32BK, kk = i % kF32BK;
        Bs[kk][nn] = (nn < valid && k0 + kk < Kr) ? B[static_cast<int64_t>(nn) * ldb + k0 + kk]
                                                  : 0.f;
      }
      __syncthreads();
#pragma unroll
      for (int kk = 0; kk < kF32BK; ++kk) {
        float av[4], bv[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) av[i] = As[kk][ty * 4 + i];
#pragma unroll
        for (int j = 0; j < 4; ++j) bv[j] = Bs[kk][tx * 4 + j];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
      }
      __syncthreads();
    }
  }

#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t m = m0 + ty * 4 + i;
    if (m >= a.M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int c = tx * 4 + j;
      if (c >= valid) continue;
      float v = acc[i][j];
      const int64_t prow = a.out_remap ? seq_row_f32(a, m) : m;
      const int64_t off = prow * ld + out0 + c;
      if (a.partials != nullptr) {
        a.partials[off] = v;
        continue;
      }
      if (a.bias != nullptr) v += a.bias[bias0 + c];
      if (a.mode == 0) v = apply_act(v, a.act);
      if (a.mode == 1 && a.residual != nullptr) v += a.residual[off];
      a.y[off] = v;
    }
  }
}

}  // namespace tpl
