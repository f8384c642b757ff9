// gemm_fp32.cuh -- fp32 column- and row-parallel linears on the CUDA cores.
//
// fp32 in / fp32 out must meet a 1e-5 relative error, which rules out TF32 or
// bf16 tensor-core inputs; these shapes are small (the tiny TP MLP: 32 tokens),
// so the kernel is built for latency: 32 x 32 output tiles, 32-wide K steps
// loaded as float4 with the next step prefetched into registers while the
// current one is multiplied, and the K range of a tile split over a thread-block
// cluster of up to 8 CTAs (grid z).  Each CTA of the cluster sums its K steps in
// order into a register accumulator; CTA 0 then adds the other CTAs' partial
// tiles, read from their shared memory, in cluster order and runs the epilogue,
// so the result is deterministic and no global scratch is needed.  Same
// semantics as the bf16 kernel: column mode maps output columns through the
// partition pieces and fuses bias + activation; row mode accumulates the ranks'
// partial products in rank order (K steps are ordered rank by rank) and fuses
// bias + residual.
#pragma once

#include <cooperative_groups.h>

#include "common.cuh"
#include "ptx.cuh"

namespace tpl {

constexpr int kF32BM = 32, kF32BN = 32, kF32BK = 32, kF32Threads = 256;
constexpr int kF32MaxSplit = 8;  // CTAs of one cluster sharing a tile's K range
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
  int32_t k_steps;  // 32-wide K steps of one tile (row mode: summed over ranks r0 .. r1-1)
  int32_t vec;      // every row start of A and B is 16-byte aligned (float4 loads)
};

__device__ __forceinline__ int64_t seq_row_f32(const F32Args& a, int64_t m) {
  const int64_t b = m / a.sp_seq, t = m - b * a.sp_seq;
  const int64_t r = t / a.sp_seg, tl = t - r * a.sp_seg;
  return (r * a.sp_batch + b) * a.sp_seg + tl;
}

// The A (activation) and B (weight) pointers, leading dimensions and width of
// K step `s` of a tile; row mode walks the ranks r0 .. r1-1 in order.
struct F32Step {
  const float* A;
  const float* B;
  int64_t lda, ldb;
  int k0, kr;
};

__device__ __forceinline__ F32Step f32_step(const F32Args& a, int s, int wrow0) {
  F32Step st;
  if (a.mode == 0) {
    st.A = a.x;
    st.B = a.w + static_cast<int64_t>(wrow0) * a.K;
    st.lda = st.ldb = a.K;
    st.kr = a.K;
    st.k0 = s * kF32BK;
    return st;
  }
  int r = a.r0;
  for (;;) {
    const int kr = static_cast<int>(a.koff[r + 1] - a.koff[r]);
    const int n = (kr + kF32BK - 1) / kF32BK;
    if (s < n || r + 1 >= a.r1) {
      st.A = a.h + a.M * a.koff[r];
      st.B = a.w + static_cast<int64_t>(a.N) * a.koff[r] + static_cast<int64_t>(wrow0) * kr;
      st.lda = st.ldb = kr;
      st.kr = kr;
      st.k0 = s * kF32BK;
      return st;
    }
    s -= n;
    ++r;
  }
}

// One thread's four K-consecutive values of a 32 x 32 operand tile (rows of
// A or B), zero outside the tile's valid rows and the step's K width.
__device__ __forceinline__ float4 f32_load4(const float* base, int64_t ld, int64_t row, bool row_ok,
                                            int k, int kr, bool vec) {
  float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
  if (!row_ok) return v;
  const float* p = base + row * ld + k;
  if (vec && k + 4 <= kr) return __ldg(reinterpret_cast<const float4*>(p));
  if (k + 0 < kr) v.x = __ldg(p + 0);
  if (k + 1 < kr) v.y = __ldg(p + 1);
  if (k + 2 < kr) v.z = __ldg(p + 2);
  if (k + 3 < kr) v.w = __ldg(p + 3);
  return v;
}

__global__ void __launch_bounds__(kF32Threads) gemm_fp32_simt(const __grid_constant__ F32Args a) {
  __shared__ float As[kF32BK][kF32BM + 1];
  __shared__ float Bs[kF32BK][kF32BN + 1];
  __shared__ float Part[kF32BM * kF32BN];  // this CTA's partial tile, read by CTA 0 of the cluster
  const int tid = threadIdx.x;
  const int tx = tid % 16, ty = tid / 16;       // 2 x 2 outputs: rows 2 ty.., columns 2 tx..
  const int lr = tid / 8, lk = (tid % 8) * 4;   // loader: row lr, K offset lk (4 floats)
  const int nt = blockIdx.x;
  const int64_t m0 = static_cast<int64_t>(blockIdx.y) * kF32BM;
  const int split = gridDim.z, z = blockIdx.z;
  ptx::griddep_wait();
  ptx::griddep_launch_dependents();

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

  // This CTA's K steps [s0, s1) of the tile.
  const int s0 = static_cast<int>(static_cast<int64_t>(a.k_steps) * z / split);
  const int s1 = static_cast<int>(static_cast<int64_t>(a.k_steps) * (z + 1) / split);

  const int64_t gm = m0 + lr;
  const bool a_ok = gm < a.M;
  const int64_t am = (a.a_remap && a_ok) ? seq_row_f32(a, gm) : gm;
  const bool b_ok = lr < valid;

  float acc[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
  float4 ra = make_float4(0.f, 0.f, 0.f, 0.f), rb = ra;
  if (s0 < s1) {
    const F32Step st = f32_step(a, s0, wrow0);
    ra = f32_load4(st.A, st.lda, am, a_ok, st.k0 + lk, st.kr, a.vec);
    rb = f32_load4(st.B, st.ldb, lr, b_ok, st.k0 + lk, st.kr, a.vec);
  }
  for (int s = s0; s < s1; ++s) {
    As[lk + 0][lr] = ra.x;
    As[lk + 1][lr] = ra.y;
    As[lk + 2][lr] = ra.z;
    As[lk + 3][lr] = ra.w;
    Bs[lk + 0][lr] = rb.x;
    Bs[lk + 1][lr] = rb.y;
    Bs[lk + 2][lr] = rb.z;
    Bs[lk + 3][lr] = rb.w;
    __syncthreads();
    if (s + 1 < s1) {  // the next step's operands travel while this one is multiplied
      const F32Step st = f32_step(a, s + 1, wrow0);
      ra = f32_load4(st.A, st.lda, am, a_ok, st.k0 + lk, st.kr, a.vec);
      rb = f32_load4(st.B, st.ldb, lr, b_ok, st.k0 + lk, st.kr, a.vec);
    }
#pragma unroll
    for (int kk = 0; kk < kF32BK; ++kk) {
      const float a0 = As[kk][2 * ty], a1 = As[kk][2 * ty + 1];
      const float b0 = Bs[kk][2 * tx], b1 = Bs[kk][2 * tx + 1];
      acc[0][0] = fmaf(a0, b0, acc[0][0]);
      acc[0][1] = fmaf(a0, b1, acc[0][1]);
      acc[1][0] = fmaf(a1, b0, acc[1][0]);
      acc[1][1] = fmaf(a1, b1, acc[1][1]);
    }
    __syncthreads();
  }

  if (split > 1) {
    // Partial tiles of the cluster's CTAs, summed by CTA 0 in cluster order.
    namespace cg = cooperative_groups;
    cg::cluster_group cl = cg::this_cluster();
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
      for (int j = 0; j < 2; ++j) Part[(2 * ty + i) * kF32BN + 2 * tx + j] = acc[i][j];
    cl.sync();
    if (z == 0) {
      for (int q = 1; q < split; ++q) {
        const float* rp = cl.map_shared_rank(Part, q);
#pragma unroll
        for (int i = 0; i < 2; ++i)
#pragma unroll
          for (int j = 0; j < 2; ++j) acc[i][j] += rp[(2 * ty + i) * kF32BN + 2 * tx + j];
      }
    }
    cl.sync();  // CTA 0 has read every partial before any CTA leaves
    if (z != 0) return;
  }

#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int64_t m = m0 + 2 * ty + i;
    if (m >= a.M) continue;
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int c = 2 * tx + j;
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
