// gemm_bf16.cuh -- persistent, warp-specialised tcgen05 GEMM for the column-
// and row-parallel linears (bf16 in, fp32 accumulate in TMEM, fused epilogue).
//
// Column mode (DeepSpeed SubParamLinearLayer.forward, nanotron c_fc): the
// output columns of every rank's shard are a list of pieces, each a run of
// consecutive fused-weight rows.  Pieces are cut into 128-column half blocks;
// a 128x256 tile pairs two consecutive half blocks, whose weight rows are
// fetched by two TMA boxes with independent row coordinates.  So the fused
// QKV weight is read in place, in its own order, with no gather pass, and a
// tile may hold the k piece of a rank in one half and its v piece in the other.
// The epilogue adds the bias (indexed by weight row), applies GELU and stores
// bf16 straight into the rank's shard.
//
// Row mode (google-research o_wo section, nanotron c_proj): the K loop runs
// over ranks r0..r1-1 and, inside each, over that rank's contraction slice,
// all into the same TMEM accumulator.  The cross-shard partial-sum reduction
// is therefore the accumulation itself, in rank order, in fp32.  The epilogue
// adds bias and residual and stores bf16 (or, for the unreduced check, stores
// one rank's fp32 partial).
//
// Roles (320 threads, one CTA per SM): warp 0 issues TMA loads into a
// kStages-deep shared-memory ring; warp 1 issues tcgen05.mma (one elected
// lane) into one of two TMEM accumulators; warps 2..9 drain the other
// accumulator through tcgen05.ld -- each owns one TMEM lane quarter (32 rows)
// and one 128-column half -- so the epilogue of tile i overlaps the MMAs of
// tile i+1, with two epilogue warps per SM sub-partition to hide latency.
#pragma once

#include "common.cuh"
#include "ptx.cuh"
#include "trace.cuh"

namespace tpl {

constexpr int kBM = 128;
constexpr int kHalfN = 128;
constexpr int kBK = 64;  // 64 bf16 = one 128-byte swizzle row
constexpr int kStages = 4;
constexpr int kABytes = kBM * kBK * 2;
constexpr int kBHalfBytes = kHalfN * kBK * 2;
constexpr int kStageBytes = kABytes + 2 * kBHalfBytes;
constexpr int kMaxPieces = 64;
constexpr int kEpiWarps = 8;  // two per TMEM lane quarter: one per 128-column half
constexpr int kGemmThreads = 64 + 32 * kEpiWarps;
constexpr int kAccCols = 256;  // fp32 columns of one accumulator
constexpr int kBiasSmemBytes = kEpiWarps * kHalfN * 4;
constexpr int kGemmSmemBytes = kStages * kStageBytes + kBiasSmemBytes + 1024 + 256;

// kModeSwiglu: a column-parallel projection over a fused [wi0; wi1] weight
// whose tiles pair a 128-column half block of wi0 with the same half block of
// wi1, so the epilogue holds both operands of silu(a) * b (google-research
// "SwiGLU" section) and writes 128 output columns per tile.
enum GemmMode : int { kModeColumn = 0, kModeRow = 1, kModeSwiglu = 2 };

struct ColPiece {
  int64_t out_off;   // element offset in y of (row 0, first column of the piece)
  int32_t src_row;   // first fused-weight row; also the fused-bias index
  int32_t src_row1;  // SwiGLU mode: first wi1 row of the piece
  int32_t width;     // columns in the piece
  int32_t ld;        // row stride (elements) of the rank's shard
  int32_t hb_begin;  // first 128-column half block (SwiGLU mode: first tile)
  int32_t pad_;
};

constexpr int kMaxPeers = 64;   // TPL_MAX_TP
constexpr int kMaxGather = 16;  // ranks a column GEMM can read A from (TPL_MAX_GATHER)

struct GemmArgs {
  CUtensorMap tmA;  // column: X {K, M};      row: H  {Kr, M, tp} of ranks 0 .. r_split-1
  CUtensorMap tmB;  // column: W {K, rows};   row: W2 {Kr, N, tp} of ranks 0 .. r_split-1
  CUtensorMap tmA2;  // row mode, ranks r_split .. tp-1 (a second contraction width)
  CUtensorMap tmB2;
  int32_t mode;
  int32_t act;
  int32_t M;
  int32_t k_iters;  // 64-wide K blocks per rank (column mode: of K)
  int32_t r0, r1;   // row mode: ranks accumulated
  int32_t m_blocks, n_tiles, num_tiles, group_m;
  int32_t n_halves;
  int32_t vec_store;  // every output row start is 16-byte aligned
  // K order of a tile: with k_serp set, a CTA pair walks K backwards on its
  // odd tiles, so a tile wave starts on the K slices the wave before it read
  // last (still in L2) when the two waves share operand blocks.
  int32_t k_serp;
  uint32_t trace_seq;  // launch number for the optional timing records (trace.cuh)
  // Fused RMSNorm (column mode, google-research allgather_layernorm): A is
  // the raw x and the norm's scale is folded into the weight, so row m of the
  // output is act(norm_rs[m] * (x W'^T)[m] + b).  Before its first epilogue,
  // every CTA's epilogue warps compute norm_rs[m] = rsqrt(mean(x[m]^2) + eps)
  // for their share of the rows (in fp32, from bf16 x) and raise norm_flag[m]
  // to norm_epoch (a value fresh to every launch, so a flag left by an earlier
  // launch never matches); an epilogue scales row m once its flag is up.
  int32_t norm;
  uint32_t norm_epoch;
  float norm_eps;
  const __nv_bfloat16* norm_x;  // x [M][k_iters * 64 >= K] rows, row stride norm_ld
  int32_t norm_K, norm_ld;
  float* norm_rs;        // [M]
  uint32_t* norm_flag;   // [M]
  int32_t n_pieces;
  ColPiece pieces[kMaxPieces];
  const __nv_bfloat16* bias;
  __nv_bfloat16* y;
  int32_t N;  // row mode output width
  const __nv_bfloat16* residual;
  float* partials;  // row mode: store this launch's fp32 sum here instead of y
  // Sequence parallelism (nanotron "MLP Module": [batch, seq // tp, hidden] per
  // rank): logical row m = b * seq + t lives at physical row
  // (t / seg * batch + b) * seg + t % seg, seg = seq / tp (rank-major slices).
  int32_t sp_batch, sp_seq, sp_seg;
  int32_t a_remap;    // A rows are read from the rank-major layout (all-gather)
  int32_t out_remap;  // output (and residual) rows use it (reduce-scatter)
  // Row mode with two contraction widths: ranks below r_split use tmA/tmB and
  // k_iters K blocks, the others tmA2/tmB2 and k_iters2 (r_split = tp if equal).
  int32_t r_split, k_iters2;
  // Peer scatter (row mode, one rank's shard of a row-parallel linear split
  // over GPUs): token m = b * sp_seq + t belongs to rank t / sp_seg and lands
  // in slot src_rank of that rank's receive buffer [tp][sp_batch][sp_seg][N],
  // at peer[t / sp_seg] (another GPU's memory for every rank but this one).
  int32_t scatter, src_rank;
  __nv_bfloat16* peer[kMaxPeers];
  // Peer gather (column mode, one rank's column shard of a linear split over
  // GPUs, fed by every rank's token slice): the A row of token
  // m = b * sp_seq + t is row b * sp_seg + t % sp_seg of rank t / sp_seg's slice
  // [sp_batch][sp_seg][K], loaded through tmGather[t / sp_seg] (a map of another
  // GPU's memory for every rank but this one; plain TMA loads, no multicast).
  int32_t a_gather;
  CUtensorMap tmGather[kMaxGather];
};

// Row mode: the rank and K block of K step ki of a tile.
__device__ __forceinline__ void row_pos(const GemmArgs& a, int ki, int& rr, int& kb) {
  const int n1 = max(0, min(a.r1, a.r_split) - a.r0) * a.k_iters;
  if (ki < n1) {
    rr = a.r0 + ki / a.k_iters;
    kb = ki - (rr - a.r0) * a.k_iters;
  } else {
    const int first2 = max(a.r0, a.r_split);
    const int k2 = ki - n1;
    rr = first2 + k2 / a.k_iters2;
    kb = k2 - (rr - first2) * a.k_iters2;
  }
}

// The fused RMSNorm's statistics: rows [r0, r1) of x for this CTA's 256
// epilogue threads, 4 adjacent lanes per row (each a quarter of the row's
// 16-byte vectors, summed in a fixed order), 64 rows per pass.
__device__ __forceinline__ void norm_stats(const GemmArgs& a, int r0, int r1, int tid) {
  const int sub = tid & 3;
  const int nv = a.norm_K / 8;
  for (int base = r0; base < r1; base += 64) {
    const int m = base + (tid >> 2);
    float ss = 0.0f;
    if (m < r1) {
      const uint4* row = reinterpret_cast<const uint4*>(a.norm_x + static_cast<int64_t>(m) *
                                                                       a.norm_ld);
      int v = sub;
      for (; v + 28 < nv; v += 32) {  // 8 vectors of this lane in flight
        uint4 q[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) q[u] = __ldg(row + v + 4 * u);
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const float f0 = bf16_lo(q[u].x), f1 = bf16_hi(q[u].x), f2 = bf16_lo(q[u].y),
                      f3 = bf16_hi(q[u].y), f4 = bf16_lo(q[u].z), f5 = bf16_hi(q[u].z),
                      f6 = bf16_lo(q[u].w), f7 = bf16_hi(q[u].w);
          ss = fmaf(f0, f0, ss); ss = fmaf(f1, f1, ss); ss = fmaf(f2, f2, ss);
          ss = fmaf(f3, f3, ss); ss = fmaf(f4, f4, ss); ss = fmaf(f5, f5, ss);
          ss = fmaf(f6, f6, ss); ss = fmaf(f7, f7, ss);
        }
      }
      for (; v < nv; v += 4) {
        const uint4 q = __ldg(row + v);
        const float f0 = bf16_lo(q.x), f1 = bf16_hi(q.x), f2 = bf16_lo(q.y), f3 = bf16_hi(q.y),
                    f4 = bf16_lo(q.z), f5 = bf16_hi(q.z), f6 = bf16_lo(q.w), f7 = bf16_hi(q.w);
        ss = fmaf(f0, f0, ss); ss = fmaf(f1, f1, ss); ss = fmaf(f2, f2, ss);
        ss = fmaf(f3, f3, ss); ss = fmaf(f4, f4, ss); ss = fmaf(f5, f5, ss);
        ss = fmaf(f6, f6, ss); ss = fmaf(f7, f7, ss);
      }
    }
    ss += __shfl_xor_sync(0xffffffffu, ss, 1);
    ss += __shfl_xor_sync(0xffffffffu, ss, 2);
    if (m < r1 && sub == 0) {
      a.norm_rs[m] = rsqrtf(ss / static_cast<float>(a.norm_K) + a.norm_eps);
      __threadfence();
      ptx::st_release_gpu(a.norm_flag + m, a.norm_epoch);
    }
  }
}

// 1 / rms of row m for the fused RMSNorm, once its flag is up (bounded wait).
__device__ __forceinline__ bool norm_row_scale(const GemmArgs& a, int m, float& rs,
                                               volatile int* abort_flag) {
  rs = 1.0f;
  if (m >= a.M) return true;
  if (!ptx::flag_wait(a.norm_flag + m, a.norm_epoch, abort_flag)) return false;
  rs = __ldcg(a.norm_rs + m);
  return true;
}

// Number of 64-wide K steps of one tile.
__device__ __forceinline__ int k_steps(const GemmArgs& a) {
  if (a.mode != kModeRow) return a.k_iters;
  const int n1 = max(0, min(a.r1, a.r_split) - a.r0);
  const int n2 = max(0, a.r1 - max(a.r0, a.r_split));
  return n1 * a.k_iters + n2 * a.k_iters2;
}

__device__ __forceinline__ int seq_row(const GemmArgs& a, int m) {
  const unsigned b = static_cast<unsigned>(m) / static_cast<unsigned>(a.sp_seq);
  const unsigned t = static_cast<unsigned>(m) - b * static_cast<unsigned>(a.sp_seq);
  const unsigned r = t / static_cast<unsigned>(a.sp_seg);
  const unsigned tl = t - r * static_cast<unsigned>(a.sp_seg);
  return static_cast<int>((r * static_cast<unsigned>(a.sp_batch) + b) *
                              static_cast<unsigned>(a.sp_seg) + tl);
}

// Physical output row of logical row m (rank-major when the output is scattered).
__device__ __forceinline__ int out_row(const GemmArgs& a, int m) {
  return a.out_remap ? seq_row(a, m) : m;
}

// Tensor map and row holding the A row of logical row m (column mode).
__device__ __forceinline__ const CUtensorMap* a_source(const GemmArgs& a, int m, int& arow) {
  if (!a.a_gather) {
    arow = a.a_remap ? seq_row(a, m) : m;
    return &a.tmA;
  }
  const unsigned seq = static_cast<unsigned>(a.sp_seq), seg = static_cast<unsigned>(a.sp_seg);
  const unsigned b = static_cast<unsigned>(m) / seq;
  const unsigned t = static_cast<unsigned>(m) - b * seq;
  const unsigned q = t / seg;
  arow = static_cast<int>(b * seg + (t - q * seg));
  return &a.tmGather[q];
}

// Output base and row of logical row m: this launch's y, or in peer-scatter
// mode the receive buffer of the rank that owns the token (see GemmArgs).
__device__ __forceinline__ __nv_bfloat16* out_base(const GemmArgs& a, int m, int& prow) {
  if (!a.scatter) {
    prow = out_row(a, m);
    return a.y;
  }
  const unsigned seq = static_cast<unsigned>(a.sp_seq), seg = static_cast<unsigned>(a.sp_seg);
  const unsigned b = static_cast<unsigned>(m) / seq;
  const unsigned t = static_cast<unsigned>(m) - b * seq;
  const unsigned q = t / seg;
  prow = static_cast<int>((static_cast<unsigned>(a.src_rank) * static_cast<unsigned>(a.sp_batch) +
                           b) * seg + (t - q * seg));
  return a.peer[q];
}

struct HalfInfo {
  int32_t brow;     // weight row (column mode) or output column (row mode) of column 0
  int32_t valid;    // columns of the half block that exist
  int64_t out_off;  // element offset in the output of (row 0, column 0)
  int32_t ld;       // output row stride
  int32_t bias_off;
};

__device__ __forceinline__ HalfInfo decode_half(const GemmArgs& a, int hb) {
  HalfInfo h;
  if (a.mode == kModeSwiglu) {
    // Half 0 of tile t is the wi0 block, half 1 the matching wi1 block.
    const int t = hb >> 1;
    int p = 0;
    while (p + 1 < a.n_pieces && a.pieces[p + 1].hb_begin <= t) ++p;
    const ColPiece& pc = a.pieces[p];
    const int local = (t - pc.hb_begin) * kHalfN;
    h.brow = ((hb & 1) ? pc.src_row1 : pc.src_row) + local;
    h.valid = min(kHalfN, pc.width - local);
    h.out_off = pc.out_off + local;
    h.ld = pc.ld;
    h.bias_off = 0;
  } else if (a.mode == kModeColumn) {
    int p = 0;
    while (p + 1 < a.n_pieces && a.pieces[p + 1].hb_begin <= hb) ++p;
    const ColPiece& pc = a.pieces[p];
    const int local = (hb - pc.hb_begin) * kHalfN;
    h.brow = pc.src_row + local;
    h.valid = min(kHalfN, pc.width - local);
    h.out_off = pc.out_off + local;
    h.ld = pc.ld;
    h.bias_off = pc.src_row + local;
  } else {
    const int col = hb * kHalfN;
    h.brow = col;
    h.valid = min(kHalfN, a.N - col);
    h.out_off = col;
    h.ld = a.N;
    h.bias_off = col;
  }
  return h;
}

__device__ __forceinline__ void tile_coords(const GemmArgs& a, int t, int& mb, int& nt) {
  const int per_group = a.group_m * a.n_tiles;
  const int g = t / per_group;
  const int first_m = g * a.group_m;
  const int gsize = min(a.m_blocks - first_m, a.group_m);
  const int tin = t - g * per_group;
  mb = first_m + tin % gsize;
  nt = tin / gsize;
}

// Bias of the 32 output columns of a half block starting at col0 (0 past its
// valid columns), read straight from global memory: every lane of a warp asks
// for the same addresses, so the loads are broadcasts.
__device__ __forceinline__ void load_bias_chunk(const GemmArgs& a, const HalfInfo& h, int col0,
                                                float (&bv)[32]) {
  const int nvalid = min(32, h.valid - col0);
  const __nv_bfloat16* b = a.bias + h.bias_off + col0;
  if (nvalid == 32 && (reinterpret_cast<uintptr_t>(b) & 15u) == 0) {
#pragma unroll
    for (int j = 0; j < 32; j += 8) {
      const uint4 q = __ldg(reinterpret_cast<const uint4*>(b + j));
      bv[j + 0] = bf16_lo(q.x); bv[j + 1] = bf16_hi(q.x);
      bv[j + 2] = bf16_lo(q.y); bv[j + 3] = bf16_hi(q.y);
      bv[j + 4] = bf16_lo(q.z); bv[j + 5] = bf16_hi(q.z);
      bv[j + 6] = bf16_lo(q.w); bv[j + 7] = bf16_hi(q.w);
    }
  } else {
#pragma unroll
    for (int j = 0; j < 32; ++j) bv[j] = (j < nvalid) ? bf16_to_f(b[j]) : 0.0f;
  }
}

// Epilogue of 32 accumulator columns of one row; bv holds the chunk's bias,
// rs the row's fused-RMSNorm factor (1 without it).
__device__ __forceinline__ void store_chunk(const GemmArgs& a, const HalfInfo& h, int m, int prow,
                                            __nv_bfloat16* ybase, int col0,
                                            const uint32_t (&r)[32], const float (&bv)[32],
                                            float rs = 1.0f) {
  const int nvalid = min(32, h.valid - col0);
  float v[32];
#pragma unroll
  for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]) * rs;

  if (a.mode == kModeRow && a.partials != nullptr) {
    float* dst = a.partials + static_cast<int64_t>(m) * h.ld + h.out_off + col0;
    if (nvalid == 32 && a.vec_store) {
#pragma unroll
      for (int j = 0; j < 32; j += 4)
        *reinterpret_cast<float4*>(dst + j) = make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]);
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j)
        if (j < nvalid) dst[j] = v[j];
    }
    return;
  }

  if (a.bias != nullptr) {
#pragma unroll
    for (int j = 0; j < 32; ++j) v[j] += bv[j];
  }
  if (a.act != TPL_ACT_NONE) {
#pragma unroll
    for (int j = 0; j < 32; ++j) v[j] = apply_act_fast(v[j], a.act);
  }
  const int64_t off = static_cast<int64_t>(prow) * h.ld + h.out_off + col0;
  if (a.residual != nullptr) {
    const __nv_bfloat16* res = a.residual + off;
    if (nvalid == 32 && a.vec_store) {
#pragma unroll
      for (int j = 0; j < 32; j += 8) {
        const uint4 q = *reinterpret_cast<const uint4*>(res + j);
        v[j + 0] += bf16_lo(q.x); v[j + 1] += bf16_hi(q.x);
        v[j + 2] += bf16_lo(q.y); v[j + 3] += bf16_hi(q.y);
        v[j + 4] += bf16_lo(q.z); v[j + 5] += bf16_hi(q.z);
        v[j + 6] += bf16_lo(q.w); v[j + 7] += bf16_hi(q.w);
      }
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j)
        if (j < nvalid) v[j] += bf16_to_f(res[j]);
    }
  }
  __nv_bfloat16* dst = ybase + off;
  if (nvalid == 32 && a.vec_store) {
#pragma unroll
    for (int j = 0; j < 32; j += 8) {
      uint4 q;
      q.x = pack_bf16x2(v[j + 0], v[j + 1]);
      q.y = pack_bf16x2(v[j + 2], v[j + 3]);
      q.z = pack_bf16x2(v[j + 4], v[j + 5]);
      q.w = pack_bf16x2(v[j + 6], v[j + 7]);
      *reinterpret_cast<uint4*>(dst + j) = q;
    }
  } else {
#pragma unroll
    for (int j = 0; j < 32; ++j)
      if (j < nvalid) dst[j] = __float2bfloat16_rn(v[j]);
  }
}

__device__ __forceinline__ float silu_fast(float v) { return __fdividef(v, 1.0f + __expf(-v)); }

// SwiGLU epilogue of 32 output columns of one row: silu(a) * b, stored bf16.
__device__ __forceinline__ void store_swiglu_chunk(const GemmArgs& a, const HalfInfo& h, int m,
                                                   int col0, const uint32_t (&ra)[32],
                                                   const uint32_t (&rb)[32]) {
  const int nvalid = min(32, h.valid - col0);
  float v[32];
#pragma unroll
  for (int j = 0; j < 32; ++j) v[j] = silu_fast(__uint_as_float(ra[j])) * __uint_as_float(rb[j]);
  __nv_bfloat16* dst = a.y + static_cast<int64_t>(m) * h.ld + h.out_off + col0;
  if (nvalid == 32 && a.vec_store) {
#pragma unroll
    for (int j = 0; j < 32; j += 8) {
      uint4 q;
      q.x = pack_bf16x2(v[j + 0], v[j + 1]);
      q.y = pack_bf16x2(v[j + 2], v[j + 3]);
      q.z = pack_bf16x2(v[j + 4], v[j + 5]);
      q.w = pack_bf16x2(v[j + 6], v[j + 7]);
      *reinterpret_cast<uint4*>(dst + j) = q;
    }
  } else {
#pragma unroll
    for (int j = 0; j < 32; ++j)
      if (j < nvalid) dst[j] = __float2bfloat16_rn(v[j]);
  }
}

// SwiGLU tile epilogue for one warp: TMEM columns 0..127 hold a = X wi0^T and
// 128..255 hold b = X wi1^T for the same 128 output columns; epilogue warp
// half hh writes output columns 64 hh .. 64 hh + 63.
__device__ __forceinline__ void swiglu_epilogue(const GemmArgs& a, int nt, int m, int hh,
                                                uint32_t tmem_row) {
  const HalfInfo h0 = decode_half(a, 2 * nt);
#pragma unroll
  for (int c = 0; c < 2; ++c) {
    const int col0 = hh * 64 + c * 32;
    if (col0 >= h0.valid) continue;
    uint32_t ra[32], rb[32];
    ptx::tmem_ld32(tmem_row + col0, ra);
    ptx::tmem_ld32(tmem_row + kHalfN + col0, rb);
    ptx::tmem_ld_wait();
    if (m < a.M) store_swiglu_chunk(a, h0, m, col0, ra, rb);
  }
}

__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_bf16_tcgen05(const __grid_constant__ GemmArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  float* bias_smem = reinterpret_cast<float*>(smem + kStages * kStageBytes);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kStages * kStageBytes + kBiasSmemBytes);
  uint64_t* empty = full + kStages;
  uint64_t* tfull = empty + kStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      ptx::mbar_init(&full[s], 1);
      ptx::mbar_init(&empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(&tfull[i], 1);
      ptx::mbar_init(&tempty[i], kEpiWarps);
    }
    ptx::mbar_init(drain, 1);
    *abort_flag = 0;
    ptx::fence_barrier_init();
    ptx::prefetch_tmap(&a.tmA);
    ptx::prefetch_tmap(&a.tmB);
    if (a.mode == kModeRow && a.r_split < a.r1) {
      ptx::prefetch_tmap(&a.tmA2);
      ptx::prefetch_tmap(&a.tmB2);
    }
  }
  if (warp == 1) {
    ptx::tmem_alloc(tmem_slot, 2 * kAccCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // the prologue above overlaps the previous kernel's tail; global memory after
  ptx::griddep_wait();
  ptx::griddep_launch_dependents();
  const TraceStamp trace = trace_begin();

  const int k_total = k_steps(a);

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < a.num_tiles; t += gridDim.x) {
        int mb, nt;
        tile_coords(a, t, mb, nt);
        const bool has1 = 2 * nt + 1 < a.n_halves;
        const HalfInfo h0 = decode_half(a, 2 * nt);
        const HalfInfo h1 = has1 ? decode_half(a, 2 * nt + 1) : h0;
        const uint32_t bytes = kABytes + (has1 ? 2 : 1) * kBHalfBytes;
        int arow;
        const CUtensorMap* mAcol = a_source(a, mb * kBM, arow);
        int rr = a.r0, kb = 0;  // row mode: rank and K block of the next step
        for (int ki = 0; ki < k_total; ++ki) {
          if (!ptx::mbar_wait(&empty[stage], phase ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          uint8_t* sA = smem + stage * kStageBytes;
          uint8_t* sB = sA + kABytes;
          ptx::mbar_arrive_expect_tx(&full[stage], bytes);
          if (a.mode != kModeRow) {
            const int kc = ki * kBK;
            ptx::tma_load_2d_nohint(sA, mAcol, &full[stage], kc, arow);
            ptx::tma_load_2d_nohint(sB, &a.tmB, &full[stage], kc, h0.brow);
            if (has1) ptx::tma_load_2d_nohint(sB + kBHalfBytes, &a.tmB, &full[stage], kc, h1.brow);
          } else {
            const bool g2 = rr >= a.r_split;  // second contraction width
            const CUtensorMap* mA = g2 ? &a.tmA2 : &a.tmA;
            const CUtensorMap* mB = g2 ? &a.tmB2 : &a.tmB;
            const int rc = g2 ? rr - a.r_split : rr;
            ptx::tma_load_3d_nohint(sA, mA, &full[stage], kb * kBK, mb * kBM, rc);
            ptx::tma_load_3d_nohint(sB, mB, &full[stage], kb * kBK, h0.brow, rc);
            if (has1)
              ptx::tma_load_3d_nohint(sB + kBHalfBytes, mB, &full[stage], kb * kBK, h1.brow, rc);
            if (++kb == (g2 ? a.k_iters2 : a.k_iters)) {
              kb = 0;
              ++rr;
            }
          }
          ++issued;
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {
        *abort_flag = 1;
        record_timeout();
        // Let the copies already in flight land before the CTA exits.
        const int back = issued < kStages ? issued : kStages;
        int s = stage;
        uint32_t ph = phase;
        volatile int no_abort = 0;
        for (int i = 0; i < back; ++i) {
          if (--s < 0) {
            s = kStages - 1;
            ph ^= 1u;
          }
          ptx::mbar_wait(&full[s], ph, &no_abort, 200000000ull);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // One thread issues every MMA: no warp-wide synchronisation per stage.
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      bool any_mma = false;
      int it = 0;
      for (int t = blockIdx.x; ok && t < a.num_tiles; t += gridDim.x, ++it) {
        int mb, nt;
        tile_coords(a, t, mb, nt);
        const bool has1 = 2 * nt + 1 < a.n_halves;
        const uint32_t idesc =
            has1 ? ptx::idesc_bf16(kBM, 2 * kHalfN) : ptx::idesc_bf16(kBM, kHalfN);
        const int acc = it & 1;
        const uint32_t acc_phase = (it >> 1) & 1;
        if (!ptx::mbar_wait(&tempty[acc], acc_phase ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * kAccCols;
        for (int ki = 0; ki < k_total; ++ki) {
          if (!ptx::mbar_wait(&full[stage], phase, abort_flag)) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          const uint32_t sA = ptx::smem_u32(smem + stage * kStageBytes);
          const uint64_t adesc = ptx::sdesc_kmajor_sw128(sA);
          const uint64_t bdesc = ptx::sdesc_kmajor_sw128(sA + kABytes);
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk)
            ptx::umma_bf16(d_tmem, adesc + 2 * kk, bdesc + 2 * kk, idesc, (ki | kk) != 0);
          ptx::umma_commit(&empty[stage]);
          any_mma = true;
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        ptx::umma_commit(&tfull[acc]);
      }
      if (!ok) {
        *abort_flag = 1;
        record_timeout();
        if (any_mma) {
          volatile int no_abort = 0;
          ptx::umma_commit(drain);
          ptx::mbar_wait(drain, 0, &no_abort, 200000000ull);
        }
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int ew = warp - 2;    // 0 .. kEpiWarps-1
    const int q = warp & 3;     // TMEM lane quarter this warp may access
    const int hh = ew >> 2;     // 128-column half of the accumulator it drains
    const int row = q * 32 + lane;
    float* bias_s = bias_smem + ew * kHalfN;
    int it = 0;
    if (a.norm) {
      const int per = (a.M + gridDim.x - 1) / gridDim.x;
      const int r0 = min(a.M, static_cast<int>(blockIdx.x) * per);
      norm_stats(a, r0, min(a.M, r0 + per), ew * 32 + lane);
    }
    for (int t = blockIdx.x; t < a.num_tiles; t += gridDim.x, ++it) {
      int mb, nt;
      tile_coords(a, t, mb, nt);
      const bool active = (hh == 0) || (2 * nt + 1 < a.n_halves);
      const int acc = it & 1;
      const uint32_t acc_phase = (it >> 1) & 1;
      HalfInfo h;
      if (active) {
        h = decode_half(a, 2 * nt + hh);
        if (a.bias != nullptr) {
          // This warp's 128 bias values, read once per tile while the MMAs run.
          for (int i = lane; i < kHalfN; i += 32)
            bias_s[i] = (i < h.valid) ? bf16_to_f(a.bias[h.bias_off + i]) : 0.0f;
          __syncwarp();
        }
      }
      int w_ok = 1;
      if (lane == 0) w_ok = ptx::mbar_wait(&tfull[acc], acc_phase, abort_flag);
      if (!__shfl_sync(0xffffffffu, w_ok, 0)) {
        if (lane == 0) {
          *abort_flag = 1;
          record_timeout();
        }
        break;
      }
      ptx::tc_fence_after();
      if (a.mode == kModeSwiglu) {
        swiglu_epilogue(a, nt, mb * kBM + row, hh,
                        tmem_base + ((q * 32u) << 16) + acc * kAccCols);
      } else if (active) {
        const int m = mb * kBM + row;
        int prow;
        __nv_bfloat16* const yb = out_base(a, m, prow);
        float rs = 1.0f;
        if (a.norm && !__all_sync(0xffffffffu, norm_row_scale(a, m, rs, abort_flag))) {
          if (lane == 0) {
            *abort_flag = 1;
            record_timeout();
          }
          break;
        }
        for (int c = 0; c < kHalfN / 32; ++c) {
          uint32_t r[32];
          ptx::tmem_ld32(tmem_base + ((q * 32u) << 16) + acc * kAccCols + hh * kHalfN + c * 32, r);
          ptx::tmem_ld_wait();
          if (m < a.M && c * 32 < h.valid) {
            float bv[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) bv[j] = bias_s[c * 32 + j];
            store_chunk(a, h, m, prow, yb, c * 32, r, bv, rs);
          }
        }
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&tempty[acc]);
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0) trace_end(trace, kTraceGemm, a.trace_seq);
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem_base, 2 * kAccCols);
  }
}

}  // namespace tpl
