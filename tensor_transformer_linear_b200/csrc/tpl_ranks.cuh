// tpl_ranks.cuh -- the TP linears split over GPUs, one process per GPU (the
// google-research row-parallel "{YZ unreduced}" partial and its reduction;
// nanotron "MLP Module": [batch, seq // tp, hidden] per rank after c_proj;
// Tenstorrent LMHead1D: every device's argmax candidates combined at the end).
//
//   tpl_column_linear_gather  this rank's shard of a column-parallel linear over
//       the all-gathered tokens: the GEMM's A tiles are TMA-loaded straight
//       from the rank that owns the tokens (peer memory), so the all-gather
//       overlaps the GEMM tile by tile.
//   tpl_row_linear_scatter  this rank's shard of the row-parallel linear.  The
//       GEMM epilogue writes each output row straight into the receive buffer
//       of the rank that owns the token (a peer pointer for every other rank),
//       so the exchange of partials overlaps the GEMM tile by tile.
//   tpl_reduce_slots        once every rank's scatter has completed, a rank sums
//       its tp slots (in rank order, fp32) plus bias and residual: its token
//       slice of the reduced output (the reduce-scatter).
//   tpl_reduce_slots_rmsnorm  the same sum, plus the RMSNorm of the result (the
//       next layer's normalised input) in the same pass over the row.
//   tpl_reduce_slots_allgather  the same sum, stored into every rank's full
//       [batch * seq][N] output at the rank's token rows (peer stores), so that
//       once every rank has run it, every rank holds the whole reduced output:
//       with the scatter before it, an all-reduce of the partials.
//   tpl_argmax_merge        the per-rank LM-head candidates, gathered, reduced to
//       the global argmax (ties to the lowest global id).
//
// Included at the end of tpl_api.cu (one translation unit with its helpers).
#pragma once

#include "common.cuh"

namespace tpl {

constexpr int kReduceThreads = 256;

// y[i] = bf16(sum_{s < tp} recv[s][i] + bias[i % N] + residual[i]) over the
// rows * N elements of one rank's slice; kVec: 8 elements per thread (N % 8 == 0,
// 16-byte aligned buffers).
template <bool kVec>
__global__ void __launch_bounds__(kReduceThreads)
    reduce_slots_kernel(const __nv_bfloat16* __restrict__ recv, int tp, int64_t total, int N,
                        const __nv_bfloat16* __restrict__ bias,
                        const __nv_bfloat16* __restrict__ residual, __nv_bfloat16* y) {
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x * (kVec ? 8 : 1);
  for (int64_t i = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) * (kVec ? 8 : 1);
       i < total; i += stride) {
    if (kVec) {
      float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      for (int s = 0; s < tp; ++s) {
        const uint4 q = __ldcs(reinterpret_cast<const uint4*>(recv + s * total + i));
        acc[0] += bf16_lo(q.x); acc[1] += bf16_hi(q.x);
        acc[2] += bf16_lo(q.y); acc[3] += bf16_hi(q.y);
        acc[4] += bf16_lo(q.z); acc[5] += bf16_hi(q.z);
        acc[6] += bf16_lo(q.w); acc[7] += bf16_hi(q.w);
      }
      if (bias != nullptr) {
        const uint4 q = __ldg(reinterpret_cast<const uint4*>(bias + i % N));
        acc[0] += bf16_lo(q.x); acc[1] += bf16_hi(q.x);
        acc[2] += bf16_lo(q.y); acc[3] += bf16_hi(q.y);
        acc[4] += bf16_lo(q.z); acc[5] += bf16_hi(q.z);
        acc[6] += bf16_lo(q.w); acc[7] += bf16_hi(q.w);
      }
      if (residual != nullptr) {
        const uint4 q = *reinterpret_cast<const uint4*>(residual + i);
        acc[0] += bf16_lo(q.x); acc[1] += bf16_hi(q.x);
        acc[2] += bf16_lo(q.y); acc[3] += bf16_hi(q.y);
        acc[4] += bf16_lo(q.z); acc[5] += bf16_hi(q.z);
        acc[6] += bf16_lo(q.w); acc[7] += bf16_hi(q.w);
      }
      uint4 o;
      o.x = pack_bf16x2(acc[0], acc[1]);
      o.y = pack_bf16x2(acc[2], acc[3]);
      o.z = pack_bf16x2(acc[4], acc[5]);
      o.w = pack_bf16x2(acc[6], acc[7]);
      *reinterpret_cast<uint4*>(y + i) = o;
    } else {
      float acc = 0.f;
      for (int s = 0; s < tp; ++s) acc += bf16_to_f(recv[s * total + i]);
      if (bias != nullptr) acc += bf16_to_f(bias[i % N]);
      if (residual != nullptr) acc += bf16_to_f(residual[i]);
      y[i] = __float2bfloat16_rn(acc);
    }
  }
}

// reduce_slots_kernel for one row, then the RMSNorm of the rounded result: one
// CTA per row, of up to kRowThreads threads, thread t owning the row's 16-byte
// vectors t, t + blockDim, ... (VPT of them at most) in registers between the
// two halves.  A thread loads all of a vector's slots (up to kSlots at a time)
// before adding any, in rank order, so a row's loads are in flight together:
// with a few rows per SM, the kernel would otherwise wait on one load round
// trip per slot.  y may alias residual; xn aliases nothing.
constexpr int kRowThreads = 256;

template <int VPT>
__global__ void __launch_bounds__(kRowThreads, VPT <= 2 ? 4 : (VPT <= 4 ? 2 : 1))
    reduce_slots_rmsnorm_kernel(const __nv_bfloat16* __restrict__ recv, int tp, int64_t rows,
                                int N, const __nv_bfloat16* __restrict__ bias,
                                const __nv_bfloat16* residual, __nv_bfloat16* y,
                                const float* __restrict__ scale, int centered, float eps,
                                __nv_bfloat16* __restrict__ xn) {
  __shared__ float part[kRowThreads / 32];
  constexpr int kSlots = 8;
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  const int nthr = blockDim.x;
  const int nvec = N / 8;
  const int64_t total = rows * N;
  const float inv_n = 1.0f / static_cast<float>(N);
  for (int64_t row = blockIdx.x; row < rows; row += gridDim.x) {
    uint4 q[VPT];
    float ss = 0.f;
    const int64_t base = row * N;
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
      const int v = tid + nthr * i;
      if (v < nvec) {
        const int64_t e = base + static_cast<int64_t>(v) * 8;
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        for (int s0 = 0; s0 < tp; s0 += kSlots) {
          uint4 r[kSlots];
#pragma unroll
          for (int j = 0; j < kSlots; ++j)
            if (s0 + j < tp)
              r[j] = __ldcs(reinterpret_cast<const uint4*>(recv + (s0 + j) * total + e));
#pragma unroll
          for (int j = 0; j < kSlots; ++j) {   // added in rank order
            if (s0 + j < tp) {
              acc[0] += bf16_lo(r[j].x); acc[1] += bf16_hi(r[j].x);
              acc[2] += bf16_lo(r[j].y); acc[3] += bf16_hi(r[j].y);
              acc[4] += bf16_lo(r[j].z); acc[5] += bf16_hi(r[j].z);
              acc[6] += bf16_lo(r[j].w); acc[7] += bf16_hi(r[j].w);
            }
          }
        }
        if (bias != nullptr) {
          const uint4 r = __ldg(reinterpret_cast<const uint4*>(bias + v * 8));
          acc[0] += bf16_lo(r.x); acc[1] += bf16_hi(r.x);
          acc[2] += bf16_lo(r.y); acc[3] += bf16_hi(r.y);
          acc[4] += bf16_lo(r.z); acc[5] += bf16_hi(r.z);
          acc[6] += bf16_lo(r.w); acc[7] += bf16_hi(r.w);
        }
        if (residual != nullptr) {
          const uint4 r = *reinterpret_cast<const uint4*>(residual + e);
          acc[0] += bf16_lo(r.x); acc[1] += bf16_hi(r.x);
          acc[2] += bf16_lo(r.y); acc[3] += bf16_hi(r.y);
          acc[4] += bf16_lo(r.z); acc[5] += bf16_hi(r.z);
          acc[6] += bf16_lo(r.w); acc[7] += bf16_hi(r.w);
        }
        q[i].x = pack_bf16x2(acc[0], acc[1]);
        q[i].y = pack_bf16x2(acc[2], acc[3]);
        q[i].z = pack_bf16x2(acc[4], acc[5]);
        q[i].w = pack_bf16x2(acc[6], acc[7]);
        *reinterpret_cast<uint4*>(y + e) = q[i];
        float f[8];
        VecTraits<__nv_bfloat16>::unpack(q[i], f);
#pragma unroll
        for (int k = 0; k < 8; ++k) ss = fmaf(f[k], f[k], ss);
      }
    }
    ss = warp_sum(ss);
    if (lane == 0) part[w] = ss;
    __syncthreads();
    float tot = 0.f;
    for (int i = 0; i < (nthr >> 5); ++i) tot += part[i];
    __syncthreads();  // part[] is rewritten by the next row
    const float rinv = rsqrtf(tot * inv_n + eps);
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
      const int v = tid + nthr * i;
      if (v < nvec) {
        float f[8];
        VecTraits<__nv_bfloat16>::unpack(q[i], f);
        if (scale != nullptr) {
          const float4* s4 = reinterpret_cast<const float4*>(scale + v * 8);
#pragma unroll
          for (int e4 = 0; e4 < 2; ++e4) {
            float4 sc = __ldg(s4 + e4);
            if (centered) {
              sc.x += 1.f; sc.y += 1.f; sc.z += 1.f; sc.w += 1.f;
            }
            f[4 * e4 + 0] = f[4 * e4 + 0] * rinv * sc.x;
            f[4 * e4 + 1] = f[4 * e4 + 1] * rinv * sc.y;
            f[4 * e4 + 2] = f[4 * e4 + 2] * rinv * sc.z;
            f[4 * e4 + 3] = f[4 * e4 + 3] * rinv * sc.w;
          }
        } else {
#pragma unroll
          for (int k = 0; k < 8; ++k) f[k] *= rinv;
        }
        __stcs(reinterpret_cast<uint4*>(xn + row * N) + v,
               VecTraits<__nv_bfloat16>::pack(f));
      }
    }
  }
}

struct PeerOut {
  __nv_bfloat16* y[kMaxPeers];
};

// The slice sum of reduce_slots_kernel, stored into every rank's full output:
// slice element i (row i / N = b * seg + t, column i % N) goes to full row
// b * seq + rank * seg + t of out.y[0 .. tp).  residual, if given, is the
// rank's own full [batch * seq][N] residual stream, read at that full row, and
// may alias out.y[rank].  kVec as in reduce_slots_kernel.
template <bool kVec>
__global__ void __launch_bounds__(kReduceThreads)
    reduce_slots_allgather_kernel(const __nv_bfloat16* __restrict__ recv, int tp, int64_t total,
                                  int N, int seg, int seq, int rank,
                                  const __nv_bfloat16* __restrict__ bias,
                                  const __nv_bfloat16* residual, const PeerOut out) {
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x * (kVec ? 8 : 1);
  for (int64_t i = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) * (kVec ? 8 : 1);
       i < total; i += stride) {
    const int64_t row = i / N;
    const int64_t col = i - row * N;
    const int64_t b = row / seg;
    const int64_t dst = (b * seq + static_cast<int64_t>(rank) * seg + (row - b * seg)) * N + col;
    if (kVec) {
      float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      for (int s = 0; s < tp; ++s) {
        const uint4 q = __ldcs(reinterpret_cast<const uint4*>(recv + s * total + i));
        acc[0] += bf16_lo(q.x); acc[1] += bf16_hi(q.x);
        acc[2] += bf16_lo(q.y); acc[3] += bf16_hi(q.y);
        acc[4] += bf16_lo(q.z); acc[5] += bf16_hi(q.z);
        acc[6] += bf16_lo(q.w); acc[7] += bf16_hi(q.w);
      }
      if (bias != nullptr) {
        const uint4 q = __ldg(reinterpret_cast<const uint4*>(bias + col));
        acc[0] += bf16_lo(q.x); acc[1] += bf16_hi(q.x);
        acc[2] += bf16_lo(q.y); acc[3] += bf16_hi(q.y);
        acc[4] += bf16_lo(q.z); acc[5] += bf16_hi(q.z);
        acc[6] += bf16_lo(q.w); acc[7] += bf16_hi(q.w);
      }
      if (residual != nullptr) {
        const uint4 q = *reinterpret_cast<const uint4*>(residual + dst);
        acc[0] += bf16_lo(q.x); acc[1] += bf16_hi(q.x);
        acc[2] += bf16_lo(q.y); acc[3] += bf16_hi(q.y);
        acc[4] += bf16_lo(q.z); acc[5] += bf16_hi(q.z);
        acc[6] += bf16_lo(q.w); acc[7] += bf16_hi(q.w);
      }
      uint4 o;
      o.x = pack_bf16x2(acc[0], acc[1]);
      o.y = pack_bf16x2(acc[2], acc[3]);
      o.z = pack_bf16x2(acc[4], acc[5]);
      o.w = pack_bf16x2(acc[6], acc[7]);
      for (int q = 0; q < tp; ++q) *reinterpret_cast<uint4*>(out.y[q] + dst) = o;
    } else {
      float acc = 0.f;
      for (int s = 0; s < tp; ++s) acc += bf16_to_f(recv[s * total + i]);
      if (bias != nullptr) acc += bf16_to_f(bias[col]);
      if (residual != nullptr) acc += bf16_to_f(residual[dst]);
      const __nv_bfloat16 o = __float2bfloat16_rn(acc);
      for (int q = 0; q < tp; ++q) out.y[q][dst] = o;
    }
  }
}

// ids[b] = the global id of the best candidate over ranks: rank s's candidate
// for row b is (shard_max[s][b], s * id_stride + shard_idx[s][b]); a negative
// shard_idx is "no candidate".  Larger logit wins, then the lower global id.
__global__ void argmax_merge_kernel(const float* shard_max, const int32_t* shard_idx, int tp,
                                    int B, int64_t id_stride, int32_t* ids) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= B) return;
  float best = 0.f;
  int64_t best_id = -1;
  for (int s = 0; s < tp; ++s) {
    const int32_t local = shard_idx[static_cast<int64_t>(s) * B + b];
    if (local < 0) continue;
    const float v = shard_max[static_cast<int64_t>(s) * B + b];
    const int64_t gid = s * id_stride + local;
    if (best_id < 0 || v > best || (v == best && gid < best_id)) {
      best = v;
      best_id = gid;
    }
  }
  ids[b] = static_cast<int32_t>(best_id);
}

}  // namespace tpl

namespace {

tpl_status column_gather(const tpl_partition* p, void* const* peer_x, int32_t tp, int64_t batch,
                         int64_t seq, int64_t K, const void* w, const void* bias, tpl_act act,
                         void* y, void* stream) {
  if (p == nullptr || peer_x == nullptr) return TPL_ERR_NULL;
  if (!act_ok(act)) return TPL_ERR_DTYPE;
  tpl_status s = check_partition(p);
  if (s != TPL_OK) return s;
  if (tp > TPL_MAX_GATHER) return TPL_ERR_UNSUPPORTED;
  SeqPar sp;
  if ((s = seqpar_of(batch, seq, tp, &sp)) != TPL_OK) return s;
  if (K < 1 || K > INT32_MAX) return TPL_ERR_SHAPE;
  // A tiles are 128-row TMA boxes that must each come from one rank's slice.
  if (sp.seg % tpl::kBM != 0) return TPL_ERR_UNSUPPORTED;
  if (w == nullptr || y == nullptr) return TPL_ERR_NULL;
  for (int q = 0; q < tp; ++q)
    if (peer_x[q] == nullptr) return TPL_ERR_NULL;
  GatherA ga;
  ga.tp = tp;
  ga.gather = peer_x;
  return column_bf16(p, peer_x[0], batch * seq, K, w, bias, act, y,
                     static_cast<cudaStream_t>(stream), sp, &ga);
}

tpl_status row_scatter(const void* h, int64_t K, int64_t batch, int64_t seq, int64_t N,
                       const void* w, int32_t rank, int32_t tp, void* const* peer,
                       void* stream) {
  if (peer == nullptr) return TPL_ERR_NULL;
  SeqPar sp;
  tpl_status s = seqpar_of(batch, seq, tp, &sp);
  if (s != TPL_OK) return s;
  if (rank < 0 || rank >= tp || K < 1 || K > INT32_MAX || N < 1 || N > INT32_MAX)
    return TPL_ERR_SHAPE;
  if (h == nullptr || w == nullptr) return TPL_ERR_NULL;
  for (int q = 0; q < tp; ++q) {
    if (peer[q] == nullptr) return TPL_ERR_NULL;
    if (!aligned(peer[q], 2)) return TPL_ERR_ALIGN;
  }
  PeerScatter ps;
  ps.src_rank = rank;
  ps.tp = tp;
  ps.peer = peer;
  const int64_t kw[1] = {K};
  return row_bf16(h, kw, 1, batch * seq, N, w, nullptr, nullptr, nullptr, nullptr,
                  static_cast<cudaStream_t>(stream), sp, &ps);
}

}  // namespace

extern "C" {

tpl_status tpl_column_linear_gather(const tpl_partition* p, void* const* peer_x, int32_t tp,
                                    int64_t batch, int64_t seq, int64_t K, const void* w,
                                    const void* bias, tpl_act act, void* y, void* stream) {
  return column_gather(p, peer_x, tp, batch, seq, K, w, bias, act, y, stream);
}

tpl_status tpl_row_linear_scatter(const void* h, int64_t K, int64_t batch, int64_t seq, int64_t N,
                                  const void* w, int32_t rank, int32_t tp, void* const* peer,
                                  void* stream) {
  return row_scatter(h, K, batch, seq, N, w, rank, tp, peer, stream);
}


tpl_status tpl_reduce_slots(const void* recv, int32_t tp, int64_t rows, int64_t N,
                            const void* bias, const void* residual, void* y, void* stream) {
  if (tp < 1 || tp > TPL_MAX_TP || rows < 0 || N < 1 || N > INT32_MAX) return TPL_ERR_SHAPE;
  // every element index of recv, tp * rows * N, must fit an int64_t
  if (rows > INT64_MAX / (N * tp)) return TPL_ERR_SHAPE;
  if (rows == 0) return TPL_OK;
  if (recv == nullptr || y == nullptr) return TPL_ERR_NULL;
  if (!aligned(recv, 2) || !aligned(y, 2) || (bias && !aligned(bias, 2)) ||
      (residual && !aligned(residual, 2)))
    return TPL_ERR_ALIGN;
  DeviceInfo* dev = nullptr;
  tpl_status s = device_info(&dev);
  if (s != TPL_OK) return s;
  const int64_t total = rows * N;
  const bool vec = (N % 8 == 0) && aligned(recv, 16) && aligned(y, 16) &&
                   (bias == nullptr || aligned(bias, 16)) &&
                   (residual == nullptr || aligned(residual, 16));
  const int64_t per_block = static_cast<int64_t>(tpl::kReduceThreads) * (vec ? 8 : 1);
  const int grid = static_cast<int>(std::min<int64_t>((total + per_block - 1) / per_block,
                                                      static_cast<int64_t>(dev->sm_count) * 8));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const auto* rv = static_cast<const __nv_bfloat16*>(recv);
  const auto* bv = static_cast<const __nv_bfloat16*>(bias);
  const auto* res = static_cast<const __nv_bfloat16*>(residual);
  auto* yv = static_cast<__nv_bfloat16*>(y);
  const int Ni = static_cast<int>(N);
  if (vec)
    tpl::reduce_slots_kernel<true><<<grid, tpl::kReduceThreads, 0, st>>>(rv, tp, total, Ni, bv, res, yv);
  else
    tpl::reduce_slots_kernel<false><<<grid, tpl::kReduceThreads, 0, st>>>(rv, tp, total, Ni, bv, res, yv);
  return launched();
}

tpl_status tpl_reduce_slots_rmsnorm(const void* recv, int32_t tp, int64_t rows, int64_t N,
                                    const void* bias, const void* residual, void* y,
                                    const float* scale, int32_t centered, float eps, void* xn,
                                    void* stream) {
  if (tp < 1 || tp > TPL_MAX_TP || rows < 0 || N < 1 || N > INT32_MAX || !(eps >= 0.0f))
    return TPL_ERR_SHAPE;
  if (rows > INT64_MAX / (N * tp)) return TPL_ERR_SHAPE;
  if (rows == 0) return TPL_OK;
  if (recv == nullptr || y == nullptr || xn == nullptr) return TPL_ERR_NULL;
  if (N % 8 != 0 || !aligned(recv, 16) || !aligned(y, 16) || !aligned(xn, 16) ||
      (bias && !aligned(bias, 16)) || (residual && !aligned(residual, 16)) ||
      (scale && !aligned(scale, 16)))
    return TPL_ERR_ALIGN;
  const int64_t nvec = N / 8;
  const int64_t vpt = (nvec + tpl::kRowThreads - 1) / tpl::kRowThreads;
  if (vpt > 8) return TPL_ERR_UNSUPPORTED;  // N > 16384: more than the registers hold
  // threads per row: one vector per thread up to N = 2048, then up to 8 each
  const int tc = static_cast<int>(std::min<int64_t>(tpl::kRowThreads, (nvec + 31) / 32 * 32));
  const int grid = static_cast<int>(std::min<int64_t>(rows, INT32_MAX));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const auto* rv = static_cast<const __nv_bfloat16*>(recv);
  const auto* bv = static_cast<const __nv_bfloat16*>(bias);
  const auto* res = static_cast<const __nv_bfloat16*>(residual);
  auto* yv = static_cast<__nv_bfloat16*>(y);
  auto* xv = static_cast<__nv_bfloat16*>(xn);
  const int Ni = static_cast<int>(N);
  if (vpt <= 1)
    tpl::reduce_slots_rmsnorm_kernel<1><<<grid, tc, 0, st>>>(rv, tp, rows, Ni, bv, res, yv, scale,
                                                             centered, eps, xv);
  else if (vpt <= 2)
    tpl::reduce_slots_rmsnorm_kernel<2><<<grid, tc, 0, st>>>(rv, tp, rows, Ni, bv, res, yv, scale,
                                                             centered, eps, xv);
  else if (vpt <= 4)
    tpl::reduce_slots_rmsnorm_kernel<4><<<grid, tc, 0, st>>>(rv, tp, rows, Ni, bv, res, yv, scale,
                                                             centered, eps, xv);
  else
    tpl::reduce_slots_rmsnorm_kernel<8><<<grid, tc, 0, st>>>(rv, tp, rows, Ni, bv, res, yv, scale,
                                                             centered, eps, xv);
  return launched();
}

tpl_status tpl_reduce_slots_allgather(const void* recv, int32_t tp, int64_t batch, int64_t seq,
                                      int64_t N, const void* bias, const void* residual,
                                      int32_t rank, void* const* peer_y, void* stream) {
  SeqPar sp;
  tpl_status s = seqpar_of(batch, seq, tp, &sp);
  if (s != TPL_OK) return s;
  if (rank < 0 || rank >= tp || N < 1 || N > INT32_MAX) return TPL_ERR_SHAPE;
  // every element index of the full output, batch * seq * N, must fit an int64_t
  if (static_cast<int64_t>(sp.batch) * sp.seq > INT64_MAX / N) return TPL_ERR_SHAPE;
  if (recv == nullptr || peer_y == nullptr) return TPL_ERR_NULL;
  bool vec = (N % 8 == 0) && aligned(recv, 16) && (bias == nullptr || aligned(bias, 16)) &&
             (residual == nullptr || aligned(residual, 16));
  tpl::PeerOut out{};
  for (int q = 0; q < tp; ++q) {
    if (peer_y[q] == nullptr) return TPL_ERR_NULL;
    if (!aligned(peer_y[q], 2)) return TPL_ERR_ALIGN;
    vec = vec && aligned(peer_y[q], 16);
    out.y[q] = static_cast<__nv_bfloat16*>(peer_y[q]);
  }
  if (!aligned(recv, 2) || (bias && !aligned(bias, 2)) || (residual && !aligned(residual, 2)))
    return TPL_ERR_ALIGN;
  DeviceInfo* dev = nullptr;
  if ((s = device_info(&dev)) != TPL_OK) return s;
  const int64_t total = static_cast<int64_t>(sp.batch) * sp.seg * N;  // this rank's slice
  const int64_t per_block = static_cast<int64_t>(tpl::kReduceThreads) * (vec ? 8 : 1);
  const int grid = static_cast<int>(std::min<int64_t>((total + per_block - 1) / per_block,
                                                      static_cast<int64_t>(dev->sm_count) * 8));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const auto* rv = static_cast<const __nv_bfloat16*>(recv);
  const auto* bv = static_cast<const __nv_bfloat16*>(bias);
  const auto* res = static_cast<const __nv_bfloat16*>(residual);
  const int Ni = static_cast<int>(N);
  if (vec)
    tpl::reduce_slots_allgather_kernel<true><<<grid, tpl::kReduceThreads, 0, st>>>(
        rv, tp, total, Ni, sp.seg, sp.seq, rank, bv, res, out);
  else
    tpl::reduce_slots_allgather_kernel<false><<<grid, tpl::kReduceThreads, 0, st>>>(
        rv, tp, total, Ni, sp.seg, sp.seq, rank, bv, res, out);
  return launched();
}

tpl_status tpl_argmax_merge(const float* shard_max, const int32_t* shard_idx, int32_t tp,
                            int64_t B, int64_t id_stride, int32_t* ids, void* stream) {
  if (tp < 1 || tp > TPL_MAX_TP || B < 1 || B > INT32_MAX || id_stride < 1 ||
      id_stride * tp > INT32_MAX)
    return TPL_ERR_SHAPE;
  if (shard_max == nullptr || shard_idx == nullptr || ids == nullptr) return TPL_ERR_NULL;
  if (!aligned(shard_max, 4) || !aligned(shard_idx, 4) || !aligned(ids, 4)) return TPL_ERR_ALIGN;
  const int Bi = static_cast<int>(B);
  tpl::argmax_merge_kernel<<<(Bi + 127) / 128, 128, 0, static_cast<cudaStream_t>(stream)>>>(
      shard_max, shard_idx, tp, Bi, id_stride, ids);
  return launched();
}

}  // extern "C"
