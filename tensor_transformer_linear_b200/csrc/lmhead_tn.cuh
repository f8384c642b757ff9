// lmhead_tn.cuh -- the decode LM head of lmhead.cuh with the operands the
// other way round, for batches of up to 32 rows (Tenstorrent LMHead1D;
// google-research unembed_manual computes the logits in fp32).
//
// In lmhead_argmax_tcgen05 a slab of W is the M = 128 operand and the batch
// the N operand, so every tcgen05.mma covers 128 vocab rows x 16 K.  An MMA
// costs about the same number of SM cycles whatever its N, so at B = 32 that
// kernel needs about 260k SM cycles per launch: HBM-bound only while the SM
// clock stays above about 1.6 GHz.  Here the batch is the M operand and a
// slab of up to 256 vocab rows is the N operand, so one MMA covers up to 256
// vocab rows x 16 K.  By default each CTA owns one contiguous vocab range
// (V / grid rows, +1 for the first V % grid CTAs) cut into 256-row slabs and
// one shorter last slab: for V = 128256 on 148 SMs, 4 x 256 MMAs per CTA,
// against 7 x 256 for swap-AB and 5 x 256 for uniform 176-row slabs dealt out
// in turn (LmArgs::ranged = 0, which the kernel also runs).
//
// kM is the height of the A operand: 128, or 64 (half the A bytes the tensor
// core reads from shared memory per MMA, and more stages in the same space).
// Stage s of the TMA ring holds the A operand [kM][64] (the batch tile in rows
// 0..31, rows past B zero-filled by the copy, rows 32..kM-1 zeroed once at the
// start, so the MMA's unused rows multiply zeros), then the W tile
// [slab_rows][64] (a short last slab fills its first rows; the MMA's columns
// past the slab's rows are never read).  D is [kM rows][N] fp32 in TMEM, two
// buffers of 256 columns.  For
// kM = 128, D row i is TMEM lane i; for kM = 64, rows 0-15 are lanes 0-15 and
// rows 16-31 lanes 32-47 (16 lanes of each 32-lane quarter).  The epilogue
// warps (warp q reads lane quarter q) walk each finished slab's columns in
// ascending vocab id, keep the best (logit, id) of the current shard per batch
// row and fold it into the workspace with atomicMax when the shard changes and
// at the slab's end.  The last CTA finalises as in lmhead.cuh.
//
// Warps: 0 .. E-1 epilogue (E = 1 for kM = 128, 2 for kM = 64), E TMA
// producer, E + 1 MMA issuer (and TMEM owner).
#pragma once

#include "common.cuh"
#include "lmhead.cuh"
#include "ptx.cuh"
#include "trace.cuh"

namespace tpl {

constexpr int kLmTnXBytes = 32 * kLmBK * 2;  // the batch tile a stage loads (4 KB)
constexpr int kLmTnAccCols = 256;            // TMEM columns per accumulator buffer

template <int kM>
struct LmTn {
  static constexpr int kEpi = kM == 128 ? 1 : 2;           // epilogue warps
  static constexpr int kLaneRows = kM == 128 ? 32 : 16;    // batch rows per epilogue warp
  static constexpr int kThreads = 32 * (kEpi + 2);
  static constexpr int kABytes = kM * kLmBK * 2;           // A operand of a stage
};

// Slab s of this CTA: its first vocab row and its rows; false past the last.
// Uniform slabs (ranged = 0) are dealt out in turn; with ranged = 1 the CTA
// walks its own contiguous range (LmArgs).
__device__ __forceinline__ bool lm_tn_slab(const LmArgs& a, int s, int& row0, int& rows) {
  if (!a.ranged) {
    const int g = static_cast<int>(blockIdx.x) + s * static_cast<int>(gridDim.x);
    if (g >= a.n_slabs) return false;
    row0 = g * a.slab_rows;
    rows = min(a.slab_rows, a.V - row0);
    return true;
  }
  const int c = static_cast<int>(blockIdx.x);
  const int r0 = c * a.range_base + min(c, a.range_rem);
  const int r1 = r0 + a.range_base + (c < a.range_rem ? 1 : 0);
  row0 = r0 + s * a.slab_rows;
  if (row0 >= r1) return false;
  rows = min(a.slab_rows, r1 - row0);
  return true;
}

// A ranged CTA's short last slab goes through tmWt and an MMA of N = tail_n.
__device__ __forceinline__ bool lm_tn_is_tail(const LmArgs& a, int rows) {
  return a.ranged && rows < a.slab_rows;
}

__device__ __forceinline__ void lm_tn_flush(const LmArgs& a, int b, int shard, float v, int id) {
  if (id >= 0) atomicMax(&a.keys[shard * a.B + b], make_key(v, id));
}

template <int kM>
__global__ void __launch_bounds__(LmTn<kM>::kThreads, 1)
    lmhead_argmax_tn(const __grid_constant__ LmArgs a) {
  using C = LmTn<kM>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + a.stages * a.stage_bytes);
  uint64_t* empty = full + kLmMaxStages;
  uint64_t* tfull = empty + kLmMaxStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* last_flag = abort_flag + 1;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int S = a.stages;
  constexpr int kProd = C::kEpi, kMma = C::kEpi + 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      ptx::mbar_init(&full[s], 1);
      ptx::mbar_init(&empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(&tfull[i], 1);
      ptx::mbar_init(&tempty[i], C::kEpi);
    }
    ptx::mbar_init(drain, 1);
    *abort_flag = 0;
    *last_flag = 0;
    ptx::fence_barrier_init();
    ptx::prefetch_tmap(&a.tmW);
    ptx::prefetch_tmap(&a.tmX);
  }
  if (warp == kMma) {
    ptx::tmem_alloc(tmem_slot, a.tmem_cols);
    ptx::tmem_relinquish();
  }
  // rows 32..kM-1 of every stage's A operand: zero, never written again
  for (int s = 0; s < S; ++s) {
    uint4* z = reinterpret_cast<uint4*>(smem + s * a.stage_bytes + kLmTnXBytes);
    for (int i = threadIdx.x; i < (C::kABytes - kLmTnXBytes) / 16; i += C::kThreads)
      z[i] = make_uint4(0u, 0u, 0u, 0u);
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // visible to the tensor core
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // the prologue above overlaps the previous kernel's tail; global memory after
  ptx::griddep_wait();
  ptx::griddep_launch_dependents();
  const TraceStamp trace = trace_begin();

  if (warp == kProd) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      const uint64_t pol_w = ptx::policy_evict_first();
      const uint64_t pol_x = ptx::policy_evict_last();
      int stage = 0, issued = 0;
      uint32_t phase = 0;
      bool ok = true;
      int row0, rows;
      for (int s = 0; ok && lm_tn_slab(a, s, row0, rows); ++s) {
        const bool tail = lm_tn_is_tail(a, rows);
        const CUtensorMap* mw = tail ? &a.tmWt : &a.tmW;
        const uint32_t bytes = static_cast<uint32_t>(
            kLmTnXBytes + (tail ? a.tail_rows : a.slab_rows) * kLmBK * 2);
        for (int kb = 0; kb < a.k_iters; ++kb) {
          if (!ptx::mbar_wait(&empty[stage], phase ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          uint8_t* st = smem + stage * a.stage_bytes;
          ptx::mbar_arrive_expect_tx(&full[stage], bytes);
          ptx::tma_load_2d(st, &a.tmX, &full[stage], kb * kLmBK, 0, pol_x);
          ptx::tma_load_2d(st + C::kABytes, mw, &full[stage], kb * kLmBK, row0, pol_w);
          ++issued;
          if (++stage == S) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {
        *abort_flag = 1;
        record_timeout();
        // wait (bounded) for the copies still in flight before the CTA exits
        const int back = issued < S ? issued : S;
        int s = stage;
        uint32_t ph = phase;
        volatile int no_abort = 0;
        for (int i = 0; i < back; ++i) {
          if (--s < 0) {
            s = S - 1;
            ph ^= 1u;
          }
          ptx::mbar_wait(&full[s], ph, &no_abort, 200000000ull);
        }
      }
    }
  } else if (warp == kMma) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc_slab = ptx::idesc_bf16(kM, a.slab_rows);
      const uint32_t idesc_tail = ptx::idesc_bf16(kM, a.ranged ? a.tail_n : a.slab_rows);
      int stage = 0, it = 0;
      uint32_t phase = 0;
      bool ok = true, any_mma = false;
      int row0, rows;
      for (int s = 0; ok && lm_tn_slab(a, s, row0, rows); ++s, ++it) {
        const uint32_t idesc = lm_tn_is_tail(a, rows) ? idesc_tail : idesc_slab;
        const int acc = it & 1;
        const uint32_t acc_phase = (it >> 1) & 1;
        if (!ptx::mbar_wait(&tempty[acc], acc_phase ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * kLmTnAccCols;
        for (int kb = 0; kb < a.k_iters; ++kb) {
          if (!ptx::mbar_wait(&full[stage], phase, abort_flag)) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          const uint32_t st = ptx::smem_u32(smem + stage * a.stage_bytes);
          const uint64_t adesc = ptx::sdesc_kmajor_sw128(st);                // batch rows
          const uint64_t bdesc = ptx::sdesc_kmajor_sw128(st + C::kABytes);  // vocab rows
#pragma unroll
          for (int kk = 0; kk < kLmBK / 16; ++kk)
            ptx::umma_bf16(d_tmem, adesc + 2 * kk, bdesc + 2 * kk, idesc, (kb | kk) != 0);
          ptx::umma_commit(&empty[stage]);
          any_mma = true;
          if (++stage == S) {
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
    // warp q reads TMEM lane quarter q; its lane l holds batch row
    // q * kLaneRows + l for l < kLaneRows
    const int b = warp * C::kLaneRows + lane;
    const bool row_ok = lane < C::kLaneRows && b < a.B;
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    int it = 0;
    bool ok = true;
    int row0, rows;
    for (int s = 0; lm_tn_slab(a, s, row0, rows); ++s, ++it) {
      const int acc = it & 1;
      const uint32_t acc_phase = (it >> 1) & 1;
      int w_ok = 1;
      if (lane == 0) w_ok = ptx::mbar_wait(&tfull[acc], acc_phase, abort_flag);
      if (!__shfl_sync(0xffffffffu, w_ok, 0)) {
        if (lane == 0) {
          *abort_flag = 1;
          record_timeout();
        }
        ok = false;
        break;
      }
      ptx::tc_fence_after();
      const int slab0 = row0;
      const int row_end = row0 + rows;  // ids at or past it are not this slab's
      int cur = slab0 / a.shard;        // shard of the running best
      int next = (cur + 1) * a.shard;   // first id of the next shard
      float best = 0.f;
      int best_id = -1;
      for (int c = 0; c < rows; c += 16) {
        uint32_t r[16];
        tmem_ld16(tmem_base + lane_base + static_cast<uint32_t>(acc * kLmTnAccCols + c), r);
        ptx::tmem_ld_wait();
        if (!row_ok) continue;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int v = slab0 + c + j;
          if (v >= row_end) break;
          const float f = __uint_as_float(r[j]);
          if (a.logits != nullptr) a.logits[static_cast<int64_t>(b) * a.V + v] = f;
          if (v >= next) {  // ascending ids: the previous shard is complete in this slab
            lm_tn_flush(a, b, cur, best, best_id);
            cur = v / a.shard;
            next = (cur + 1) * a.shard;
            best_id = -1;
          }
          if (best_id < 0 || f > best) {  // ties keep the lower id
            best = f;
            best_id = v;
          }
        }
      }
      if (row_ok) lm_tn_flush(a, b, cur, best, best_id);
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&tempty[acc]);
    }

    // ------------------------------------------------ completion: last CTA
    __threadfence();
    asm volatile("bar.sync 1, %0;" ::"n"(32 * C::kEpi) : "memory");
    if (threadIdx.x == 0) *last_flag = (atomicAdd(a.counter, 1u) == gridDim.x - 1) ? 1 : 0;
    asm volatile("bar.sync 1, %0;" ::"n"(32 * C::kEpi) : "memory");
    if (*last_flag && ok && !*abort_flag) {
      __threadfence();
      for (int bb = threadIdx.x; bb < a.B; bb += 32 * C::kEpi) {
        unsigned long long best_key = 0ull;
        for (int s = 0; s < a.tp; ++s) {
          unsigned long long* kp = &a.keys[s * a.B + bb];
          const unsigned long long k = __ldcg(kp);
          if (k == 0ull) {
            a.shard_max[s * a.B + bb] = -__int_as_float(0x7f800000);
            a.shard_idx[s * a.B + bb] = -1;
          } else {
            a.shard_max[s * a.B + bb] = key_float(static_cast<uint32_t>(k >> 32));
            a.shard_idx[s * a.B + bb] =
                static_cast<int32_t>(0xFFFFFFFFu - static_cast<uint32_t>(k & 0xFFFFFFFFull));
          }
          best_key = k > best_key ? k : best_key;
          *kp = 0ull;
        }
        a.ids[bb] = best_key == 0ull
                        ? -1
                        : static_cast<int32_t>(0xFFFFFFFFu -
                                               static_cast<uint32_t>(best_key & 0xFFFFFFFFull));
      }
      if (threadIdx.x == 0) *a.counter = 0u;
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0) trace_end(trace, kTraceLmHead, a.trace_seq);
  if (warp == kMma) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem_base, a.tmem_cols);
  }
}

}  // namespace tpl
