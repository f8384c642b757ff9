// lmhead.cuh -- decode LM head over a vocab-sharded weight with the per-shard
// and the global argmax fused in (Tenstorrent LMHead1D; google-research
// unembed_manual computes the logits in fp32).
//
// The weight is read exactly once, so the kernel is an HBM stream.  Its
// arithmetic (2 * B * K FLOP per weight row, 32 FLOP per byte at B = 32) is
// still too much for the CUDA cores at HBM speed, so the dot products run on
// the tensor cores with the operands swapped: A = a 128-row vocab slab of W
// (TMA-streamed, evict-first), B = the whole batch x (re-read from L2,
// evict-last), D = 128 x Bpad fp32 logits in TMEM.  Each CTA walks its slabs
// through a deep TMA ring; the epilogue warps turn each finished slab into
// per-(shard, row) 64-bit keys (order-preserving logit bits, inverted id) and
// fold them into the workspace with atomicMax, which also resolves ties to the
// lowest id.  Each epilogue warp transposes its 32 x 16 logit tiles through
// shared memory so that one lane scans one batch row with float compares, and
// folds its winners into the workspace with one atomic instruction per tile:
// the epilogue stays a small fraction of a slab's streaming time and leaves
// issue slots to the producer and MMA warps.  The last CTA to finish writes
// shard_max / shard_idx / ids and zeroes the workspace for the next call.
#pragma once

#include "common.cuh"
#include "ptx.cuh"
#include "trace.cuh"

namespace tpl {

constexpr int kLmRows = 128;
constexpr int kLmBK = 64;
constexpr int kLmThreads = 192;
constexpr int kLmABytes = kLmRows * kLmBK * 2;
constexpr int kLmMaxStages = 12;
constexpr int kLmTbufWarp = 16 * 33;  // floats of one epilogue warp's transpose tile
constexpr int kLmTbufBytes = 4 * kLmTbufWarp * 4;

struct LmArgs {
  CUtensorMap tmW;  // {K, V}, box {64, slab_rows}
  CUtensorMap tmX;  // {K, B}, box {64, Npad}
  int32_t B, Npad, K, k_iters;
  int32_t V, tp, shard;
  int32_t n_slabs;
  int32_t slab_rows;  // vocab rows per slab (<= 128; the MMA tile rows beyond it are ignored)
  int32_t stages, stage_bytes;
  uint32_t tmem_cols;
  float* logits;
  float* shard_max;
  int32_t* shard_idx;
  int32_t* ids;
  unsigned long long* keys;  // [tp][B], zero on entry and on exit
  unsigned int* counter;
  uint32_t trace_seq;  // launch number for the optional timing records (trace.cuh)
  int32_t tn;          // 128 or 64: run lmhead_argmax_tn<tn> (lmhead_tn.cuh); 0: this kernel
  // lmhead_argmax_tn only.  ranged = 0: slab g covers rows [g slab_rows, ...)
  // and CTA c takes slabs c, c + grid, ...  ranged = 1: CTA c owns the
  // contiguous rows [c range_base + min(c, range_rem), + range_base + (c <
  // range_rem)), cut into slabs of slab_rows (= 256) and one shorter last slab,
  // loaded through tmWt (box {64, tail_rows}) and multiplied with N = tail_n.
  int32_t ranged, range_base, range_rem, tail_rows, tail_n;
  CUtensorMap tmWt;
};

// Order-preserving map of a float onto uint32 (larger float -> larger key).
__device__ __forceinline__ uint32_t float_key(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_float(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}
// 0 is reserved for "no candidate"; every real (logit, id) pair maps above it.
__device__ __forceinline__ unsigned long long make_key(float f, int32_t id) {
  return (static_cast<unsigned long long>(float_key(f)) << 32) |
         static_cast<unsigned long long>(0xFFFFFFFFu - static_cast<uint32_t>(id));
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
}

__global__ void __launch_bounds__(kLmThreads, 1) lmhead_argmax_tcgen05(const __grid_constant__ LmArgs a) {
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
  float* tbuf = reinterpret_cast<float*>(smem + a.stages * a.stage_bytes + 256);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int S = a.stages;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      ptx::mbar_init(&full[s], 1);
      ptx::mbar_init(&empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(&tfull[i], 1);
      ptx::mbar_init(&tempty[i], 4);
    }
    ptx::mbar_init(drain, 1);
    *abort_flag = 0;
    *last_flag = 0;
    ptx::fence_barrier_init();
    ptx::prefetch_tmap(&a.tmW);
    ptx::prefetch_tmap(&a.tmX);
  }
  if (warp == 1) {
    ptx::tmem_alloc(tmem_slot, a.tmem_cols);
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

  if (warp == 0) {
    if (lane == 0) {
      const uint64_t pol_w = ptx::policy_evict_first();
      const uint64_t pol_x = ptx::policy_evict_last();
      const uint32_t bytes =
          static_cast<uint32_t>(a.slab_rows * kLmBK * 2 + a.stage_bytes - kLmABytes);
      int stage = 0, issued = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int slab = blockIdx.x; ok && slab < a.n_slabs; slab += gridDim.x) {
        for (int kb = 0; kb < a.k_iters; ++kb) {
          if (!ptx::mbar_wait(&empty[stage], phase ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          uint8_t* sW = smem + stage * a.stage_bytes;
          ptx::mbar_arrive_expect_tx(&full[stage], bytes);
          ptx::tma_load_2d(sW, &a.tmW, &full[stage], kb * kLmBK, slab * a.slab_rows, pol_w);
          ptx::tma_load_2d(sW + kLmABytes, &a.tmX, &full[stage], kb * kLmBK, 0, pol_x);
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
  } else if (warp == 1) {
    // One thread issues every MMA: no warp-wide synchronisation per stage.
    if (lane == 0) {
      const uint32_t idesc = ptx::idesc_bf16(kLmRows, a.Npad);
      int stage = 0, it = 0;
      uint32_t phase = 0;
      bool ok = true, any_mma = false;
      for (int slab = blockIdx.x; ok && slab < a.n_slabs; slab += gridDim.x, ++it) {
        const int acc = it & 1;
        const uint32_t acc_phase = (it >> 1) & 1;
        if (!ptx::mbar_wait(&tempty[acc], acc_phase ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * (a.tmem_cols / 2);
        for (int kb = 0; kb < a.k_iters; ++kb) {
          if (!ptx::mbar_wait(&full[stage], phase, abort_flag)) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          const uint32_t sW = ptx::smem_u32(smem + stage * a.stage_bytes);
          const uint64_t adesc = ptx::sdesc_kmajor_sw128(sW);
          const uint64_t bdesc = ptx::sdesc_kmajor_sw128(sW + kLmABytes);
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
    const int q = warp & 3;
    int it = 0;
    bool ok = true;
    for (int slab = blockIdx.x; slab < a.n_slabs; slab += gridDim.x, ++it) {
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
      const int slab0 = slab * a.slab_rows;              // first vocab id of the slab
      const int row0 = slab0 + q * 32;                   // first vocab id of this warp
      const int row_end = min(slab0 + a.slab_rows, a.V);  // ids at or past it are not this slab's
      const int v = row0 + lane;
      const bool valid = v < row_end;
      const bool warp_live = row0 < row_end;
      const int s_first = min(row0, row_end - 1) / a.shard;
      const int s_last = min(row0 + 31, row_end - 1) / a.shard;
      const int split = (s_first + 1) * a.shard;  // first id of the next shard
      float* tb = tbuf + (warp - 2) * kLmTbufWarp;
      const int col = lane & 15, half = lane >> 4;
      for (int c = 0; c < a.Npad; c += 16) {
        uint32_t r[16];
        tmem_ld16(tmem_base + ((q * 32u) << 16) + acc * (a.tmem_cols / 2) + c, r);
        ptx::tmem_ld_wait();
        if (!warp_live) continue;
        if (a.logits != nullptr && valid) {
#pragma unroll
          for (int j = 0; j < 16; ++j)
            if (c + j < a.B) a.logits[static_cast<int64_t>(c + j) * a.V + v] = __uint_as_float(r[j]);
        }
        if (s_last > s_first + 1) {
          // Shards narrower than a warp (tiny vocabularies): one atomic per logit.
          if (valid) {
#pragma unroll
            for (int j = 0; j < 16; ++j)
              if (c + j < a.B)
                atomicMax(&a.keys[(v / a.shard) * a.B + c + j], make_key(__uint_as_float(r[j]), v));
          }
          continue;
        }
        // Transpose the warp's 32 rows x 16 columns through shared memory so that
        // each lane scans one column (batch row) over 16 vocab rows with plain
        // float compares, ascending ids first (ties keep the lowest id).
#pragma unroll
        for (int j = 0; j < 16; ++j) tb[j * 33 + lane] = __uint_as_float(r[j]);
        __syncwarp();
        float bv0 = 0.0f, bv1 = 0.0f;
        int bi0 = -1, bi1 = -1;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int rr = half * 16 + i;
          const int vv = row0 + rr;
          const float f = tb[col * 33 + rr];
          if (vv < row_end) {
            if (vv < split) {
              if (bi0 < 0 || f > bv0) { bv0 = f; bi0 = vv; }
            } else {
              if (bi1 < 0 || f > bv1) { bv1 = f; bi1 = vv; }
            }
          }
        }
        __syncwarp();
        // Lanes l and l ^ 16 hold the two row halves of the same column.
        {
          const float ov = __shfl_xor_sync(0xffffffffu, bv0, 16);
          const int oi = __shfl_xor_sync(0xffffffffu, bi0, 16);
          if (oi >= 0 && (bi0 < 0 || ov > bv0 || (ov == bv0 && oi < bi0))) { bv0 = ov; bi0 = oi; }
          const float ov1 = __shfl_xor_sync(0xffffffffu, bv1, 16);
          const int oi1 = __shfl_xor_sync(0xffffffffu, bi1, 16);
          if (oi1 >= 0 && (bi1 < 0 || ov1 > bv1 || (ov1 == bv1 && oi1 < bi1))) { bv1 = ov1; bi1 = oi1; }
        }
        const int b = c + col;
        if (half == 0 && b < a.B) {
          if (bi0 >= 0) atomicMax(&a.keys[s_first * a.B + b], make_key(bv0, bi0));
          if (bi1 >= 0) atomicMax(&a.keys[(s_first + 1) * a.B + b], make_key(bv1, bi1));
        }
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&tempty[acc]);
    }

    // ------------------------------------------------ completion: last CTA
    __threadfence();
    asm volatile("bar.sync 1, 128;" ::: "memory");
    if (warp == 2 && lane == 0) {
      const unsigned prev = atomicAdd(a.counter, 1u);
      *last_flag = (prev == gridDim.x - 1) ? 1 : 0;
    }
    asm volatile("bar.sync 1, 128;" ::: "memory");
    if (*last_flag && ok && !*abort_flag) {
      __threadfence();
      const int t = threadIdx.x - 64;
      for (int b = t; b < a.B; b += 128) {
        unsigned long long best = 0ull;
        for (int s = 0; s < a.tp; ++s) {
          unsigned long long* kp = &a.keys[s * a.B + b];
          const unsigned long long k = __ldcg(kp);
          if (k == 0ull) {
            a.shard_max[s * a.B + b] = -__int_as_float(0x7f800000);
            a.shard_idx[s * a.B + b] = -1;
          } else {
            a.shard_max[s * a.B + b] = key_float(static_cast<uint32_t>(k >> 32));
            a.shard_idx[s * a.B + b] =
                static_cast<int32_t>(0xFFFFFFFFu - static_cast<uint32_t>(k & 0xFFFFFFFFull));
          }
          best = k > best ? k : best;
          *kp = 0ull;
        }
        a.ids[b] = best == 0ull ? -1
                                : static_cast<int32_t>(0xFFFFFFFFu -
                                                       static_cast<uint32_t>(best & 0xFFFFFFFFull));
      }
      if (t == 0) *a.counter = 0u;
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0) trace_end(trace, kTraceLmHead, a.trace_seq);
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem_base, a.tmem_cols);
  }
}

}  // namespace tpl
