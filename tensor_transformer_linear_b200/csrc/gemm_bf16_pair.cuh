// gemm_bf16_pair.cuh -- the column/row-parallel GEMM of gemm_bf16.cuh on a CTA
// pair (cluster of 2, one TPC) with tcgen05.mma.cta_group::2.
//
// A 256 x 256 output tile is computed by one MMA instruction stream issued from
// the even CTA: each CTA stages its own 128 rows of A and one 128-column half
// block of B (the same half-block pairing as the single-CTA kernel), so every
// CTA moves 32 KB per 64-wide K step for a 128 x 256 slice of output instead of
// 48 KB -- a third less shared-memory fill and L2 traffic per FLOP.  Each CTA's
// TMEM receives its 128 rows of the accumulator; both CTAs run the same fused
// epilogue on their rows.
//
// Synchronisation (all mbarrier waits bounded, see ptx::mbar_wait):
//   full[s]   lives in the even CTA; its producer arrives once with the bytes of
//             both CTAs' loads, and both CTAs' TMA loads complete on it.
//   empty[s]  one per CTA; the MMA thread's commit is multicast to both.
//   tfull[a]  one per CTA; commit multicast at the end of each tile.
//   tempty[a] lives in the even CTA; all 16 epilogue warps of the pair arrive.
// Every thread of both CTAs reaches the final cluster barrier, so neither CTA
// leaves (or frees TMEM) while the pair still uses it.
#pragma once

#include "gemm_bf16.cuh"

namespace tpl {

constexpr int kPairStages = 7;
constexpr int kPairStageBytes = kABytes + kBHalfBytes;  // per CTA
constexpr int kPairBM = 2 * kBM;                        // tile rows over the pair
constexpr int kGemmPairSmemBytes = kPairStages * kPairStageBytes + 1024 + 256;

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kGemmThreads, 1)
    gemm_bf16_tcgen05_pair(const __grid_constant__ GemmArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kPairStages * kPairStageBytes);
  uint64_t* empty = full + kPairStages;
  uint64_t* tfull = empty + kPairStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = ptx::cluster_ctarank();
  const bool leader = (rank == 0);
  const int pair = blockIdx.x >> 1;
  const int npairs = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kPairStages; ++s) {
      ptx::mbar_init(&full[s], 1);
      ptx::mbar_init(&empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(&tfull[i], 1);
      ptx::mbar_init(&tempty[i], 2 * kEpiWarps);
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
    ptx::tmem_alloc_pair(tmem_slot, 2 * kAccCols);
    ptx::tmem_relinquish_pair();
  }
  ptx::tc_fence_before();
  __syncwarp();
  ptx::cluster_sync();  // barriers initialised and TMEM allocated in both CTAs
  ptx::tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // the prologue above overlaps the previous kernel's tail; global memory after
  ptx::griddep_wait();
  ptx::griddep_launch_dependents();
  const TraceStamp trace = trace_begin();

  const int k_total = k_steps(a);
  const uint32_t full_lead = ptx::mapa_shared(&full[0], 0);      // full[s] at + 8 s
  const uint32_t tempty_lead = ptx::mapa_shared(&tempty[0], 0);  // tempty[a] at + 8 a

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int it = 0;
      for (int t = pair; ok && t < a.num_tiles; t += npairs, ++it) {
        int mb, nt;
        tile_coords(a, t, mb, nt);
        const bool has1 = 2 * nt + 1 < a.n_halves;
        // This CTA's half of B; an odd last half is padded with the even one.
        const HalfInfo h = decode_half(a, (rank == 1 && has1) ? 2 * nt + 1 : 2 * nt);
        const int m_row = mb * kPairBM + static_cast<int>(rank) * kBM;
        int arow;
        const CUtensorMap* mAcol = a_source(a, m_row, arow);
        const bool rev = a.k_serp && (it & 1);
        // row mode: rank and K block of the next step (walking backwards when rev)
        int rr = 0, kb = 0;
        if (a.mode == kModeRow) row_pos(a, rev ? k_total - 1 : 0, rr, kb);
        for (int kstep = 0; kstep < k_total; ++kstep) {
          const int ki = rev ? k_total - 1 - kstep : kstep;
          if (!ptx::mbar_wait(&empty[stage], phase ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          if (leader) ptx::mbar_arrive_expect_tx(&full[stage], 2 * kPairStageBytes);
          uint8_t* sA = smem + stage * kPairStageBytes;
          uint8_t* sB = sA + kABytes;
          const uint32_t bar = full_lead + 8u * stage;
          if (a.mode != kModeRow) {
            const int kc = ki * kBK;
            ptx::tma_load_2d_pair(sA, mAcol, bar, kc, arow);
            ptx::tma_load_2d_pair(sB, &a.tmB, bar, kc, h.brow);
          } else {
            const bool g2 = rr >= a.r_split;  // second contraction width
            const CUtensorMap* mA = g2 ? &a.tmA2 : &a.tmA;
            const CUtensorMap* mB = g2 ? &a.tmB2 : &a.tmB;
            const int rc = g2 ? rr - a.r_split : rr;
            ptx::tma_load_3d_pair(sA, mA, bar, kb * kBK, m_row, rc);
            ptx::tma_load_3d_pair(sB, mB, bar, kb * kBK, h.brow, rc);
            if (!rev) {
              if (++kb == (g2 ? a.k_iters2 : a.k_iters)) {
                kb = 0;
                ++rr;
              }
            } else if (--kb < 0) {
              --rr;
              kb = (rr >= a.r_split ? a.k_iters2 : a.k_iters) - 1;
            }
          }
          if (++stage == kPairStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {
        *abort_flag = 1;
        record_timeout();
        __nanosleep(100000);  // let copies already in flight land before the final barrier
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && leader) {
      const uint32_t idesc = ptx::idesc_bf16(kPairBM, 2 * kHalfN);
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      bool any_mma = false;
      int it = 0;
      for (int t = pair; ok && t < a.num_tiles; t += npairs, ++it) {
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
          const uint32_t sA = ptx::smem_u32(smem + stage * kPairStageBytes);
          const uint64_t adesc = ptx::sdesc_kmajor_sw128(sA);
          const uint64_t bdesc = ptx::sdesc_kmajor_sw128(sA + kABytes);
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk)
            ptx::umma_bf16_pair(d_tmem, adesc + 2 * kk, bdesc + 2 * kk, idesc, (ki | kk) != 0);
          ptx::umma_commit_pair(&empty[stage], 0x3);
          any_mma = true;
          if (++stage == kPairStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        ptx::umma_commit_pair(&tfull[acc], 0x3);
      }
      if (!ok) {
        *abort_flag = 1;
        record_timeout();
        if (any_mma) {
          volatile int no_abort = 0;
          ptx::umma_commit_pair(drain, 0x1);
          ptx::mbar_wait(drain, 0, &no_abort, 200000000ull);
        }
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int ew = warp - 2;
    const int q = warp & 3;
    const int hh = ew >> 2;
    const int row = q * 32 + lane;
    int it = 0;
    if (a.norm) {
      const int per = (a.M + gridDim.x - 1) / gridDim.x;
      const int r0 = min(a.M, static_cast<int>(blockIdx.x) * per);
      norm_stats(a, r0, min(a.M, r0 + per), ew * 32 + lane);
    }
    for (int t = pair; t < a.num_tiles; t += npairs, ++it) {
      int mb, nt;
      tile_coords(a, t, mb, nt);
      const bool active = (hh == 0) || (2 * nt + 1 < a.n_halves);
      const int acc = it & 1;
      const uint32_t acc_phase = (it >> 1) & 1;
      HalfInfo h;
      if (active) h = decode_half(a, 2 * nt + hh);
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
        swiglu_epilogue(a, nt, mb * kPairBM + static_cast<int>(rank) * kBM + row, hh,
                        tmem_base + ((q * 32u) << 16) + acc * kAccCols);
      } else if (active) {
        const int m = mb * kPairBM + static_cast<int>(rank) * kBM + row;
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
          float bv[32];
          if (a.bias != nullptr && c * 32 < h.valid) load_bias_chunk(a, h, c * 32, bv);
          uint32_t r[32];
          ptx::tmem_ld32(tmem_base + ((q * 32u) << 16) + acc * kAccCols + hh * kHalfN + c * 32, r);
          ptx::tmem_ld_wait();
          if (m < a.M && c * 32 < h.valid) store_chunk(a, h, m, prow, yb, c * 32, r, bv, rs);
        }
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive_cluster(tempty_lead + 8u * acc);
    }
  }

  ptx::tc_fence_before();
  __syncwarp();
  ptx::cluster_sync();  // every MMA, remote arrival and epilogue of the pair is done
  if (threadIdx.x == 0) trace_end(trace, kTraceGemmPair, a.trace_seq);
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc_pair(tmem_base, 2 * kAccCols);
  }
}

}  // namespace tpl
