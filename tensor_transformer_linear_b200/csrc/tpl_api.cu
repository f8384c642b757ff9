// tpl_api.cu -- the extern "C" entry points declared in include/tpl.h:
// argument validation, the sub-parameter partition, TMA descriptor encoding and
// kernel launches on the caller's stream.  Every computational step runs in
// the kernels included below; there is no host or library fallback.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <vector>

#include "tpl.h"
#include "common.cuh"
#include "gemm_bf16.cuh"
#include "gemm_bf16_pair.cuh"
#include "gemm_fp32.cuh"
#include "lmhead.cuh"
#include "lmhead_tn.cuh"
#include "mlp_fp32.cuh"
#include "norm_fold.cuh"
#include "rmsnorm.cuh"

namespace {

using tpl::ColPiece;
using tpl::F32Piece;

std::atomic<uint64_t> g_launch_count{0};

constexpr int kMaxDevices = 64;

struct DeviceInfo {
  int sm_count = 0;
  bool gemm_attr = false;
  bool lm_attr = false;
  bool mlp_attr = false;
  int mlp_clusters = -1;  // clusters of the fused fp32 MLP that fit at once (-1: not asked yet)
  uint32_t epoch = 0;  // last flag epoch handed to a launch on this device
};

std::mutex g_mu;
DeviceInfo g_dev[kMaxDevices];

tpl_status device_info(DeviceInfo** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return TPL_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceInfo& d = g_dev[dev];
  if (d.sm_count == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      return TPL_ERR_CUDA;
    int major = 0, minor = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    if (major != 10 || minor != 0) return TPL_ERR_UNSUPPORTED;  // built for sm_100a only
    d.sm_count = n;
  }
  if (!d.gemm_attr) {
    if (cudaFuncSetAttribute(tpl::gemm_bf16_tcgen05, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             tpl::kGemmSmemBytes) != cudaSuccess)
      return TPL_ERR_CUDA;
    if (cudaFuncSetAttribute(tpl::gemm_bf16_tcgen05_pair,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             tpl::kGemmPairSmemBytes) != cudaSuccess)
      return TPL_ERR_CUDA;
    d.gemm_attr = true;
  }
  if (!d.lm_attr) {
    if (cudaFuncSetAttribute(tpl::lmhead_argmax_tcgen05,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024) != cudaSuccess ||
        cudaFuncSetAttribute(tpl::lmhead_argmax_tn<128>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024) != cudaSuccess ||
        cudaFuncSetAttribute(tpl::lmhead_argmax_tn<64>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024) != cudaSuccess)
      return TPL_ERR_CUDA;
    d.lm_attr = true;
  }
  if (!d.mlp_attr) {
    if (cudaFuncSetAttribute(tpl::mlp_fp32_fused, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             227 * 1024) != cudaSuccess ||
        cudaFuncSetAttribute(tpl::mlp_fp32_fused,
                             cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess)
      return TPL_ERR_CUDA;
    d.mlp_attr = true;
  }
  *out = &d;
  return TPL_OK;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// bf16 tensor map, 128-byte swizzle, box {64, rows[, 1]}.
tpl_status encode_bf16(CUtensorMap* m, const void* base, int rank, const uint64_t* dims,
                       const uint64_t* strides, uint32_t box_rows) {
  auto fn = encode_fn();
  if (fn == nullptr) return TPL_ERR_CUDA;
  const cuuint32_t box[3] = {64, box_rows, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, static_cast<cuuint32_t>(rank),
                  const_cast<void*>(base), reinterpret_cast<const cuuint64_t*>(dims),
                  reinterpret_cast<const cuuint64_t*>(strides), box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? TPL_OK : TPL_ERR_CUDA;
}

inline bool aligned(const void* p, uintptr_t a) {
  return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0;
}

tpl_status launched() {
  g_launch_count.fetch_add(1, std::memory_order_relaxed);
  return cudaGetLastError() == cudaSuccess ? TPL_OK : TPL_ERR_CUDA;
}

// Integer tuning override from the environment (default when unset).
int env_int(const char* name, int dflt) {
  const char* e = std::getenv(name);
  return (e != nullptr && e[0] != '\0') ? std::atoi(e) : dflt;
}

// A fresh epoch for the flags of one launch (never 0, so zeroed flags never match).
uint32_t next_epoch(DeviceInfo* dev) {
  std::lock_guard<std::mutex> lk(g_mu);
  if (++dev->epoch == 0) dev->epoch = 1;
  return dev->epoch;
}

// Kernels of the path are launched as programmatic dependents of the work
// before them on the stream (CUDA programmatic dependent launch): a kernel's
// CTAs start their prologue (barrier init, TMEM allocation, descriptor
// prefetch) on SMs the previous kernel has left, and wait in griddep_wait
// until it has completed.  TPL_PDL=0 launches them plainly.
bool pdl_enabled() {
  static const bool on = env_int("TPL_PDL", 1) != 0;
  return on;
}

template <typename... KArgs, typename... Args>
tpl_status launch_ex(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                     cudaStream_t st, Args... args) {
  cudaLaunchConfig_t cfg;
  std::memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  if (pdl_enabled()) {
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
  }
  if (cudaLaunchKernelEx(&cfg, kern, args...) != cudaSuccess) return TPL_ERR_CUDA;
  return launched();
}

// CTA pairs (tcgen05 cta_group::2, 256-row tiles) unless M fits one 128-row
// block or TPL_GEMM_CTA_PAIRS=0 asks for the single-CTA kernel.
bool use_cta_pairs(int64_t M) {
  const char* e = std::getenv("TPL_GEMM_CTA_PAIRS");
  if (e != nullptr && e[0] == '0') return false;
  return M > tpl::kBM;
}

// Fills the tile counts of `a` (n_tiles / n_halves already set) and launches
// the GEMM on a single CTA per tile or on CTA pairs.
tpl_status launch_gemm(tpl::GemmArgs& a, int64_t M, DeviceInfo* dev, cudaStream_t st) {
  const bool pairs = use_cta_pairs(M) && dev->sm_count >= 2;
  const int64_t bm = pairs ? tpl::kPairBM : tpl::kBM;
  a.m_blocks = static_cast<int32_t>((M + bm - 1) / bm);
  // Tile raster: groups of group_m m-blocks, n-tiles swept inside a group.
  // Measured on the MLP and fused-QKV shapes: column mode (K = 4096) reads the
  // least from DRAM with 16 m-blocks of 256 rows (a wave then shares x and
  // each weight block across its tiles: c_fc 1.84x -> 1.31x its algorithmic
  // bytes, 696 -> 686 us); row mode (K = 14336, a wave's operand blocks about
  // fill L2) with 8 m-blocks and the K order reversed on every other tile,
  // so consecutive waves meet in L2 (1.09 -> 0.96 GB read).
  // Column mode on CTA pairs: the largest group (at most 16) whose A slabs fit
  // in 32 MB, so they stay in L2 while the group sweeps its n-tiles: 16 at
  // K = 4096, 8 at K = 8192 (the 4-layer stack, whose c_fc has K = 8192, ran at
  // 1172 TFLOP/s with 8 and 1131 with 16).
  const bool row = a.mode == tpl::kModeRow;
  int group = 16;
  if (pairs && row) {
    group = 8;
  } else if (pairs) {
    const int64_t slab = static_cast<int64_t>(tpl::kPairBM) * a.k_iters * tpl::kBK * 2;
    while (group > 1 && group * slab > (int64_t{32} << 20)) group /= 2;
  }
  a.group_m = env_int("TPL_GEMM_GROUP_M", group);
  a.k_serp = pairs ? env_int("TPL_GEMM_KSERP", row ? 1 : 0) : 0;
  const int64_t tiles = static_cast<int64_t>(a.m_blocks) * a.n_tiles;
  if (tiles > INT32_MAX) return TPL_ERR_SHAPE;
  a.num_tiles = static_cast<int32_t>(tiles);
  if (a.norm) a.norm_epoch = next_epoch(dev);
  a.trace_seq = static_cast<uint32_t>(g_launch_count.load(std::memory_order_relaxed));
  if (pairs) {
    const int64_t npairs = std::min<int64_t>(tiles, dev->sm_count / 2);
    const int grid = 2 * static_cast<int>(npairs);
    return launch_ex(tpl::gemm_bf16_tcgen05_pair, dim3(grid), dim3(tpl::kGemmThreads),
                     tpl::kGemmPairSmemBytes, st, a);
  }
  const int grid = static_cast<int>(std::min<int64_t>(tiles, dev->sm_count));
  return launch_ex(tpl::gemm_bf16_tcgen05, dim3(grid), dim3(tpl::kGemmThreads),
                   tpl::kGemmSmemBytes, st, a);
}

tpl_status check_partition(const tpl_partition* p) {
  if (p->tp_size < 1 || p->tp_size > TPL_MAX_TP || p->n_sub < 1 || p->n_sub > TPL_MAX_SUB)
    return TPL_ERR_SHAPE;
  if (p->logical_out < 1 || p->logical_out > INT32_MAX) return TPL_ERR_SHAPE;
  for (int r = 0; r < p->tp_size; ++r) {
    if (p->shard_width[r] < 1 || p->shard_width[r] > INT32_MAX || p->shard_base[r] < 0)
      return TPL_ERR_SHAPE;
    for (int j = 0; j < p->n_sub; ++j) {
      const int64_t w = p->width[r][j], s = p->src_off[r][j], d = p->dst_off[r][j];
      if (w < 1 || s < 0 || d < 0 || s + w > p->logical_out || d + w > p->shard_width[r])
        return TPL_ERR_SHAPE;
    }
  }
  return TPL_OK;
}

int act_ok(int act) {
  return act == TPL_ACT_NONE || act == TPL_ACT_GELU_ERF || act == TPL_ACT_GELU_TANH;
}

// Sequence-parallel row layout (rank-major token slices); all zero = plain rows.
struct SeqPar {
  int32_t batch = 0, seq = 0, seg = 0;
  int32_t a_remap = 0, out_remap = 0;
};

// One rank's shard of a row-parallel linear split over GPUs: its output rows go
// to the receive buffers of the ranks that own the tokens (peer[q], [tp] bases).
struct PeerScatter {
  int32_t src_rank = 0;
  int32_t tp = 0;
  void* const* peer = nullptr;
};

template <typename Args>
void set_seqpar(Args& a, const SeqPar& sp) {
  a.sp_batch = sp.batch;
  a.sp_seq = sp.seq;
  a.sp_seg = sp.seg;
  a.a_remap = sp.a_remap;
  a.out_remap = sp.out_remap;
}

// ------------------------------------------------------------------ column

// The fused RMSNorm of a column linear (tpl_column_linear_rmsnorm): per-row
// factors and their flags in the caller's workspace.
struct NormFuse {
  float eps = 0.0f;
  float* rs = nullptr;
  uint32_t* flag = nullptr;
};

// Token slices of the A operand held by several ranks (peer gather): rank q's
// slice [batch][seq/tp][K] at gather[q], q < tp.
struct GatherA {
  int32_t tp = 0;
  void* const* gather = nullptr;
};

tpl_status column_bf16(const tpl_partition* p, const void* x, int64_t M, int64_t K, const void* w,
                       const void* bias, int act, void* y, cudaStream_t st,
                       const SeqPar& sp = SeqPar{}, const GatherA* ga = nullptr,
                       const NormFuse* nf = nullptr) {
  if ((K % 8) != 0 || !aligned(x, 16) || !aligned(w, 16) || !aligned(y, 2) ||
      (bias != nullptr && !aligned(bias, 2)))
    return TPL_ERR_ALIGN;
  if (ga != nullptr)
    for (int q = 0; q < ga->tp; ++q)
      if (!aligned(ga->gather[q], 16)) return TPL_ERR_ALIGN;
  DeviceInfo* dev = nullptr;
  tpl_status s = device_info(&dev);
  if (s != TPL_OK) return s;

  tpl::GemmArgs a;
  std::memset(&a, 0, sizeof(a));
  if (ga == nullptr) {
    const uint64_t dims[2] = {static_cast<uint64_t>(K), static_cast<uint64_t>(M)};
    const uint64_t str[1] = {static_cast<uint64_t>(K) * 2};
    if ((s = encode_bf16(&a.tmA, x, 2, dims, str, tpl::kBM)) != TPL_OK) return s;
  } else {
    const uint64_t dims[2] = {static_cast<uint64_t>(K),
                              static_cast<uint64_t>(sp.batch) * static_cast<uint64_t>(sp.seg)};
    const uint64_t str[1] = {static_cast<uint64_t>(K) * 2};
    for (int q = 0; q < ga->tp; ++q)
      if ((s = encode_bf16(&a.tmGather[q], ga->gather[q], 2, dims, str, tpl::kBM)) != TPL_OK)
        return s;
    a.tmA = a.tmGather[0];
    a.a_gather = 1;
  }
  {
    const uint64_t dims[2] = {static_cast<uint64_t>(K), static_cast<uint64_t>(p->logical_out)};
    const uint64_t str[1] = {static_cast<uint64_t>(K) * 2};
    if ((s = encode_bf16(&a.tmB, w, 2, dims, str, tpl::kHalfN)) != TPL_OK) return s;
  }
  a.mode = tpl::kModeColumn;
  a.act = act;
  a.M = static_cast<int32_t>(M);
  if (nf != nullptr) {
    a.norm = 1;
    a.norm_eps = nf->eps;
    a.norm_x = static_cast<const __nv_bfloat16*>(x);
    a.norm_K = static_cast<int32_t>(K);
    a.norm_ld = static_cast<int32_t>(K);
    a.norm_rs = nf->rs;
    a.norm_flag = nf->flag;
  }
  set_seqpar(a, sp);
  a.k_iters = static_cast<int32_t>((K + tpl::kBK - 1) / tpl::kBK);
  a.bias = static_cast<const __nv_bfloat16*>(bias);
  a.y = static_cast<__nv_bfloat16*>(y);

  std::vector<ColPiece> pieces;
  for (int r = 0; r < p->tp_size; ++r)
    for (int j = 0; j < p->n_sub; ++j) {
      ColPiece c;
      c.out_off = M * p->shard_base[r] + p->dst_off[r][j];
      c.src_row = static_cast<int32_t>(p->src_off[r][j]);
      c.width = static_cast<int32_t>(p->width[r][j]);
      c.ld = static_cast<int32_t>(p->shard_width[r]);
      c.hb_begin = 0;
      pieces.push_back(c);
    }
  for (size_t b = 0; b < pieces.size(); b += tpl::kMaxPieces) {
    const size_t e = std::min(pieces.size(), b + tpl::kMaxPieces);
    int hb = 0;
    bool vec = aligned(y, 16);
    a.n_pieces = static_cast<int32_t>(e - b);
    for (size_t i = b; i < e; ++i) {
      ColPiece c = pieces[i];
      c.hb_begin = hb;
      hb += (c.width + tpl::kHalfN - 1) / tpl::kHalfN;
      vec = vec && (c.out_off % 8 == 0) && (c.ld % 8 == 0);
      a.pieces[i - b] = c;
    }
    a.n_halves = hb;
    a.vec_store = vec ? 1 : 0;
    a.n_tiles = (hb + 1) / 2;
    if ((s = launch_gemm(a, M, dev, st)) != TPL_OK) return s;
  }
  return TPL_OK;
}

// Launches the fp32 kernel over n_tiles x mb output tiles, splitting each
// tile's K steps over a cluster of up to 8 CTAs (grid z) when there are too
// few tiles to fill the GPU (the tiny MLP: 32 and 8 tiles).
tpl_status launch_fp32(const tpl::F32Args& a, int64_t mb, cudaStream_t st) {
  const int64_t tiles = static_cast<int64_t>(a.n_tiles) * mb;
  int split = 1;
  while (split < tpl::kF32MaxSplit && tiles * split < 128 && split * 2 <= a.k_steps) split *= 2;
  cudaLaunchConfig_t cfg;
  std::memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = dim3(static_cast<unsigned>(a.n_tiles), static_cast<unsigned>(mb),
                     static_cast<unsigned>(split));
  cfg.blockDim = dim3(tpl::kF32Threads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = static_cast<unsigned>(split);
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (pdl_enabled()) {
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.numAttrs = 2;
  }
  if (cudaLaunchKernelEx(&cfg, tpl::gemm_fp32_simt, a) != cudaSuccess) return TPL_ERR_CUDA;
  return launched();
}

// 32-wide K steps of ranks r0 .. r1-1 (row mode).
int32_t fp32_row_steps(const tpl::F32Args& a) {
  int64_t n = 0;
  for (int r = a.r0; r < a.r1; ++r)
    n += (a.koff[r + 1] - a.koff[r] + tpl::kF32BK - 1) / tpl::kF32BK;
  return static_cast<int32_t>(n);
}

tpl_status column_fp32(const tpl_partition* p, const void* x, int64_t M, int64_t K, const void* w,
                       const void* bias, int act, void* y, cudaStream_t st,
                       const SeqPar& sp = SeqPar{}) {
  if (!aligned(x, 4) || !aligned(w, 4) || !aligned(y, 4) || (bias && !aligned(bias, 4)))
    return TPL_ERR_ALIGN;
  tpl::F32Args a;
  std::memset(&a, 0, sizeof(a));
  a.mode = 0;
  a.act = act;
  a.M = M;
  set_seqpar(a, sp);
  a.K = static_cast<int32_t>(K);
  a.x = static_cast<const float*>(x);
  a.w = static_cast<const float*>(w);
  a.bias = static_cast<const float*>(bias);
  a.y = static_cast<float*>(y);
  a.k_steps = static_cast<int32_t>((K + tpl::kF32BK - 1) / tpl::kF32BK);
  a.vec = (K % 4 == 0 && aligned(x, 16) && aligned(w, 16)) ? 1 : 0;
  std::vector<F32Piece> pieces;
  for (int r = 0; r < p->tp_size; ++r)
    for (int j = 0; j < p->n_sub; ++j) {
      F32Piece c;
      c.out_off = M * p->shard_base[r] + p->dst_off[r][j];
      c.src_row = static_cast<int32_t>(p->src_off[r][j]);
      c.width = static_cast<int32_t>(p->width[r][j]);
      c.ld = static_cast<int32_t>(p->shard_width[r]);
      c.nt_begin = 0;
      pieces.push_back(c);
    }
  const int64_t mb = (M + tpl::kF32BM - 1) / tpl::kF32BM;
  if (mb > 65535) return TPL_ERR_SHAPE;
  for (size_t b = 0; b < pieces.size(); b += tpl::kF32MaxPieces) {
    const size_t e = std::min(pieces.size(), b + tpl::kF32MaxPieces);
    int nt = 0;
    a.n_pieces = static_cast<int32_t>(e - b);
    for (size_t i = b; i < e; ++i) {
      F32Piece c = pieces[i];
      c.nt_begin = nt;
      nt += (c.width + tpl::kF32BN - 1) / tpl::kF32BN;
      a.pieces[i - b] = c;
    }
    a.n_tiles = nt;
    tpl_status s = launch_fp32(a, mb, st);
    if (s != TPL_OK) return s;
  }
  return TPL_OK;
}

// --------------------------------------------------------------------- row

tpl_status row_bf16(const void* h, const int64_t* k_w, int tp, int64_t M, int64_t N, const void* w,
                    const void* bias, const void* residual, void* y, float* partials,
                    cudaStream_t st, const SeqPar& sp = SeqPar{},
                    const PeerScatter* ps = nullptr) {
  for (int r = 0; r < tp; ++r)
    if (k_w[r] % 8 != 0) return TPL_ERR_ALIGN;
  if (!aligned(h, 16) || !aligned(w, 16) || !aligned(y, 2) || (bias && !aligned(bias, 2)) ||
      (residual && !aligned(residual, 2)) || (partials && !aligned(partials, 4)))
    return TPL_ERR_ALIGN;
  // Up to two contiguous groups of equal contraction width: the shape of every
  // partition from tpl_partition_subparams (remainder units on the lowest ranks).
  const int64_t Kr = k_w[0];
  int split = tp;
  for (int r = 1; r < tp; ++r)
    if (k_w[r] != Kr) {
      split = r;
      break;
    }
  const int64_t Kr2 = split < tp ? k_w[split] : Kr;
  for (int r = split; r < tp; ++r)
    if (k_w[r] != Kr2) return TPL_ERR_UNSUPPORTED;
  DeviceInfo* dev = nullptr;
  tpl_status s = device_info(&dev);
  if (s != TPL_OK) return s;

  tpl::GemmArgs a;
  std::memset(&a, 0, sizeof(a));
  auto encode_group = [&](CUtensorMap* mh, CUtensorMap* mw, int64_t kr, int64_t ranks,
                          int64_t first) -> tpl_status {
    const char* hb = static_cast<const char*>(h) + M * first * Kr * 2;
    const char* wb = static_cast<const char*>(w) + N * first * Kr * 2;
    const uint64_t dh[3] = {static_cast<uint64_t>(kr), static_cast<uint64_t>(M),
                            static_cast<uint64_t>(ranks)};
    const uint64_t sh[2] = {static_cast<uint64_t>(kr) * 2, static_cast<uint64_t>(M * kr) * 2};
    tpl_status st2 = encode_bf16(mh, hb, 3, dh, sh, tpl::kBM);
    if (st2 != TPL_OK) return st2;
    const uint64_t dw[3] = {static_cast<uint64_t>(kr), static_cast<uint64_t>(N),
                            static_cast<uint64_t>(ranks)};
    const uint64_t sw[2] = {static_cast<uint64_t>(kr) * 2, static_cast<uint64_t>(N * kr) * 2};
    return encode_bf16(mw, wb, 3, dw, sw, tpl::kHalfN);
  };
  if ((s = encode_group(&a.tmA, &a.tmB, Kr, split, 0)) != TPL_OK) return s;
  if (split < tp && (s = encode_group(&a.tmA2, &a.tmB2, Kr2, tp - split, split)) != TPL_OK)
    return s;
  a.mode = tpl::kModeRow;
  a.M = static_cast<int32_t>(M);
  set_seqpar(a, sp);
  a.N = static_cast<int32_t>(N);
  a.k_iters = static_cast<int32_t>((Kr + tpl::kBK - 1) / tpl::kBK);
  a.k_iters2 = static_cast<int32_t>((Kr2 + tpl::kBK - 1) / tpl::kBK);
  a.r_split = split;
  a.n_halves = static_cast<int32_t>((N + tpl::kHalfN - 1) / tpl::kHalfN);
  a.n_tiles = (a.n_halves + 1) / 2;
  a.y = static_cast<__nv_bfloat16*>(y);

  // The fused path: all ranks accumulate into one accumulator.
  a.r0 = 0;
  a.r1 = tp;
  a.bias = static_cast<const __nv_bfloat16*>(bias);
  a.residual = static_cast<const __nv_bfloat16*>(residual);
  a.partials = nullptr;
  a.vec_store = (N % 8 == 0 && aligned(y, 16) && (residual == nullptr || aligned(residual, 16)));
  if (ps != nullptr) {
    a.scatter = 1;
    a.src_rank = ps->src_rank;
    bool vec = (N % 8 == 0);
    for (int q = 0; q < ps->tp; ++q) {
      a.peer[q] = static_cast<__nv_bfloat16*>(ps->peer[q]);
      vec = vec && aligned(ps->peer[q], 16);
    }
    a.vec_store = vec ? 1 : 0;
  }
  if ((s = launch_gemm(a, M, dev, st)) != TPL_OK) return s;

  if (partials != nullptr) {
    a.bias = nullptr;
    a.residual = nullptr;
    a.vec_store = (N % 4 == 0 && aligned(partials, 16)) ? 1 : 0;
    for (int r = 0; r < tp; ++r) {
      a.r0 = r;
      a.r1 = r + 1;
      a.partials = partials + static_cast<int64_t>(r) * M * N;
      if ((s = launch_gemm(a, M, dev, st)) != TPL_OK) return s;
    }
  }
  return TPL_OK;
}

tpl_status row_fp32(const void* h, const int64_t* k_w, int tp, int64_t M, int64_t N, const void* w,
                    const void* bias, const void* residual, void* y, float* partials,
                    cudaStream_t st, const SeqPar& sp = SeqPar{}) {
  if (!aligned(h, 4) || !aligned(w, 4) || !aligned(y, 4) || (bias && !aligned(bias, 4)) ||
      (residual && !aligned(residual, 4)) || (partials && !aligned(partials, 4)))
    return TPL_ERR_ALIGN;
  tpl::F32Args a;
  std::memset(&a, 0, sizeof(a));
  a.mode = 1;
  a.M = M;
  set_seqpar(a, sp);
  a.N = static_cast<int32_t>(N);
  a.h = static_cast<const float*>(h);
  a.w = static_cast<const float*>(w);
  a.y = static_cast<float*>(y);
  a.koff[0] = 0;
  bool vec = aligned(h, 16) && aligned(w, 16);
  for (int r = 0; r < tp; ++r) {
    a.koff[r + 1] = a.koff[r] + k_w[r];
    vec = vec && (k_w[r] % 4 == 0);
  }
  a.vec = vec ? 1 : 0;
  a.n_tiles = static_cast<int32_t>((N + tpl::kF32BN - 1) / tpl::kF32BN);
  const int64_t mb = (M + tpl::kF32BM - 1) / tpl::kF32BM;
  if (mb > 65535) return TPL_ERR_SHAPE;
  a.r0 = 0;
  a.r1 = tp;
  a.k_steps = fp32_row_steps(a);
  a.bias = static_cast<const float*>(bias);
  a.residual = static_cast<const float*>(residual);
  tpl_status s = launch_fp32(a, mb, st);
  if (s != TPL_OK) return s;
  if (partials != nullptr) {
    a.bias = nullptr;
    a.residual = nullptr;
    for (int r = 0; r < tp; ++r) {
      a.r0 = r;
      a.r1 = r + 1;
      a.k_steps = fp32_row_steps(a);
      a.partials = partials + static_cast<int64_t>(r) * M * N;
      if ((s = launch_fp32(a, mb, st)) != TPL_OK) return s;
    }
  }
  return TPL_OK;
}

// ----------------------------------------------------------------- rmsnorm

template <typename T>
tpl_status rmsnorm_launch(const void* x, int64_t M, int64_t H, const float* scale, int centered,
                          float eps, void* y, cudaStream_t st) {
  DeviceInfo* dev = nullptr;
  tpl_status s = device_info(&dev);
  if (s != TPL_OK) return s;
  constexpr int P = tpl::VecTraits<T>::kPer;
  const int64_t rows_per_block = tpl::kNormWarps;
  const int64_t blocks = std::min<int64_t>((M + rows_per_block - 1) / rows_per_block,
                                           static_cast<int64_t>(dev->sm_count) * 16);
  const T* xp = static_cast<const T*>(x);
  T* yp = static_cast<T*>(y);
  const bool vec = (H % P == 0) && aligned(x, 16) && aligned(y, 16) &&
                   (scale == nullptr || aligned(scale, 16));
  const int64_t lanes_vec = (H / P + 31) / 32;  // vectors per lane
  const int64_t cta_vec = (H / P + tpl::kNormCtaThreads - 1) / tpl::kNormCtaThreads;
  const int g = static_cast<int>(blocks);
  const int t = tpl::kNormWarps * 32;
  const int Hi = static_cast<int>(H);
  if (vec && H / P >= 2 * tpl::kNormCtaThreads && cta_vec <= 16) {
    // Wide rows: a CTA per row (the block scheduler balances rows over SMs as
    // CTAs finish), up to 16 CTAs resident per SM.
    const int gc = static_cast<int>(std::min<int64_t>(M, INT32_MAX));
    const int tc = tpl::kNormCtaThreads;
    if (cta_vec <= 2)
      s = launch_ex(tpl::rmsnorm_cta<T, 2>, dim3(gc), dim3(tc), 0, st, xp, yp, scale,
                    centered, eps, M, Hi);
    else if (cta_vec <= 4)
      s = launch_ex(tpl::rmsnorm_cta<T, 4>, dim3(gc), dim3(tc), 0, st, xp, yp, scale,
                    centered, eps, M, Hi);
    else if (cta_vec <= 8)
      s = launch_ex(tpl::rmsnorm_cta<T, 8>, dim3(gc), dim3(tc), 0, st, xp, yp, scale,
                    centered, eps, M, Hi);
    else
      s = launch_ex(tpl::rmsnorm_cta<T, 16>, dim3(gc), dim3(tc), 0, st, xp, yp, scale,
                    centered, eps, M, Hi);
  } else if (vec && lanes_vec <= 32) {
    if (lanes_vec <= 1)
      s = launch_ex(tpl::rmsnorm_reg<T, 1>, dim3(g), dim3(t), 0, st, xp, yp, scale,
                    centered, eps, M, Hi);
    else if (lanes_vec <= 2)
      s = launch_ex(tpl::rmsnorm_reg<T, 2>, dim3(g), dim3(t), 0, st, xp, yp, scale,
                    centered, eps, M, Hi);
    else if (lanes_vec <= 4)
      s = launch_ex(tpl::rmsnorm_reg<T, 4>, dim3(g), dim3(t), 0, st, xp, yp, scale,
                    centered, eps, M, Hi);
    else if (lanes_vec <= 8)
      s = launch_ex(tpl::rmsnorm_reg<T, 8>, dim3(g), dim3(t), 0, st, xp, yp, scale,
                    centered, eps, M, Hi);
    else if (lanes_vec <= 16)
      s = launch_ex(tpl::rmsnorm_reg<T, 16>, dim3(g), dim3(t), 0, st, xp, yp, scale,
                    centered, eps, M, Hi);
    else
      s = launch_ex(tpl::rmsnorm_reg<T, 32>, dim3(g), dim3(t), 0, st, xp, yp, scale,
                    centered, eps, M, Hi);
  } else {
    s = launch_ex(tpl::rmsnorm_generic<T>, dim3(g), dim3(t), 0, st, xp, yp, scale, centered, eps,
                  M, H);
  }
  return s;
}

}  // namespace

// ======================================================================
// extern "C" entry points
// ======================================================================

extern "C" {

const char* tpl_status_string(tpl_status s) {
  switch (s) {
    case TPL_OK: return "TPL_OK";
    case TPL_ERR_NULL: return "TPL_ERR_NULL: a required pointer is NULL";
    case TPL_ERR_SHAPE: return "TPL_ERR_SHAPE: a size is out of range or sizes disagree";
    case TPL_ERR_INDIVISIBLE: return "TPL_ERR_INDIVISIBLE: the partition leaves a rank empty";
    case TPL_ERR_DTYPE: return "TPL_ERR_DTYPE: unknown dtype or activation";
    case TPL_ERR_ALIGN: return "TPL_ERR_ALIGN: pointer or row stride breaks the 16-byte rule";
    case TPL_ERR_CUDA: return "TPL_ERR_CUDA: a CUDA call failed";
    case TPL_ERR_TIMEOUT: return "TPL_ERR_TIMEOUT: a kernel gave up waiting on its pipeline";
    case TPL_ERR_UNSUPPORTED: return "TPL_ERR_UNSUPPORTED: outside what this library implements";
  }
  return "unknown tpl_status";
}

uint64_t tpl_launch_count(void) { return g_launch_count.load(std::memory_order_relaxed); }

tpl_status tpl_partition_subparams(const int64_t* sub_sizes, int32_t n_sub, int32_t tp_size,
                                   int64_t align, tpl_partition* out) {
  if (sub_sizes == nullptr || out == nullptr) return TPL_ERR_NULL;
  if (tp_size < 1 || tp_size > TPL_MAX_TP || n_sub < 1 || n_sub > TPL_MAX_SUB || align < 1)
    return TPL_ERR_SHAPE;
  int64_t total = 0;
  for (int j = 0; j < n_sub; ++j) {
    if (sub_sizes[j] < 1 || sub_sizes[j] > INT32_MAX) return TPL_ERR_SHAPE;
    if (sub_sizes[j] % align != 0) return TPL_ERR_INDIVISIBLE;
    total += sub_sizes[j];
  }
  if (total > INT32_MAX) return TPL_ERR_SHAPE;
  tpl_partition p;
  std::memset(&p, 0, sizeof(p));
  p.tp_size = tp_size;
  p.n_sub = n_sub;
  p.logical_out = total;
  int64_t sub_start = 0;
  for (int j = 0; j < n_sub; ++j) {
    const int64_t units = sub_sizes[j] / align;
    int64_t row = sub_start;
    for (int r = 0; r < tp_size; ++r) {
      const int64_t u = units / tp_size + (r < units % tp_size ? 1 : 0);
      if (u == 0) return TPL_ERR_INDIVISIBLE;
      p.width[r][j] = u * align;
      p.src_off[r][j] = row;
      row += p.width[r][j];
    }
    sub_start += sub_sizes[j];
  }
  int64_t base = 0;
  for (int r = 0; r < tp_size; ++r) {
    int64_t col = 0;
    for (int j = 0; j < n_sub; ++j) {
      p.dst_off[r][j] = col;
      col += p.width[r][j];
    }
    p.shard_width[r] = col;
    p.shard_base[r] = base;
    base += col;
  }
  *out = p;
  return TPL_OK;
}

tpl_status tpl_column_linear(const tpl_partition* p, const void* x, int64_t M, int64_t K,
                             const void* w, const void* bias, tpl_dtype dt, tpl_act act, void* y,
                             void* stream) {
  if (p == nullptr) return TPL_ERR_NULL;
  if ((dt != TPL_FP32 && dt != TPL_BF16) || !act_ok(act)) return TPL_ERR_DTYPE;
  tpl_status s = check_partition(p);
  if (s != TPL_OK) return s;
  if (M < 0 || K < 1 || M > INT32_MAX || K > INT32_MAX) return TPL_ERR_SHAPE;
  if (M == 0) return TPL_OK;
  if (x == nullptr || w == nullptr || y == nullptr) return TPL_ERR_NULL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return dt == TPL_BF16 ? column_bf16(p, x, M, K, w, bias, act, y, st)
                        : column_fp32(p, x, M, K, w, bias, act, y, st);
}

tpl_status tpl_row_linear_reduce(const void* h, const int64_t* k_w, int32_t tp, int64_t M,
                                 int64_t N, const void* w, const void* bias, const void* residual,
                                 tpl_dtype dt, void* y, float* partials, void* stream) {
  if (k_w == nullptr) return TPL_ERR_NULL;
  if (dt != TPL_FP32 && dt != TPL_BF16) return TPL_ERR_DTYPE;
  if (tp < 1 || tp > TPL_MAX_TP || M < 0 || N < 1 || M > INT32_MAX || N > INT32_MAX)
    return TPL_ERR_SHAPE;
  int64_t ktot = 0;
  for (int r = 0; r < tp; ++r) {
    if (k_w[r] < 1 || k_w[r] > INT32_MAX) return TPL_ERR_SHAPE;
    ktot += k_w[r];
  }
  if (ktot > INT32_MAX) return TPL_ERR_SHAPE;
  if (M == 0) return TPL_OK;
  if (h == nullptr || w == nullptr || y == nullptr) return TPL_ERR_NULL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return dt == TPL_BF16 ? row_bf16(h, k_w, tp, M, N, w, bias, residual, y, partials, st)
                        : row_fp32(h, k_w, tp, M, N, w, bias, residual, y, partials, st);
}

static size_t round256(size_t n) { return (n + 255) / 256 * 256; }

tpl_status tpl_column_linear_rmsnorm_workspace_size(int64_t M, size_t* bytes) {
  if (bytes == nullptr) return TPL_ERR_NULL;
  if (M < 0 || M > INT32_MAX) return TPL_ERR_SHAPE;
  *bytes = 2 * round256(static_cast<size_t>(M) * 4);
  return TPL_OK;
}

tpl_status tpl_column_linear_rmsnorm(const tpl_partition* p, const void* x, int64_t M, int64_t K,
                                     const void* w, const void* bias, float eps, tpl_act act,
                                     void* y, void* workspace, size_t ws_bytes, void* stream) {
  if (p == nullptr) return TPL_ERR_NULL;
  if (!act_ok(act)) return TPL_ERR_DTYPE;
  tpl_status s = check_partition(p);
  if (s != TPL_OK) return s;
  if (M < 0 || K < 1 || M > INT32_MAX || K > INT32_MAX || !(eps >= 0.0f)) return TPL_ERR_SHAPE;
  if (M == 0) return TPL_OK;
  if (x == nullptr || w == nullptr || y == nullptr || workspace == nullptr) return TPL_ERR_NULL;
  if (!aligned(workspace, 256)) return TPL_ERR_ALIGN;
  size_t need = 0;
  if ((s = tpl_column_linear_rmsnorm_workspace_size(M, &need)) != TPL_OK) return s;
  if (ws_bytes < need) return TPL_ERR_SHAPE;
  NormFuse nf;
  nf.eps = eps;
  nf.rs = static_cast<float*>(workspace);
  nf.flag = reinterpret_cast<uint32_t*>(static_cast<char*>(workspace) +
                                        round256(static_cast<size_t>(M) * 4));
  return column_bf16(p, x, M, K, w, bias, act, y, static_cast<cudaStream_t>(stream), SeqPar{},
                     nullptr, &nf);
}

tpl_status tpl_fold_norm_scale(const void* w, int64_t rows, int64_t K, const float* scale,
                               int32_t centered, void* w_out, void* stream) {
  if (rows < 0 || K < 1 || rows > INT32_MAX || K > INT32_MAX) return TPL_ERR_SHAPE;
  if (rows == 0) return TPL_OK;
  if (w == nullptr || scale == nullptr || w_out == nullptr) return TPL_ERR_NULL;
  if (K % 8 != 0 || !aligned(w, 16) || !aligned(w_out, 16) || !aligned(scale, 16))
    return TPL_ERR_ALIGN;
  DeviceInfo* dev = nullptr;
  tpl_status s = device_info(&dev);
  if (s != TPL_OK) return s;
  const int64_t vecs = rows * (K / 8);
  const int grid = static_cast<int>(std::min<int64_t>((vecs + 255) / 256,
                                                      static_cast<int64_t>(dev->sm_count) * 8));
  tpl::fold_norm_scale_kernel<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const __nv_bfloat16*>(w), rows, K, scale, centered,
      static_cast<__nv_bfloat16*>(w_out));
  return launched();
}

tpl_status tpl_rmsnorm(const void* x, int64_t M, int64_t H, const float* scale, int32_t centered,
                       float eps, tpl_dtype dt, void* y, void* stream) {
  if (dt != TPL_FP32 && dt != TPL_BF16) return TPL_ERR_DTYPE;
  if (M < 0 || H < 1 || H > INT32_MAX || !(eps >= 0.0f)) return TPL_ERR_SHAPE;
  if (M == 0) return TPL_OK;
  if (x == nullptr || y == nullptr) return TPL_ERR_NULL;
  if (!aligned(x, dt == TPL_BF16 ? 2 : 4) || !aligned(y, dt == TPL_BF16 ? 2 : 4) ||
      (scale && !aligned(scale, 4)))
    return TPL_ERR_ALIGN;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return dt == TPL_BF16 ? rmsnorm_launch<__nv_bfloat16>(x, M, H, scale, centered, eps, y, st)
                        : rmsnorm_launch<float>(x, M, H, scale, centered, eps, y, st);
}

static tpl_status lm_layout(int64_t B, int64_t V, int32_t tp, int32_t n_chunks, int64_t* shard) {
  if (B < 1 || B > 256 || V < 1 || V > INT32_MAX || tp < 1 || tp > TPL_MAX_TP || n_chunks < 1)
    return TPL_ERR_SHAPE;
  const int64_t sh = (V + tp - 1) / tp;
  const int64_t cap = (sh + n_chunks - 1) / n_chunks;
  const int64_t num_splits = (sh + cap - 1) / cap;
  const int64_t last = sh - std::min(sh, cap) * (num_splits - 1);
  if (num_splits != n_chunks || last <= 0) return TPL_ERR_SHAPE;
  *shard = sh;
  return TPL_OK;
}

tpl_status tpl_lmhead_workspace_size(int64_t B, int64_t V, int32_t tp, int32_t n_chunks,
                                     size_t* bytes) {
  if (bytes == nullptr) return TPL_ERR_NULL;
  int64_t shard = 0;
  tpl_status s = lm_layout(B, V, tp, n_chunks, &shard);
  if (s != TPL_OK) return s;
  const size_t raw = static_cast<size_t>(tp) * static_cast<size_t>(B) * 8 + 16;
  *bytes = (raw + 255) / 256 * 256;
  return TPL_OK;
}

}  // extern "C"

namespace {

// Every check of an LM-head call and the kernel's arguments (tensor maps
// included), with nothing enqueued; `scratch` is the keys + counter area of
// `ws_bytes` bytes (the caller's workspace or the library's fixed array).
// The transposed decode LM head (lmhead_tn.cuh) for batches of up to 32 rows,
// with a 64-row A operand (TPL_LMHEAD_TN=2, the default) or a 128-row one (1);
// TPL_LMHEAD_TN=0 keeps the swap-AB kernel for every batch.  Measured on one
// B200 at B = 32: even with swap-AB at a 1.8 GHz SM clock (within 1-3 us of
// 158 us), 18-29 us faster at 1.2-1.4 GHz.  Returns the A operand height, or 0.
int lmhead_tn_rows() {
  static const int v = env_int("TPL_LMHEAD_TN", 2);
  return v == 1 ? 128 : (v == 2 ? 64 : 0);
}

tpl_status lmhead_prepare(const void* x, int64_t B, int64_t K, const void* w, int64_t V,
                          int32_t tp, int32_t n_chunks, float* logits, float* shard_max,
                          int32_t* shard_idx, int32_t* ids, void* scratch, size_t ws_bytes,
                          tpl::LmArgs* a, int* smem, int* grid) {
  if (x == nullptr || w == nullptr || shard_max == nullptr || shard_idx == nullptr ||
      ids == nullptr || scratch == nullptr)
    return TPL_ERR_NULL;
  int64_t shard = 0;
  tpl_status s = lm_layout(B, V, tp, n_chunks, &shard);
  if (s != TPL_OK) return s;
  if (K < 1 || K > INT32_MAX) return TPL_ERR_SHAPE;
  size_t need = 0;
  tpl_lmhead_workspace_size(B, V, tp, n_chunks, &need);
  if (ws_bytes < need) return TPL_ERR_SHAPE;
  if (K % 8 != 0 || !aligned(x, 16) || !aligned(w, 16) || !aligned(scratch, 16) ||
      (logits && !aligned(logits, 4)) || !aligned(shard_max, 4) || !aligned(shard_idx, 4) ||
      !aligned(ids, 4))
    return TPL_ERR_ALIGN;
  DeviceInfo* dev = nullptr;
  if ((s = device_info(&dev)) != TPL_OK) return s;

  std::memset(a, 0, sizeof(*a));
  a->B = static_cast<int32_t>(B);
  a->Npad = static_cast<int32_t>((B + 15) / 16 * 16);
  // Slab height: the fewest rounds of at most 128-row slabs over the SMs, then
  // the shortest slab that still covers V in that many rounds, so every CTA
  // streams (nearly) the same number of rows.
  {
    const int64_t sms = dev->sm_count;
    const int64_t rounds = (V + sms * tpl::kLmRows - 1) / (sms * tpl::kLmRows);
    a->slab_rows = static_cast<int32_t>((V + sms * rounds - 1) / (sms * rounds));
  }
  {
    const uint64_t dims[2] = {static_cast<uint64_t>(K), static_cast<uint64_t>(V)};
    const uint64_t str[1] = {static_cast<uint64_t>(K) * 2};
    if ((s = encode_bf16(&a->tmW, w, 2, dims, str, static_cast<uint32_t>(a->slab_rows))) !=
        TPL_OK)
      return s;
  }
  {
    const uint64_t dims[2] = {static_cast<uint64_t>(K), static_cast<uint64_t>(B)};
    const uint64_t str[1] = {static_cast<uint64_t>(K) * 2};
    if ((s = encode_bf16(&a->tmX, x, 2, dims, str, static_cast<uint32_t>(a->Npad))) != TPL_OK)
      return s;
  }
  a->K = static_cast<int32_t>(K);
  a->k_iters = static_cast<int32_t>((K + tpl::kLmBK - 1) / tpl::kLmBK);
  a->V = static_cast<int32_t>(V);
  a->tp = tp;
  a->shard = static_cast<int32_t>(shard);
  a->n_slabs = static_cast<int32_t>((V + a->slab_rows - 1) / a->slab_rows);
  a->stage_bytes = tpl::kLmABytes + a->Npad * tpl::kLmBK * 2;
  const int budget = 227 * 1024 - 1024 - 256 - tpl::kLmTbufBytes;
  a->stages = std::min(tpl::kLmMaxStages, budget / a->stage_bytes);
  if (a->stages < 2) return TPL_ERR_UNSUPPORTED;
  uint32_t cols = 32;
  while (cols < static_cast<uint32_t>(2 * a->Npad)) cols <<= 1;
  a->tmem_cols = cols;
  a->logits = logits;
  a->shard_max = shard_max;
  a->shard_idx = shard_idx;
  a->ids = ids;
  a->keys = static_cast<unsigned long long*>(scratch);
  a->counter = reinterpret_cast<unsigned int*>(static_cast<char*>(scratch) +
                                               static_cast<size_t>(tp) * B * 8);
  *smem = a->stages * a->stage_bytes + 1024 + 256 + tpl::kLmTbufBytes;
  *grid = std::min(a->n_slabs, dev->sm_count);
  if (B <= 32 && lmhead_tn_rows() != 0) {
    // The batch as the M operand, vocab slabs as N (lmhead_tn.cuh).  An MMA
    // costs about the same whatever its N, so by default every CTA owns one
    // contiguous vocab range cut into 256-row slabs and one shorter last slab:
    // for V = 128256 on 148 SMs, 866-867 rows per CTA in 3 x 256 + 98/99, so
    // 4 x 256 MMAs per CTA instead of 5 x 256 with uniform slabs.
    // TPL_LMHEAD_RANGES=0: uniform slabs of 16..256 rows (a multiple of 16)
    // dealt out in turn, the height that gives the busiest CTA the fewest rows
    // (176 rows, 729 slabs, 880 rows on the busiest CTA).
    const int64_t sms = dev->sm_count;
    a->tn = lmhead_tn_rows();
    const uint64_t wd[2] = {static_cast<uint64_t>(K), static_cast<uint64_t>(V)};
    const uint64_t xd[2] = {static_cast<uint64_t>(K), static_cast<uint64_t>(B)};
    const uint64_t str[1] = {static_cast<uint64_t>(K) * 2};
    a->ranged = env_int("TPL_LMHEAD_RANGES", 1) != 0 ? 1 : 0;
    if (a->ranged) {
      const int64_t g = std::min<int64_t>(V, sms);
      a->range_base = static_cast<int32_t>(V / g);
      a->range_rem = static_cast<int32_t>(V % g);
      a->slab_rows = 256;
      // the longest last slab of any CTA (ranges of range_base or range_base + 1 rows)
      int64_t tail = a->range_base % 256;
      if (a->range_rem > 0 && (a->range_base + 1) % 256 > tail) tail = (a->range_base + 1) % 256;
      a->tail_rows = static_cast<int32_t>(tail > 0 ? tail : 256);
      a->tail_n = (a->tail_rows + 15) / 16 * 16;
      if ((s = encode_bf16(&a->tmWt, w, 2, wd, str, static_cast<uint32_t>(a->tail_rows))) !=
          TPL_OK)
        return s;
      a->n_slabs = static_cast<int32_t>(g);  // ranges, one per CTA
    } else {
      int64_t best_rows = INT64_MAX, best_r = 16;
      for (int64_t r = 256; r >= 16; r -= 16) {
        const int64_t slabs = (V + r - 1) / r;
        const int64_t busiest = (slabs + sms - 1) / sms * r;
        if (busiest < best_rows) {
          best_rows = busiest;
          best_r = r;
        }
      }
      a->slab_rows = static_cast<int32_t>(best_r);
      a->n_slabs = static_cast<int32_t>((V + a->slab_rows - 1) / a->slab_rows);
    }
    if ((s = encode_bf16(&a->tmW, w, 2, wd, str, static_cast<uint32_t>(a->slab_rows))) != TPL_OK)
      return s;
    if ((s = encode_bf16(&a->tmX, x, 2, xd, str, 32u)) != TPL_OK) return s;
    // the A operand (a->tn rows) and the W tile
    a->stage_bytes = a->tn * tpl::kLmBK * 2 + (a->slab_rows * tpl::kLmBK * 2 + 1023) / 1024 * 1024;
    a->stages = std::min(tpl::kLmMaxStages, (227 * 1024 - 1024 - 256) / a->stage_bytes);
    if (a->stages < 2) return TPL_ERR_UNSUPPORTED;
    a->tmem_cols = 2 * tpl::kLmTnAccCols;
    *smem = a->stages * a->stage_bytes + 1024 + 256;
    *grid = std::min(a->n_slabs, dev->sm_count);
  }
  return TPL_OK;
}

tpl_status lmhead_launch(const tpl::LmArgs& args, int smem, int grid, cudaStream_t st) {
  tpl::LmArgs a = args;
  a.trace_seq = static_cast<uint32_t>(g_launch_count.load(std::memory_order_relaxed));
  if (a.tn == 64)
    return launch_ex(tpl::lmhead_argmax_tn<64>, dim3(grid), dim3(tpl::LmTn<64>::kThreads),
                     static_cast<size_t>(smem), st, a);
  if (a.tn == 128)
    return launch_ex(tpl::lmhead_argmax_tn<128>, dim3(grid), dim3(tpl::LmTn<128>::kThreads),
                     static_cast<size_t>(smem), st, a);
  return launch_ex(tpl::lmhead_argmax_tcgen05, dim3(grid), dim3(tpl::kLmThreads),
                   static_cast<size_t>(smem), st, a);
}

}  // namespace

extern "C" {

tpl_status tpl_lmhead_argmax(const void* x, int64_t B, int64_t K, const void* w, int64_t V,
                             int32_t tp, int32_t n_chunks, float* logits, float* shard_max,
                             int32_t* shard_idx, int32_t* ids, void* workspace, size_t ws_bytes,
                             void* stream) {
  tpl::LmArgs a;
  int smem = 0, grid = 0;
  tpl_status s = lmhead_prepare(x, B, K, w, V, tp, n_chunks, logits, shard_max, shard_idx, ids,
                                workspace, ws_bytes, &a, &smem, &grid);
  if (s != TPL_OK) return s;
  return lmhead_launch(a, smem, grid, static_cast<cudaStream_t>(stream));
}

tpl_status tpl_tp_mlp_fp32(const float* x, int64_t M, int64_t H, const float* w1,
                          const float* b1, int64_t I, int32_t tp, tpl_act act, const float* w2,
                          const float* b2, const float* residual, float* y, void* stream) {
  if (act != TPL_ACT_NONE && act != TPL_ACT_GELU_ERF && act != TPL_ACT_GELU_TANH)
    return TPL_ERR_DTYPE;
  if (M < 0 || H < 1 || I < 1 || tp < 1 || tp > TPL_MAX_TP || H > INT32_MAX || I > INT32_MAX)
    return TPL_ERR_SHAPE;
  if (I % tp != 0) return TPL_ERR_INDIVISIBLE;
  // slices of I / 16 columns, each inside one rank's shard; 16-byte vectors
  if (tpl::kMlpSlices % tp != 0 || I % (4 * tpl::kMlpSlices) != 0 ||
      H % tpl::kMlpSlices != 0 || H % 4 != 0)
    return TPL_ERR_UNSUPPORTED;
  const int hc = static_cast<int>(I / tpl::kMlpSlices);
  const int64_t smem = tpl::mlp_smem_floats(static_cast<int>(H), hc) * 4;
  if (smem > 227 * 1024) return TPL_ERR_UNSUPPORTED;
  const int64_t mtiles = (M + tpl::kMlpRows - 1) / tpl::kMlpRows;
  if (mtiles > 65535) return TPL_ERR_SHAPE;
  if (M == 0) return TPL_OK;
  if (x == nullptr || w1 == nullptr || w2 == nullptr || y == nullptr) return TPL_ERR_NULL;
  if (!aligned(x, 16) || !aligned(w1, 16) || !aligned(w2, 16) || !aligned(y, 16) ||
      (b1 && !aligned(b1, 4)) || (b2 && !aligned(b2, 4)) || (residual && !aligned(residual, 4)))
    return TPL_ERR_ALIGN;
  DeviceInfo* dev = nullptr;
  tpl_status s = device_info(&dev);
  if (s != TPL_OK) return s;
  cudaLaunchConfig_t cfg;
  std::memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = dim3(tpl::kMlpSlices, static_cast<unsigned>(mtiles));
  cfg.blockDim = dim3(tpl::kMlpThreads);
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  cfg.stream = static_cast<cudaStream_t>(stream);
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = tpl::kMlpSlices;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  {
    // a 16-CTA cluster of this shared-memory size must fit one GPC of the device
    std::lock_guard<std::mutex> lk(g_mu);
    if (dev->mlp_clusters < 0) {
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, tpl::mlp_fp32_fused, &cfg) != cudaSuccess) n = 0;
      dev->mlp_clusters = n;
    }
    if (dev->mlp_clusters == 0) return TPL_ERR_UNSUPPORTED;
  }
  if (pdl_enabled()) {
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.numAttrs = 2;
  }
  tpl::MlpArgs a;
  a.x = x;
  a.w1 = w1;
  a.b1 = b1;
  a.w2 = w2;
  a.b2 = b2;
  a.residual = residual;
  a.y = y;
  a.M = M;
  a.H = static_cast<int32_t>(H);
  a.I = static_cast<int32_t>(I);
  a.kr = static_cast<int32_t>(I / tp);
  a.hc = hc;
  a.act = act;
  if (cudaLaunchKernelEx(&cfg, tpl::mlp_fp32_fused, a) != cudaSuccess) return TPL_ERR_CUDA;
  return launched();
}

tpl_status tpl_trace_set(void* buffer, int64_t capacity) {
  static_assert(sizeof(tpl::TraceRecord) == sizeof(tpl_trace_record), "record layout");
  static_assert(sizeof(tpl::TraceHeader) == TPL_TRACE_HEADER_BYTES, "header layout");
  tpl::TraceHeader* h = nullptr;
  if (buffer != nullptr) {
    if (capacity <= 0 || capacity > static_cast<int64_t>(UINT32_MAX)) return TPL_ERR_SHAPE;
    if (reinterpret_cast<uintptr_t>(buffer) % 16 != 0) return TPL_ERR_ALIGN;
    tpl::TraceHeader hdr{};
    hdr.capacity = static_cast<uint32_t>(capacity);
    if (cudaMemcpy(buffer, &hdr, sizeof(hdr), cudaMemcpyHostToDevice) != cudaSuccess)
      return TPL_ERR_CUDA;
    h = static_cast<tpl::TraceHeader*>(buffer);
  }
  if (cudaMemcpyToSymbol(tpl::g_trace, &h, sizeof(h)) != cudaSuccess) return TPL_ERR_CUDA;
  return cudaDeviceSynchronize() == cudaSuccess ? TPL_OK : TPL_ERR_CUDA;
}

tpl_status tpl_get_device_status(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return TPL_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, tpl::g_status_word, sizeof(int)) != cudaSuccess)
    return TPL_ERR_CUDA;
  if (v != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(tpl::g_status_word, &zero, sizeof(int)) != cudaSuccess)
      return TPL_ERR_CUDA;
    return static_cast<tpl_status>(v);
  }
  return TPL_OK;
}

}  // extern "C"

// ======================================================================
// LM head with library-owned scratch, for callers that cannot allocate
// ======================================================================

// Scratch of tpl_lmhead_argmax_static: per-(shard, row) keys and the
// completion counter.  A device global, so no call allocates; every GPU that
// loads the library holds it until the process exits.
static __device__ __align__(256) unsigned char g_lmhead_scratch[TPL_LMHEAD_STATIC_SCRATCH_BYTES];

namespace {

std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices];
unsigned long long g_scratch_ctx[kMaxDevices];

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

// Unique id (never reused within the process) of the CUDA context current on
// this thread; false if there is none yet.
bool current_context_id(unsigned long long* id) {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess && q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrentFn>(p);
    if (cudaGetDriverEntryPointByVersion("cuCtxGetId", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess && q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(p);
  });
  CUcontext ctx = nullptr;
  if (get_current == nullptr || get_id == nullptr || get_current(&ctx) != CUDA_SUCCESS ||
      ctx == nullptr)
    return false;
  return get_id(ctx, id) == CUDA_SUCCESS;
}

// Device address of g_lmhead_scratch on the current device.  In host code the
// array's name is only a host-side stand-in, so the kernel must be given this
// address instead.  It is looked up once per device and looked up again when
// the device's context has changed since (after cudaDeviceReset, the next
// call maps the array in the new context).
tpl_status lmhead_scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return TPL_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  unsigned long long ctx = 0;
  const bool have_ctx = current_context_id(&ctx);
  if (g_scratch_addr[dev] == nullptr || !have_ctx || ctx != g_scratch_ctx[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_lmhead_scratch) != cudaSuccess || p == nullptr)
      return TPL_ERR_CUDA;
    g_scratch_addr[dev] = p;
    g_scratch_ctx[dev] = current_context_id(&ctx) ? ctx : 0ull;
  }
  *out = g_scratch_addr[dev];
  return TPL_OK;
}

}  // namespace

extern "C" tpl_status tpl_lmhead_argmax_static(const void* x, int64_t B, int64_t K, const void* w,
                                               int64_t V, int32_t tp, int32_t n_chunks,
                                               float* logits, float* shard_max,
                                               int32_t* shard_idx, int32_t* ids, void* stream) {
  if (x == nullptr || w == nullptr || shard_max == nullptr || shard_idx == nullptr ||
      ids == nullptr)
    return TPL_ERR_NULL;
  size_t need = 0;
  tpl_status s = tpl_lmhead_workspace_size(B, V, tp, n_chunks, &need);
  if (s != TPL_OK) return s;
  if (need > static_cast<size_t>(TPL_LMHEAD_STATIC_SCRATCH_BYTES)) return TPL_ERR_SHAPE;
  void* scratch = nullptr;
  if ((s = lmhead_scratch_address(&scratch)) != TPL_OK) return s;
  // Every check of tpl_lmhead_argmax, and the kernel's arguments, before
  // anything is enqueued: a rejected call enqueues nothing, not even the clear.
  tpl::LmArgs a;
  int smem = 0, grid = 0;
  s = lmhead_prepare(x, B, K, w, V, tp, n_chunks, logits, shard_max, shard_idx, ids, scratch,
                     static_cast<size_t>(TPL_LMHEAD_STATIC_SCRATCH_BYTES), &a, &smem, &grid);
  if (s != TPL_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // The array keeps the previous call's contents: start this call from zero.
  if (cudaMemsetAsync(scratch, 0, need, st) != cudaSuccess) return TPL_ERR_CUDA;
  return lmhead_launch(a, smem, grid, st);
}

// Entry points of the next rows (same translation unit).
#include "tpl_next.cuh"
// The TP linears split over GPUs (same translation unit).
#include "tpl_ranks.cuh"
