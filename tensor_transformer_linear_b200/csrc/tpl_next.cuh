// tpl_next.cuh -- entry points of the path's next rows: sequence-parallel
// reduce-scatter / all-gather layouts around the TP linears, the fused SwiGLU
// column linear and the vocab-sharded embedding lookup.  Included at the end
// of tpl_api.cu (one translation unit with the helpers it uses).
#pragma once

#include "embed.cuh"

namespace {

tpl_status seqpar_of(int64_t batch, int64_t seq, int32_t tp, SeqPar* sp) {
  if (batch < 1 || seq < 1 || tp < 1 || tp > TPL_MAX_TP) return TPL_ERR_SHAPE;
  if (seq % tp != 0) return TPL_ERR_INDIVISIBLE;
  if (batch * seq > INT32_MAX) return TPL_ERR_SHAPE;
  sp->batch = static_cast<int32_t>(batch);
  sp->seq = static_cast<int32_t>(seq);
  sp->seg = static_cast<int32_t>(seq / tp);
  return TPL_OK;
}

}  // namespace

extern "C" {

tpl_status tpl_row_linear_reduce_scatter(const void* h, const int64_t* k_w, int32_t tp,
                                         int64_t batch, int64_t seq, int64_t N, const void* w,
                                         const void* bias, const void* residual, tpl_dtype dt,
                                         void* y, void* stream) {
  if (k_w == nullptr) return TPL_ERR_NULL;
  if (dt != TPL_FP32 && dt != TPL_BF16) return TPL_ERR_DTYPE;
  SeqPar sp;
  tpl_status s = seqpar_of(batch, seq, tp, &sp);
  if (s != TPL_OK) return s;
  sp.out_remap = 1;
  if (N < 1 || N > INT32_MAX) return TPL_ERR_SHAPE;
  int64_t ktot = 0;
  for (int r = 0; r < tp; ++r) {
    if (k_w[r] < 1 || k_w[r] > INT32_MAX) return TPL_ERR_SHAPE;
    ktot += k_w[r];
  }
  if (ktot > INT32_MAX) return TPL_ERR_SHAPE;
  if (h == nullptr || w == nullptr || y == nullptr) return TPL_ERR_NULL;
  const int64_t M = batch * seq;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return dt == TPL_BF16 ? row_bf16(h, k_w, tp, M, N, w, bias, residual, y, nullptr, st, sp)
                        : row_fp32(h, k_w, tp, M, N, w, bias, residual, y, nullptr, st, sp);
}

tpl_status tpl_column_linear_allgather(const tpl_partition* p, const void* x, int64_t batch,
                                       int64_t seq, int64_t K, const void* w, const void* bias,
                                       tpl_dtype dt, tpl_act act, void* y, void* stream) {
  if (p == nullptr) return TPL_ERR_NULL;
  if ((dt != TPL_FP32 && dt != TPL_BF16) || !act_ok(act)) return TPL_ERR_DTYPE;
  tpl_status s = check_partition(p);
  if (s != TPL_OK) return s;
  SeqPar sp;
  if ((s = seqpar_of(batch, seq, p->tp_size, &sp)) != TPL_OK) return s;
  sp.a_remap = 1;
  if (K < 1 || K > INT32_MAX) return TPL_ERR_SHAPE;
  if (x == nullptr || w == nullptr || y == nullptr) return TPL_ERR_NULL;
  // The tensor-core path reads A in 128-row TMA boxes that must stay inside one
  // rank's token slice.
  if (dt == TPL_BF16 && sp.seg % tpl::kBM != 0) return TPL_ERR_UNSUPPORTED;
  const int64_t M = batch * seq;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return dt == TPL_BF16 ? column_bf16(p, x, M, K, w, bias, act, y, st, sp)
                        : column_fp32(p, x, M, K, w, bias, act, y, st, sp);
}

tpl_status tpl_swiglu_column_linear(const void* x, int64_t M, int64_t K, const void* w, int64_t F,
                                    int32_t tp, tpl_dtype dt, void* h, void* stream) {
  if (dt != TPL_FP32 && dt != TPL_BF16) return TPL_ERR_DTYPE;
  if (dt != TPL_BF16) return TPL_ERR_UNSUPPORTED;
  if (tp < 1 || tp > TPL_MAX_TP || M < 0 || M > INT32_MAX || K < 1 || K > INT32_MAX || F < 1 ||
      2 * F > INT32_MAX)
    return TPL_ERR_SHAPE;
  tpl_partition part;
  tpl_status s = tpl_partition_subparams(&F, 1, tp, 1, &part);
  if (s != TPL_OK) return s;
  if (M == 0) return TPL_OK;
  if (x == nullptr || w == nullptr || h == nullptr) return TPL_ERR_NULL;
  if ((K % 8) != 0 || !aligned(x, 16) || !aligned(w, 16) || !aligned(h, 2)) return TPL_ERR_ALIGN;
  DeviceInfo* dev = nullptr;
  if ((s = device_info(&dev)) != TPL_OK) return s;

  tpl::GemmArgs a;
  std::memset(&a, 0, sizeof(a));
  {
    const uint64_t dims[2] = {static_cast<uint64_t>(K), static_cast<uint64_t>(M)};
    const uint64_t str[1] = {static_cast<uint64_t>(K) * 2};
    if ((s = encode_bf16(&a.tmA, x, 2, dims, str, tpl::kBM)) != TPL_OK) return s;
  }
  {
    const uint64_t dims[2] = {static_cast<uint64_t>(K), static_cast<uint64_t>(2 * F)};
    const uint64_t str[1] = {static_cast<uint64_t>(K) * 2};
    if ((s = encode_bf16(&a.tmB, w, 2, dims, str, tpl::kHalfN)) != TPL_OK) return s;
  }
  a.mode = tpl::kModeSwiglu;
  a.act = TPL_ACT_NONE;
  a.M = static_cast<int32_t>(M);
  a.k_iters = static_cast<int32_t>((K + tpl::kBK - 1) / tpl::kBK);
  a.y = static_cast<__nv_bfloat16*>(h);
  int tiles = 0;
  bool vec = aligned(h, 16);
  a.n_pieces = tp;
  for (int r = 0; r < tp; ++r) {
    ColPiece c;
    std::memset(&c, 0, sizeof(c));
    c.out_off = M * part.shard_base[r];
    c.src_row = static_cast<int32_t>(part.src_off[r][0]);
    c.src_row1 = static_cast<int32_t>(F + part.src_off[r][0]);
    c.width = static_cast<int32_t>(part.width[r][0]);
    c.ld = static_cast<int32_t>(part.shard_width[r]);
    c.hb_begin = tiles;
    tiles += (c.width + tpl::kHalfN - 1) / tpl::kHalfN;
    vec = vec && (c.out_off % 8 == 0) && (c.ld % 8 == 0);
    a.pieces[r] = c;
  }
  a.n_tiles = tiles;
  a.n_halves = 2 * tiles;
  a.vec_store = vec ? 1 : 0;
  return launch_gemm(a, M, dev, static_cast<cudaStream_t>(stream));
}

tpl_status tpl_embedding_lookup(const int32_t* ids, int64_t n, const void* table, int64_t V,
                                int64_t H, int32_t tp, tpl_dtype dt, void* out, void* stream) {
  if (dt != TPL_FP32 && dt != TPL_BF16) return TPL_ERR_DTYPE;
  if (n < 0 || V < 1 || V > INT32_MAX || H < 1 || H > INT32_MAX || tp < 1 || tp > TPL_MAX_TP)
    return TPL_ERR_SHAPE;
  if (n == 0) return TPL_OK;
  if (ids == nullptr || table == nullptr || out == nullptr) return TPL_ERR_NULL;
  const uintptr_t es = dt == TPL_BF16 ? 2 : 4;
  if (!aligned(ids, 4) || !aligned(table, es) || !aligned(out, es)) return TPL_ERR_ALIGN;
  DeviceInfo* dev = nullptr;
  tpl_status s = device_info(&dev);
  if (s != TPL_OK) return s;
  const int64_t shard = (V + tp - 1) / tp;
  const int per = dt == TPL_BF16 ? 8 : 4;
  const bool vec = (H % per == 0) && aligned(table, 16) && aligned(out, 16);
  const int64_t blocks = std::min<int64_t>((n + tpl::kEmbedWarps - 1) / tpl::kEmbedWarps,
                                           static_cast<int64_t>(dev->sm_count) * 16);
  const int g = static_cast<int>(blocks), t = tpl::kEmbedWarps * 32;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (dt == TPL_BF16) {
    const auto* tb = static_cast<const __nv_bfloat16*>(table);
    auto* o = static_cast<__nv_bfloat16*>(out);
    if (vec)
      tpl::embedding_lookup_kernel<__nv_bfloat16, true><<<g, t, 0, st>>>(ids, n, tb, V, H, tp, shard, o);
    else
      tpl::embedding_lookup_kernel<__nv_bfloat16, false><<<g, t, 0, st>>>(ids, n, tb, V, H, tp, shard, o);
  } else {
    const auto* tb = static_cast<const float*>(table);
    auto* o = static_cast<float*>(out);
    if (vec)
      tpl::embedding_lookup_kernel<float, true><<<g, t, 0, st>>>(ids, n, tb, V, H, tp, shard, o);
    else
      tpl::embedding_lookup_kernel<float, false><<<g, t, 0, st>>>(ids, n, tb, V, H, tp, shard, o);
  }
  return launched();
}

}  // extern "C"

// ======================================================================
// Self-test of the bounded pipeline waits
// ======================================================================

namespace tpl {

// One thread waits, with the same bounded wait every pipeline of this library
// uses, on an mbarrier that nothing ever arrives on; when the limit runs out
// it records TPL_ERR_TIMEOUT in the status word and returns normally.
__global__ void selftest_wait_timeout_kernel(uint64_t limit_ns, int* waited) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    ptx::mbar_init(&bar, 1);
    abort_flag = 0;
    ptx::fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const uint64_t t0 = ptx::globaltimer();
    if (!ptx::mbar_wait(&bar, 0, &abort_flag, limit_ns)) record_timeout();
    if (waited != nullptr) *waited = static_cast<int>((ptx::globaltimer() - t0) / 1000);
  }
}

}  // namespace tpl

extern "C" tpl_status tpl_selftest_wait_timeout(uint64_t limit_ns, int32_t* waited_us,
                                                void* stream) {
  if (limit_ns == 0 || limit_ns > 1000000000ull) return TPL_ERR_SHAPE;
  if (waited_us != nullptr && !aligned(waited_us, 4)) return TPL_ERR_ALIGN;
  tpl::selftest_wait_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
      limit_ns, waited_us);
  return launched();
}
