// embed.cuh -- vocab-sharded embedding lookup (google-research embed_manual,
// 'embed' scope): every rank r owns table rows r*shard .. (r+1)*shard, looks up
// one_x = id - r*shard, keeps the row where 0 <= one_x < its row count, and the
// embedding is the sum over ranks.  On one GPU all shards are local, so exactly
// one rank contributes for an id in [0, V) and none for any other id.
//
// HBM-bound gather: one warp per token, 16-byte vectors when the row allows,
// fp32 accumulation over the (masked) shards, one rounding on store.
#pragma once

#include "common.cuh"
#include "rmsnorm.cuh"  // VecTraits

namespace tpl {

constexpr int kEmbedWarps = 8;
constexpr int kEmbedBatch = 8;  // 16-byte vectors per lane in flight

template <typename T, bool kVec>
__global__ void __launch_bounds__(kEmbedWarps * 32)
    embedding_lookup_kernel(const int32_t* __restrict__ ids, int64_t n, const T* __restrict__ table,
                            int64_t V, int64_t H, int tp, int64_t shard, T* __restrict__ out) {
  using VT = VecTraits<T>;
  constexpr int P = VT::kPer;
  const int lane = threadIdx.x & 31;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * kEmbedWarps + (threadIdx.x >> 5); i < n;
       i += static_cast<int64_t>(gridDim.x) * kEmbedWarps) {
    const int64_t id = ids[i];
    // The rank whose shard holds this id, if any (the others are masked to 0).
    int64_t row = -1;
    for (int r = 0; r < tp; ++r) {
      const int64_t start = static_cast<int64_t>(r) * shard;
      const int64_t rows = max(static_cast<int64_t>(0), min(shard, V - start));
      const int64_t local = id - start;
      if (local >= 0 && local < rows) row = start + local;
    }
    T* dst = out + i * H;
    if (kVec) {
      // kEmbedBatch vectors per lane are loaded before any is stored, so a warp
      // keeps kEmbedBatch * 512 bytes of the row in flight.
      const int64_t nv = H / P;
      const uint4* src = reinterpret_cast<const uint4*>(table + (row < 0 ? 0 : row) * H);
      for (int64_t v0 = lane; v0 < nv; v0 += 32 * kEmbedBatch) {
        uint4 q[kEmbedBatch];
#pragma unroll
        for (int u = 0; u < kEmbedBatch; ++u) {
          const int64_t v = v0 + 32 * u;
          q[u] = (row >= 0 && v < nv) ? __ldcs(src + v) : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int u = 0; u < kEmbedBatch; ++u) {
          const int64_t v = v0 + 32 * u;
          if (v < nv) {
            float f[P], acc[P];
            VT::unpack(q[u], f);
#pragma unroll
            for (int e = 0; e < P; ++e) acc[e] = 0.0f + f[e];
            __stcs(reinterpret_cast<uint4*>(dst) + v, VT::pack(acc));
          }
        }
      }
    } else {
      for (int64_t c = lane; c < H; c += 32) {
        float acc = 0.0f;
        if (row >= 0) acc += VT::load1(table + row * H + c);
        VT::store1(dst + c, acc);
      }
    }
  }
}

}  // namespace tpl
