// trace.cuh -- optional per-CTA timing records of the tensor-core kernels.
//
// When a trace buffer is installed (tpl_trace_set), thread 0 of every CTA of
// the GEMM and LM-head kernels appends one record when the CTA finishes: the
// launch's sequence number, the kernel kind, the CTA index, %globaltimer (ns)
// when the CTA passed its wait on the previous kernel and when it finished,
// and the SM cycles (%clock64) between the two.  cycles / (t1 - t0) is the SM
// clock the CTA actually ran at, which the host cannot read for a launch of a
// few hundred microseconds (nvidia-smi and NVML report a sampled clock).
// With no buffer installed the cost is one load of a device pointer per CTA.
#pragma once

#include <cstdint>

#include "ptx.cuh"

namespace tpl {

enum TraceKind : uint16_t { kTraceGemm = 1, kTraceGemmPair = 2, kTraceLmHead = 3 };

struct TraceRecord {   // 32 bytes; layout mirrored by tpl_trace_record in include/tpl.h
  uint32_t seq;        // the launch's number in the library's launch counter
  uint16_t kind;       // TraceKind
  uint16_t cta;        // blockIdx.x
  uint64_t t0_ns, t1_ns;
  uint64_t cycles;
};

struct TraceHeader {   // 16 bytes, followed by `capacity` records
  uint32_t count;      // records claimed so far (may exceed capacity: the rest were dropped)
  uint32_t capacity;
  uint32_t pad[2];
};

__device__ TraceHeader* g_trace;  // null: tracing off

struct TraceStamp {
  long long c0;
  uint64_t t0;
};

__device__ __forceinline__ TraceStamp trace_begin() {
  TraceStamp s;
  s.c0 = clock64();
  s.t0 = ptx::globaltimer();
  return s;
}

// Called by one thread of the CTA after its last global store.
__device__ __forceinline__ void trace_end(const TraceStamp& s, uint16_t kind, uint32_t seq) {
  TraceHeader* h = *const_cast<TraceHeader* volatile*>(&g_trace);
  if (h == nullptr) return;
  const long long c1 = clock64();
  const uint64_t t1 = ptx::globaltimer();
  const uint32_t i = atomicAdd(&h->count, 1u);
  if (i >= h->capacity) return;
  TraceRecord* r = reinterpret_cast<TraceRecord*>(h + 1) + i;
  r->seq = seq;
  r->kind = kind;
  r->cta = static_cast<uint16_t>(blockIdx.x);
  r->t0_ns = s.t0;
  r->t1_ns = t1;
  r->cycles = static_cast<uint64_t>(c1 - s.c0);
}

}  // namespace tpl
