// Phase traces of the tensor-core kernels, compiled in only when MOBA_TRACE
// is defined (the separate libmoba_trace.so build; the ordinary library
// carries none of it): lane 0 of every warp of one chosen CTA of one chosen
// kernel records (SM clock, event id, argument) into a caller-provided
// device buffer, one region per warp, with plain stores (no atomics on the
// timed path). Every MOBA_TRACE_* macro expands to nothing otherwise.
//
// Device symbols cannot be shared between the library's files (they are
// compiled without relocatable device code), so each traced file holds its
// own copy of the target description; a host-side registry in api.cu sets
// every copy when moba_trace_arm() is called.
#pragma once

#ifdef MOBA_TRACE
#include <cuda_runtime.h>
#include <stdint.h>

namespace moba {
namespace trace {

struct Target {
  unsigned long long* buf;  // [kMaxWarps][cap][2]: clock64, id | arg << 32
  int* counts;              // [kMaxWarps] records written per warp
  int cap;                  // records per warp
  int cta;                  // blockIdx.x of the CTA that records
  int kernel;               // which kernel records (Kernel below)
};

enum Kernel { kGateNet = 1, kAttnHist = 2, kAttnCur = 3, kAttnDense = 4 };
constexpr int kMaxWarps = 16;

// Host registry (api.cu): every traced file registers a setter of its copy.
void add_setter(cudaError_t (*fn)(const Target&));

namespace {
__device__ Target d_target;
cudaError_t set_target(const Target& t) { return cudaMemcpyToSymbol(d_target, &t, sizeof t); }
struct Registrar {
  Registrar() { add_setter(&set_target); }
} registrar;
}  // namespace

__device__ __forceinline__ bool armed(int kernel) {
  return d_target.buf != nullptr && d_target.kernel == kernel && (int)blockIdx.x == d_target.cta;
}

__device__ __forceinline__ void record(int& n, int id, int arg) {
  if (n < d_target.cap) {
    unsigned long long* p =
        d_target.buf + ((size_t)(threadIdx.x >> 5) * d_target.cap + n) * 2;
    p[0] = (unsigned long long)clock64();
    p[1] = (unsigned long long)(unsigned)id | ((unsigned long long)(unsigned)arg << 32);
  }
  ++n;
}

}  // namespace trace
}  // namespace moba

#define MOBA_TRACE_STATE(kernel)                                                          \
  const bool trace_on_ = moba::trace::armed(kernel) && (threadIdx.x & 31) == 0;          \
  int trace_n_ = 0
#define MOBA_TRACE(id, arg)                                       \
  do {                                                            \
    if (trace_on_) moba::trace::record(trace_n_, (id), (arg));    \
  } while (0)
#define MOBA_TRACE_END()                                                                   \
  do {                                                                                     \
    if (trace_on_) moba::trace::d_target.counts[threadIdx.x >> 5] = trace_n_;             \
  } while (0)
#else
#define MOBA_TRACE_STATE(kernel) \
  do {                           \
  } while (0)
#define MOBA_TRACE(id, arg) \
  do {                      \
  } while (0)
#define MOBA_TRACE_END() \
  do {                   \
  } while (0)
#endif
