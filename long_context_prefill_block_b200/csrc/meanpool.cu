// Block mean-pooling of keys (PaperTrace "2.1.3 MoBA", section 1, eq. 3):
// kbar_i = (1/B) * sum of the raw keys of block i, one routing vector per
// (sequence, block, kv head), fp32. Keys packed [T][Hkv][d] or, for decode
// caches, head-major [Hkv][T][d].
//
// One CTA per (block, sequence, kv head). Each thread owns 16 bytes of a key
// row (8 bf16 or 4 fp32 elements); a row is read by D*size/16 consecutive
// threads, so every warp load is contiguous 128-256 B. Rows of one block are
// spread over the CTA's row groups, summed in registers and reduced once in
// shared memory: K is read exactly once (HBM-bound).
//
// Incremental form (section 5.1, long outputs need incremental means): with
// cu_new, sequence b only recomputes the blocks that hold its last
// n_b = cu_new[b+1] - cu_new[b] positions (the tokens just appended to its
// cache); CTA x of the sequence takes the x-th of those blocks.
#include "common.cuh"

namespace moba {
namespace {

constexpr int kThreads = 256;

template <typename T, int D>
__global__ void __launch_bounds__(kThreads) meanpool_kernel(Dims dm, const T* __restrict__ k,
                                                            const int32_t* __restrict__ cu,
                                                            const int32_t* __restrict__ cu_new,
                                                            float* __restrict__ kbar,
                                                            int* status) {
  constexpr int VEC = Vec16<T>::N;   // elements per 16-byte load
  constexpr int TPR = D / VEC;       // threads per key row
  constexpr int RG = kThreads / TPR; // rows in flight
  __shared__ float red[RG][D + 1];

  const int b = blockIdx.y, g = blockIdx.z;
  int i = blockIdx.x;
  int64_t start;
  int len;
  const bool ok = seq_bounds(dm, cu, b, start, len, status);
  if (cu_new) {
    if (!ok) return;
    const int n = cu_new[b + 1] - cu_new[b];
    if (n < 0 || n > len) {
      set_status(status, kStInvalidArg);
      return;
    }
    if (n == 0) return;
    i += (len - n) / dm.B;
    if (i * dm.B >= len) return;
  }
  const int j0 = i * dm.B;
  const int j1 = ok ? min(len, j0 + dm.B) : j0;
  const int lane = threadIdx.x % TPR, rg = threadIdx.x / TPR;

  float acc[VEC];
#pragma unroll
  for (int e = 0; e < VEC; ++e) acc[e] = 0.f;
  // unrolled so that several rows' loads are in flight per thread
#pragma unroll 8
  for (int j = j0 + rg; j < j1; j += RG) {
    float x[VEC];
    Vec16<T>::load(k + kv_row(dm, start + j, g) + lane * VEC, x);
#pragma unroll
    for (int e = 0; e < VEC; ++e) acc[e] += x[e];
  }
#pragma unroll
  for (int e = 0; e < VEC; ++e) red[rg][lane * VEC + e] = acc[e];
  __syncthreads();
  if (threadIdx.x < D) {
    float s = 0.f;
#pragma unroll 8
    for (int r = 0; r < RG; ++r) s += red[r][threadIdx.x];
    const int n = j1 - j0;
    kbar[(((int64_t)b * dm.nb + i) * dm.Hkv + g) * D + threadIdx.x] = n > 0 ? s / (float)n : 0.f;
  }
}

template <typename T, int D>
cudaError_t run(const Dims& dm, const void* k, const int32_t* cu, const int32_t* cu_new,
                int nblk, float* kbar, int* status, cudaStream_t st) {
  dim3 grid(nblk, dm.batch, dm.Hkv);
  meanpool_kernel<T, D><<<grid, kThreads, 0, st>>>(dm, static_cast<const T*>(k), cu, cu_new, kbar,
                                                   status);
  return cudaGetLastError();
}

cudaError_t launch(const Dims& dm, const void* k, const int32_t* cu, const int32_t* cu_new,
                   int nblk, float* kbar, int* status, cudaStream_t st) {
  if (dm.batch == 0 || nblk == 0) return cudaSuccess;
  if (dm.dtype == kBF16)
    return dm.d == 128 ? run<__nv_bfloat16, 128>(dm, k, cu, cu_new, nblk, kbar, status, st)
                       : run<__nv_bfloat16, 64>(dm, k, cu, cu_new, nblk, kbar, status, st);
  return dm.d == 128 ? run<float, 128>(dm, k, cu, cu_new, nblk, kbar, status, st)
                     : run<float, 64>(dm, k, cu, cu_new, nblk, kbar, status, st);
}

}  // namespace

cudaError_t launch_meanpool(const Dims& dm, const void* k, const int32_t* cu, float* kbar,
                            int* status, cudaStream_t st) {
  return launch(dm, k, cu, nullptr, dm.nb, kbar, status, st);
}

cudaError_t launch_meanpool_update(const Dims& dm, const void* k, const int32_t* cu,
                                   const int32_t* cu_new, int max_new, float* kbar, int* status,
                                   cudaStream_t st) {
  if (max_new <= 0) return cudaSuccess;
  // n new positions touch at most ceil((n - 1) / B) + 1 blocks
  const int64_t nblk = (int64_t)(max_new - 1) / dm.B + 2;
  return launch(dm, k, cu, cu_new, (int)(nblk < dm.nb ? nblk : dm.nb), kbar, status, st);
}

}  // namespace moba
