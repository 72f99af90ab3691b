// Own-block routing score by prefix mean (PaperTrace "2.1.3 MoBA", section
// 5.2, the paragraph on causal blocks: the full mean of the query's own block
// holds keys after the query, so a gate that scores the own block uses the
// mean of its keys up to the query instead). For query p of block c:
//   own[t][h] = q_{t,h} . (1/(p - cB + 1)) sum_{j=cB..p} k_j      (fp32)
// The gate then ranks it against the earlier blocks' q . kbar_i.
//
// Two launches, both over (32-row chunk of a block, sequence, kv head), so
// that every CTA does one short piece of work and the grid fills the GPU:
//   chunk_sum_kernel  sums the keys of each chunk (fp32) into a scratch table;
//   own_dot_kernel    starts from the sum of the block's earlier chunks, turns
//                     its own chunk into running prefix sums in shared memory
//                     and dots each prefix row with the q rows of the group
//                     (a warp per (row, q head), D/32 columns per lane).
// K is read twice and Q once (HBM-bound); the chunk sums stay in L2.
#include "common.cuh"

namespace moba {
namespace {

constexpr int kThreads = 128;
constexpr int kRows = kOwnChunkRows;  // rows per chunk

// PL consecutive elements (PL * sizeof(T) bytes, aligned to that) widened to fp32.
template <typename T, int PL>
__device__ __forceinline__ void load_pl(const T* p, float (&x)[PL]) {
  if constexpr (sizeof(T) == 2) {
    if constexpr (PL == 4) {
      const uint2 w = *reinterpret_cast<const uint2*>(p);
      x[0] = __uint_as_float(w.x << 16);
      x[1] = __uint_as_float(w.x & 0xffff0000u);
      x[2] = __uint_as_float(w.y << 16);
      x[3] = __uint_as_float(w.y & 0xffff0000u);
    } else {
      const uint32_t w = *reinterpret_cast<const uint32_t*>(p);
      x[0] = __uint_as_float(w << 16);
      x[1] = __uint_as_float(w & 0xffff0000u);
    }
  } else {
#pragma unroll
    for (int u = 0; u < PL; ++u) x[u] = to_f32(p[u]);
  }
}

// Rows [r0, r1) of chunk x (block i, chunk ch of the block) of a sequence of
// len tokens, or false if the chunk starts past the sequence's end.
__device__ __forceinline__ bool chunk_rows(const Dims& dm, int x, int len, int& i, int& ch, int& r0,
                                           int& r1) {
  const int cpb = own_chunks_per_block(dm);
  i = x / cpb;
  ch = x % cpb;
  r0 = i * dm.B + ch * kRows;
  if (r0 >= len) return false;
  r1 = min(min(r0 + kRows, (i + 1) * dm.B), len);
  return true;
}

// First float of the chunk sum of (sequence b, block i, chunk ch, kv head g).
__device__ __forceinline__ int64_t chunk_slot(const Dims& dm, int b, int i, int ch, int g) {
  return ((((int64_t)b * dm.nb + i) * own_chunks_per_block(dm) + ch) * dm.Hkv + g) * dm.d;
}

template <typename T, int D>
__global__ void __launch_bounds__(kThreads) chunk_sum_kernel(Dims dm, const T* __restrict__ k,
                                                             const int32_t* __restrict__ cu,
                                                             float* __restrict__ csum,
                                                             int* status) {
  constexpr int VEC = Vec16<T>::N, TPR = D / VEC, RG = kThreads / TPR;
  __shared__ float red[RG][D + 1];
  const int b = blockIdx.y, g = blockIdx.z;
  int64_t start;
  int len, i, ch, r0, r1;
  if (!seq_bounds(dm, cu, b, start, len, status)) return;
  if (!chunk_rows(dm, blockIdx.x, len, i, ch, r0, r1)) return;
  const int lane = threadIdx.x % TPR, rg = threadIdx.x / TPR;
  float acc[VEC];
#pragma unroll
  for (int e = 0; e < VEC; ++e) acc[e] = 0.f;
#pragma unroll
  for (int j = r0 + rg; j < r1; j += RG) {
    float x[VEC];
    Vec16<T>::load(k + ((start + j) * dm.Hkv + g) * (int64_t)D + lane * VEC, x);
#pragma unroll
    for (int e = 0; e < VEC; ++e) acc[e] += x[e];
  }
#pragma unroll
  for (int e = 0; e < VEC; ++e) red[rg][lane * VEC + e] = acc[e];
  __syncthreads();
  if (threadIdx.x < D) {
    float s = 0.f;
#pragma unroll
    for (int r = 0; r < RG; ++r) s += red[r][threadIdx.x];
    csum[chunk_slot(dm, b, i, ch, g) + threadIdx.x] = s;
  }
}

template <typename T, int D>
__global__ void __launch_bounds__(kThreads) own_dot_kernel(Dims dm, const T* __restrict__ q,
                                                           const T* __restrict__ k,
                                                           const int32_t* __restrict__ cu,
                                                           const float* __restrict__ csum,
                                                           float* __restrict__ own) {
  __shared__ __align__(16) float ks[kRows][D];
  constexpr int VEC = Vec16<T>::N, TPR = D / VEC;  // 16-byte loads per key row
  constexpr int PL = D / 32;                       // columns per lane in the dot products
  const int b = blockIdx.y, g = blockIdx.z;
  int64_t start;
  int len, i, ch, r0, r1;
  if (!seq_bounds(dm, cu, b, start, len, nullptr)) return;
  if (!chunk_rows(dm, blockIdx.x, len, i, ch, r0, r1)) return;
  const int nr = r1 - r0, j0 = i * dm.B;
  const int grp = dm.Hq / dm.Hkv;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int e = threadIdx.x; e < kRows * TPR; e += kThreads) {
    const int r = e / TPR, l = e % TPR;
    float x[VEC];
    if (r < nr) {
      Vec16<T>::load(k + ((start + r0 + r) * dm.Hkv + g) * (int64_t)D + l * VEC, x);
    } else {
#pragma unroll
      for (int u = 0; u < VEC; ++u) x[u] = 0.f;
    }
#pragma unroll
    for (int u = 0; u < VEC; u += 4)
      *reinterpret_cast<float4*>(&ks[r][l * VEC + u]) = make_float4(x[u], x[u + 1], x[u + 2], x[u + 3]);
  }
  // column x: the keys of the block's earlier chunks, then the running sum
  float carry = 0.f;
  if (threadIdx.x < D) {
    const float* src = csum + chunk_slot(dm, b, i, 0, g) + threadIdx.x;
    const int64_t stride = (int64_t)dm.Hkv * D;
#pragma unroll 4
    for (int c2 = 0; c2 < ch; ++c2) carry += src[c2 * stride];
  }
  __syncthreads();
  if (threadIdx.x < D) {
    for (int r = 0; r < nr; ++r) {
      carry += ks[r][threadIdx.x];
      ks[r][threadIdx.x] = carry;
    }
  }
  __syncthreads();
  // independent iterations: several q rows in flight per warp
#pragma unroll 4
  for (int e = warp; e < nr * grp; e += kThreads / 32) {
    const int r = e / grp, h = g * grp + e % grp;
    const int64_t t = start + r0 + r;
    float qv[PL];
    load_pl<T, PL>(q + (t * dm.Hq + h) * (int64_t)D + lane * PL, qv);
    float acc = 0.f;
#pragma unroll
    for (int u = 0; u < PL; ++u) acc = fmaf(qv[u], ks[r][lane * PL + u], acc);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (lane == 0) own[t * dm.Hq + h] = acc / (float)(r0 + r - j0 + 1);
  }
}

template <typename T, int D>
cudaError_t run(const Dims& dm, const void* q, const void* k, const int32_t* cu, float* own,
                float* csum, int* status, cudaStream_t st) {
  dim3 grid(dm.nb * own_chunks_per_block(dm), dm.batch, dm.Hkv);
  chunk_sum_kernel<T, D><<<grid, kThreads, 0, st>>>(dm, static_cast<const T*>(k), cu, csum,
                                                    status);
  own_dot_kernel<T, D><<<grid, kThreads, 0, st>>>(dm, static_cast<const T*>(q),
                                                  static_cast<const T*>(k), cu, csum, own);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_own_score(const Dims& dm, const void* q, const void* k, const int32_t* cu,
                             float* own, float* csum, int* status, cudaStream_t st) {
  if (dm.batch == 0 || dm.nb == 0) return cudaSuccess;
  if ((int64_t)dm.nb * own_chunks_per_block(dm) > INT32_MAX) return cudaErrorInvalidValue;
  if (dm.dtype == kBF16)
    return dm.d == 128 ? run<__nv_bfloat16, 128>(dm, q, k, cu, own, csum, status, st)
                       : run<__nv_bfloat16, 64>(dm, q, k, cu, own, csum, status, st);
  return dm.d == 128 ? run<float, 128>(dm, q, k, cu, own, csum, status, st)
                     : run<float, 64>(dm, q, k, cu, own, csum, status, st);
}

}  // namespace moba
