// Branch-free sorting networks on 16 keys, in registers (compile-time
// indices only), for the gate's top-k selection. Keys are 32-bit unsigned
// integers or fp32 values (compared with float max / min; keys are never
// NaN).
//
// oe_sort16: Batcher's odd-even merge sort (63 compare-exchanges),
// descending: v[0] ends up the largest. merge_top16: given two descending
// lists of 16, leaves the 16 largest of their union in the first, descending
// (elementwise max of the first with the second reversed gives a bitonic
// sequence holding the 16 largest; a bitonic merger of 32 compare-exchanges
// sorts it). Each compare-exchange is one max and one min.
//
// __host__ __device__ so the networks can be checked exhaustively on the host
// (0-1 principle: a network sorts every input iff it sorts every 0/1 input).
#pragma once

#include <math.h>
#include <stdint.h>
#include <string.h>

namespace moba {
namespace net {

__host__ __device__ __forceinline__ uint32_t kmax(uint32_t a, uint32_t b) { return a > b ? a : b; }
__host__ __device__ __forceinline__ uint32_t kmin(uint32_t a, uint32_t b) { return a > b ? b : a; }
__host__ __device__ __forceinline__ float kmax(float a, float b) { return fmaxf(a, b); }
__host__ __device__ __forceinline__ float kmin(float a, float b) { return fminf(a, b); }

template <typename K>
__host__ __device__ __forceinline__ void cx(K& a, K& b) {
  const K hi = kmax(a, b);
  const K lo = kmin(a, b);
  a = hi;
  b = lo;
}

// Merges the two sorted halves of v[LO .. LO+N) taking every R-th element.
template <int LO, int N, int R, typename K>
__host__ __device__ __forceinline__ void oe_merge(K (&v)[16]) {
  constexpr int M = 2 * R;
  if constexpr (M < N - 1) {
    oe_merge<LO, N, M>(v);
    oe_merge<LO + R, N, M>(v);
#pragma unroll
    for (int i = LO + R; i + R < LO + N; i += M) cx(v[i], v[i + R]);
  } else {
    cx(v[LO], v[LO + R]);
  }
}

template <int LO, int N, typename K>
__host__ __device__ __forceinline__ void oe_sort(K (&v)[16]) {
  if constexpr (N > 1) {
    oe_sort<LO, N / 2>(v);
    oe_sort<LO + N / 2, N / 2>(v);
    oe_merge<LO, N, 1>(v);
  }
}

template <typename K>
__host__ __device__ __forceinline__ void oe_sort16(K (&v)[16]) {
  oe_sort<0, 16>(v);
}

// l, g sorted descending; l <- the 16 largest of l and g, descending.
template <typename K>
__host__ __device__ __forceinline__ void merge_top16(K (&l)[16], const K (&g)[16]) {
#pragma unroll
  for (int i = 0; i < 16; ++i) l[i] = kmax(l[i], g[15 - i]);
#pragma unroll
  for (int s = 8; s >= 1; s >>= 1)
#pragma unroll
    for (int i = 0; i < 16; ++i)
      if ((i & s) == 0) cx(l[i], l[i + s]);
}

__host__ __device__ __forceinline__ uint32_t float_bits(float s) {
#ifdef __CUDA_ARCH__
  return __float_as_uint(s);
#else
  uint32_t u;
  memcpy(&u, &s, sizeof u);
  return u;
#endif
}

__host__ __device__ __forceinline__ float bits_float(uint32_t u) {
#ifdef __CUDA_ARCH__
  return __uint_as_float(u);
#else
  float s;
  memcpy(&s, &u, sizeof s);
  return s;
#endif
}

// Selection key of score s of block i (0 <= i < 256), as an fp32 value:
// the score (-0 first turned into +0) with its lowest 8 mantissa bits
// replaced by the block index -- 255 - i for a non-negative score, i for a
// negative one -- so that under the float order a larger key is a larger
// score or, between scores that agree in all but those 8 bits (within 2^-15
// of each other, relative; 2^-141 absolute among subnormals), the lower
// block. Empty slots use -inf, below every finite key.
__host__ __device__ __forceinline__ float order_key(float s, int i) {
  const uint32_t u = float_bits(s + 0.0f);
  const uint32_t low = (u >> 31) ? (uint32_t)i : (uint32_t)(255 - i);
  return bits_float((u & 0xFFFFFF00u) | low);
}

__host__ __device__ __forceinline__ int key_block(float key) {
  const uint32_t u = float_bits(key);
  return (u >> 31) ? (int)(u & 0xFFu) : 255 - (int)(u & 0xFFu);
}

}  // namespace net
}  // namespace moba
