// Branch-free sorting networks on 16 unsigned 32-bit keys, in registers
// (compile-time indices only), for the gate's top-k selection.
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

#include <stdint.h>
#include <string.h>

namespace moba {
namespace net {

__host__ __device__ __forceinline__ void cx(uint32_t& a, uint32_t& b) {
  const uint32_t hi = a > b ? a : b;
  const uint32_t lo = a > b ? b : a;
  a = hi;
  b = lo;
}

// Merges the two sorted halves of v[LO .. LO+N) taking every R-th element.
template <int LO, int N, int R>
__host__ __device__ __forceinline__ void oe_merge(uint32_t (&v)[16]) {
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

template <int LO, int N>
__host__ __device__ __forceinline__ void oe_sort(uint32_t (&v)[16]) {
  if constexpr (N > 1) {
    oe_sort<LO, N / 2>(v);
    oe_sort<LO + N / 2, N / 2>(v);
    oe_merge<LO, N, 1>(v);
  }
}

__host__ __device__ __forceinline__ void oe_sort16(uint32_t (&v)[16]) { oe_sort<0, 16>(v); }

// l, g sorted descending; l <- the 16 largest of l and g, descending.
__host__ __device__ __forceinline__ void merge_top16(uint32_t (&l)[16], const uint32_t (&g)[16]) {
#pragma unroll
  for (int i = 0; i < 16; ++i) l[i] = l[i] > g[15 - i] ? l[i] : g[15 - i];
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

// Selection key of score s of block i (0 <= i < 256): the score's bits made
// order-preserving as an unsigned integer (negative values inverted, the
// sign bit set on the others; -0 first turned into +0), the lowest 8 bits
// then replaced by 255 - i. A larger key is a larger score or, between
// scores that agree in their top 24 order bits (within 2^-15 of each
// other, relative; 2^-141 absolute among subnormals), the lower block. Empty slots use key 0, below every
// finite score.
__host__ __device__ __forceinline__ uint32_t order_key(float s, int i) {
  const uint32_t u = float_bits(s + 0.0f);
  const uint32_t ord = u ^ ((uint32_t)((int32_t)u >> 31) | 0x80000000u);
  return (ord & 0xFFFFFF00u) | (uint32_t)(255 - i);
}

__host__ __device__ __forceinline__ int key_block(uint32_t key) { return 255 - (int)(key & 0xFFu); }

}  // namespace net
}  // namespace moba
