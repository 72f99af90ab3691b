// Online-softmax merge of the partial results of one query (PaperTrace
// "2.1.3 MoBA", section 2 eq. 7-8): each slot holds a normalised partial
// o_j = u_j / l_j and lse_j = m_j + log l_j over a disjoint part of the
// query's candidate keys (the own block, and each chosen earlier block).
// With m = max_j lse_j and w_j = exp(lse_j - m):
//   l = sum_j w_j,   o = sum_j w_j o_j / l,   lse = m + log l,
// which is eq. (7)-(8) written with lse (u_j = o_j l_j, l_j = exp(lse_j - m_j))
// and equals ONE softmax over the union of the candidates -- never a sum of
// separately normalised outputs. The result is written in the original
// (token, head) order, which undoes the regrouping.
//
// One warp per (token, head); each lane owns D/32 consecutive columns, so
// every partial row is read with one coalesced 512-byte (D=128) access.
#include <cmath>

#include "common.cuh"

namespace moba {
namespace {

constexpr int kWarps = 4;

template <typename T, int D>
__global__ void __launch_bounds__(kWarps * 32)
merge_kernel(Dims dm, Chunk ch, const int32_t* __restrict__ idx, const int32_t* __restrict__ cu,
             const void* __restrict__ part_o, const float* __restrict__ part_lse,
             T* __restrict__ out, float* __restrict__ lse_out) {
  constexpr int PL = D / 32;  // columns per lane
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.y, hl = blockIdx.z, h = ch.h0 + hl;
  const int64_t start = cu[b];
  const int len = cu[b + 1] - cu[b];
  if (len < 0 || len > dm.max_seqlen) return;
  const int p = blockIdx.x * kWarps + warp;
  if (p >= len) return;
  const int64_t t = start + p;
  const int c = p / dm.B;
  const int32_t* row = idx + (t * dm.Hq + h) * (int64_t)dm.topk;
  const int64_t prow0 = (t * ch.nq + hl) * (int64_t)dm.topk;
  const int64_t nr = (int64_t)ch.nq * dm.topk;

  float m = -INFINITY;
  for (int r = 0; r < dm.topk; ++r) {
    const int e = row[r];
    if (e >= 0 && e <= c) m = fmaxf(m, part_lse[part_lse_at(part_row(prow0 + r, nr))]);
  }
  float acc[PL];
#pragma unroll
  for (int u = 0; u < PL; ++u) acc[u] = 0.f;
  float l = 0.f;
  for (int r = 0; r < dm.topk; ++r) {
    const int e = row[r];
    if (!(e >= 0 && e <= c)) continue;
    const PartRow pr = part_row(prow0 + r, nr);
    const float w = expf(part_lse[part_lse_at(pr)] - m);
    l += w;
    // lane's PL columns lie inside one 32-byte piece (partials in T)
    constexpr int PE = 32 / (int)sizeof(T);
    const T* src = part_piece<T>(part_o, pr, D, lane * PL / PE) + (lane * PL) % PE;
#pragma unroll
    for (int u = 0; u < PL; ++u) acc[u] = fmaf(w, to_f32(src[u]), acc[u]);
  }
  const float inv_l = 1.f / l;
  T* dst = out + (t * dm.Hq + h) * (int64_t)D + lane * PL;
#pragma unroll
  for (int u = 0; u < PL; ++u) dst[u] = from_f32<T>(acc[u] * inv_l);
  if (lse_out && lane == 0) lse_out[t * dm.Hq + h] = m + logf(l);
}

template <typename T, int D>
cudaError_t run(const Dims& dm, const Chunk& ch, const int32_t* idx, const int32_t* cu,
                const Partials& pt, void* out, float* lse, cudaStream_t st) {
  dim3 grid((dm.max_seqlen + kWarps - 1) / kWarps, dm.batch, ch.nq);
  merge_kernel<T, D><<<grid, kWarps * 32, 0, st>>>(dm, ch, idx, cu, pt.o, pt.lse,
                                                   static_cast<T*>(out), lse);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_merge(const Dims& dm, const Chunk& ch, const int32_t* idx, const int32_t* cu,
                         const Partials& pt, void* out, float* lse, cudaStream_t st) {
  if (dm.batch == 0 || dm.max_seqlen == 0) return cudaSuccess;
  if (dm.dtype == kBF16)
    return dm.d == 128 ? run<__nv_bfloat16, 128>(dm, ch, idx, cu, pt, out, lse, st)
                       : run<__nv_bfloat16, 64>(dm, ch, idx, cu, pt, out, lse, st);
  return dm.d == 128 ? run<float, 128>(dm, ch, idx, cu, pt, out, lse, st)
                     : run<float, 64>(dm, ch, idx, cu, pt, out, lse, st);
}

}  // namespace moba
