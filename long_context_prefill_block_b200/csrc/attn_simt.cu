// Portable SIMT attention kernels (fp32 FMA), used for fp32 inputs, for
// block sizes the tensor-core path does not take, and as the comparison
// dense kernel at fp32. Three row sources share one body:
//   HIST  : a tile of regrouped (query, head, slot) rows against the B raw
//           keys of one earlier block, non-causal (PaperTrace "2.1.3 MoBA",
//           section 2 eq. 6);
//   CUR   : consecutive query rows against their own block, causal (eq. 5);
//   DENSE : consecutive query rows against every earlier key (eq. 1, causal).
// HIST and CUR write a normalised partial result o = u / l and its
// log-sum-exp m + log l per slot; the merge kernel combines the slots by
// eq. (7)-(8). DENSE writes the final output.
//
// Layout of work: 32 rows per CTA, 4 threads per row, each thread owning
// D/4 columns in float4 groups at 4*part + 16*j (conflict-free shared reads);
// keys and values stream through shared memory 32 at a time; each chunk is
// folded into the running (m, l, o) with one rescale (online softmax).
#include <cmath>

#include "common.cuh"

namespace moba {
namespace {

enum Mode { HIST = 0, CUR = 1, DENSE = 2 };
constexpr int kTM = kSimtTileM;  // rows per CTA
constexpr int kThreads = kTM * 4;
constexpr int kKC = 32;          // keys per shared-memory chunk

template <typename T, int D, int MODE>
__global__ void __launch_bounds__(kThreads)
attn_simt(Dims dm, Chunk ch, const T* __restrict__ q, const T* __restrict__ k,
          const T* __restrict__ v, const int32_t* __restrict__ cu,
          const int32_t* __restrict__ list_off, const int32_t* __restrict__ pairs,
          const int4* __restrict__ tiles, const int32_t* __restrict__ tile_count,
          const int32_t* __restrict__ idx, void* __restrict__ part_o,
          float* __restrict__ part_lse, T* __restrict__ out, float* __restrict__ lse_out) {
  __shared__ __align__(16) float ks[kKC][D + 4];
  __shared__ __align__(16) float vs[kKC][D + 4];
  __shared__ int s_lo, s_hi;
  constexpr int NG = D / 16;  // float4 groups per thread

  const int rloc = threadIdx.x >> 2, part = threadIdx.x & 3;
  const int grp = dm.Hq / dm.Hkv;
  int b, g;
  bool valid = false;
  int64_t t = 0, prow = 0;
  int h = 0, lo = 0, hi = -1;

  if (MODE == HIST) {
    if ((int)blockIdx.x >= *tile_count) return;
    const int4 tl = tiles[blockIdx.x];
    const int L = tl.x;
    const int e = L % dm.nb;
    const int gl = (L / dm.nb) % ch.ng;
    b = L / (dm.nb * ch.ng);
    g = ch.g0 + gl;
    const int count = tl.z;
    const int r = tl.y + rloc;
    valid = r < count;
    if (valid) {
      prow = pairs[tl.w + r];
      const int64_t th = prow / dm.topk;
      t = th / ch.nq;
      h = ch.h0 + (int)(th % ch.nq);
    }
    lo = e * dm.B;
    hi = lo + dm.B - 1;
  } else {
    b = blockIdx.y;
    h = (MODE == CUR ? ch.h0 : 0) + blockIdx.z;
    g = h / grp;
    const int64_t st = cu[b];
    const int len = cu[b + 1] - cu[b];
    if (len < 0 || len > dm.max_seqlen) return;
    if ((int)blockIdx.x * kTM >= len) return;
    const int p = blockIdx.x * kTM + rloc;
    valid = p < len;
    t = st + p;
    const int c = p / dm.B;
    lo = MODE == CUR ? c * dm.B : 0;
    hi = p;
    if (MODE == CUR && valid) {
      const int32_t* row = idx + (t * dm.Hq + h) * (int64_t)dm.topk;
      int slot = -1;
      for (int r = 0; r < dm.topk; ++r)
        if (row[r] == c && slot < 0) slot = r;
      valid = slot >= 0;
      prow = (t * ch.nq + (h - ch.h0)) * (int64_t)dm.topk + (slot < 0 ? 0 : slot);
    }
  }
  const int64_t start = cu[b];

  // Key window of the CTA: the union of its rows' windows.
  if (threadIdx.x == 0) {
    s_lo = 0x7fffffff;
    s_hi = -1;
  }
  __syncthreads();
  if (valid && part == 0) {
    atomicMin(&s_lo, lo);
    atomicMax(&s_hi, hi);
  }
  __syncthreads();
  const int klo = s_lo, khi = s_hi;

  float qr[NG * 4];
  if (valid) {
    const T* src = q + (t * dm.Hq + h) * (int64_t)D;
#pragma unroll
    for (int j = 0; j < NG; ++j)
#pragma unroll
      for (int u = 0; u < 4; ++u) qr[j * 4 + u] = to_f32(src[part * 4 + 16 * j + u]);
  } else {
#pragma unroll
    for (int j = 0; j < NG * 4; ++j) qr[j] = 0.f;
  }
  const float scale = rsqrtf((float)D);
  float m_run = -INFINITY, l_run = 0.f;
  float o[NG * 4];
#pragma unroll
  for (int j = 0; j < NG * 4; ++j) o[j] = 0.f;

  constexpr int VEC = Vec16<T>::N, TPR = D / VEC;
  for (int k0 = klo; k0 <= khi; k0 += kKC) {
    __syncthreads();
    for (int e = threadIdx.x; e < kKC * TPR; e += kThreads) {
      const int r = e / TPR, l = e % TPR;
      const int j = k0 + r;
      float xk[VEC], xv[VEC];
      if (j <= khi) {
        const int64_t off = ((start + j) * dm.Hkv + g) * (int64_t)D + l * VEC;
        Vec16<T>::load(k + off, xk);
        Vec16<T>::load(v + off, xv);
      } else {
#pragma unroll
        for (int u = 0; u < VEC; ++u) xk[u] = xv[u] = 0.f;
      }
#pragma unroll
      for (int u = 0; u < VEC; ++u) {
        ks[r][l * VEC + u] = xk[u];
        vs[r][l * VEC + u] = xv[u];
      }
    }
    __syncthreads();
    float s[kKC];
    float m_chunk = -INFINITY;
#pragma unroll
    for (int jj = 0; jj < kKC; ++jj) {
      float acc = 0.f;
#pragma unroll
      for (int j = 0; j < NG; ++j) {
        const float4 w = *reinterpret_cast<const float4*>(&ks[jj][part * 4 + 16 * j]);
        acc = fmaf(qr[j * 4 + 0], w.x, acc);
        acc = fmaf(qr[j * 4 + 1], w.y, acc);
        acc = fmaf(qr[j * 4 + 2], w.z, acc);
        acc = fmaf(qr[j * 4 + 3], w.w, acc);
      }
      acc += __shfl_xor_sync(0xffffffffu, acc, 1);
      acc += __shfl_xor_sync(0xffffffffu, acc, 2);
      const int key = k0 + jj;
      s[jj] = (valid && key >= lo && key <= hi) ? acc * scale : -INFINITY;
      m_chunk = fmaxf(m_chunk, s[jj]);
    }
    if (m_chunk == -INFINITY) continue;
    const float m_new = fmaxf(m_run, m_chunk);
    const float corr = expf(m_run - m_new);
    l_run *= corr;
#pragma unroll
    for (int j = 0; j < NG * 4; ++j) o[j] *= corr;
#pragma unroll
    for (int jj = 0; jj < kKC; ++jj) {
      const float pw = expf(s[jj] - m_new);
      l_run += pw;
#pragma unroll
      for (int j = 0; j < NG; ++j) {
        const float4 w = *reinterpret_cast<const float4*>(&vs[jj][part * 4 + 16 * j]);
        o[j * 4 + 0] = fmaf(pw, w.x, o[j * 4 + 0]);
        o[j * 4 + 1] = fmaf(pw, w.y, o[j * 4 + 1]);
        o[j * 4 + 2] = fmaf(pw, w.z, o[j * 4 + 2]);
        o[j * 4 + 3] = fmaf(pw, w.w, o[j * 4 + 3]);
      }
    }
    m_run = m_new;
  }
  if (!valid || l_run <= 0.f) return;
  const float inv_l = 1.f / l_run;
  const float lse = m_run + logf(l_run);
  if (MODE == DENSE) {
    T* dst = out + (t * dm.Hq + h) * (int64_t)D;
#pragma unroll
    for (int j = 0; j < NG; ++j)
#pragma unroll
      for (int u = 0; u < 4; ++u) dst[part * 4 + 16 * j + u] = from_f32<T>(o[j * 4 + u] * inv_l);
    if (lse_out && part == 0) lse_out[t * dm.Hq + h] = lse;
  } else {
    const PartRow pr = part_row(prow, (int64_t)ch.nq * dm.topk);
    constexpr int PE = 32 / (int)sizeof(T);  // values per 32-byte piece
#pragma unroll
    for (int j = 0; j < NG; ++j) {
      const int x0 = part * 4 + 16 * j;  // four columns inside one piece
      T* dst = part_piece<T>(part_o, pr, D, x0 / PE) + x0 % PE;
#pragma unroll
      for (int u = 0; u < 4; ++u) dst[u] = from_f32<T>(o[j * 4 + u] * inv_l);
    }
    if (part == 0) part_lse[part_lse_at(pr)] = lse;
  }
}

template <typename T, int D, int MODE>
cudaError_t run(dim3 grid, cudaStream_t st, const Dims& dm, const Chunk& ch, const void* q,
                const void* k, const void* v, const int32_t* cu, const Regroup* rg,
                const int32_t* idx, const Partials* pt, void* out, float* lse) {
  attn_simt<T, D, MODE><<<grid, kThreads, 0, st>>>(
      dm, ch, static_cast<const T*>(q), static_cast<const T*>(k), static_cast<const T*>(v), cu,
      rg ? rg->list_off : nullptr, rg ? rg->pairs : nullptr, rg ? rg->tiles : nullptr,
      rg ? rg->tile_off + ch.n_lists : nullptr, idx, pt ? pt->o : nullptr,
      pt ? pt->lse : nullptr, static_cast<T*>(out), lse);
  return cudaGetLastError();
}

template <int MODE>
cudaError_t dispatch(dim3 grid, cudaStream_t st, const Dims& dm, const Chunk& ch, const void* q,
                     const void* k, const void* v, const int32_t* cu, const Regroup* rg,
                     const int32_t* idx, const Partials* pt, void* out, float* lse) {
  if (dm.dtype == kBF16)
    return dm.d == 128
               ? run<__nv_bfloat16, 128, MODE>(grid, st, dm, ch, q, k, v, cu, rg, idx, pt, out, lse)
               : run<__nv_bfloat16, 64, MODE>(grid, st, dm, ch, q, k, v, cu, rg, idx, pt, out, lse);
  return dm.d == 128 ? run<float, 128, MODE>(grid, st, dm, ch, q, k, v, cu, rg, idx, pt, out, lse)
                     : run<float, 64, MODE>(grid, st, dm, ch, q, k, v, cu, rg, idx, pt, out, lse);
}

}  // namespace

cudaError_t launch_history_simt(const Dims& dm, const Chunk& ch, const void* q, const void* k,
                                const void* v, const int32_t* cu, const Regroup& rg,
                                const Partials& pt, cudaStream_t st) {
  if (rg.max_tiles == 0) return cudaSuccess;
  dim3 grid((unsigned)rg.max_tiles);
  return dispatch<HIST>(grid, st, dm, ch, q, k, v, cu, &rg, nullptr, &pt, nullptr, nullptr);
}

cudaError_t launch_current_simt(const Dims& dm, const Chunk& ch, const void* q, const void* k,
                                const void* v, const int32_t* cu, const int32_t* idx,
                                const Partials& pt, cudaStream_t st) {
  if (dm.batch == 0 || dm.max_seqlen == 0) return cudaSuccess;
  dim3 grid((dm.max_seqlen + kTM - 1) / kTM, dm.batch, ch.nq);
  return dispatch<CUR>(grid, st, dm, ch, q, k, v, cu, nullptr, idx, &pt, nullptr, nullptr);
}

cudaError_t launch_dense_simt(const Dims& dm, const void* q, const void* k, const void* v,
                              const int32_t* cu, void* out, float* lse, cudaStream_t st) {
  if (dm.batch == 0 || dm.max_seqlen == 0) return cudaSuccess;
  Chunk ch{0, dm.Hkv, 0, dm.Hq, 0, kTM};
  dim3 grid((dm.max_seqlen + kTM - 1) / kTM, dm.batch, dm.Hq);
  return dispatch<DENSE>(grid, st, dm, ch, q, k, v, cu, nullptr, nullptr, nullptr, out, lse);
}

}  // namespace moba
