// The parameter-free MoBA gate with causal block mask, forced own block and
// top-k (PaperTrace "2.1.3 MoBA", section 1 eq. 3, section 2, section 2.1):
//   s_i = q . kbar_i for the blocks i < c wholly before the query's block c;
//   blocks after c are never chosen and the full mean of block c (which
//   would include future keys) is never scored; block c is always chosen and
//   uses one of the k slots; the other min(k-1, c) slots take the highest
//   s_i, equal scores going to the lower block index.
//
// Scores are fp32 FMA (q widened from bf16, kbar fp32): the near-tie band of
// the parity check is 1e-4 relative and bf16/tf32 products would flip far
// more ranks than that. One CTA scores 64 consecutive queries of one
// (sequence, head) against the earlier blocks in chunks of 32: a register-
// tiled fp32 GEMM (each thread 4 queries x 2 blocks, operands in shared
// memory) writes the chunk's scores to shared memory, then 4 threads per
// query scan them into sorted register lists of their best KM >= k-1
// blocks; at the end the four lists are merged by warp shuffles.
//
// Own-block variant (section 5.2, causal blocks): with dm.prefix the own
// block c is not forced but scored by its prefix mean (own[t][h], from
// launch_own_score) and competes for the k slots: the k best of blocks
// 0..c win, equal scores going to the lower index, so c loses a tie. Block
// c is in iff fewer than k earlier blocks score at least as high, i.e.
// unless c >= k and the k-th best earlier block scores >= own.
#include <climits>
#include <cmath>

#include "common.cuh"

namespace moba {
namespace {

constexpr int kQ = 64;        // queries per CTA
constexpr int kThreads = 256; // 4 threads per query in the selection phase
constexpr int kCh = 32;       // kbar rows per shared-memory chunk

__device__ __forceinline__ bool better(float s, int i, float t, int j) {
  return s > t || (s == t && i < j);
}

template <int KM>
__device__ __forceinline__ void insert(float (&ts)[KM], int (&ti)[KM], float s, int i) {
#pragma unroll
  for (int j = 0; j < KM; ++j) {
    if (better(s, i, ts[j], ti[j])) {
      const float fs = ts[j];
      const int fi = ti[j];
      ts[j] = s;
      ti[j] = i;
      s = fs;
      i = fi;
    }
  }
}

template <typename T, int D, int KM>
__global__ void __launch_bounds__(kThreads) gate_kernel(Dims dm, const T* __restrict__ q,
                                                        const float* __restrict__ kbar,
                                                        const float* __restrict__ own,
                                                        const int32_t* __restrict__ cu,
                                                        int32_t* __restrict__ idx, int* status) {
  extern __shared__ __align__(16) float gsm[];
  float(*qs)[D + 4] = reinterpret_cast<float(*)[D + 4]>(gsm);                     // [kQ]
  float(*kb)[D + 4] = reinterpret_cast<float(*)[D + 4]>(gsm + kQ * (D + 4));      // [kCh]
  float(*sc)[kCh + 1] = reinterpret_cast<float(*)[kCh + 1]>(gsm + (kQ + kCh) * (D + 4));

  // blockIdx.z: the q head, or with shared routing the kv head, whose group
  // of nh q heads is scored by the sum of their q rows (the mean's ranking)
  const int b = blockIdx.y, grp = dm.Hq / dm.Hkv;
  const int g = dm.shared ? (int)blockIdx.z : (int)blockIdx.z / grp;
  const int h0 = dm.shared ? g * grp : (int)blockIdx.z, nh = dm.shared ? grp : 1;
  int64_t start;
  int len;
  if (!seq_bounds(dm, cu, b, start, len, status)) return;
  const int p0 = blockIdx.x * kQ;
  if (p0 >= len) return;

  constexpr int VEC = Vec16<T>::N, TPR = D / VEC;
  for (int e = threadIdx.x; e < kQ * TPR; e += kThreads) {
    const int r = e / TPR, l = e % TPR;
    float x[VEC];
#pragma unroll
    for (int u = 0; u < VEC; ++u) x[u] = 0.f;
    if (p0 + r < len) {
      for (int hh = 0; hh < nh; ++hh) {
        float y[VEC];
        Vec16<T>::load(q + ((start + p0 + r) * dm.Hq + h0 + hh) * (int64_t)D + l * VEC, y);
#pragma unroll
        for (int u = 0; u < VEC; ++u) x[u] += y[u];
      }
    }
#pragma unroll
    for (int u = 0; u < VEC; ++u) qs[r][l * VEC + u] = x[u];
  }

  // selection mapping: query qi, quarter `part` of every chunk
  const int qi = threadIdx.x >> 2, part = threadIdx.x & 3;
  // GEMM mapping: queries ty + 16 i (i < 4), blocks tx + 16 j (j < 2)
  const int ty = threadIdx.x >> 4, tx = threadIdx.x & 15;
  const int p = p0 + qi;
  const bool valid = p < len;
  const int c = valid ? p / dm.B : 0;
  const int cmax = (min(p0 + kQ, len) - 1) / dm.B;  // blocks any query of the tile may score

  float ts[KM];
  int ti[KM];
#pragma unroll
  for (int j = 0; j < KM; ++j) {
    ts[j] = -INFINITY;
    ti[j] = INT_MAX;
  }

  for (int base = 0; base < cmax; base += kCh) {
    __syncthreads();
    const int nblk = min(kCh, cmax - base);
    for (int e = threadIdx.x; e < kCh * (D / 4); e += kThreads) {
      const int r = e / (D / 4), l = e % (D / 4);
      float4 w = make_float4(0.f, 0.f, 0.f, 0.f);
      if (r < nblk)
        w = __ldg(reinterpret_cast<const float4*>(
            kbar + (((int64_t)b * dm.nb + base + r) * dm.Hkv + g) * D + l * 4));
      *reinterpret_cast<float4*>(&kb[r][l * 4]) = w;
    }
    __syncthreads();
    float acc[4][2];
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[i][0] = acc[i][1] = 0.f;
#pragma unroll 4
    for (int x4 = 0; x4 < D / 4; ++x4) {
      float4 qv[4], kv[2];
#pragma unroll
      for (int i = 0; i < 4; ++i) qv[i] = reinterpret_cast<const float4*>(qs[ty + 16 * i])[x4];
#pragma unroll
      for (int j = 0; j < 2; ++j) kv[j] = reinterpret_cast<const float4*>(kb[tx + 16 * j])[x4];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          acc[i][j] = fmaf(qv[i].x, kv[j].x, acc[i][j]);
          acc[i][j] = fmaf(qv[i].y, kv[j].y, acc[i][j]);
          acc[i][j] = fmaf(qv[i].z, kv[j].z, acc[i][j]);
          acc[i][j] = fmaf(qv[i].w, kv[j].w, acc[i][j]);
        }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 2; ++j) sc[ty + 16 * i][tx + 16 * j] = acc[i][j];
    __syncthreads();
#pragma unroll
    for (int u = 0; u < kCh / 4; ++u) {
      const int jj = part + 4 * u;
      const int i = base + jj;
      if (jj < nblk && i < c) insert<KM>(ts, ti, sc[qi][jj], i);
    }
  }

  // Merge the four lists of each query: round r takes the best head.
  const int need = hist_slots(dm);
  float kth = -INFINITY;  // score of the k-th best earlier block (prefix variant)
  int sel[KM];
#pragma unroll
  for (int r = 0; r < KM; ++r) {
    sel[r] = INT_MAX;
    if (r < need) {
      float bs = ts[0];
      int bi = ti[0], owner = part;
#pragma unroll
      for (int off = 1; off <= 2; off <<= 1) {
        const float os = __shfl_xor_sync(0xffffffffu, bs, off);
        const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
        const int oo = __shfl_xor_sync(0xffffffffu, owner, off);
        if (better(os, oi, bs, bi)) {
          bs = os;
          bi = oi;
          owner = oo;
        }
      }
      if (owner == part) {
#pragma unroll
        for (int j = 0; j + 1 < KM; ++j) {
          ts[j] = ts[j + 1];
          ti[j] = ti[j + 1];
        }
        ts[KM - 1] = -INFINITY;
        ti[KM - 1] = INT_MAX;
      }
      if (r < c) sel[r] = bi;
      if (r == dm.topk - 1) kth = bs;
    }
  }
  // the own block: forced, or in unless k earlier blocks score at least as high
  bool own_in = true;
  if (dm.prefix && valid) {
    float so = 0.f;
    for (int hh = 0; hh < nh; ++hh) so += own[(start + p) * dm.Hq + h0 + hh];
    own_in = !(c >= dm.topk && kth >= so);
  }
  const int hsel = valid ? (own_in ? min(dm.topk - 1, c) : dm.topk) : 0;
#pragma unroll
  for (int r = 0; r < KM; ++r)
    if (r >= hsel) sel[r] = INT_MAX;
  if (part != 0 || !valid) return;
  // ascending order of the chosen earlier blocks
#pragma unroll
  for (int a = 0; a < KM; ++a) {
#pragma unroll
    for (int j = 0; j + 1 < KM - a; ++j) {
      if (sel[j] > sel[j + 1]) {
        const int x = sel[j];
        sel[j] = sel[j + 1];
        sel[j + 1] = x;
      }
    }
  }
  for (int hh = 0; hh < nh; ++hh) {
    if (!MOBA_CHECK(start + p < dm.T && h0 + hh < dm.Hq, status)) break;
    int32_t* row = idx + ((start + p) * dm.Hq + h0 + hh) * (int64_t)dm.topk;
#pragma unroll
    for (int r = 0; r <= KM; ++r) {
      if (r < dm.topk)
        row[r] = r < hsel ? sel[r < KM ? r : KM - 1] : (r == hsel && own_in ? c : -1);
    }
  }
}

template <typename T, int D, int KM>
cudaError_t run(const Dims& dm, const void* q, const float* kbar, const float* own,
                const int32_t* cu, int32_t* idx, int* status, cudaStream_t st) {
  dim3 grid((dm.max_seqlen + kQ - 1) / kQ, dm.batch, dm.shared ? dm.Hkv : dm.Hq);
  const size_t smem = sizeof(float) * ((kQ + kCh) * (D + 4) + kQ * (kCh + 1));
  cudaError_t e = cudaFuncSetAttribute(gate_kernel<T, D, KM>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  gate_kernel<T, D, KM><<<grid, kThreads, smem, st>>>(dm, static_cast<const T*>(q), kbar, own,
                                                      cu, idx, status);
  return cudaGetLastError();
}

template <typename T, int D>
cudaError_t by_k(const Dims& dm, const void* q, const float* kbar, const float* own,
                 const int32_t* cu, int32_t* idx, int* status, cudaStream_t st) {
  const int need = hist_slots(dm);
  if (need <= 1) return run<T, D, 1>(dm, q, kbar, own, cu, idx, status, st);
  if (need <= 2) return run<T, D, 2>(dm, q, kbar, own, cu, idx, status, st);
  if (need <= 4) return run<T, D, 4>(dm, q, kbar, own, cu, idx, status, st);
  if (need <= 8) return run<T, D, 8>(dm, q, kbar, own, cu, idx, status, st);
  if (need <= 16) return run<T, D, 16>(dm, q, kbar, own, cu, idx, status, st);
  return run<T, D, 32>(dm, q, kbar, own, cu, idx, status, st);
}

}  // namespace

cudaError_t launch_gate(const Dims& dm, const void* q, const float* kbar, const float* own,
                        const int32_t* cu, int32_t* idx, int* status, cudaStream_t st) {
  if (dm.batch == 0 || dm.max_seqlen == 0) return cudaSuccess;
  if (gate_tc_supported(dm)) return launch_gate_tc(dm, q, kbar, own, cu, idx, status, st);
  if (dm.dtype == kBF16)
    return dm.d == 128 ? by_k<__nv_bfloat16, 128>(dm, q, kbar, own, cu, idx, status, st)
                       : by_k<__nv_bfloat16, 64>(dm, q, kbar, own, cu, idx, status, st);
  return dm.d == 128 ? by_k<float, 128>(dm, q, kbar, own, cu, idx, status, st)
                     : by_k<float, 64>(dm, q, kbar, own, cu, idx, status, st);
}

}  // namespace moba
