// Backward pass of MoBA attention (PaperTrace "2.1.3 MoBA", section 5.3:
// the hard top-k indices only build the mask and pass no gradient to the
// routing scores; the loss flows back along the Q/K/V that were read).
// Gradients of L = sum(dO . O) per query row with candidate keys J,
// logits s_j = q.k_j / sqrt(d), P_j = softmax_J(s)_j:
//   dP_j = dO . v_j,  D = sum_j P_j dP_j = dO . O,  dS_j = P_j (dP_j - D)
//   dq = sum_j dS_j k_j / sqrt(d),  dk_j += dS_j q / sqrt(d),  dv_j += P_j dO
// with P recomputed from the forward's log-sum-exp (P_j = exp(s_j - lse)).
//
// Block-major, like the forward: one CTA per (list of queries that chose a
// history block, 64-key tile of that block) and one per (own block, kv head,
// 64-key tile); each CTA keeps its keys' dk, dv in registers while it walks
// its query rows 32 at a time, so each (block, kv head, key tile) is written
// by exactly one CTA per kernel; every query row's dq gathers contributions
// from several CTAs and is added atomically (fp32). fp32 FMA throughout.
#include "common.cuh"

namespace moba {
namespace {

constexpr int kThreads = 256;
constexpr int KT = 64;  // keys per CTA
constexpr int RC = 32;  // query rows per step
enum { HIST = 0, CUR = 1 };

template <int D>
struct BwdSmem {
  // padded rows of 16-byte multiples: 8 lanes reading keys kg, kg + 8, ... at
  // one column touch 8 distinct 4-bank groups
  static constexpr int LD = D + 4;
  static constexpr size_t bytes = sizeof(int64_t) * RC +
                                  sizeof(float) * (2 * KT * LD + 2 * RC * LD + 2 * RC * (KT + 1) +
                                                   3 * RC);
};

struct BwdArgs {
  Dims dm;
  Chunk ch;
  const void* q;
  const void* k;
  const void* v;
  const void* dout;
  const float* lse;   // [T][Hq], natural log
  const float* Dsum;  // [T][Hq], dO . O
  const int32_t* cu;
  const int32_t* idx;  // [T][Hq][k] index rows (own-block rows of the prefix-mean gate)
  const int32_t* list_off;
  const int32_t* pairs;
  float* dq;  // [T][Hq][d]
  float* dk;  // [T][Hkv][d]
  float* dv;  // [T][Hkv][d]
  int* status;
};

// D = dO . O per (token, head): one warp per row.
template <typename T, int D>
__global__ void __launch_bounds__(kThreads) bwd_dot_kernel(int64_t rows, const T* __restrict__ dout,
                                                           const T* __restrict__ out,
                                                           float* __restrict__ Dsum) {
  const int64_t row = (int64_t)blockIdx.x * (kThreads / 32) + threadIdx.x / 32;
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  float acc = 0.f;
  for (int x = lane; x < D; x += 32)
    acc += to_f32(dout[row * D + x]) * to_f32(out[row * D + x]);
#pragma unroll
  for (int off = 16; off; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (lane == 0) Dsum[row] = acc;
}

template <typename T, int D, int MODE>
__global__ void __launch_bounds__(kThreads) bwd_block_kernel(const BwdArgs a) {
  using S = BwdSmem<D>;
  constexpr int LD = S::LD;
  extern __shared__ int64_t sm_raw[];
  int64_t* qrow_s = sm_raw;  // q row (t * Hq + h) of each step row
  float* sm = reinterpret_cast<float*>(sm_raw + RC);
  float(*Ks)[LD] = reinterpret_cast<float(*)[LD]>(sm);
  float(*Vs)[LD] = reinterpret_cast<float(*)[LD]>(sm + KT * LD);
  float(*Qs)[LD] = reinterpret_cast<float(*)[LD]>(sm + 2 * KT * LD);
  float(*Os)[LD] = reinterpret_cast<float(*)[LD]>(sm + 2 * KT * LD + RC * LD);  // dO rows
  float(*Pm)[KT + 1] = reinterpret_cast<float(*)[KT + 1]>(sm + 2 * KT * LD + 2 * RC * LD);
  float(*Sm)[KT + 1] = reinterpret_cast<float(*)[KT + 1]>(sm + 2 * KT * LD + 2 * RC * LD +
                                                           RC * (KT + 1));  // dS
  float* lse_s = sm + 2 * KT * LD + 2 * RC * LD + 2 * RC * (KT + 1);
  float* D_s = lse_s + RC;
  int* pos_s = reinterpret_cast<int*>(D_s + RC);  // row position (CUR), or -1: no row

  const Dims& dm = a.dm;
  const int tid = threadIdx.x;
  const int grp = dm.Hq / dm.Hkv;
  const float scale = rsqrtf((float)D);
  const int kt = blockIdx.y;

  // ---- this CTA's keys and rows
  int b, g, blk;
  int64_t n_rows;
  int64_t row0 = 0;  // HIST: first entry in the list
  if (MODE == HIST) {
    const int L = blockIdx.x;
    blk = L % dm.nb;
    g = a.ch.g0 + (L / dm.nb) % a.ch.ng;
    b = L / (dm.nb * a.ch.ng);
    row0 = a.list_off[L];
    n_rows = a.list_off[L + 1] - row0;
  } else {
    blk = blockIdx.x % dm.nb;
    g = (blockIdx.x / dm.nb) % dm.Hkv;
    b = blockIdx.x / (dm.nb * dm.Hkv);
    n_rows = 0;
  }
  int64_t start;
  int len;
  if (!seq_bounds(dm, a.cu, b, start, len, nullptr)) return;
  const int k0 = blk * dm.B + kt * KT;                      // first key position
  const int k1 = min(min(k0 + KT, (blk + 1) * dm.B), len);  // one past the last
  if (k0 >= k1) return;
  int p_first = 0;
  if (MODE == CUR) {
    // queries of the block at or after the tile's first key, every head of the group
    p_first = k0;
    const int p_end = min((blk + 1) * dm.B, len);
    n_rows = (int64_t)(p_end - p_first) * grp;
  }
  if (n_rows <= 0) return;

  // ---- keys and values of the tile, fp32
  constexpr int VEC = Vec16<T>::N, TPR = D / VEC;
  for (int e = tid; e < KT * TPR; e += kThreads) {
    const int r = e / TPR, l = e % TPR;
    float xk[VEC], xv[VEC];
    if (k0 + r < k1) {
      const int64_t off = ((start + k0 + r) * dm.Hkv + g) * (int64_t)D + l * VEC;
      Vec16<T>::load(static_cast<const T*>(a.k) + off, xk);
      Vec16<T>::load(static_cast<const T*>(a.v) + off, xv);
    } else {
#pragma unroll
      for (int u = 0; u < VEC; ++u) xk[u] = xv[u] = 0.f;
    }
#pragma unroll
    for (int u = 0; u < VEC; ++u) {
      Ks[r][l * VEC + u] = xk[u];
      Vs[r][l * VEC + u] = xv[u];
    }
  }

  // dk, dv of key kk (0..63), dims [x0, x0 + D/4)
  const int kk = tid >> 2, x0 = (tid & 3) * (D / 4);
  float dk[D / 4], dv[D / 4];
#pragma unroll
  for (int x = 0; x < D / 4; ++x) dk[x] = dv[x] = 0.f;

  for (int64_t c0 = 0; c0 < n_rows; c0 += RC) {
    __syncthreads();
    // ---- rows c0 .. c0 + RC: q, dO, lse, D
    if (tid < RC) {
      const int64_t i = c0 + tid;
      int pos = -1;
      int64_t qrow = 0;
      if (i < n_rows) {
        if (MODE == HIST) {
          const int64_t prow = a.pairs[row0 + i];
          const int64_t th = prow / dm.topk;
          const int64_t t = th / a.ch.nq;
          const int h = a.ch.h0 + (int)(th % a.ch.nq);
          qrow = t * dm.Hq + h;
          pos = 0;  // every key of a history block is visible
        } else {
          const int p = p_first + (int)(i / grp);
          const int h = g * grp + (int)(i % grp);
          qrow = (start + p) * dm.Hq + h;
          // a row whose own block lost the prefix-mean gate reads none of it
          pos = reads_own(dm, a.idx + qrow * dm.topk, p / dm.B) ? p : -1;
        }
        lse_s[tid] = a.lse[qrow];
        D_s[tid] = a.Dsum[qrow];
      }
      pos_s[tid] = pos;
      qrow_s[tid] = qrow;
    }
    __syncthreads();
    for (int e = tid; e < RC * TPR; e += kThreads) {
      const int r = e / TPR, l = e % TPR;
      float xq[VEC], xo[VEC];
      if (pos_s[r] >= 0) {
        const int64_t qrow = qrow_s[r];
        Vec16<T>::load(static_cast<const T*>(a.q) + qrow * D + l * VEC, xq);
        Vec16<T>::load(static_cast<const T*>(a.dout) + qrow * D + l * VEC, xo);
      } else {
#pragma unroll
        for (int u = 0; u < VEC; ++u) xq[u] = xo[u] = 0.f;
      }
#pragma unroll
      for (int u = 0; u < VEC; ++u) {
        Qs[r][l * VEC + u] = xq[u];
        Os[r][l * VEC + u] = xo[u];
      }
    }
    __syncthreads();
    // ---- S = Q K^T and dP = dO V^T: row r, keys kg, kg + 8, ..., kg + 56;
    // 16-byte shared-memory reads along d
    {
      const int r = tid >> 3, kg = tid & 7;
      float s[8], dp[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) s[u] = dp[u] = 0.f;
#pragma unroll 2
      for (int x = 0; x < D; x += 4) {
        const float4 q4 = *reinterpret_cast<const float4*>(&Qs[r][x]);
        const float4 o4 = *reinterpret_cast<const float4*>(&Os[r][x]);
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const float4 k4 = *reinterpret_cast<const float4*>(&Ks[kg + 8 * u][x]);
          const float4 v4 = *reinterpret_cast<const float4*>(&Vs[kg + 8 * u][x]);
          s[u] = fmaf(q4.x, k4.x, fmaf(q4.y, k4.y, fmaf(q4.z, k4.z, fmaf(q4.w, k4.w, s[u]))));
          dp[u] = fmaf(o4.x, v4.x, fmaf(o4.y, v4.y, fmaf(o4.z, v4.z, fmaf(o4.w, v4.w, dp[u]))));
        }
      }
      const int pos = pos_s[r];
      const float l = lse_s[r], dd = D_s[r];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int kp = k0 + kg + 8 * u;  // key position
        const bool vis = pos >= 0 && kp < k1 && (MODE == HIST || kp <= pos);
        const float p = vis ? __expf(s[u] * scale - l) : 0.f;
        Pm[r][kg + 8 * u] = p;
        Sm[r][kg + 8 * u] = p * (dp[u] - dd);  // dS
      }
    }
    __syncthreads();
    // ---- dV += P^T dO, dK += dS^T Q for key kk, dims x0 ..
#pragma unroll 2
    for (int r = 0; r < RC; ++r) {
      const float p = Pm[r][kk], ds = Sm[r][kk];
#pragma unroll
      for (int x = 0; x < D / 4; x += 4) {
        const float4 o4 = *reinterpret_cast<const float4*>(&Os[r][x0 + x]);
        const float4 q4 = *reinterpret_cast<const float4*>(&Qs[r][x0 + x]);
        dv[x] = fmaf(p, o4.x, dv[x]);
        dv[x + 1] = fmaf(p, o4.y, dv[x + 1]);
        dv[x + 2] = fmaf(p, o4.z, dv[x + 2]);
        dv[x + 3] = fmaf(p, o4.w, dv[x + 3]);
        dk[x] = fmaf(ds, q4.x, dk[x]);
        dk[x + 1] = fmaf(ds, q4.y, dk[x + 1]);
        dk[x + 2] = fmaf(ds, q4.z, dk[x + 2]);
        dk[x + 3] = fmaf(ds, q4.w, dk[x + 3]);
      }
    }
    // ---- dQ = dS K for row r = tid / 8, dims (tid % 8) * D/8 ..
    {
      const int r = tid >> 3, xq = (tid & 7) * (D / 8);
      if (pos_s[r] >= 0) {
        float dq[D / 8];
#pragma unroll
        for (int x = 0; x < D / 8; ++x) dq[x] = 0.f;
#pragma unroll 4
        for (int j = 0; j < KT; ++j) {
          const float ds = Sm[r][j];
#pragma unroll
          for (int x = 0; x < D / 8; x += 4) {
            const float4 k4 = *reinterpret_cast<const float4*>(&Ks[j][xq + x]);
            dq[x] = fmaf(ds, k4.x, dq[x]);
            dq[x + 1] = fmaf(ds, k4.y, dq[x + 1]);
            dq[x + 2] = fmaf(ds, k4.z, dq[x + 2]);
            dq[x + 3] = fmaf(ds, k4.w, dq[x + 3]);
          }
        }
        float* dst = a.dq + qrow_s[r] * D + xq;
#pragma unroll
        for (int x = 0; x < D / 8; ++x) atomicAdd(dst + x, dq[x] * scale);
      }
    }
  }
  // ---- this (block, kv head, key tile)'s dk, dv: one writer per kernel
  if (k0 + kk < k1) {
    const int64_t off = ((start + k0 + kk) * dm.Hkv + g) * (int64_t)D + x0;
#pragma unroll
    for (int x = 0; x < D / 4; ++x) {
      a.dk[off + x] += dk[x] * scale;
      a.dv[off + x] += dv[x];
    }
  }
}

template <typename T, int D>
cudaError_t run_dot(const Dims& dm, const void* out, const void* dout, float* Dsum,
                    cudaStream_t st) {
  const int64_t rows = (int64_t)dm.T * dm.Hq;
  if (rows <= 0) return cudaSuccess;
  bwd_dot_kernel<T, D><<<(unsigned)((rows + 7) / 8), kThreads, 0, st>>>(
      rows, static_cast<const T*>(dout), static_cast<const T*>(out), Dsum);
  return cudaGetLastError();
}

template <typename T, int D>
cudaError_t run(const BwdArgs& a, int n_lists, cudaStream_t st) {
  const Dims& dm = a.dm;
  cudaError_t e;
  const size_t smem = BwdSmem<D>::bytes;
  if ((e = cudaFuncSetAttribute(bwd_block_kernel<T, D, HIST>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)))
    return e;
  if ((e = cudaFuncSetAttribute(bwd_block_kernel<T, D, CUR>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)))
    return e;
  const unsigned kts = (unsigned)((dm.B + KT - 1) / KT);
  if (n_lists > 0) {
    bwd_block_kernel<T, D, HIST><<<dim3((unsigned)n_lists, kts), kThreads, smem, st>>>(a);
    if ((e = cudaGetLastError())) return e;
  }
  const int64_t own = (int64_t)dm.batch * dm.Hkv * dm.nb;
  if (own > 0) {
    bwd_block_kernel<T, D, CUR><<<dim3((unsigned)own, kts), kThreads, smem, st>>>(a);
    if ((e = cudaGetLastError())) return e;
  }
  return cudaSuccess;
}

}  // namespace

cudaError_t launch_bwd_dot(const Dims& dm, const void* out, const void* dout, float* Dsum,
                           cudaStream_t st) {
  if (dm.dtype == kBF16)
    return dm.d == 128 ? run_dot<__nv_bfloat16, 128>(dm, out, dout, Dsum, st)
                       : run_dot<__nv_bfloat16, 64>(dm, out, dout, Dsum, st);
  return dm.d == 128 ? run_dot<float, 128>(dm, out, dout, Dsum, st)
                     : run_dot<float, 64>(dm, out, dout, Dsum, st);
}

cudaError_t launch_backward(const Dims& dm, const Chunk& ch, const void* q, const void* k,
                            const void* v, const void* dout, const float* lse, const float* Dsum,
                            const int32_t* cu, const int32_t* idx, const Regroup& rg, float* dq,
                            float* dk, float* dv, int* status, cudaStream_t st) {
  if (dm.batch == 0 || dm.max_seqlen == 0) return cudaSuccess;
  BwdArgs a{};
  a.dm = dm;
  a.ch = ch;
  a.q = q;
  a.k = k;
  a.v = v;
  a.dout = dout;
  a.lse = lse;
  a.Dsum = Dsum;
  a.cu = cu;
  a.idx = idx;
  a.list_off = rg.list_off;
  a.pairs = rg.pairs;
  a.dq = dq;
  a.dk = dk;
  a.dv = dv;
  a.status = status;
  if (dm.dtype == kBF16)
    return dm.d == 128 ? run<__nv_bfloat16, 128>(a, ch.n_lists, st)
                       : run<__nv_bfloat16, 64>(a, ch.n_lists, st);
  return dm.d == 128 ? run<float, 128>(a, ch.n_lists, st)
                     : run<float, 64>(a, ch.n_lists, st);
}

}  // namespace moba
