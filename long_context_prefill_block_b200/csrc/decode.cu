// Decode step (PaperTrace "2.1.3 MoBA", section 5.1 on long outputs --
// incremental block means and logical block numbers -- and section 5.4:
// decoding asks only a few queries per step and is bound by the KV reads and
// the launches, not by arithmetic).
//
// Request r's cache holds tokens cu[r] .. cu[r+1]-1 (length L_r, the new
// tokens' keys included); its n_r = cu_q[r+1] - cu_q[r] queries sit at the
// last positions L_r - n_r .. L_r - 1. Each query gets the prefill forward's
// result for its position: gate over the complete earlier blocks by their
// means (fp32), own block forced and counted in k, top-(k-1) of the rest
// (ties to the lower index), one softmax over the chosen keys, causal in the
// own block. Block ids are logical: block i of a request covers its
// positions iB .. iB+B-1, wherever its cache starts.
//
// Two launches, both SIMT (a query row against its keys is a matrix-vector
// product: HBM-bound, no tensor-core shape):
//   decode_gate_kernel  one CTA per (query, head), 8 warps: a warp reads a
//                       block mean with one coalesced 16-bytes-per-lane load,
//                       reduces the dot product with q by shuffles, and the
//                       lane owning the block keeps it in a sorted list; each
//                       warp picks its k-1 best by rounds of warp arg-max,
//                       and warp 0 merges the warps' lists the same way;
//   decode_attn_kernel  split-K over the chosen keys: one CTA per (query,
//                       q head, chosen block, chunk of <= 512 keys) keeps an
//                       online softmax (m, l, o) per group of lanes that share
//                       a key row, merges them and writes a normalised partial
//                       (o, lse); the row's last CTA to finish (an arrival
//                       counter, zeroed by the gate) merges the partials by
//                       eq. (7)-(8) written with lse and writes the output.
#include <climits>
#include <cmath>

#include "common.cuh"

namespace moba {
namespace {

constexpr int kGateWarps = 8;
constexpr int kAttnThreads = 256;
constexpr int kAttnWarps = kAttnThreads / 32;

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

// Request, cache start, cache length and position of query qi; false (and a
// status code) if cu_q does not describe a valid set of trailing queries.
__device__ __forceinline__ bool decode_position(const Dims& dm, const int32_t* __restrict__ cu,
                                                const int32_t* __restrict__ cu_q, int qi, int& r,
                                                int64_t& start, int& len, int& p, int* status) {
  int lo = 0, hi = dm.batch;  // largest r with cu_q[r] <= qi
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (cu_q[mid] <= qi) lo = mid;
    else hi = mid - 1;
  }
  r = lo;
  const int n = r < dm.batch ? cu_q[r + 1] - cu_q[r] : 0;
  if (r >= dm.batch || qi >= cu_q[r + 1] || !seq_bounds(dm, cu, r, start, len, status) || n > len) {
    set_status(status, kStInvalidArg);
    return false;
  }
  p = len - n + (qi - cu_q[r]);
  return true;
}

template <typename T, int D, int KM>
__global__ void __launch_bounds__(kGateWarps * 32)
decode_gate_kernel(Dims dm, const T* __restrict__ q, const float* __restrict__ kbar,
                   const int32_t* __restrict__ cu, const int32_t* __restrict__ cu_q,
                   int32_t* __restrict__ idx, int* __restrict__ arrivals, int* status) {
  __shared__ __align__(16) float qs[D];
  __shared__ float ws[kGateWarps][KM];
  __shared__ int wi[kGateWarps][KM];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int H = dm.shared ? dm.Hkv : dm.Hq;  // routing units per query
  const int qi = blockIdx.x / H, u = blockIdx.x % H;
  int r, len, p;
  int64_t start;
  if (!decode_position(dm, cu, cu_q, qi, r, start, len, p, status)) return;  // whole CTA
  const int grp = dm.Hq / dm.Hkv;
  const int g = dm.shared ? u : u / grp;
  const int h0 = dm.shared ? u * grp : u, nh = dm.shared ? grp : 1;
  // the query (with shared routing the sum of the group's queries: it ranks
  // the blocks as their mean does)
  for (int x = tid; x < D; x += kGateWarps * 32) {
    float s = 0.f;
    for (int j = 0; j < nh; ++j) s += to_f32(q[((int64_t)qi * dm.Hq + h0 + j) * D + x]);
    qs[x] = s;
  }
  // the attention kernel's split counters of these rows start at zero
  if (tid < nh) arrivals[(int64_t)qi * dm.Hq + h0 + tid] = 0;
  __syncthreads();
  const int c = p / dm.B;
  float ts[KM];
  int ti[KM];
#pragma unroll
  for (int j = 0; j < KM; ++j) {
    ts[j] = -INFINITY;
    ti[j] = INT_MAX;
  }
  // Warp-cooperative scores: LPB lanes read one block mean together (16
  // bytes each, one coalesced read of the block's d values), the dot product
  // is reduced over those lanes, and one of them (by step) keeps the score
  // in its sorted list. GU steps' loads are in flight together.
  constexpr int LPB = D / 4;     // lanes per block mean
  constexpr int BPS = 32 / LPB;  // block means a warp reads per step
  constexpr int GU = 8;
  const int grp_i = lane / LPB, sub = lane % LPB;
  const float4 qv = reinterpret_cast<const float4*>(qs)[sub];
  const int stride = kGateWarps * BPS;
  const int nsteps = (c + stride - 1) / stride;
  for (int s0 = 0; s0 < nsteps; s0 += GU) {
    float4 kv[GU];
#pragma unroll
    for (int u = 0; u < GU; ++u) {
      const int i = (s0 + u) * stride + warp * BPS + grp_i;
      kv[u] = i < c ? __ldg(reinterpret_cast<const float4*>(
                              kbar + (((int64_t)r * dm.nb + i) * dm.Hkv + g) * D) + sub)
                    : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int u = 0; u < GU; ++u) {
      float acc = fmaf(kv[u].w, qv.w, fmaf(kv[u].z, qv.z, fmaf(kv[u].y, qv.y, kv[u].x * qv.x)));
#pragma unroll
      for (int off = LPB / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
      const int st = s0 + u;
      const int i = st * stride + warp * BPS + grp_i;
      if (i < c && sub == st % LPB) insert<KM>(ts, ti, acc, i);
    }
  }
  // each warp: k-1 rounds of arg-max over the heads of its 32 sorted lists
  const int need = dm.topk - 1, hsel = min(need, c);
#pragma unroll
  for (int rr = 0; rr < KM; ++rr) {
    if (rr < need) {
      float bs = ts[0];
      int bi = ti[0], owner = lane;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        const float os = __shfl_xor_sync(0xffffffffu, bs, off);
        const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
        const int oo = __shfl_xor_sync(0xffffffffu, owner, off);
        if (better(os, oi, bs, bi)) {
          bs = os;
          bi = oi;
          owner = oo;
        }
      }
      if (owner == lane) {
#pragma unroll
        for (int j = 0; j + 1 < KM; ++j) {
          ts[j] = ts[j + 1];
          ti[j] = ti[j + 1];
        }
        ts[KM - 1] = -INFINITY;
        ti[KM - 1] = INT_MAX;
      }
      if (lane == 0) {
        ws[warp][rr] = bs;
        wi[warp][rr] = bi;
      }
    }
  }
  __syncthreads();
  if (warp != 0) return;
  // the warps' lists into one, by warp 0: each lane holds up to KC of the
  // candidates in a sorted list, then k-1 rounds of warp arg-max
  constexpr int KC = (kGateWarps * KM + 31) / 32;
  float cs[KC];
  int ci[KC];
#pragma unroll
  for (int j = 0; j < KC; ++j) {
    cs[j] = -INFINITY;
    ci[j] = INT_MAX;
  }
  for (int e = lane; e < kGateWarps * need; e += 32) insert<KC>(cs, ci, ws[e / need][e % need], wi[e / need][e % need]);
  float fs[KM];
  int fi[KM];
#pragma unroll
  for (int rr = 0; rr < KM; ++rr) {
    fs[rr] = -INFINITY;
    fi[rr] = INT_MAX;
    if (rr < need) {
      float bs = cs[0];
      int bi = ci[0], owner = lane;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        const float os = __shfl_xor_sync(0xffffffffu, bs, off);
        const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
        const int oo = __shfl_xor_sync(0xffffffffu, owner, off);
        if (better(os, oi, bs, bi)) {
          bs = os;
          bi = oi;
          owner = oo;
        }
      }
      if (owner == lane) {
#pragma unroll
        for (int j = 0; j + 1 < KC; ++j) {
          cs[j] = cs[j + 1];
          ci[j] = ci[j + 1];
        }
        cs[KC - 1] = -INFINITY;
        ci[KC - 1] = INT_MAX;
      }
      fs[rr] = bs;
      fi[rr] = bi;
    }
  }
  if (lane != 0) return;
  int sel[KM];
#pragma unroll
  for (int j = 0; j < KM; ++j) sel[j] = j < hsel ? fi[j] : INT_MAX;
#pragma unroll
  for (int a = 0; a < KM; ++a)
#pragma unroll
    for (int j = 0; j + 1 < KM - a; ++j)
      if (sel[j] > sel[j + 1]) {
        const int x = sel[j];
        sel[j] = sel[j + 1];
        sel[j + 1] = x;
      }
  for (int j = 0; j < nh; ++j) {
    int32_t* row = idx + ((int64_t)qi * dm.Hq + h0 + j) * dm.topk;
#pragma unroll
    for (int rr = 0; rr <= KM; ++rr)
      if (rr < dm.topk) row[rr] = rr < hsel ? sel[rr < KM ? rr : KM - 1] : (rr == hsel ? c : -1);
  }
}

// 16 raw bytes as fp32: 8 bf16 or 4 fp32 values.
template <typename T>
__device__ __forceinline__ void unpack16(const uint4& r, float* out) {
  const uint32_t w[4] = {r.x, r.y, r.z, r.w};
  if constexpr (sizeof(T) == 2) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      out[2 * i] = __uint_as_float(w[i] << 16);
      out[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i) out[i] = __uint_as_float(w[i]);
  }
}

// Keys per split: at most 512, never across a block boundary.
__host__ __device__ inline int split_keys(const Dims& dm) { return dm.B < 512 ? dm.B : 512; }
__host__ __device__ inline int splits_per_block(const Dims& dm) {
  return (dm.B + split_keys(dm) - 1) / split_keys(dm);
}
__host__ __device__ inline int splits_per_row(const Dims& dm) {
  return dm.topk * splits_per_block(dm);
}

// One CTA per (split s, q head h, query qi): blockIdx.x = qi * splits + s. Lanes are grouped LPK to a key
// row (16 bytes of the row per lane); each group walks keys
// lo + group, lo + group + groups, ... with an online softmax in the log2
// domain (logits pre-scaled by log2(e)/sqrt(d)), U keys per step so that
// several rows' loads are in flight.
template <typename T, int D>
__global__ void __launch_bounds__(kAttnThreads)
decode_attn_kernel(Dims dm, const T* __restrict__ q, const T* __restrict__ k,
                   const T* __restrict__ v, const int32_t* __restrict__ cu,
                   const int32_t* __restrict__ cu_q, const int32_t* __restrict__ idx,
                   float* __restrict__ part_o, float* __restrict__ part_lse,
                   int* __restrict__ arrivals, T* __restrict__ out, float* __restrict__ lse_out) {
  constexpr int EPL = Vec16<T>::N;  // elements per lane
  constexpr int LPK = D / EPL;      // lanes per key row
  constexpr int GPW = 32 / LPK;     // key groups per warp
  constexpr int G = GPW * kAttnWarps;
  // 4 rows per step keeps the kernel at 63 registers, 4 CTAs per SM: more
  // warps with loads in flight beat more loads per warp (8 rows: 74
  // registers, 3 CTAs per SM, 657 against 583 us for four queries at the
  // million-token cache)
  constexpr int U = 4;
  __shared__ float wm[kAttnWarps], wl[kAttnWarps];
  __shared__ __align__(16) float wo[kAttnWarps][D];
  const int S = splits_per_row(dm);
  const int s = (int)(blockIdx.x % S), qi = (int)(blockIdx.x / S), h = blockIdx.y;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t row = (int64_t)qi * dm.Hq + h, prow = row * S + s;
  int r, len, p;
  int64_t start;
  int lo = 0, hi = 0;
  if (decode_position(dm, cu, cu_q, qi, r, start, len, p, nullptr)) {
    const int c = p / dm.B, spb = splits_per_block(dm), kc = split_keys(dm);
    const int e = idx[((int64_t)qi * dm.Hq + h) * dm.topk + s / spb];
    if (e >= 0 && e <= c) {
      const int b0 = e * dm.B, b1 = e < c ? b0 + dm.B : p + 1;
      lo = b0 + (s % spb) * kc;
      hi = min(lo + kc, b1);
    }
  }
  if (lo >= hi) {  // no keys in this split (uniform over the CTA)
    if (tid == 0) part_lse[prow] = -INFINITY;
  } else {
  const int g = h / (dm.Hq / dm.Hkv);
  const int grp_id = warp * GPW + lane / LPK, sub = lane % LPK;
  const float sl2 = 1.4426950408889634f * rsqrtf((float)D);
  float qv[EPL];
  Vec16<T>::load(q + ((int64_t)qi * dm.Hq + h) * D + sub * EPL, qv);
#pragma unroll
  for (int x = 0; x < EPL; ++x) qv[x] *= sl2;
  float m = -INFINITY, l = 0.f, o[EPL];
#pragma unroll
  for (int x = 0; x < EPL; ++x) o[x] = 0.f;
  const T* kbase = k + kv_row(dm, start, g) + sub * EPL;
  const T* vbase = v + kv_row(dm, start, g) + sub * EPL;
  // row stride of the cache: a head-major cache keeps one head's rows
  // contiguous, so a split streams consecutive rows
  const int64_t rs = dm.kv_hm ? (int64_t)D : (int64_t)dm.Hkv * D;
  // The trip count is the same for every lane (the shuffles need all 32).
  // A step loads U rows per lane group as raw 16-byte vectors (all 2U loads
  // in flight together), then folds them into the softmax with one rescale.
  for (int base = lo; base < hi; base += U * G) {
    uint4 kr[U], vr[U];
#pragma unroll
    for (int uu = 0; uu < U; ++uu) {
      const int j = base + grp_id + uu * G;
      const int jj = j < hi ? j : lo;  // a row in range; its value is not used
      kr[uu] = __ldg(reinterpret_cast<const uint4*>(kbase + jj * rs));
      vr[uu] = __ldg(reinterpret_cast<const uint4*>(vbase + jj * rs));
    }
    float d[U];
    float mn = m;
#pragma unroll
    for (int uu = 0; uu < U; ++uu) {
      float kx[EPL];
      unpack16<T>(kr[uu], kx);
      float acc = 0.f;
#pragma unroll
      for (int x = 0; x < EPL; ++x) acc = fmaf(qv[x], kx[x], acc);
#pragma unroll
      for (int off = LPK / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
      d[uu] = base + grp_id + uu * G < hi ? acc : -INFINITY;
      mn = fmaxf(mn, d[uu]);
    }
    if (mn == -INFINITY) continue;  // this group has no key in the step
    const float corr = exp2f(m - mn);
    l *= corr;
#pragma unroll
    for (int x = 0; x < EPL; ++x) o[x] *= corr;
#pragma unroll
    for (int uu = 0; uu < U; ++uu) {
      const float w = exp2f(d[uu] - mn);
      float vx[EPL];
      unpack16<T>(vr[uu], vx);
      l += w;
#pragma unroll
      for (int x = 0; x < EPL; ++x) o[x] = fmaf(w, vx[x], o[x]);
    }
    m = mn;
  }
  // merge the lane groups of the warp (groups that saw no key have m = -inf)
#pragma unroll
  for (int off = LPK; off < 32; off <<= 1) {
    const float mo = __shfl_xor_sync(0xffffffffu, m, off);
    const float lo2 = __shfl_xor_sync(0xffffffffu, l, off);
    const float mn = fmaxf(m, mo);
    const float a = mn == -INFINITY ? 0.f : exp2f(m - mn);
    const float b = mn == -INFINITY ? 0.f : exp2f(mo - mn);
    l = l * a + lo2 * b;
#pragma unroll
    for (int x = 0; x < EPL; ++x) {
      const float ox = __shfl_xor_sync(0xffffffffu, o[x], off);
      o[x] = o[x] * a + ox * b;
    }
    m = mn;
  }
  if (lane < LPK) {
#pragma unroll
    for (int x = 0; x < EPL; ++x) wo[warp][sub * EPL + x] = o[x];
    if (lane == 0) {
      wm[warp] = m;
      wl[warp] = l;
    }
  }
  __syncthreads();
  float M = -INFINITY;
#pragma unroll
  for (int w = 0; w < kAttnWarps; ++w) M = fmaxf(M, wm[w]);
  float L = 0.f;
#pragma unroll
  for (int w = 0; w < kAttnWarps; ++w) L += wm[w] == -INFINITY ? 0.f : wl[w] * exp2f(wm[w] - M);
  for (int x = tid; x < D; x += kAttnThreads) {
    float acc = 0.f;
#pragma unroll
    for (int w = 0; w < kAttnWarps; ++w)
      if (wm[w] != -INFINITY) acc = fmaf(wo[w][x], exp2f(wm[w] - M), acc);
    part_o[prow * D + x] = acc / L;
  }
  if (tid == 0) part_lse[prow] = (M + log2f(L)) * 0.6931471805599453f;
  }
  // The last split of the row to arrive merges them all (eq. 7-8 written
  // with lse: w_s = exp(lse_s - max lse), o = sum_s w_s o_s / sum_s w_s).
  // No CTA waits for another: the others have written their partials and
  // left.
  __shared__ int last;
  __threadfence();
  __syncthreads();
  if (tid == 0) last = atomicAdd(&arrivals[row], 1) == S - 1;
  __syncthreads();
  if (!last) return;
  __threadfence();
  const float* ls = part_lse + row * S;
  float M = -INFINITY;
  for (int s2 = tid; s2 < S; s2 += kAttnThreads) M = fmaxf(M, __ldcg(ls + s2));
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
  if (lane == 0) wm[warp] = M;
  __syncthreads();
#pragma unroll
  for (int w = 0; w < kAttnWarps; ++w) M = fmaxf(M, wm[w]);
  // warp w takes splits w, w + 8, ...: a lane holds four columns of the row,
  // loads are branch-free (a split without keys gets weight 0; its partial
  // row is never written, so its value is masked, not multiplied)
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  float Lw = 0.f;
  const bool cols = lane * 4 < D;
#pragma unroll 4
  for (int s2 = warp; s2 < S; s2 += kAttnWarps) {
    const float lv = __ldcg(ls + s2);
    const bool on = lv != -INFINITY;
    const float w = on ? expf(lv - M) : 0.f;
    Lw += w;
    if (cols) {
      const float4 ov = __ldcg(reinterpret_cast<const float4*>(part_o + (row * S + s2) * D) + lane);
      acc.x += on ? w * ov.x : 0.f;
      acc.y += on ? w * ov.y : 0.f;
      acc.z += on ? w * ov.z : 0.f;
      acc.w += on ? w * ov.w : 0.f;
    }
  }
  __syncthreads();  // wo, wl are free again
  if (cols) *reinterpret_cast<float4*>(&wo[warp][lane * 4]) = acc;
  if (lane == 0) wl[warp] = Lw;
  __syncthreads();
  for (int x = tid; x < D; x += kAttnThreads) {
    float O = 0.f, L = 0.f;
#pragma unroll
    for (int w = 0; w < kAttnWarps; ++w) {
      O += wo[w][x];
      L += wl[w];
    }
    out[row * D + x] = from_f32<T>(O / L);
    if (x == 0 && lse_out) lse_out[row] = M + logf(L);
  }
}

template <typename T, int D, int KM>
cudaError_t run_gate(const Dims& dm, int nq, const void* q, const float* kbar, const int32_t* cu,
                     const int32_t* cu_q, int32_t* idx, int* arrivals, int* status,
                     cudaStream_t st) {
  const int64_t items = (int64_t)nq * (dm.shared ? dm.Hkv : dm.Hq);
  if (items > INT32_MAX) return cudaErrorInvalidValue;
  decode_gate_kernel<T, D, KM><<<(unsigned)items, kGateWarps * 32, 0, st>>>(
      dm, static_cast<const T*>(q), kbar, cu, cu_q, idx, arrivals, status);
  return cudaGetLastError();
}

template <typename T, int D>
cudaError_t run(const Dims& dm, int nq, const void* q, const void* k, const void* v,
                const int32_t* cu, const int32_t* cu_q, const float* kbar, int32_t* idx,
                float* part_o, float* part_lse, int* arrivals, void* out, float* lse, int* status,
                cudaStream_t st) {
  cudaError_t e;
  const int need = dm.topk - 1;
  if (need <= 1) e = run_gate<T, D, 1>(dm, nq, q, kbar, cu, cu_q, idx, arrivals, status, st);
  else if (need <= 2) e = run_gate<T, D, 2>(dm, nq, q, kbar, cu, cu_q, idx, arrivals, status, st);
  else if (need <= 4) e = run_gate<T, D, 4>(dm, nq, q, kbar, cu, cu_q, idx, arrivals, status, st);
  else if (need <= 8) e = run_gate<T, D, 8>(dm, nq, q, kbar, cu, cu_q, idx, arrivals, status, st);
  else if (need <= 16) e = run_gate<T, D, 16>(dm, nq, q, kbar, cu, cu_q, idx, arrivals, status, st);
  else e = run_gate<T, D, 32>(dm, nq, q, kbar, cu, cu_q, idx, arrivals, status, st);
  if (e != cudaSuccess) return e;
  if ((int64_t)splits_per_row(dm) * nq > INT32_MAX) return cudaErrorInvalidValue;
  dim3 grid((unsigned)(splits_per_row(dm) * nq), (unsigned)dm.Hq);
  decode_attn_kernel<T, D><<<grid, kAttnThreads, 0, st>>>(
      dm, static_cast<const T*>(q), static_cast<const T*>(k), static_cast<const T*>(v), cu, cu_q,
      idx, part_o, part_lse, arrivals, static_cast<T*>(out), lse);
  return cudaGetLastError();
}

}  // namespace

size_t decode_partial_rows(const Dims& dm, int n_queries) {
  return (size_t)n_queries * dm.Hq * splits_per_row(dm);
}

cudaError_t launch_decode(const Dims& dm, int n_queries, const void* q, const void* k,
                          const void* v, const int32_t* cu, const int32_t* cu_q, const float* kbar,
                          int32_t* idx, float* part_o, float* part_lse, int* arrivals, void* out,
                          float* lse, int* status, cudaStream_t st) {
  if (dm.batch == 0 || n_queries == 0) return cudaSuccess;
  if (dm.dtype == kBF16)
    return dm.d == 128 ? run<__nv_bfloat16, 128>(dm, n_queries, q, k, v, cu, cu_q, kbar, idx,
                                                 part_o, part_lse, arrivals, out, lse, status, st)
                       : run<__nv_bfloat16, 64>(dm, n_queries, q, k, v, cu, cu_q, kbar, idx,
                                                part_o, part_lse, arrivals, out, lse, status, st);
  return dm.d == 128 ? run<float, 128>(dm, n_queries, q, k, v, cu, cu_q, kbar, idx, part_o,
                                       part_lse, arrivals, out, lse, status, st)
                     : run<float, 64>(dm, n_queries, q, k, v, cu, cu_q, kbar, idx, part_o,
                                      part_lse, arrivals, out, lse, status, st);
}

}  // namespace moba
