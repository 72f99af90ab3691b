// Tensor-core form of the MoBA gate (PaperTrace "2.1.3 MoBA", section 1
// eq. 3, section 2, section 2.1): the scores s_i = q . kbar_i of a tile of
// 128 queries of one head against the blocks of its sequence are one
// tcgen05 contraction; the causal block mask, the forced own block and the
// top-k run in the epilogue, one query row per thread (TMEM lane = row).
//
// Scores as exact as an fp32 dot product from bf16 tensor cores: q is bf16
// (exact), and each fp32 kbar element is split into three bf16 terms,
// kbar = h + m + l with h = bf16(kbar), m = bf16(kbar - h), l = bf16(kbar -
// h - m) (both differences are exact in fp32), so the three products q.h +
// q.m + q.l, accumulated in fp32 in TMEM, carry kbar to 2^-24 relative, as
// the fp32 path does.
//
// Persistent CTAs walk work items (sequence, kv head, query tile, q head of
// the group) in that order: a CTA splits the kbar rows of its (sequence, kv
// head) into shared memory once and reuses them for every q head and query
// tile of the group; the next tile's Q is fetched by TMA while the current
// one is selected.
#include <climits>
#include <mutex>

#include "tc_ptx.cuh"

namespace moba {
namespace {

using namespace tc;

constexpr int kThreads = 256;                // row r: threads r and r + 128
constexpr int kTileRows = 128;               // queries per tile
constexpr uint32_t kQHalf = 128 * 128;       // one 64-column half of a Q tile
constexpr uint32_t kQTile = 2 * kQHalf;
constexpr int kMaxBlocks = 256;              // MMA N limit
constexpr int kCuSmem = 257;                 // sequence offsets kept in shared memory (batch <= 256)

struct GateArgs {
  Dims dm;
  const float* kbar;
  const float* own;  // own-block scores [T][Hq] of the prefix-mean gate, else unused
  const int32_t* cu;
  int32_t* idx;
  int* status;
  int groups;      // batch * Hkv (sequence, kv head) groups
  int ipg;         // items per group: query tiles per sequence * q heads per kv head
  int cpg;         // CTAs per group (0: each CTA takes whole groups, round robin)
  int nbp;         // blocks per sequence rounded up to a multiple of 16
  int qbuf;        // Q buffers (1 or 2)
  uint32_t tmem_cols;
  uint32_t merge_col;  // TMEM column of the second thread's list (scores, then indices)
};

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

// Insertion during a thread's own scan: indices only grow, so an equal score
// never displaces an earlier (lower) block.
template <int KM>
__device__ __forceinline__ void insert_scan(float (&ts)[KM], int (&ti)[KM], float s, int i) {
#pragma unroll
  for (int j = 0; j < KM; ++j) {
    if (s > ts[j]) {
      const float fs = ts[j];
      const int fi = ti[j];
      ts[j] = s;
      ti[j] = i;
      s = fs;
      i = fi;
    }
  }
}

struct Item {
  int b, g, h, p0;
  int64_t start;
  int len;
};

__device__ __forceinline__ Item decode(const GateArgs& a, const int32_t* cu, int it) {
  const Dims& dm = a.dm;
  const int grp = dm.Hq / dm.Hkv;
  const int per_tile = dm.shared ? 1 : grp;  // items per (query tile, kv head)
  const int nqt = (dm.max_seqlen + kTileRows - 1) / kTileRows;
  Item x;
  const int hl = it % per_tile;
  int rest = it / per_tile;
  const int qt = rest % nqt;
  rest /= nqt;
  x.g = rest % dm.Hkv;
  x.b = rest / dm.Hkv;
  x.h = x.g * grp + hl;
  x.p0 = qt * kTileRows;
  x.start = cu[x.b];
  x.len = cu[x.b + 1] - cu[x.b];
  return x;
}

// Item of this CTA's s-th slot, or -1 past its last. With more groups than
// CTAs a CTA takes whole groups; otherwise cpg CTAs share a group, taking
// every cpg-th item, so each sees early and late query tiles alike (the
// later a tile, the more blocks its rows score).
__device__ __forceinline__ int item_of(const GateArgs& a, int s) {
  if (a.cpg == 0) {
    const int gi = blockIdx.x + (s / a.ipg) * gridDim.x;
    return gi < a.groups ? gi * a.ipg + s % a.ipg : -1;
  }
  const int gi = blockIdx.x / a.cpg, j = blockIdx.x % a.cpg;
  const int64_t w = j + (int64_t)s * a.cpg;
  return (gi < a.groups && w < a.ipg) ? gi * a.ipg + (int)w : -1;
}

// First item at slot s or later whose query tile holds at least one query
// (s is moved to its slot), or -1.
__device__ __forceinline__ int next_valid(const GateArgs& a, const int32_t* cu, int& s) {
  for (;; ++s) {
    const int it = item_of(a, s);
    if (it < 0) return -1;
    const Item x = decode(a, cu, it);
    if (x.len > 0 && x.len <= a.dm.max_seqlen && x.p0 < x.len) return it;
  }
}

// PFX: the own block is scored by its prefix mean (compiled separately, so
// the forced-own-block kernel carries none of that code)
template <int KM, bool PFX>
__global__ void __launch_bounds__(kThreads, KM <= 4 ? 3 : 1)
gate_tc_kernel(const __grid_constant__ CUtensorMap tmq, const GateArgs a) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t q_full[2], mma_done;
  __shared__ uint32_t tmem_base;
  __shared__ int abort_flag;
  __shared__ int32_t cu_s[kCuSmem];
  const Dims& dm = a.dm;
  const int tid = threadIdx.x, warp = tid >> 5;

  const uint32_t sbase = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const uint32_t sQ = sbase;                          // Q[qbuf]
  const uint32_t sK = sbase + a.qbuf * kQTile;        // kbar terms [3][2 halves][nbp][128 B]
  const uint32_t kTermHalf = (uint32_t)a.nbp * 128u;  // bytes of one 64-column half of a term

  const bool cu_in_smem = dm.batch + 1 <= kCuSmem;
  if (cu_in_smem)
    for (int i = tid; i <= dm.batch; i += kThreads) cu_s[i] = a.cu[i];
  const int32_t* cu = cu_in_smem ? cu_s : a.cu;
  if (tid == 0) {
    mbar_init(&q_full[0], 1);
    mbar_init(&q_full[1], 1);
    mbar_init(&mma_done, 1);
    abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 0) {
    tmem_alloc(&tmem_base, a.tmem_cols);
    tmem_relinquish();
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tmem = tmem_base;
  volatile int* abort = &abort_flag;
  int* status = a.status;

  // Q tiles per item: with shared routing every q head of the group, whose
  // scores accumulate in TMEM (their sum ranks like their mean)
  const int nh = dm.shared ? dm.Hq / dm.Hkv : 1;
  auto issue_q = [&](int it, int hh, uint32_t buf) {
    const Item x = decode(a, cu, it);
    mbar_expect_tx(&q_full[buf], kQTile);
    const int z = (int)(x.start + x.p0);
    tma_load_3d(sQ + buf * kQTile, &tmq, &q_full[buf], 0, x.h + hh, z);
    tma_load_3d(sQ + buf * kQTile + kQHalf, &tmq, &q_full[buf], 64, x.h + hh, z);
  };

  int slot = 0;
  int it = next_valid(a, cu, slot);
  uint32_t nq = 0, nmma = 0;  // Q tiles requested / consumed so far; MMA groups
  uint32_t n_issued = 0;
  if (it >= 0 && tid == 0) {
    issue_q(it, 0, 0);
    n_issued = 1;
  }
  int cur_b = -1, cur_g = -1;
  bool ok = true;
  while (ok && it >= 0) {
    const Item x = decode(a, cu, it);
    if (x.b != cur_b || x.g != cur_g) {
      // split this (sequence, kv head)'s kbar rows into the three bf16 terms,
      // K-major, 128-byte swizzle (the layout a TMA tile of them would have)
      __syncthreads();
      for (int e = tid; e < a.nbp * 32; e += kThreads) {
        const int i = e >> 5, d = (e & 31) * 4;
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        if (i < dm.nb)
          v = *reinterpret_cast<const float4*>(
              a.kbar + (((int64_t)x.b * dm.nb + i) * dm.Hkv + x.g) * 128 + d);
        const float vv[4] = {v.x, v.y, v.z, v.w};
        uint32_t w[3][2];
#pragma unroll
        for (int u = 0; u < 4; u += 2) {
          float hi[2], mid[2], lo[2];
#pragma unroll
          for (int q = 0; q < 2; ++q) {
            const float f = vv[u + q];
            hi[q] = __bfloat162float(__float2bfloat16_rn(f));
            const float r1 = f - hi[q];
            mid[q] = __bfloat162float(__float2bfloat16_rn(r1));
            lo[q] = r1 - mid[q];
          }
          w[0][u >> 1] = pack_bf16x2(hi[0], hi[1]);
          w[1][u >> 1] = pack_bf16x2(mid[0], mid[1]);
          w[2][u >> 1] = pack_bf16x2(lo[0], lo[1]);
        }
        const uint32_t off = (uint32_t)(d >> 6) * kTermHalf + (uint32_t)i * 128u +
                             ((((uint32_t)(d & 63) >> 3) ^ ((uint32_t)i & 7u)) << 4) +
                             (uint32_t)(d & 7) * 2u;
#pragma unroll
        for (int t = 0; t < 3; ++t)
          asm volatile("st.shared.v2.b32 [%0], {%1, %2};" ::"r"(sK + t * 2 * kTermHalf + off),
                       "r"(w[t][0]), "r"(w[t][1])
                       : "memory");
      }
      fence_proxy_async_smem();
      __syncthreads();
      cur_b = x.b;
      cur_g = x.g;
    }
    // blocks any row of the tile may choose: i < c(p) <= c_max
    const int c_max = (min(x.p0 + kTileRows, x.len) - 1) / dm.B;
    const int N = ((c_max + 15) / 16) * 16;
    int nslot = slot + 1;
    const int nxt = next_valid(a, cu, nslot);
    for (int hh = 0; ok && hh < nh; ++hh) {
      const uint32_t qb = nq % a.qbuf;
      ok = mbar_wait(&q_full[qb], (nq / a.qbuf) & 1, abort, status);
      if (!ok) break;
      ++nq;
      if (N > 0 && tid == 0) {
        fence_after_sync();
        const uint32_t idesc = idesc_bf16(kTileRows, N, false, false);
#pragma unroll 1
        for (int t = 0; t < 3; ++t)
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t ko = (kk >> 2) * kQHalf + (kk & 3) * 32;
            const uint64_t ad = desc_sw128(sQ + qb * kQTile + ko, 16, 1024);
            const uint64_t bd = desc_sw128(
                sK + t * 2 * kTermHalf + (kk >> 2) * kTermHalf + (kk & 3) * 32, 16, 1024);
            mma_ss(tmem, ad, bd, idesc, (hh > 0 || t > 0 || kk > 0) ? 1u : 0u);
          }
        commit(&mma_done);
      }
      // the next Q tile: this item's next head, else the next item's first
      const bool more = hh + 1 < nh;
      const bool has_next = more || nxt >= 0;
      if (a.qbuf == 2 && tid == 0 && has_next) {
        // the other buffer's last reader (the previous tile's MMA) is done
        issue_q(more ? it : nxt, more ? hh + 1 : 0, n_issued % 2);
        ++n_issued;
      }
      if (N > 0) {
        ok = mbar_wait(&mma_done, nmma & 1, abort, status);
        ++nmma;
        if (!ok) break;
        fence_after_sync();
      }
      if (a.qbuf == 1 && tid == 0 && has_next) {
        issue_q(more ? it : nxt, more ? hh + 1 : 0, 0);
        ++n_issued;
      }
    }
    if (!ok) break;
    // ---- selection: row rr of the tile (TMEM lane rr); thread rr scans the
    // even 32-column chunks of the candidates, thread rr + 128 the odd ones,
    // then the first merges the second's list
    const int rr = tid & (kTileRows - 1), part = tid >> 7;
    const int p = x.p0 + rr;
    const bool valid = p < x.len;
    const int c = valid ? p / dm.B : 0;
    float ts[KM];
    int ti[KM];
#pragma unroll
    for (int j = 0; j < KM; ++j) {
      ts[j] = -INFINITY;
      ti[j] = INT_MAX;
    }
    const int cw = __reduce_max_sync(0xffffffffu, c);  // columns this warp needs
    const uint32_t taddr = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    for (int cb = part; cb * 32 < cw; cb += 2) {
      if (KM <= 4) {
        uint32_t rr[32];
        tmem_ld32(taddr + cb * 32, rr);
        tmem_wait_ld();
#pragma unroll
        for (int xx = 0; xx < 32; ++xx) {
          const int i = cb * 32 + xx;
          if (cb * 32 + xx >= cw) break;  // past every row's candidates in this warp
          if (i < c) insert_scan<KM>(ts, ti, __uint_as_float(rr[xx]), i);
        }
      } else {
        // long lists: four columns per step, so the unrolled insertion code
        // stays small enough for the instruction cache
#pragma unroll 1
        for (int x4 = 0; x4 < 8 && cb * 32 + x4 * 4 < cw; ++x4) {
          uint32_t rr[4];
          tmem_ld4(taddr + cb * 32 + x4 * 4, rr);
          tmem_wait_ld();
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int i = cb * 32 + x4 * 4 + u;
            if (i < c) insert_scan<KM>(ts, ti, __uint_as_float(rr[u]), i);
          }
        }
      }
    }
    // the second thread's list goes through TMEM (same lane, spare columns)
    constexpr int MW = KM < 16 ? 16 : KM;
    const uint32_t tm_s = taddr + a.merge_col, tm_i = tm_s + MW;
    if (part == 1) {
#pragma unroll
      for (int c16 = 0; c16 < MW / 16; ++c16) {
        uint32_t vs[16], vi[16];
#pragma unroll
        for (int u = 0; u < 16; ++u) {
          const int j = c16 * 16 + u;
          vs[u] = __float_as_uint(j < KM ? ts[j < KM ? j : 0] : -INFINITY);
          vi[u] = (uint32_t)(j < KM ? ti[j < KM ? j : 0] : INT_MAX);
        }
        tmem_st16(tm_s + c16 * 16, vs);
        tmem_st16(tm_i + c16 * 16, vi);
      }
      tmem_wait_st();
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    if (part == 0) {
#pragma unroll
      for (int c16 = 0; c16 < MW / 16; ++c16) {
        uint32_t vs[16], vi[16];
        tmem_ld16(tm_s + c16 * 16, vs);
        tmem_ld16(tm_i + c16 * 16, vi);
        tmem_wait_ld();
#pragma unroll
        for (int u = 0; u < 16; ++u)
          if (c16 * 16 + u < KM) insert<KM>(ts, ti, __uint_as_float(vs[u]), (int)vi[u]);
      }
    }
    if (part == 0 && valid) {
      // the own block: forced, or (prefix mean) in unless k earlier blocks
      // score at least as high; it loses ties, being the highest index
      bool own_in = true;
      if (PFX && c >= dm.topk) {
        float kth = -INFINITY, so = 0.f;
#pragma unroll
        for (int j = 0; j < KM; ++j)
          if (j == dm.topk - 1) kth = ts[j];
        for (int hh = 0; hh < nh; ++hh) so += a.own[(x.start + p) * dm.Hq + x.h + hh];
        own_in = !(kth >= so);
      }
      const int hsel = own_in ? min(dm.topk - 1, c) : dm.topk;
      int sel[KM];
#pragma unroll
      for (int r = 0; r < KM; ++r) sel[r] = r < hsel ? ti[r] : INT_MAX;
      // ascending order of the chosen earlier blocks
#pragma unroll
      for (int q = 0; q < KM; ++q)
#pragma unroll
        for (int j = 0; j + 1 < KM - q; ++j)
          if (sel[j] > sel[j + 1]) {
            const int s = sel[j];
            sel[j] = sel[j + 1];
            sel[j + 1] = s;
          }
      for (int hh = 0; hh < nh; ++hh) {
        if (!MOBA_CHECK(x.start + p < dm.T && x.h + hh < dm.Hq, status)) break;
        int32_t* row = a.idx + ((x.start + p) * dm.Hq + x.h + hh) * (int64_t)dm.topk;
        for (int r = 0; r < dm.topk; ++r)
          row[r] = r < hsel ? sel[r < KM ? r : KM - 1] : (r == hsel && own_in ? c : -1);
      }
    }
    // TMEM and this Q buffer are free again
    fence_before_sync();
    __syncthreads();
    it = nxt;
    slot = nslot;
  }
  if (!ok) *abort = 1;
  __syncthreads();
  if (tid == 0) {
    // let every copy and MMA issued land before the CTA exits
    for (uint32_t x = nq; x < n_issued; ++x) mbar_drain(&q_full[x % a.qbuf], (x / a.qbuf) & 1);
    commit(&mma_done);
    mbar_drain(&mma_done, nmma & 1);
  }
  fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    fence_after_sync();
    tmem_dealloc(tmem, a.tmem_cols);
  }
}

constexpr int kMaxSmem = 232448;  // 227 KB per CTA

// CTAs of gate_tc_kernel<KM, PFX> per SM at `smem` bytes of dynamic shared
// memory, bounded by registers and shared memory (counted here from the
// kernel's attributes, asked once per device and remembered).
template <int KM, bool PFX>
cudaError_t occupancy(int* n, size_t smem) {
  static std::mutex mu;
  static cudaFuncAttributes attrs[kMaxDevices];
  static bool have[kMaxDevices] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  if (!have[dev]) {
    if ((e = cudaFuncGetAttributes(&attrs[dev], gate_tc_kernel<KM, PFX>))) return e;
    // allow all the dynamic shared memory the static part leaves
    if ((e = cudaFuncSetAttribute(gate_tc_kernel<KM, PFX>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  kMaxSmem - (int)attrs[dev].sharedSizeBytes)))
      return e;
    have[dev] = true;
  }
  const cudaFuncAttributes& fa = attrs[dev];
  const size_t per_cta = smem + fa.sharedSizeBytes;
  if (per_cta > (size_t)kMaxSmem) {
    *n = 0;
    return cudaSuccess;
  }
  constexpr size_t kSmemPerSM = 233472;  // 228 KB, of which 1 KB is reserved per CTA
  int by_smem = (int)(kSmemPerSM / (per_cta + 1024));
  const int regs = ((fa.numRegs + 7) / 8) * 8;
  int by_regs = regs > 0 ? 65536 / (regs * kThreads) : 1;
  *n = by_smem < by_regs ? by_smem : by_regs;
  return cudaSuccess;
}

template <int KM, bool PFX>
cudaError_t run(const CUtensorMap& mq, const GateArgs& a, size_t smem, int grid, cudaStream_t st) {
  gate_tc_kernel<KM, PFX><<<grid, kThreads, smem, st>>>(mq, a);
  return cudaGetLastError();
}

}  // namespace

bool gate_tc_supported(const Dims& dm) {
  return dm.dtype == kBF16 && dm.d == 128 && dm.nb <= kMaxBlocks && dm.topk <= 33;
}

namespace {
template <bool PFX>
cudaError_t launch_impl(const Dims& dm, const void* q, const float* kbar, const float* own,
                        const int32_t* cu, int32_t* idx, int* status, cudaStream_t st) {
  if (dm.batch == 0 || dm.max_seqlen == 0) return cudaSuccess;
  GateArgs a{};
  a.dm = dm;
  a.kbar = kbar;
  a.own = own;
  a.cu = cu;
  a.idx = idx;
  a.status = status;
  const int nqt = (dm.max_seqlen + kTileRows - 1) / kTileRows;
  const int64_t ipg = (int64_t)nqt * (dm.shared ? 1 : dm.Hq / dm.Hkv);
  if ((int64_t)dm.batch * dm.Hkv * ipg > INT_MAX) return cudaErrorInvalidValue;
  a.groups = dm.batch * dm.Hkv;
  a.ipg = (int)ipg;
  a.nbp = ((dm.nb + 15) / 16) * 16;
  const int need = hist_slots(dm);
  const int km = need <= 1 ? 1 : need <= 2 ? 2 : need <= 4 ? 4 : need <= 8 ? 8 : need <= 16 ? 16 : 32;
  const size_t fixed = 1024 + (size_t)3 * 2 * a.nbp * 128;
  constexpr size_t kSmemMax = kMaxSmem;
  // accumulator columns (read 32 at a time), then the merge lists
  a.merge_col = (uint32_t)((a.nbp + 31) / 32) * 32;
  uint32_t cols = 32;
  while (cols < a.merge_col + 2u * (km < 16 ? 16u : (uint32_t)km)) cols <<= 1;
  if (cols > 512) return cudaErrorInvalidConfiguration;
  a.tmem_cols = cols;
  // CTAs per SM: shared memory (as the occupancy calculator counts it) and
  // the 512 TMEM columns both bound it. A second Q buffer (prefetch) is used
  // only where it costs no CTA per SM.
  const int need_km = km;
  auto per_sm_of = [&](int qbuf) {
    const size_t smem = fixed + (size_t)qbuf * kQTile;
    if (smem > kSmemMax) return 0;
    int n = 0;
    cudaError_t e2;
    switch (need_km) {
      case 1: e2 = occupancy<1, PFX>(&n, smem); break;
      case 2: e2 = occupancy<2, PFX>(&n, smem); break;
      case 4: e2 = occupancy<4, PFX>(&n, smem); break;
      case 8: e2 = occupancy<8, PFX>(&n, smem); break;
      case 16: e2 = occupancy<16, PFX>(&n, smem); break;
      default: e2 = occupancy<32, PFX>(&n, smem); break;
    }
    if (e2 != cudaSuccess) return 0;
    if (n > (int)(512 / cols)) n = (int)(512 / cols);
    return n;
  };
  a.qbuf = per_sm_of(2) >= per_sm_of(1) && per_sm_of(2) > 0 ? 2 : 1;
  const size_t smem = fixed + (size_t)a.qbuf * kQTile;
  const int per_sm = per_sm_of(a.qbuf);
  if (per_sm < 1) return cudaErrorInvalidConfiguration;
  const int target = sm_count() * per_sm;
  int grid;
  if (a.groups >= target) {
    a.cpg = 0;
    grid = target;
  } else {
    a.cpg = target / a.groups;
    if (a.cpg > a.ipg) a.cpg = a.ipg;
    grid = a.groups * a.cpg;
  }
  CUtensorMap mq;
  cudaError_t e = make_head_map(&mq, q, dm.T, dm.Hq, kTileRows);
  if (e != cudaSuccess) return e;
  if (need <= 1) return run<1, PFX>(mq, a, smem, grid, st);
  if (need <= 2) return run<2, PFX>(mq, a, smem, grid, st);
  if (need <= 4) return run<4, PFX>(mq, a, smem, grid, st);
  if (need <= 8) return run<8, PFX>(mq, a, smem, grid, st);
  if (need <= 16) return run<16, PFX>(mq, a, smem, grid, st);
  return run<32, PFX>(mq, a, smem, grid, st);
}

}  // namespace

cudaError_t launch_gate_tc(const Dims& dm, const void* q, const float* kbar, const float* own,
                           const int32_t* cu, int32_t* idx, int* status, cudaStream_t st) {
  if (gate_net_supported(dm)) return launch_gate_net(dm, q, kbar, cu, idx, status, st);
  return dm.prefix ? launch_impl<true>(dm, q, kbar, own, cu, idx, status, st)
                   : launch_impl<false>(dm, q, kbar, own, cu, idx, status, st);
}

}  // namespace moba
