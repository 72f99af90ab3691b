// Tensor-core backward of MoBA attention (PaperTrace "2.1.3 MoBA", section
// 5.3: the hard top-k passes no gradient; the loss flows back along the
// Q/K/V that were read), bf16 inputs, d = 128, B % 128 == 0.
//
// Same decomposition as the SIMT backward: one CTA per (regroup list of a
// history block, 128-key tile) and one per (own block, kv head, 128-key
// tile), each walking its query rows 128 at a time. Per row tile, five
// tcgen05 contractions (M = N = K = 128, fp32 accumulation in TMEM):
//   S  = Q K^T,  dP = dO V^T                     (TMEM columns 0, 128)
//   P  = exp(S / sqrt(d) - lse), dS = P (dP - D) (threads, one row each;
//        written to shared memory as bf16, [rows][keys], 128-byte swizzle)
//   dV += P^T dO, dK += dS^T Q                    (TMEM 256, 384; A operands
//        are the P / dS tiles read M-major, i.e. transposed)
//   dQ  = dS K                                    (TMEM 0, reusing S)
// dQ leaves by fp32 atomics (several key tiles add into one row); the
// tile's dK, dV leave once, at the end, added to the fp32 outputs.
#include "tc_ptx.cuh"

namespace moba {

bool bwd_tc_supported(const Dims& dm) {
  return dm.dtype == kBF16 && dm.d == 128 && dm.B % 128 == 0;
}

namespace {

using namespace tc;

enum { HIST = 0, CUR = 1 };
constexpr int kThreads = 128;  // thread r: tile row r, TMEM lane r
constexpr int TM = 128;        // query rows per tile
constexpr int TN = 128;        // keys per CTA
constexpr int D = 128;
constexpr uint32_t kHalf = 128 * 128;  // one 64-column half of a 128-row bf16 tile
constexpr uint32_t kTile = 2 * kHalf;
// shared memory: K, V (loaded once), Q, dO (per row tile), P, dS
constexpr uint32_t kK = 0, kV = kTile, kQ = 2 * kTile, kO = 3 * kTile, kP = 4 * kTile,
                   kS = 5 * kTile;
constexpr uint32_t kSmemBytes = 6 * kTile + 1024;
constexpr uint32_t kTmemCols = 512;  // S / dQ 0, dP 128, dV 256, dK 384
constexpr uint32_t kIdescNN = idesc_bf16(TM, TN, false, false);  // both operands K-major
constexpr uint32_t kIdescTB = idesc_bf16(TM, TN, true, true);    // A and B M/N-major
constexpr uint32_t kIdescKB = idesc_bf16(TM, TN, false, true);   // A K-major, B N-major

struct Args {
  Dims dm;
  Chunk ch;
  const __nv_bfloat16* q;
  const __nv_bfloat16* dout;
  const float* lse;
  const float* Dsum;
  const int32_t* cu;
  const int32_t* idx;  // [T][Hq][k] index rows (own-block rows of the prefix-mean gate)
  const int32_t* list_off;
  const int32_t* pairs;
  float* dq;
  float* dk;
  float* dv;
  int* status;
};

// Row-major bf16 row (128 elements = 256 bytes) into the swizzled layout the
// MMA reads: two 64-column halves, 128-byte rows, 16-byte chunks XOR row % 8.
__device__ __forceinline__ uint32_t swz(uint32_t base, int row, int c16) {
  return base + (c16 >> 3) * kHalf + row * 128 + ((((uint32_t)c16 & 7u) ^ ((uint32_t)row & 7u)) << 4);
}

template <int MODE>
__global__ void __launch_bounds__(kThreads, 1)
bwd_tc_kernel(const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv,
              const Args a) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t kv_full, mma_bar;
  __shared__ uint32_t tmem_base;
  __shared__ int abort_flag;
  __shared__ int64_t qrow_s[TM];
  __shared__ int pos_s[TM];
  const Dims& dm = a.dm;
  const int tid = threadIdx.x, warp = tid >> 5;
  const int grp = dm.Hq / dm.Hkv;
  const int kt = blockIdx.y;

  int b, g, blk;
  int64_t n_rows, row0 = 0;
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
  const int64_t start = a.cu[b];
  const int len = a.cu[b + 1] - a.cu[b];
  if (len < 0 || len > dm.max_seqlen) return;
  const int k0 = blk * dm.B + kt * TN;
  const int k1 = min(k0 + TN, len);
  if (k0 >= k1) return;
  int p_first = 0;
  if (MODE == CUR) {
    p_first = k0;
    n_rows = (int64_t)(min((blk + 1) * dm.B, len) - p_first) * grp;
  }
  if (n_rows <= 0) return;

  const uint32_t sbase = (smem_u32(smem_raw) + 1023u) & ~1023u;
  if (tid == 0) {
    mbar_init(&kv_full, 1);
    mbar_init(&mma_bar, 1);
    abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 0) {
    tmem_alloc(&tmem_base, kTmemCols);
    tmem_relinquish();
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tmem = tmem_base;
  volatile int* abort = &abort_flag;
  int* status = a.status;
  const uint32_t lane_addr = static_cast<uint32_t>(warp * 32) << 16;
  const float scale = rsqrtf((float)D);

  // K and V of the tile: TMA, two 64-column halves each
  if (tid == 0) {
    mbar_expect_tx(&kv_full, 2 * kTile);
    const int z = (int)(start + k0);
    tma_load_3d(sbase + kK, &tmk, &kv_full, 0, g, z);
    tma_load_3d(sbase + kK + kHalf, &tmk, &kv_full, 64, g, z);
    tma_load_3d(sbase + kV, &tmv, &kv_full, 0, g, z);
    tma_load_3d(sbase + kV + kHalf, &tmv, &kv_full, 64, g, z);
  }
  bool ok = __syncthreads_and(mbar_wait(&kv_full, 0, abort, status));
  uint32_t nmma = 0;

  // Row metadata of a tile (q row id, position, lse, D) and the cp.async of
  // its Q and dO rows. The next tile's metadata is read while the current
  // tile's MMAs run, and its rows are requested as soon as the Q / dO
  // buffers are free, so both latencies hide behind the current tile.
  const int r = tid;
  auto meta = [&](int64_t c0, int64_t& qrow, int& pos, float& lse_r, float& d_r) {
    const int64_t i = c0 + r;
    qrow = 0;
    pos = -1;
    lse_r = d_r = 0.f;
    if (i < n_rows) {
      if (MODE == HIST) {
        const int64_t th = a.pairs[row0 + i] / dm.topk;
        qrow = (th / a.ch.nq) * dm.Hq + a.ch.h0 + (int)(th % a.ch.nq);
        pos = 0;
      } else {
        const int p = p_first + (int)(i / grp);
        qrow = (start + p) * dm.Hq + g * grp + (int)(i % grp);
        // a row whose own block lost the prefix-mean gate reads none of it
        pos = reads_own(dm, a.idx + qrow * dm.topk, p / dm.B) ? p : -1;
      }
      lse_r = a.lse[qrow];
      d_r = a.Dsum[qrow];
    }
  };
  auto request = [&](int64_t qrow, int pos) {
    const __nv_bfloat16* qs = a.q + (pos >= 0 ? qrow : 0) * (int64_t)D;
    const __nv_bfloat16* os = a.dout + (pos >= 0 ? qrow : 0) * (int64_t)D;
#pragma unroll
    for (int c16 = 0; c16 < 16; ++c16) {
      cp_async16(swz(sbase + kQ, r, c16), qs + c16 * 8, pos >= 0 ? 16u : 0u);
      cp_async16(swz(sbase + kO, r, c16), os + c16 * 8, pos >= 0 ? 16u : 0u);
    }
  };
  int64_t qrow_n;
  int pos_n;
  float lse_n, d_n;
  meta(0, qrow_n, pos_n, lse_n, d_n);
  if (ok) request(qrow_n, pos_n);
  for (int64_t c0 = 0; ok && c0 < n_rows; c0 += TM) {
    const int64_t qrow = qrow_n;
    const int pos = pos_n;
    const float lse_r = lse_n, d_r = d_n;
    cp_async_wait_all();
    fence_proxy_async_smem();
    fence_before_sync();
    __syncthreads();
    // ---- S = Q K^T, dP = dO V^T
    if (tid == 0) {
      fence_after_sync();
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t off = (kk >> 2) * kHalf + (kk & 3) * 32;
        mma_ss(tmem + 0, desc_sw128(sbase + kQ + off, 16, 1024),
               desc_sw128(sbase + kK + off, 16, 1024), kIdescNN, kk > 0 ? 1u : 0u);
        mma_ss(tmem + 128, desc_sw128(sbase + kO + off, 16, 1024),
               desc_sw128(sbase + kV + off, 16, 1024), kIdescNN, kk > 0 ? 1u : 0u);
      }
      commit(&mma_bar);
    }
    ok = mbar_wait(&mma_bar, nmma & 1, abort, status);
    ++nmma;
    if (!__syncthreads_and(ok)) { ok = false; break; }
    fence_after_sync();
    // ---- P and dS of row r, to shared memory as bf16
#pragma unroll 1
    for (int c = 0; c < TN / 32; ++c) {
      uint32_t sv[32], pv[32];
      tmem_ld32(tmem + 0 + lane_addr + c * 32, sv);
      tmem_ld32(tmem + 128 + lane_addr + c * 32, pv);
      tmem_wait_ld();
      uint32_t pk[16], sk[16];
#pragma unroll
      for (int x = 0; x < 32; x += 2) {
        float p2[2], s2[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int kp = k0 + c * 32 + x + u;
          const bool vis = pos >= 0 && kp < k1 && (MODE == HIST || kp <= pos);
          const float p = vis ? __expf(__uint_as_float(sv[x + u]) * scale - lse_r) : 0.f;
          p2[u] = p;
          s2[u] = p * (__uint_as_float(pv[x + u]) - d_r);
        }
        pk[x / 2] = pack_bf16x2(p2[0], p2[1]);
        sk[x / 2] = pack_bf16x2(s2[0], s2[1]);
      }
      // 32 keys = four 16-byte chunks of the row
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        const int c16 = c * 4 + q4;
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(swz(sbase + kP, r, c16)),
                     "r"(pk[4 * q4]), "r"(pk[4 * q4 + 1]), "r"(pk[4 * q4 + 2]), "r"(pk[4 * q4 + 3])
                     : "memory");
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(swz(sbase + kS, r, c16)),
                     "r"(sk[4 * q4]), "r"(sk[4 * q4 + 1]), "r"(sk[4 * q4 + 2]), "r"(sk[4 * q4 + 3])
                     : "memory");
      }
    }
    fence_proxy_async_smem();
    fence_before_sync();
    __syncthreads();
    // ---- dV += P^T dO, dK += dS^T Q (A read M-major = transposed), dQ = dS K
    if (tid == 0) {
      fence_after_sync();
      const uint32_t acc0 = c0 > 0 ? 1u : 0u;
#pragma unroll
      for (int kk = 0; kk < TM / 16; ++kk) {
        // K dimension = tile rows, 16 per step: 16 rows x 128 B in each half
        const uint32_t roff = kk * 16 * 128;
        mma_ss(tmem + 256, desc_sw128(sbase + kP + roff, kHalf, 1024),
               desc_sw128(sbase + kO + roff, kHalf, 1024), kIdescTB, (acc0 || kk > 0) ? 1u : 0u);
        mma_ss(tmem + 384, desc_sw128(sbase + kS + roff, kHalf, 1024),
               desc_sw128(sbase + kQ + roff, kHalf, 1024), kIdescTB, (acc0 || kk > 0) ? 1u : 0u);
      }
#pragma unroll
      for (int kk = 0; kk < TN / 16; ++kk) {
        // K dimension = keys: dS K-major, K tile read N-major (d contiguous)
        const uint32_t off = (kk >> 2) * kHalf + (kk & 3) * 32;
        mma_ss(tmem + 0, desc_sw128(sbase + kS + off, 16, 1024),
               desc_sw128(sbase + kK + kk * 16 * 128, kHalf, 1024), kIdescKB, kk > 0 ? 1u : 0u);
      }
      commit(&mma_bar);
    }
    const bool more = c0 + TM < n_rows;
    if (more) meta(c0 + TM, qrow_n, pos_n, lse_n, d_n);
    ok = mbar_wait(&mma_bar, nmma & 1, abort, status);
    ++nmma;
    if (!__syncthreads_and(ok)) { ok = false; break; }
    fence_after_sync();
    // the Q and dO buffers are free: the next tile's rows may land
    if (more) request(qrow_n, pos_n);
    // ---- dq: rows through shared memory (the P and dS tiles are free now:
    // their MMAs are done), then each warp adds whole 512-byte rows with
    // 16-byte vector reductions. Row r's 16-byte chunk c sits at chunk
    // c ^ (r % 32) of its row, so neither side has bank conflicts beyond the
    // four wavefronts a 512-byte access needs.
    {
      const uint32_t st = sbase + kP;  // 128 rows x 512 bytes = the P and dS tiles
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        uint32_t v[32];
        tmem_ld32(tmem + 0 + lane_addr + c * 32, v);
        tmem_wait_ld();
#pragma unroll
        for (int x4 = 0; x4 < 8; ++x4) {
          const uint32_t chunk = (uint32_t)(c * 8 + x4) ^ ((uint32_t)r & 31u);
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(st + r * 512 + chunk * 16),
                       "r"(__float_as_uint(__uint_as_float(v[4 * x4]) * scale)),
                       "r"(__float_as_uint(__uint_as_float(v[4 * x4 + 1]) * scale)),
                       "r"(__float_as_uint(__uint_as_float(v[4 * x4 + 2]) * scale)),
                       "r"(__float_as_uint(__uint_as_float(v[4 * x4 + 3]) * scale))
                       : "memory");
        }
      }
      qrow_s[r] = qrow;
      pos_s[r] = pos;
      __syncthreads();
      const int lane = tid & 31;
#pragma unroll 4
      for (int i = 0; i < TM / 4; ++i) {
        const int row = warp * (TM / 4) + i;
        if (pos_s[row] < 0) continue;  // warp-uniform
        const uint32_t chunk = (uint32_t)lane ^ ((uint32_t)row & 31u);
        uint32_t x, y, z, w;
        asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                     : "=r"(x), "=r"(y), "=r"(z), "=r"(w)
                     : "r"(st + row * 512 + chunk * 16)
                     : "memory");
        float* dst = a.dq + qrow_s[row] * D + lane * 4;
        asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(dst),
                     "f"(__uint_as_float(x)), "f"(__uint_as_float(y)), "f"(__uint_as_float(z)),
                     "f"(__uint_as_float(w))
                     : "memory");
      }
    }
    fence_before_sync();
    __syncthreads();
  }
  cp_async_wait_all();  // an early exit may leave the next tile's rows in flight
  // ---- dK, dV of key k0 + tid (TMEM lane tid)
  if (ok) {
    const int key = k0 + tid;
    const int64_t off = ((start + key) * dm.Hkv + g) * (int64_t)D;
#pragma unroll 1
    for (int c = 0; c < D / 32; ++c) {
      uint32_t kv[32], vv[32];
      tmem_ld32(tmem + 384 + lane_addr + c * 32, kv);
      tmem_ld32(tmem + 256 + lane_addr + c * 32, vv);
      tmem_wait_ld();
      if (key < k1) {
#pragma unroll
        for (int x = 0; x < 32; ++x) {
          a.dk[off + c * 32 + x] += __uint_as_float(kv[x]) * scale;
          a.dv[off + c * 32 + x] += __uint_as_float(vv[x]);
        }
      }
    }
  } else if (tid == 0) {
    // wait until every MMA issued has finished before the TMEM is freed
    commit(&mma_bar);
    mbar_drain(&mma_bar, nmma & 1);
  }
  fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    fence_after_sync();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

cudaError_t launch_backward_tc(const Dims& dm, const Chunk& ch, const void* q, const void* k,
                               const void* v, const void* dout, const float* lse,
                               const float* Dsum, const int32_t* cu, const int32_t* idx,
                               const Regroup& rg, float* dq, float* dk, float* dv, int* status,
                               cudaStream_t st) {
  if (dm.batch == 0 || dm.max_seqlen == 0) return cudaSuccess;
  CUtensorMap mk, mv;
  cudaError_t e;
  if ((e = make_head_map(&mk, k, dm.T, dm.Hkv, TN))) return e;
  if ((e = make_head_map(&mv, v, dm.T, dm.Hkv, TN))) return e;
  Args a{};
  a.dm = dm;
  a.ch = ch;
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.dout = static_cast<const __nv_bfloat16*>(dout);
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
  if ((e = cudaFuncSetAttribute(bwd_tc_kernel<HIST>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                kSmemBytes)))
    return e;
  if ((e = cudaFuncSetAttribute(bwd_tc_kernel<CUR>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                kSmemBytes)))
    return e;
  const unsigned kts = (unsigned)(dm.B / TN);
  if (ch.n_lists > 0) {
    bwd_tc_kernel<HIST><<<dim3((unsigned)ch.n_lists, kts), kThreads, kSmemBytes, st>>>(mk, mv, a);
    if ((e = cudaGetLastError())) return e;
  }
  const int64_t own = (int64_t)dm.batch * dm.Hkv * dm.nb;
  if (own > 0) {
    bwd_tc_kernel<CUR><<<dim3((unsigned)own, kts), kThreads, kSmemBytes, st>>>(mk, mv, a);
    if ((e = cudaGetLastError())) return e;
  }
  return cudaSuccess;
}

}  // namespace moba
