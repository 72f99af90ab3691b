// Tensor-core attention for bf16, d = 128 (sm_100a: tcgen05 + TMEM + TMA).
//
// One engine serves the three places where MoBA does exact softmax
// attention (PaperTrace "2.1.3 MoBA", section 2 eq. 4-6, section 3.1):
//   HIST  : a tile of up to 128 regrouped (query, head, slot) rows that all
//           chose the same earlier block, against that block's B raw keys,
//           non-causal (eq. 6); writes a normalised partial result per slot;
//   CUR   : 128 consecutive queries of one head against their own block,
//           causal on the diagonal tile (eq. 5); writes a partial result;
//   DENSE : 128 consecutive queries against every earlier key of their
//           sequence (eq. 1, causal); writes the output.
// The partials are combined by the merge kernel with eq. (7)-(8).
//
// CTA = 6 warps, one 128-row query tile:
//   warp 0     TMA producer: K and V tiles of 128 keys (two 64-column
//              halves each, 128-byte swizzle) into a 2-stage ring;
//   warp 1     allocates 512 TMEM columns; lane 0 issues every tcgen05.mma:
//              S_j = Q K_j^T into TMEM buffer j%2 (fp32, 128 columns), then
//              O += P_{j-1} V_{j-1} with P read from TMEM (bf16 packed into
//              the first 64 columns of the S buffer it came from);
//   warps 2-5  softmax, one query row per thread (TMEM lane = row): load the
//              row of S, exponentiate in base 2, store P, keep (m, l); the
//              output accumulator O (TMEM columns 256..383) is rescaled only
//              when a row's maximum grows by more than 2^8 (values stay
//              below 256, exact in fp32), so PV never waits for a rescale in
//              the common case.
// Q rows are loaded by the softmax threads themselves (a gathered tile in
// HIST mode) straight into the swizzled shared layout the MMA reads.
//
// Every wait is bounded (tc::mbar_wait); on expiry the CTA records
// kStTimeout, drains the copies and MMAs it issued, frees its TMEM and exits.
#include <cudaTypedefs.h>

#include "tc_ptx.cuh"

namespace moba {

bool tc_supported(const Dims& dm) {
  return dm.dtype == kBF16 && dm.d == 128 && dm.B % 128 == 0;
}

namespace {

using namespace tc;

enum Mode { HIST = 0, CUR = 1, DENSE = 2 };

constexpr int TM = 128;   // query rows per tile
constexpr int TN = 128;   // keys per KV tile
constexpr int D = 128;    // head dim
constexpr int NS = 2;     // K/V ring stages
constexpr int kThreads = 192;
constexpr uint32_t kHalf = 128 * 128;      // bytes of one 64-column half of a 128-row tile
constexpr uint32_t kTile = 2 * kHalf;      // bytes of one 128 x 128 bf16 tile
constexpr uint32_t kQOff = 0;
constexpr uint32_t kKOff = kTile;
constexpr uint32_t kVOff = kKOff + NS * kTile;
constexpr uint32_t kSmemBytes = kVOff + NS * kTile + 1024;  // + 1024-byte alignment slack
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kOCol = 256;            // O accumulator columns [256, 384)
constexpr uint32_t kIdescQK = idesc_bf16(TM, TN, false, false);  // Q, K both K-major
constexpr uint32_t kIdescPV = idesc_bf16(TM, D, false, true);    // V is MN-major (d contiguous)
constexpr float kRescaleLog2 = 8.f;

struct Shared {
  uint64_t q_full;
  uint64_t k_full[NS], k_empty[NS], v_full[NS], v_empty[NS];
  uint64_t s_full[2], s_free[2], p_full[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};

struct Args {
  Dims dm;
  Chunk ch;
  const __nv_bfloat16* q;
  const int32_t* cu;
  // HIST
  const int32_t* list_off;
  const int32_t* pairs;
  const int2* tiles;
  const int32_t* tile_count;
  // CUR
  const int32_t* idx;
  // outputs
  float* part_o;
  float* part_lse;
  __nv_bfloat16* out;
  float* lse_out;
  int* status;
};

template <int MODE>
__global__ void __launch_bounds__(kThreads, 1)
attn_tc_kernel(const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv,
               const Args a) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ Shared sh;
  const Dims& dm = a.dm;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // ---- which tile ----------------------------------------------------------
  int b, g, n_kv, kv0;   // sequence, kv head, KV tiles, first key (sequence-relative)
  int p0 = 0;            // first query position (CUR / DENSE)
  int h_fixed = 0;       // q head (CUR / DENSE)
  int list = 0, row0 = 0, count = 0;
  if (a.status && *reinterpret_cast<volatile int*>(a.status) == kStTimeout) return;
  if (MODE == HIST) {
    if ((int)blockIdx.x >= *a.tile_count) return;
    const int2 tl = a.tiles[blockIdx.x];
    list = tl.x;
    row0 = tl.y;
    const int e = list % dm.nb;
    g = a.ch.g0 + (list / dm.nb) % a.ch.ng;
    b = list / (dm.nb * a.ch.ng);
    count = a.list_off[list + 1] - a.list_off[list];
    kv0 = e * dm.B;
    n_kv = dm.B / TN;
  } else {
    b = blockIdx.y;
    const int len = a.cu[b + 1] - a.cu[b];
    if (len < 0 || len > dm.max_seqlen) return;
    // longest tiles first (they end last)
    const int qt = gridDim.x - 1 - blockIdx.x;
    p0 = qt * TM;
    if (p0 >= len) return;
    h_fixed = (MODE == CUR ? a.ch.h0 : 0) + blockIdx.z;
    g = h_fixed / (dm.Hq / dm.Hkv);
    const int c = p0 / dm.B;
    kv0 = MODE == CUR ? c * dm.B : 0;
    n_kv = (p0 - kv0) / TN + 1;
  }
  const int64_t start = a.cu[b];

  const uint32_t sbase = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const uint32_t sQ = sbase + kQOff, sK = sbase + kKOff, sV = sbase + kVOff;

  if (threadIdx.x == 0) {
    mbar_init(&sh.q_full, 128);
    for (int i = 0; i < NS; ++i) {
      mbar_init(&sh.k_full[i], 1);
      mbar_init(&sh.k_empty[i], 1);
      mbar_init(&sh.v_full[i], 1);
      mbar_init(&sh.v_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sh.s_full[i], 1);
      mbar_init(&sh.s_free[i], 1);
      mbar_init(&sh.p_full[i], 128);
    }
    mbar_init(&sh.drain, 1);
    sh.abort = 0;
    mbar_fence_init();
  }
  if (warp == 1) {
    tmem_alloc(&sh.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tmem = sh.tmem_base;
  volatile int* abort = &sh.abort;

  if (warp == 0) {
    // ================= TMA producer =================
    if (lane == 0) {
      int issued_k = 0, issued_v = 0;
      for (int j = 0; j < n_kv; ++j) {
        const int st = j % NS, u = j / NS;
        const int z = (int)(start + kv0 + j * TN);
        if (u > 0 && !mbar_wait(&sh.k_empty[st], (u - 1) & 1, abort, a.status)) break;
        mbar_expect_tx(&sh.k_full[st], kTile);
        tma_load_3d(sK + st * kTile, &tmk, &sh.k_full[st], 0, g, z);
        tma_load_3d(sK + st * kTile + kHalf, &tmk, &sh.k_full[st], 64, g, z);
        issued_k = j + 1;
        if (u > 0 && !mbar_wait(&sh.v_empty[st], (u - 1) & 1, abort, a.status)) break;
        mbar_expect_tx(&sh.v_full[st], kTile);
        tma_load_3d(sV + st * kTile, &tmv, &sh.v_full[st], 0, g, z);
        tma_load_3d(sV + st * kTile + kHalf, &tmv, &sh.v_full[st], 64, g, z);
        issued_v = j + 1;
      }
      if (*abort) {
        // let the copies already issued land before the CTA exits
        for (int j = (issued_k > NS ? issued_k - NS : 0); j < issued_k; ++j)
          mbar_drain(&sh.k_full[j % NS], (j / NS) & 1);
        for (int j = (issued_v > NS ? issued_v - NS : 0); j < issued_v; ++j)
          mbar_drain(&sh.v_full[j % NS], (j / NS) & 1);
      }
    }
  } else if (warp == 1) {
    // ================= MMA issuer =================
    if (lane == 0) {
      const uint32_t tS[2] = {tmem, tmem + 128};
      const uint32_t tO = tmem + kOCol;
      bool ok = mbar_wait(&sh.q_full, 0, abort, a.status);
      auto issue_pv = [&](int jj) -> bool {
        const int st = jj % NS, bb = jj & 1;
        if (!mbar_wait(&sh.p_full[bb], (jj >> 1) & 1, abort, a.status)) return false;
        if (!mbar_wait(&sh.v_full[st], (jj / NS) & 1, abort, a.status)) return false;
        fence_after_sync();
#pragma unroll
        for (int kk = 0; kk < TN / 16; ++kk) {
          const uint64_t bd = desc_sw128(sV + st * kTile + kk * 16 * 128, kHalf, 1024);
          mma_ts(tO, tS[bb] + kk * 8, bd, kIdescPV, (jj > 0 || kk > 0) ? 1u : 0u);
        }
        commit(&sh.v_empty[st]);
        commit(&sh.s_free[bb]);
        return true;
      };
      for (int j = 0; ok && j < n_kv; ++j) {
        const int st = j % NS, bb = j & 1;
        if (!mbar_wait(&sh.k_full[st], (j / NS) & 1, abort, a.status)) { ok = false; break; }
        if (j >= 2 && !mbar_wait(&sh.s_free[bb], ((j - 2) >> 1) & 1, abort, a.status)) {
          ok = false;
          break;
        }
        fence_after_sync();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * kHalf + (kk & 3) * 32;
          const uint64_t ad = desc_sw128(sQ + off, 16, 1024);
          const uint64_t bd = desc_sw128(sK + st * kTile + off, 16, 1024);
          mma_ss(tS[bb], ad, bd, kIdescQK, kk > 0 ? 1u : 0u);
        }
        commit(&sh.s_full[bb]);
        commit(&sh.k_empty[st]);
        if (j >= 1 && !issue_pv(j - 1)) { ok = false; break; }
      }
      if (ok) ok = issue_pv(n_kv - 1);
      if (!ok) {
        // wait until every MMA issued so far has finished
        commit(&sh.drain);
        mbar_drain(&sh.drain, 0);
      }
    }
  } else {
    // ================= softmax warps 2..5 =================
    const int quarter = warp & 3;          // TMEM lanes this warp may access
    const int r = quarter * 32 + lane;     // query row of this thread
    const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
    // row identity
    bool valid = false;
    int64_t t = 0, prow = 0;
    int h = h_fixed, p = 0;
    if (MODE == HIST) {
      valid = row0 + r < count;
      if (valid) {
        prow = a.pairs[a.list_off[list] + row0 + r];
        const int64_t th = prow / dm.topk;
        t = th / a.ch.nq;
        h = a.ch.h0 + (int)(th % a.ch.nq);
      }
    } else {
      const int len = a.cu[b + 1] - a.cu[b];
      p = p0 + r;
      valid = p < len;
      t = start + p;
      if (MODE == CUR && valid) {
        const int c = p / dm.B;
        const int32_t* row = a.idx + (t * dm.Hq + h) * (int64_t)dm.topk;
        int slot = -1;
        for (int i = 0; i < dm.topk; ++i)
          if (row[i] == c && slot < 0) slot = i;
        prow = (t * a.ch.nq + (h - a.ch.h0)) * (int64_t)dm.topk + (slot < 0 ? 0 : slot);
        valid = slot >= 0;
      }
    }
    const bool has_q = MODE == HIST ? (row0 + r < count) : (p < a.cu[b + 1] - a.cu[b]);
    // ---- Q row -> swizzled shared tile (two 64-column halves)
    {
      const uint4* src = reinterpret_cast<const uint4*>(a.q + (t * dm.Hq + h) * (int64_t)D);
#pragma unroll
      for (int c16 = 0; c16 < 16; ++c16) {
        const uint4 x = has_q ? __ldg(src + c16) : make_uint4(0, 0, 0, 0);
        const uint32_t half = c16 >> 3, cc = c16 & 7;
        const uint32_t addr = sQ + half * kHalf + r * 128 + ((cc ^ (r & 7)) << 4);
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(x.x),
                     "r"(x.y), "r"(x.z), "r"(x.w)
                     : "memory");
      }
      fence_proxy_async_smem();
      mbar_arrive(&sh.q_full);
    }
    const float sl2 = rsqrtf((float)D) * 1.4426950408889634f;  // softmax scale, base 2
    float m_i = -INFINITY, l_i = 0.f;
    bool ok = true;
    for (int j = 0; j < n_kv; ++j) {
      const int bb = j & 1;
      ok = mbar_wait(&sh.s_full[bb], (j >> 1) & 1, abort, a.status);
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      fence_after_sync();
      const uint32_t tS = tmem + bb * 128 + lane_addr;
      float s[TN];
#pragma unroll
      for (int c = 0; c < TN / 32; ++c) {
        uint32_t rr[32];
        tmem_ld32(tS + c * 32, rr);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) s[c * 32 + i] = __uint_as_float(rr[i]) * sl2;
      }
      // causal mask on the diagonal tile (CUR / DENSE): key > query
      if (MODE != HIST && j == n_kv - 1) {
        const int lim = p - (kv0 + j * TN);  // last visible column
#pragma unroll
        for (int i = 0; i < TN; ++i)
          if (i > lim) s[i] = -INFINITY;
      }
      float mt = s[0];
#pragma unroll
      for (int i = 1; i < TN; ++i) mt = fmaxf(mt, s[i]);
      const bool need = mt > m_i + kRescaleLog2;
      const float m_new = need ? mt : m_i;
      if (__any_sync(0xffffffffu, need) && j > 0) {
        // O holds PV of tiles < j: wait until PV_{j-1} has landed, then rescale
        ok = mbar_wait(&sh.s_free[(j - 1) & 1], ((j - 1) >> 1) & 1, abort, a.status);
        if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
        fence_after_sync();
        const float alpha = need ? ex2(m_i - m_new) : 1.f;
        const uint32_t tO = tmem + kOCol + lane_addr;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t rr[32];
          tmem_ld32(tO + c * 32, rr);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) rr[i] = __float_as_uint(__uint_as_float(rr[i]) * alpha);
          tmem_st32(tO + c * 32, rr);
        }
        tmem_wait_st();
      }
      if (need) {
        l_i *= ex2(m_i - m_new);
        m_i = m_new;
      }
      // P = exp2(s - m) in bf16, packed two per column into the S buffer
      float rowsum = 0.f;
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t pk[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float e0 = ex2(s[c * 64 + 2 * i] - m_i);
          const float e1 = ex2(s[c * 64 + 2 * i + 1] - m_i);
          rowsum += e0 + e1;
          pk[i] = pack_bf16x2(e0, e1);
        }
        tmem_st32(tS + c * 32, pk);
      }
      tmem_wait_st();
      l_i += rowsum;
      fence_before_sync();
      mbar_arrive(&sh.p_full[bb]);
    }
    // ---- epilogue: wait for the last PV, normalise, write
    if (ok) {
      const int jl = n_kv - 1;
      ok = mbar_wait(&sh.s_free[jl & 1], (jl >> 1) & 1, abort, a.status);
      ok = __all_sync(0xffffffffu, ok);
    }
    if (ok) {
      fence_after_sync();
      const float inv_l = 1.f / l_i;
      const float lse = (m_i + log2f(l_i)) * 0.6931471805599453f;
      const uint32_t tO = tmem + kOCol + lane_addr;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t rr[32];
        tmem_ld32(tO + c * 32, rr);
        tmem_wait_ld();
        if (valid) {
          if (MODE == DENSE) {
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 16; ++i)
              pk[i] = pack_bf16x2(__uint_as_float(rr[2 * i]) * inv_l,
                                  __uint_as_float(rr[2 * i + 1]) * inv_l);
            uint4* dst = reinterpret_cast<uint4*>(a.out + (t * dm.Hq + h) * (int64_t)D + c * 32);
#pragma unroll
            for (int i = 0; i < 4; ++i)
              dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
          } else {
            float4* dst = reinterpret_cast<float4*>(a.part_o + prow * D + c * 32);
#pragma unroll
            for (int i = 0; i < 8; ++i)
              dst[i] = make_float4(__uint_as_float(rr[4 * i]) * inv_l,
                                   __uint_as_float(rr[4 * i + 1]) * inv_l,
                                   __uint_as_float(rr[4 * i + 2]) * inv_l,
                                   __uint_as_float(rr[4 * i + 3]) * inv_l);
          }
        }
      }
      if (valid) {
        if (MODE == DENSE) {
          if (a.lse_out) a.lse_out[t * dm.Hq + h] = lse;
        } else {
          a.part_lse[prow] = lse;
        }
      }
    }
  }

  fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    fence_after_sync();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ---- host side -----------------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

// [T][H][128] bf16 viewed as (x = d, y = head, z = token); box 64 x 1 x 128.
cudaError_t make_map(CUtensorMap* map, const void* base, int T, int H) {
  auto fn = encode_fn();
  if (!fn) return cudaErrorNotSupported;
  const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)T};
  const cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)H * D * 2};
  const cuuint32_t box[3] = {64, 1, (cuuint32_t)TN};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

template <int MODE>
cudaError_t launch(dim3 grid, const Args& args, const void* k, const void* v, cudaStream_t st) {
  CUtensorMap mk, mv;
  cudaError_t e;
  if ((e = make_map(&mk, k, args.dm.T, args.dm.Hkv))) return e;
  if ((e = make_map(&mv, v, args.dm.T, args.dm.Hkv))) return e;
  if ((e = cudaFuncSetAttribute(attn_tc_kernel<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                kSmemBytes)))
    return e;
  attn_tc_kernel<MODE><<<grid, kThreads, kSmemBytes, st>>>(mk, mv, args);
  return cudaGetLastError();
}

Args base_args(const Dims& dm, const Chunk& ch, const void* q, const int32_t* cu, int* status) {
  Args a{};
  a.dm = dm;
  a.ch = ch;
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.cu = cu;
  a.status = status;
  return a;
}

}  // namespace

cudaError_t launch_history_tc(const Dims& dm, const Chunk& ch, const void* q, const void* k,
                              const void* v, const int32_t* cu, const Regroup& rg,
                              const Partials& pt, int* status, cudaStream_t st) {
  if (rg.max_tiles == 0) return cudaSuccess;
  Args a = base_args(dm, ch, q, cu, status);
  a.list_off = rg.list_off;
  a.pairs = rg.pairs;
  a.tiles = rg.tiles;
  a.tile_count = rg.tile_off + ch.n_lists;
  a.part_o = pt.o;
  a.part_lse = pt.lse;
  return launch<HIST>(dim3((unsigned)rg.max_tiles), a, k, v, st);
}

cudaError_t launch_current_tc(const Dims& dm, const Chunk& ch, const void* q, const void* k,
                              const void* v, const int32_t* cu, const int32_t* idx,
                              const Partials& pt, int* status, cudaStream_t st) {
  if (dm.batch == 0 || dm.max_seqlen == 0) return cudaSuccess;
  Args a = base_args(dm, ch, q, cu, status);
  a.idx = idx;
  a.part_o = pt.o;
  a.part_lse = pt.lse;
  return launch<CUR>(dim3((dm.max_seqlen + TM - 1) / TM, dm.batch, ch.nq), a, k, v, st);
}

cudaError_t launch_dense_tc(const Dims& dm, const void* q, const void* k, const void* v,
                            const int32_t* cu, void* out, float* lse, int* status,
                            cudaStream_t st) {
  if (dm.batch == 0 || dm.max_seqlen == 0) return cudaSuccess;
  Chunk ch{0, dm.Hkv, 0, dm.Hq, 0, TM};
  Args a = base_args(dm, ch, q, cu, status);
  a.out = static_cast<__nv_bfloat16*>(out);
  a.lse_out = lse;
  return launch<DENSE>(dim3((dm.max_seqlen + TM - 1) / TM, dm.batch, dm.Hq), a, k, v, st);
}

}  // namespace moba
