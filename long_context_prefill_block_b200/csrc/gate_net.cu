// Tensor-core gate with a sorting-network top-k, for long index rows (5 to
// 15 history slots beside the forced own block, e.g. k = 12 at the
// million-token shape) and at most 256 blocks per sequence (PaperTrace
// "2.1.3 MoBA", section 1 eq. 3, section 2, section 2.1).
//
// Scores: as in the other tensor-core gate, s_i = q . kbar_i of a tile of
// 128 queries of one head against every block of its sequence is one tcgen05
// contraction with each fp32 kbar element split into three bf16 terms
// (h + m + l, exact to 2^-24 relative), accumulated in fp32 in TMEM. Here the
// Q tile is the MMA's A operand in TMEM: four loader warps read their 32
// query rows from global memory and store them into one of two TMEM Q
// buffers, so shared memory holds only the three kbar terms (192 KB at 256
// blocks) and the next tile's Q arrives while this tile's MMA runs.
//
// Selection: the 256 threads of the selection warps take two per row (TMEM
// lane = row); each copies its 16-column groups of the row's scores (every
// other group) into registers at once, which frees the accumulator for the
// next tile's MMA, and turns each score of a block i < c into an fp32 order
// key (sortnet.cuh: the score with its low 8 mantissa bits holding the
// block index; blocks >= c get -inf), compared with float max / min, which
// issue on the FMA pipes rather than the half-rate integer ALU pipe. Per
// group a 16-key odd-even merge sort, then a
// bitonic merge into the thread's running top 16; the two threads' lists
// meet through TMEM and the first thread keeps the row's top 16. Every step
// is a max/min network: no branch depends on the data, so the 32 rows of a
// warp never diverge. The chosen blocks are the top min(k-1, c) keys: the
// exact fp32 top-k, except that two scores agreeing in their top 24 order
// bits (within 2^-15 relative) rank by block index, well inside the 1e-4
// relative near-tie band within which any choice is a correct one.
//
// Roles (12 warps): warps 0-3 load Q rows into TMEM (warp w: lanes 32w..);
// lane 0 of warp 0 also issues the MMAs and commits; warps 4-7 (first
// thread of each row) and 8-11 (second thread) select. Every wait is a
// bounded mbarrier wait; on expiry the CTA records kStTimeout, drains its
// MMAs and exits.
#include <climits>
#include <mutex>

#include "sortnet.cuh"
#include "tc_ptx.cuh"
#include "trace.cuh"

namespace moba {
namespace {

using namespace tc;

constexpr int kThreads = 384;
constexpr int kRows = 128;            // queries per tile
constexpr int kMaxBlocks = 256;       // MMA N limit
constexpr int kCuSmem = 257;          // sequence offsets kept in shared memory
constexpr uint32_t kAccCol = 0;       // scores, up to 256 columns
constexpr uint32_t kQCol = 256;       // two Q buffers of 64 columns (bf16 pairs)
constexpr uint32_t kXCol = 384;       // two 16-column buffers for the list exchange
constexpr uint32_t kTmemCols = 512;
constexpr int kLaunchRegs = 168;      // 65536 / 384, rounded down to a multiple of 8
constexpr int kRegsLoad = 72;         // warps 0-3 after setmaxnreg.dec
constexpr int kRegsSel = 216;         // warps 4-11 after setmaxnreg.inc
static_assert(128 * kRegsLoad + 256 * kRegsSel <= kThreads * kLaunchRegs,
              "register split exceeds the launch allocation");

struct NetArgs {
  Dims dm;
  const __nv_bfloat16* q;
  const float* kbar;
  const int32_t* cu;
  int32_t* idx;
  int* status;
  int groups;      // batch * Hkv (sequence, kv head) groups
  int ipg;         // items per group: query tiles per sequence * q heads per item
  int cpg;         // CTAs per group (0: each CTA takes whole groups, round robin)
  int nbp;         // blocks per sequence rounded up to a multiple of 16
  int vec_rows;    // index rows may be written with 16-byte stores
};

struct Item {
  int b, g, h, p0, len;
  int64_t start;
};

__device__ __forceinline__ Item decode_item(const NetArgs& a, const int32_t* cu, int gi, int j) {
  const Dims& dm = a.dm;
  const int grp = dm.Hq / dm.Hkv;
  const int per_tile = dm.shared ? 1 : grp;
  Item x;
  x.g = gi % dm.Hkv;
  x.b = gi / dm.Hkv;
  x.h = x.g * grp + j % per_tile;
  x.p0 = (j / per_tile) * kRows;
  x.start = cu[x.b];
  x.len = cu[x.b + 1] - cu[x.b];
  return x;
}

__device__ __forceinline__ bool item_live(const NetArgs& a, const Item& x) {
  return x.len > 0 && x.len <= a.dm.max_seqlen && x.p0 < x.len;
}

// MMA width of an item: its rows choose among blocks i < c <= c_max.
__device__ __forceinline__ int item_n(const NetArgs& a, const Item& x) {
  const int c_max = (min(x.p0 + kRows, x.len) - 1) / a.dm.B;
  return ((c_max + 15) / 16) * 16;
}

// The CTA's s-th group (-1 past the last) and the first item / item stride
// it takes in each group.
__device__ __forceinline__ int group_of(const NetArgs& a, int s) {
  if (a.cpg == 0) {
    const int gi = blockIdx.x + s * gridDim.x;
    return gi < a.groups ? gi : -1;
  }
  const int gi = blockIdx.x / a.cpg;
  return (s == 0 && gi < a.groups) ? gi : -1;
}

__device__ __forceinline__ void regs_dec() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsLoad));
}
__device__ __forceinline__ void regs_inc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsSel));
}

// Splits this group's kbar rows into the three bf16 terms in shared memory,
// K-major with the 128-byte swizzle (the layout a TMA tile of them would
// have); run by the `nthr` threads whose index is t.
__device__ __forceinline__ void stage_kbar(const NetArgs& a, const Item& x0, uint32_t sK,
                                           uint32_t kTermHalf, int t, int nthr) {
  const Dims& dm = a.dm;
  for (int e = t; e < a.nbp * 32; e += nthr) {
    const int i = e >> 5, d = (e & 31) * 4;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (i < dm.nb)
      v = *reinterpret_cast<const float4*>(
          a.kbar + (((int64_t)x0.b * dm.nb + i) * dm.Hkv + x0.g) * 128 + d);
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
    for (int q = 0; q < 3; ++q)
      asm volatile("st.shared.v2.b32 [%0], {%1, %2};" ::"r"(sK + q * 2 * kTermHalf + off),
                   "r"(w[q][0]), "r"(w[q][1])
                   : "memory");
  }
}

__global__ void __launch_bounds__(kThreads, 1) gate_net_kernel(const NetArgs a) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t q_full[2], q_empty[2], acc_full, acc_empty, x_full[4][2], drain;
  __shared__ uint32_t tmem_base;
  __shared__ int abort_flag;
  __shared__ int32_t cu_s[kCuSmem];
  const Dims& dm = a.dm;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (a.status && *reinterpret_cast<volatile int*>(a.status) == kStTimeout) return;

  const uint32_t sK = (smem_u32(smem_raw) + 1023u) & ~1023u;  // kbar terms [3][2 halves][nbp][128 B]
  const uint32_t kTermHalf = (uint32_t)a.nbp * 128u;

  const bool cu_in_smem = dm.batch + 1 <= kCuSmem;
  if (cu_in_smem)
    for (int i = tid; i <= dm.batch; i += kThreads) cu_s[i] = a.cu[i];
  const int32_t* cu = cu_in_smem ? cu_s : a.cu;
  if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&q_full[i], 4);   // one arrival per loader warp
      mbar_init(&q_empty[i], 1);  // MMA commit
    }
    mbar_init(&acc_full, 1);
    mbar_init(&acc_empty, 8);  // one arrival per selection warp
    for (int i = 0; i < 4; ++i) {
      mbar_init(&x_full[i][0], 1);
      mbar_init(&x_full[i][1], 1);
    }
    mbar_init(&drain, 1);
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
  const int nh = dm.shared ? dm.Hq / dm.Hkv : 1;  // Q tiles summed per item (shared routing)
  const int j0 = a.cpg ? (int)blockIdx.x % a.cpg : 0;
  const int jstep = a.cpg ? a.cpg : 1;
  const uint32_t quarter_lanes = (uint32_t)((warp & 3) * 32) << 16;
  // phase trace (trace build only); event ids: loaders 1 item, 2 buffer free,
  // 3 tile stored; MMA issuer 4 scores free, 5 tile ready, 6 issued;
  // selection 10 scores ready, 11 scores in registers, 12 list sorted,
  // 13 lists merged, 14 row written
  MOBA_TRACE_STATE(trace::kGateNet);

  // The roles split here, at the top level, each with its own copy of the
  // group loop, so ptxas gives each role's code its own register budget.
  // Per group the roles meet twice at barrier 1 (all 384 threads): before
  // the selection warps stage the group's kbar terms (the previous group's
  // MMAs are complete: the selection warps waited for their commit) and after.
  uint32_t n_item = 0;  // items handled so far (every role counts alike)
  bool ok = true;
  if (warp < 4) {
    // ====== Q loaders (warps 0-3) + MMA issuer (lane 0 of warp 0) ======
    regs_dec();
    const int r = warp * 32 + lane;  // tile row of this thread
    uint32_t n_slot = 0;             // Q buffer slots filled so far
    for (int gs = 0;; ++gs) {
      const int gi = group_of(a, gs);
      if (gi < 0) break;
      named_bar(1, kThreads);
      named_bar(1, kThreads);
      for (int j = j0; ok && j < a.ipg; j += jstep) {
        const Item x = decode_item(a, cu, gi, j);
        if (!item_live(a, x)) continue;
        const int N = item_n(a, x);
        MOBA_TRACE(1, N);
        {
          // the next item's rows of this thread into L2 while this item loads
          int jn = j + jstep;
          while (jn < a.ipg && !item_live(a, decode_item(a, cu, gi, jn))) jn += jstep;
          if (jn < a.ipg) {
            const Item xn = decode_item(a, cu, gi, jn);
            if (xn.p0 + r < xn.len && item_n(a, xn) > 0)
              for (int hh = 0; hh < nh; ++hh) {
                const __nv_bfloat16* row = a.q + ((xn.start + xn.p0 + r) * dm.Hq + xn.h + hh) * 128;
                prefetch_l2(row);
                prefetch_l2(row + 64);
              }
          }
        }
        // every Q tile of the item: load it, then (warp 0, lane 0) issue its
        // MMAs at once, so a later tile's buffer never waits on this warp
        for (int hh = 0; ok && N > 0 && hh < nh; ++hh, ++n_slot) {
          const uint32_t b = n_slot & 1u;
          if (n_slot >= 2) {
            ok = mbar_wait(&q_empty[b], ((n_slot >> 1) - 1) & 1, abort, status);
            if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
          }
          MOBA_TRACE(2, hh);
          const int p = x.p0 + r;
          const bool has = p < x.len && MOBA_CHECK(x.start + p < dm.T && x.h + hh < dm.Hq, status);
          const __nv_bfloat16* src = a.q + ((x.start + (has ? p : 0)) * dm.Hq + x.h + hh) * 128;
          // the row in four 16-column pieces of two 32-byte loads each, one
          // piece's loads in flight while the previous piece is stored (the
          // loader warps have few registers)
          uint32_t v[2][16];
          auto load_piece = [&](int piece, uint32_t (&w)[16]) {
            uint32_t lo[8], hi[8];
            if (has) {
              ldg_v8_b32(src + piece * 32, lo);
              ldg_v8_b32(src + piece * 32 + 16, hi);
            } else {
#pragma unroll
              for (int u = 0; u < 8; ++u) lo[u] = hi[u] = 0u;
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
              w[u] = lo[u];
              w[8 + u] = hi[u];
            }
          };
          load_piece(0, v[0]);
#pragma unroll
          for (int piece = 0; piece < 4; ++piece) {
            if (piece + 1 < 4) load_piece(piece + 1, v[(piece + 1) & 1]);
            tmem_st16(tmem + quarter_lanes + kQCol + b * 64 + piece * 16, v[piece & 1]);
          }
          tmem_wait_st();
          fence_before_sync();
          __syncwarp();
          if (lane == 0) mbar_arrive(&q_full[b]);
          MOBA_TRACE(3, hh);
          if (warp == 0) {
            if (lane == 0) {
              // scores (+)= Q K^T with the three kbar terms; the first tile
              // of an item waits until the last item's scores were read out
              if (hh == 0 && n_item > 0)
                ok = mbar_wait(&acc_empty, (n_item - 1) & 1, abort, status);
              MOBA_TRACE(4, hh);
              if (ok) ok = mbar_wait(&q_full[b], (n_slot >> 1) & 1, abort, status);
              MOBA_TRACE(5, hh);
              if (ok) {
                fence_after_sync();
                const uint32_t idesc = idesc_bf16(kRows, N, false, false);
#pragma unroll 1
                for (int t = 0; t < 3; ++t)
#pragma unroll
                  for (int kk = 0; kk < 8; ++kk) {
                    const uint64_t bd = desc_sw128(
                        sK + t * 2 * kTermHalf + (kk >> 2) * kTermHalf + (kk & 3) * 32, 16, 1024);
                    mma_ts(tmem + kAccCol, tmem + kQCol + b * 64 + kk * 8, bd, idesc,
                           (hh > 0 || t > 0 || kk > 0) ? 1u : 0u);
                  }
                commit(&q_empty[b]);
                if (hh == nh - 1) commit(&acc_full);
                MOBA_TRACE(6, N);
              }
            }
            ok = __shfl_sync(0xffffffffu, ok, 0);
          }
        }
        if (ok && N == 0 && warp == 0) {
          // nothing to score: the rows take their own block alone
          if (lane == 0) {
            if (n_item > 0) ok = mbar_wait(&acc_empty, (n_item - 1) & 1, abort, status);
            if (ok) mbar_arrive(&acc_full);
          }
          ok = __shfl_sync(0xffffffffu, ok, 0);
        }
        ++n_item;
      }
    }
  } else {
    // ====== selection (warps 4-11): two threads per row ======
    regs_inc();
    const int part = (warp - 4) >> 2;  // 0: even 16-column groups, 1: odd
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    for (int gs = 0;; ++gs) {
      const int gi = group_of(a, gs);
      if (gi < 0) break;
      named_bar(1, kThreads);
      if (!*abort) {
        stage_kbar(a, decode_item(a, cu, gi, 0), sK, kTermHalf, tid - 128, kThreads - 128);
        fence_proxy_async_smem();
      }
      named_bar(1, kThreads);
      for (int j = j0; ok && j < a.ipg; j += jstep) {
        const Item x = decode_item(a, cu, gi, j);
        if (!item_live(a, x)) continue;
        const int p = x.p0 + r;
        const bool valid = p < x.len;
        const int c = valid ? p / dm.B : 0;
        ok = mbar_wait(&acc_full, n_item & 1, abort, status);
        if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
        MOBA_TRACE(10, (int)n_item);
        fence_after_sync();
        const int cw = __reduce_max_sync(0xffffffffu, c);  // columns any row of the warp needs
        uint32_t raw[8][16];
#pragma unroll
        for (int gq = 0; gq < 8; ++gq) {
          const int g = part + 2 * gq;
          if (16 * g < cw) tmem_ld16(tmem + quarter_lanes + kAccCol + 16 * g, raw[gq]);
        }
        tmem_wait_ld();
        // the scores are in registers: the next item's MMA may overwrite them
        fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty);
        MOBA_TRACE(11, cw);
        // fp32 keys compared with float max / min (sortnet.cuh)
        float list[16];
#pragma unroll
        for (int u = 0; u < 16; ++u) list[u] = -INFINITY;
        // groups below every row's own block need no mask
        const int cmin = __reduce_min_sync(0xffffffffu, valid ? c : cw);
#pragma unroll
        for (int gq = 0; gq < 8; ++gq) {
          const int g = part + 2 * gq;
          if (16 * g < cw) {
            float key[16];
            if (16 * g + 16 <= cmin) {
#pragma unroll
              for (int u = 0; u < 16; ++u) key[u] = net::order_key(__uint_as_float(raw[gq][u]), 16 * g + u);
            } else {
#pragma unroll
              for (int u = 0; u < 16; ++u) {
                const int i = 16 * g + u;
                key[u] = i < c ? net::order_key(__uint_as_float(raw[gq][u]), i) : -INFINITY;
              }
            }
            net::oe_sort16(key);
            net::merge_top16(list, key);
          }
        }
        MOBA_TRACE(12, 0);
        // the two lists of the row meet through TMEM (two buffers by item parity)
        const uint32_t par = n_item & 1u;
        const uint32_t xcol = tmem + quarter_lanes + kXCol + par * 16;
        if (part == 1) {
          uint32_t w[16];
#pragma unroll
          for (int u = 0; u < 16; ++u) w[u] = __float_as_uint(list[u]);
          tmem_st16(xcol, w);
          tmem_wait_st();
          fence_before_sync();
          __syncwarp();
          if (lane == 0) mbar_arrive(&x_full[quarter][par]);
          MOBA_TRACE(13, 0);
        } else {
          ok = mbar_wait(&x_full[quarter][par], (n_item >> 1) & 1, abort, status);
          if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
          fence_after_sync();
          uint32_t w[16];
          tmem_ld16(xcol, w);
          tmem_wait_ld();
          float other[16];
#pragma unroll
          for (int u = 0; u < 16; ++u) other[u] = __uint_as_float(w[u]);
          net::merge_top16(list, other);
          MOBA_TRACE(13, 0);
          if (valid) {
            // the top min(k-1, c) keys in ascending block order (descending
            // 255 - i, exact in fp32), then the own block c, then -1
            const int hsel = min(dm.topk - 1, c);
            float sel[16];
#pragma unroll
            for (int u = 0; u < 16; ++u)
              sel[u] = u < hsel ? (float)(255 - net::key_block(list[u])) : -1.f;
            net::oe_sort16(sel);
            int v[16];
#pragma unroll
            for (int u = 0; u < 16; ++u) v[u] = u < hsel ? 255 - (int)sel[u] : (u == hsel ? c : -1);
            for (int hh = 0; hh < nh; ++hh) {
              if (!MOBA_CHECK(x.start + p < dm.T && x.h + hh < dm.Hq, status)) break;
              int32_t* row = a.idx + ((x.start + p) * dm.Hq + x.h + hh) * (int64_t)dm.topk;
              if (a.vec_rows) {
#pragma unroll
                for (int u = 0; u < 16; u += 4)
                  if (u < dm.topk)
                    *reinterpret_cast<int4*>(row + u) = make_int4(v[u], v[u + 1], v[u + 2], v[u + 3]);
              } else {
#pragma unroll
                for (int u = 0; u < 16; ++u)
                  if (u < dm.topk) row[u] = v[u];
              }
            }
          }
        }
        MOBA_TRACE(14, 0);
        ++n_item;
      }
    }
  }
  MOBA_TRACE_END();
  if (!ok) *abort = 1;
  __syncthreads();
  if (tid == 0 && *abort) {
    // let every MMA issued land before the CTA frees its TMEM
    commit(&drain);
    mbar_drain(&drain, 0);
  }
  fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    fence_after_sync();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

bool gate_net_supported(const Dims& dm) {
  const int need = hist_slots(dm);
  return dm.dtype == kBF16 && dm.d == 128 && dm.nb <= kMaxBlocks && !dm.prefix && need >= 5 &&
         need <= 15;
}

cudaError_t launch_gate_net(const Dims& dm, const void* q, const float* kbar, const int32_t* cu,
                            int32_t* idx, int* status, cudaStream_t st) {
  if (dm.batch == 0 || dm.max_seqlen == 0) return cudaSuccess;
  NetArgs a{};
  a.dm = dm;
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.kbar = kbar;
  a.cu = cu;
  a.idx = idx;
  a.status = status;
  const int nqt = (dm.max_seqlen + kRows - 1) / kRows;
  const int64_t ipg = (int64_t)nqt * (dm.shared ? 1 : dm.Hq / dm.Hkv);
  if ((int64_t)dm.batch * dm.Hkv * ipg > INT_MAX) return cudaErrorInvalidValue;
  a.groups = dm.batch * dm.Hkv;
  a.ipg = (int)ipg;
  a.nbp = ((dm.nb + 15) / 16) * 16;
  // a row of k int32 starts on a 16-byte boundary when k % 4 == 0 and idx does
  a.vec_rows = (dm.topk % 4 == 0 && (reinterpret_cast<uintptr_t>(idx) & 15) == 0) ? 1 : 0;
  const size_t smem = 1024 + (size_t)3 * 2 * a.nbp * 128;
  // once per device: the shared memory, and the registers the setmaxnreg
  // split needs from the launch
  static std::mutex mu;
  static int ready[tc::kMaxDevices] = {};  // 0 unknown, 1 ready, -1 unusable
  int dev = 0;
  cudaError_t e;
  if ((e = cudaGetDevice(&dev))) return e;
  if (dev < 0 || dev >= tc::kMaxDevices) return cudaErrorInvalidDevice;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (ready[dev] == 0) {
      if ((e = cudaFuncSetAttribute(gate_net_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    1024 + 3 * 2 * kMaxBlocks * 128)))
        return e;
      cudaFuncAttributes fa;
      if ((e = cudaFuncGetAttributes(&fa, gate_net_kernel))) return e;
      ready[dev] = fa.numRegs * kThreads >= 128 * kRegsLoad + 256 * kRegsSel ? 1 : -1;
    }
  }
  if (ready[dev] < 0) return cudaErrorInvalidConfiguration;
  const int target = tc::sm_count();  // one CTA per SM (all 512 TMEM columns)
  int grid;
  if (a.groups >= target) {
    a.cpg = 0;
    grid = target;
  } else {
    a.cpg = target / a.groups;
    if (a.cpg > a.ipg) a.cpg = a.ipg;
    grid = a.groups * a.cpg;
  }
  gate_net_kernel<<<grid, kThreads, smem, st>>>(a);
  return cudaGetLastError();
}

}  // namespace moba
