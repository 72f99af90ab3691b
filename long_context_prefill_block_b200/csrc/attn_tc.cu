// Tensor-core attention for bf16, d = 128 (sm_100a: tcgen05 + TMEM + TMA).
//
// One engine serves the three places where MoBA does exact softmax
// attention (PaperTrace "2.1.3 MoBA", section 2 eq. 4-6, section 3.1):
//   HIST  : a tile of up to 128 regrouped (query, head, slot) rows that all
//           chose the same earlier block, against that block's B raw keys,
//           non-causal (eq. 6); writes a normalised partial result per slot;
//   CUR   : 128 consecutive queries of one head against their own block,
//           causal on the diagonal tile (eq. 5); its epilogue merges the
//           result with the rows' history partials (eq. 7-8) and writes
//           the output;
//   DENSE : 128 consecutive queries against every earlier key of their
//           sequence (eq. 1, causal); writes the output.
// HIST runs first; CUR then finds every history partial of its rows ready.
//
// Persistent CTAs (one per SM) walk a static list of work units of two
// 128-row query halves that read the same KV tiles (HIST: 256 consecutive
// rows of one block's list; CUR / DENSE: two consecutive 128-row query
// tiles, the second one seeing one more KV tile). Each KV tile (128 keys) is
// loaded once and used by both halves, which halves the shared-memory fill
// traffic per flop, and the two halves ping-pong on the tensor core: while
// one half's softmax runs, the other half's MMAs do. TMEM holds per half h
// the logits S[h] (128 fp32 columns; P overwrites its first 64 columns as
// bf16 pairs) and the accumulator O[h]. Roles (12 warps):
//   warp 0      TMA producer: K and V tiles of 128 keys (two 64-column
//               halves, 128-byte swizzle) into a 2-stage ring;
//   warps 1-2   lane 0 of warp 1 + h issues the tcgen05.mma of half h (warp
//               1 also allocates all 512 TMEM columns): S[h] = Q_h K(0)^T,
//               then per KV tile j O[h] += P_h(j) V(j) and S[h] = Q_h
//               K(j+1)^T into the same TMEM -- tcgen05.mma operations of one
//               thread run in issue order, so the PV has read P before the
//               next QK^T overwrites it. The softmax warps hand P over in
//               four quarters of 32 keys, so each quarter's PV runs while the
//               next is exponentiated. Issuing blocks for about the group's
//               execution time, hence one issuer per half;
//   warp 3      Q loader: cp.async of each half's (gathered, in HIST mode)
//               query rows into the swizzled layout the MMA reads;
//   warps 4-7   softmax + epilogue of half 0, warps 8-11 of half 1: one query
//               row per thread (TMEM lane = row), base-2 exponentials; O[h]
//               is rescaled only when a row maximum grows by more than 2^8.
//               The two halves take turns on the exponentials (shared-memory
//               counters), so one half's PV and next QK^T run on the tensor
//               core while the other half exponentiates.
// The softmax warps get most of the register file (setmaxnreg): they hold a
// whole 128-column row of S, or of O in the epilogue.
//
// Every wait is bounded (tc::mbar_wait); on expiry the CTA records
// kStTimeout, drains the copies and MMAs it issued, frees its TMEM and exits.
#include <cudaTypedefs.h>

#include <mutex>

#include "tc_ptx.cuh"
#include "trace.cuh"

namespace moba {

bool tc_supported(const Dims& dm) {
  return dm.dtype == kBF16 && dm.d == 128 && dm.B % 128 == 0;
}

namespace {

using namespace tc;

enum Mode { HIST = 0, CUR = 1, DENSE = 2 };

constexpr int TM = 128;   // query rows per half
constexpr int TN = 128;   // keys per KV tile
constexpr int D = 128;    // head dim
constexpr int NS = 2;     // K/V ring stages
constexpr int kThreads = 384;
constexpr int kLoaderThreads = 32;
constexpr int kLaunchRegs = 168;    // 65536 / 384, rounded down to a multiple of 8
constexpr int kRegsOther = 72;      // warps 0-3 after setmaxnreg.dec
constexpr int kRegsSoftmax = 216;   // warps 4-11 after setmaxnreg.inc
static_assert(128 * kRegsOther + 256 * kRegsSoftmax <= kThreads * kLaunchRegs,
              "register split exceeds the launch allocation");
constexpr uint32_t kHalf = 128 * 128;  // bytes of one 64-column half of a 128-row tile
constexpr uint32_t kTile = 2 * kHalf;  // bytes of one 128 x 128 bf16 tile
// Q buffers: the (unit, half) loads of a CTA take slots 0, 1, 2, ... in
// order; slot s uses buffer s % kQBufs. With three buffers for two halves
// the loader fills the next unit's first half while this unit still computes.
constexpr int kQBufs = 3;
constexpr uint32_t kQOff = 0;                // Q[kQBufs]
constexpr uint32_t kKOff = kQBufs * kTile;   // K[NS]
constexpr uint32_t kVOff = kKOff + NS * kTile;
constexpr uint32_t kSmemBytes = kVOff + NS * kTile + 1024;  // + 1024-byte alignment slack
constexpr int kCuSmem = 257;  // sequence offsets kept in shared memory
constexpr uint32_t kTmemCols = 512;    // S[0] 0, S[1] 128, O[0] 256, O[1] 384
constexpr uint32_t kOCol = 256;
constexpr uint32_t kIdescQK = idesc_bf16(TM, TN, false, false);  // Q, K both K-major
constexpr uint32_t kIdescPV = idesc_bf16(TM, D, false, true);    // V is MN-major (d contiguous)
constexpr float kRescaleLog2 = 8.f;
// Softmax exponentials taken off the exponential unit: of every 8 column
// pairs, this many go through ex2_poly2 on the FMA pipes.
constexpr int kPolyOf8 = 0;
// Whether the history and own-block kernels also make the two query halves
// take turns on the exponentials (the dense kernel always does).
constexpr bool kTurnsAll = true;

struct Shared {
  // per query half h
  uint64_t q_full[kQBufs], q_empty[kQBufs];
  uint64_t s_full[2], p_q[2][4], o_full[2], o_free[2];
  uint64_t k_full[NS], k_empty[NS], v_full[NS], v_empty[NS];
  uint64_t drain[2];
  uint32_t tmem_base;
  int abort;
  int exp_cnt[2];  // per half: softmax warps done with a KV tile's exponentials
  int32_t cu[kCuSmem];  // sequence offsets (batch < kCuSmem), read without global loads
};

struct Args {
  Dims dm;
  Chunk ch;
  const __nv_bfloat16* q;
  const int32_t* cu;
  int n_tiles;  // CUR / DENSE: size of the static tile space
  // HIST
  const int32_t* list_off;
  const int32_t* pairs;
  const int4* tiles;
  const int32_t* tile_count;
  // CUR
  const int32_t* idx;
  // outputs
  void* part_o;  // bf16 partial rows, interleaved layout
  float* part_lse;
  __nv_bfloat16* out;
  float* lse_out;
  int* status;
};

// A work unit: half 0 is described by the fields below; half 1 starts 128
// rows later (half_view). n[h] = KV tiles half h reads (0: half h is empty);
// the unit streams max(n[0], n[1]) KV tiles.
struct Tile {
  bool skip;
  int b, g, h, kv0, n_kv, p0, list, row0, count, base;
  int n[2];
  int64_t start;
  int4 raw;  // HIST: the tile-table entry, decoded by resolve()
};

// Unit t of the static unit space. CUR / DENSE units are ordered longest
// first so the persistent CTAs end together. A HIST unit is one 16-byte
// load of the tile table, decoded later by resolve(): the roles fetch the
// next unit's description a unit ahead, and the load must not stall them
// until the unit starts.
template <int MODE>
__device__ __forceinline__ Tile get_tile(const Args& a, const int32_t* cu, int t) {
  const Dims& dm = a.dm;
  Tile T{};
  T.skip = false;
  if (MODE == HIST) {
    T.raw = a.tiles[t];  // list, first row, list size, list base
    return T;
  }
  int m;  // the unit holds query tiles 2m and 2m + 1 (of the block / sequence)
  if (MODE == CUR) {
    const int R = dm.B / TM;                      // query tiles per block
    const int R2 = (R + 1) / 2;                   // units per block
    const int per = dm.nb * dm.batch * a.ch.nq;   // units with the same m
    m = R2 - 1 - t / per;
    int rem = t % per;
    const int c = rem / (dm.batch * a.ch.nq);
    rem %= dm.batch * a.ch.nq;
    T.b = rem / a.ch.nq;
    T.h = a.ch.h0 + rem % a.ch.nq;
    T.p0 = c * dm.B + 2 * m * TM;
    T.kv0 = c * dm.B;
    T.n[1] = 2 * m + 1 < R ? 2 * m + 2 : 0;
  } else {
    const int nqt = (dm.max_seqlen + TM - 1) / TM;
    const int nqt2 = (nqt + 1) / 2;
    const int per = dm.batch * dm.Hq;
    m = nqt2 - 1 - t / per;
    const int rem = t % per;
    T.b = rem / dm.Hq;
    T.h = rem % dm.Hq;
    T.p0 = 2 * m * TM;
    T.kv0 = 0;
    T.n[1] = 2 * m + 2;
  }
  T.n[0] = 2 * m + 1;
  T.g = T.h / (dm.Hq / dm.Hkv);
  T.start = cu[T.b];
  const int len = cu[T.b + 1] - cu[T.b];
  T.count = len;  // sequence length, for the row checks below
  T.skip = len < 0 || len > dm.max_seqlen || T.p0 >= len;
  if (T.p0 + TM >= len) T.n[1] = 0;
  T.n_kv = T.n[1] > T.n[0] ? T.n[1] : T.n[0];
  return T;
}

// Decodes a HIST unit's tile-table entry (CUR / DENSE units are complete).
template <int MODE>
__device__ __forceinline__ Tile resolve(const Args& a, const int32_t* cu, Tile T) {
  if (MODE == HIST) {
    const Dims& dm = a.dm;
    const int4 tl = T.raw;
    T.list = tl.x;
    T.row0 = tl.y;
    const int e = T.list % dm.nb;
    T.g = a.ch.g0 + (T.list / dm.nb) % a.ch.ng;
    T.b = T.list / (dm.nb * a.ch.ng);
    T.count = tl.z;
    T.base = tl.w;
    T.kv0 = e * dm.B;
    T.n_kv = dm.B / TN;
    T.n[0] = T.n_kv;
    T.n[1] = T.row0 + TM < T.count ? T.n_kv : 0;
    T.start = cu[T.b];
  }
  return T;
}

// The tile of query half h of a unit, as the row helpers below see it.
template <int MODE>
__device__ __forceinline__ Tile half_view(const Tile& T, int h) {
  Tile U = T;
  if (MODE == HIST)
    U.row0 += h * TM;
  else
    U.p0 += h * TM;
  U.n_kv = T.n[h];
  return U;
}

// Identity of query row r of a tile: the q row it reads (t * Hq + h, or -1)
// and, for outputs, the token t, head h, position p and partial row prow.
// Own-block rows (CUR): prow is the row's first partial slot, nhist the
// number of history partials before the own block's slot, and own whether
// the row reads its own block (a row whose own block lost the prefix-mean
// gate merges its history alone).
struct Row {
  bool has_q, valid, own;
  int64_t t, prow;
  int h, p, nhist;
};

template <int MODE>
__device__ __forceinline__ Row get_row(const Args& a, const Tile& T, int r) {
  const Dims& dm = a.dm;
  Row R{};
  const int64_t n_part = (int64_t)dm.T * a.ch.nq * dm.topk;  // partial rows of the pass
  if (MODE == HIST) {
    R.has_q = R.valid = T.row0 + r < T.count &&
                        MOBA_CHECK((int64_t)T.base + T.row0 + r <
                                       (int64_t)dm.T * a.ch.nq * hist_slots(dm),
                                   a.status);
    if (R.valid) {
      R.prow = a.pairs[T.base + T.row0 + r];
      R.has_q = R.valid = MOBA_CHECK(R.prow >= 0 && R.prow < n_part, a.status);
      const int64_t th = R.prow / dm.topk;
      R.t = th / a.ch.nq;
      R.h = a.ch.h0 + (int)(th % a.ch.nq);
    }
    return R;
  }
  R.h = T.h;
  R.p = T.p0 + r;
  R.has_q = R.valid = R.p < T.count && MOBA_CHECK(T.start + R.p < dm.T, a.status);
  R.t = T.start + R.p;
  if (MODE == CUR && R.valid) {
    const int c = R.p / dm.B;
    const int32_t* row = a.idx + (R.t * dm.Hq + R.h) * (int64_t)dm.topk;
    int slot = -1, n = 0;
    for (int i = 0; i < dm.topk; ++i) {
      if (row[i] == c && slot < 0) slot = i;
      n += row[i] >= 0 && row[i] < c;
    }
    R.prow = (R.t * a.ch.nq + (R.h - a.ch.h0)) * (int64_t)dm.topk;
    R.own = slot >= 0;
    R.nhist = R.own ? slot : n;
    R.valid = (R.own || dm.prefix) &&
              MOBA_CHECK(R.nhist <= dm.topk && R.prow + dm.topk <= n_part, a.status);
  }
  return R;
}

// Query row r of a tile for the loader: the q row it reads, or none.
template <int MODE>
__device__ __forceinline__ bool q_row_of(const Args& a, const Tile& T, int r, int64_t& qrow) {
  if (MODE == HIST) {
    if (T.row0 + r >= T.count) return false;
    const int64_t prow = a.pairs[T.base + T.row0 + r];
    const int64_t th = prow / a.dm.topk;
    qrow = (th / a.ch.nq) * a.dm.Hq + a.ch.h0 + (int)(th % a.ch.nq);
    return MOBA_CHECK(qrow >= 0 && qrow < (int64_t)a.dm.T * a.dm.Hq, a.status);
  }
  const int p = T.p0 + r;
  if (p >= T.count) return false;
  qrow = (T.start + p) * a.dm.Hq + T.h;
  return MOBA_CHECK(qrow < (int64_t)a.dm.T * a.dm.Hq, a.status);
}

__device__ __forceinline__ void regs_dec() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsOther));
}
__device__ __forceinline__ void regs_inc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsSoftmax));
}

template <int MODE>
__global__ void __launch_bounds__(kThreads, 1)
attn_tc_kernel(const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv,
               const Args a) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ Shared sh;
  const Dims& dm = a.dm;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (a.status && *reinterpret_cast<volatile int*>(a.status) == kStTimeout) return;
  const int n_tiles = MODE == HIST ? *a.tile_count : a.n_tiles;
  if ((int)blockIdx.x >= n_tiles) return;

  const uint32_t sbase = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const uint32_t sQ = sbase + kQOff, sK = sbase + kKOff, sV = sbase + kVOff;

  const bool cu_in_smem = dm.batch < kCuSmem;
  if (cu_in_smem)
    for (int i = threadIdx.x; i <= dm.batch; i += kThreads) sh.cu[i] = a.cu[i];
  const int32_t* cuv = cu_in_smem ? sh.cu : a.cu;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kQBufs; ++i) {
      mbar_init(&sh.q_full[i], kLoaderThreads);
      mbar_init(&sh.q_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sh.s_full[i], 1);
      for (int c = 0; c < 4; ++c) mbar_init(&sh.p_q[i][c], 128);
      mbar_init(&sh.o_full[i], 1);
      mbar_init(&sh.o_free[i], 128);
    }
    for (int i = 0; i < NS; ++i) {
      mbar_init(&sh.k_full[i], 1);
      mbar_init(&sh.k_empty[i], 2);  // one commit from each issuer
      mbar_init(&sh.v_full[i], 1);
      mbar_init(&sh.v_empty[i], 2);
    }
    mbar_init(&sh.drain[0], 1);
    mbar_init(&sh.drain[1], 1);
    sh.abort = 0;
    sh.exp_cnt[0] = sh.exp_cnt[1] = 0;
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
  int* status = a.status;
  // phase trace (trace build only); event ids: TMA producer 20 K tile issued,
  // 21 V tile issued; MMA issuers 30 unit, 31 QK issued, 32 P keys 0-63
  // ready, 33 PV issued; Q loader 40 Q half loaded; softmax 50 S ready,
  // 51 row max, 52 P keys 0-63 written, 53 P written, 54 O ready, 55 row
  // written, 56 S in registers, 58 P computed
  MOBA_TRACE_STATE(MODE == HIST ? trace::kAttnHist
                                : (MODE == CUR ? trace::kAttnCur : trace::kAttnDense));

  if (warp < 4) {
    // warps 0-3 (one warp group) give registers to the softmax warps
    regs_dec();
    if (warp == 0) {
      // ================= TMA producer: K and V tiles =================
      if (lane == 0) {
        uint32_t g = 0, nk = 0, nv = 0;
        bool ok = true;
        Tile Tnext = (int)blockIdx.x < n_tiles ? get_tile<MODE>(a, cuv, blockIdx.x) : Tile{};
        for (int t = blockIdx.x; ok && t < n_tiles; t += gridDim.x) {
          const Tile T = resolve<MODE>(a, cuv, Tnext);  // read one unit ahead
          if (t + (int)gridDim.x < n_tiles) Tnext = get_tile<MODE>(a, cuv, t + gridDim.x);
          if (T.skip) continue;
          for (int j = 0; j < T.n_kv; ++j, ++g) {
            const uint32_t st = g % NS, u = g / NS;
            const int z = (int)(T.start + T.kv0 + j * TN);
            if (u > 0 && !(ok = mbar_wait(&sh.k_empty[st], (u - 1) & 1, abort, status))) break;
            mbar_expect_tx(&sh.k_full[st], kTile);
            tma_load_3d(sK + st * kTile, &tmk, &sh.k_full[st], 0, T.g, z);
            tma_load_3d(sK + st * kTile + kHalf, &tmk, &sh.k_full[st], 64, T.g, z);
            nk = g + 1;
            MOBA_TRACE(20, j);
            if (u > 0 && !(ok = mbar_wait(&sh.v_empty[st], (u - 1) & 1, abort, status))) break;
            mbar_expect_tx(&sh.v_full[st], kTile);
            tma_load_3d(sV + st * kTile, &tmv, &sh.v_full[st], 0, T.g, z);
            tma_load_3d(sV + st * kTile + kHalf, &tmv, &sh.v_full[st], 64, T.g, z);
            nv = g + 1;
            MOBA_TRACE(21, j);
          }
        }
        if (!ok || *abort) {
          // let the copies already issued land before the CTA exits
          for (uint32_t x = nk > NS ? nk - NS : 0; x < nk; ++x)
            mbar_drain(&sh.k_full[x % NS], (x / NS) & 1);
          for (uint32_t x = nv > NS ? nv - NS : 0; x < nv; ++x)
            mbar_drain(&sh.v_full[x % NS], (x / NS) & 1);
        }
      }
    } else if (warp < 3) {
      // ====== MMA issuers: warp 1 for query half 0, warp 2 for half 1 ======
      // One thread per half: issuing a group of MMAs blocks the thread for
      // about the group's execution time, so a single issuer would make each
      // half wait behind the other's groups. Per half the order is QK(0),
      // then PV(j), QK(j + 1) for each KV tile j; K(j) and V(j) are
      // released by both issuers (empty barriers count two), also for tiles
      // a half skips.
      const int h = warp - 1;
      if (lane == 0) {
        uint32_t gk = 0;  // KV tiles streamed before this unit
        uint32_t kh = 0;  // KV tiles of this half before this unit
        uint32_t uh = 0;  // units with this half non-empty before this one
        uint32_t qs = 0;  // Q slots (loads of either half) before this unit
        bool ok = true;
        Tile Tnext = (int)blockIdx.x < n_tiles ? get_tile<MODE>(a, cuv, blockIdx.x) : Tile{};
        for (int t = blockIdx.x; ok && t < n_tiles; t += gridDim.x) {
          const Tile T = resolve<MODE>(a, cuv, Tnext);  // read one unit ahead
          if (t + (int)gridDim.x < n_tiles) Tnext = get_tile<MODE>(a, cuv, t + gridDim.x);
          if (T.skip) continue;
          const int nh = T.n[h];
          MOBA_TRACE(30, nh);
          const uint32_t qslot = qs + (h == 1 && T.n[0] > 0 ? 1u : 0u);
          const uint32_t qb = qslot % kQBufs;
          qs += (T.n[0] > 0 ? 1u : 0u) + (T.n[1] > 0 ? 1u : 0u);
          for (int j = 0; ok && j < T.n_kv; ++j) {
            const uint32_t gg = gk + j, st = gg % NS;
            // Both issuers wait for every tile, also one they skip, before
            // releasing it: an early release could complete the barrier
            // phase of an older tile that the other issuer still reads.
            if (!(ok = mbar_wait(&sh.k_full[st], (gg / NS) & 1, abort, status))) break;
            if (j < nh) {
              // S[h] = Q_h K(j)^T; S[h] holds P(j - 1) until PV(j - 1), which
              // this thread issued before
              if (j == 0 &&
                  !(ok = mbar_wait(&sh.q_full[qb], (qslot / kQBufs) & 1, abort, status)))
                break;
              fence_after_sync();
#pragma unroll
              for (int kk = 0; kk < D / 16; ++kk) {
                const uint32_t off = (kk >> 2) * kHalf + (kk & 3) * 32;
                const uint64_t ad = desc_sw128(sQ + qb * kTile + off, 16, 1024);
                const uint64_t bd = desc_sw128(sK + st * kTile + off, 16, 1024);
                mma_ss(tmem + h * 128, ad, bd, kIdescQK, kk > 0 ? 1u : 0u);
              }
              commit(&sh.s_full[h]);
              if (j == nh - 1) commit(&sh.q_empty[qb]);
              MOBA_TRACE(31, j);
            }
            commit(&sh.k_empty[st]);
            if (j < nh && j == 0 && uh > 0 &&
                !(ok = mbar_wait(&sh.o_free[h], (uh - 1) & 1, abort, status)))
              break;
            if (!(ok = mbar_wait(&sh.v_full[st], (gg / NS) & 1, abort, status))) break;
            if (j < nh) {
              // O[h] += P_h(j) V(j), P read from the first 64 columns of S[h].
              // P arrives in quarters of 32 keys (two k-steps each): each
              // quarter's PV runs while the softmax warps exponentiate the next
#pragma unroll
              for (int kk = 0; kk < TN / 16; ++kk) {
                if ((kk & 1) == 0) {
                  if (!(ok = mbar_wait(&sh.p_q[h][kk >> 1], (kh + j) & 1, abort, status))) break;
                  fence_after_sync();
                  if (kk == 0) MOBA_TRACE(32, j);
                }
                const uint64_t bd = desc_sw128(sV + st * kTile + kk * 16 * 128, kHalf, 1024);
                mma_ts(tmem + kOCol + h * 128, tmem + h * 128 + kk * 8, bd, kIdescPV,
                       (j > 0 || kk > 0) ? 1u : 0u);
              }
              if (!ok) break;
              if (j == nh - 1) commit(&sh.o_full[h]);
              MOBA_TRACE(33, j);
            }
            commit(&sh.v_empty[st]);
          }
          gk += T.n_kv;
          kh += nh;
          uh += nh > 0 ? 1u : 0u;
        }
        if (!ok) {
          // wait until every MMA this thread issued has finished
          commit(&sh.drain[h]);
          mbar_drain(&sh.drain[h], 0);
        }
      }
    } else {
      // ================= Q loader, warp 3 =================
      // The row ids of a unit (tile table -> list offset -> pairs: three
      // dependent global loads in the history kernel) are fetched one unit
      // ahead, while the current unit computes, so a freed Q buffer waits
      // only for its copies.
      constexpr int RPL = TM / kLoaderThreads;  // rows per lane and half
      const int tl = lane;
      uint32_t qs = 0;  // Q slots loaded so far
      bool ok = true;
      auto next_unit = [&](int t) {
        for (; t < n_tiles; t += gridDim.x)
          if (!get_tile<MODE>(a, cuv, t).skip) break;
        return t;
      };
      // row ids (t * Hq + h < 2^31, checked on the host) of both halves of
      // unit t, -1 where a row is empty; bit h of the result: half h reads
      auto fetch_rows = [&](int t, int32_t (&qr)[2][RPL]) {
        const Tile T = resolve<MODE>(a, cuv, get_tile<MODE>(a, cuv, t));
        int mask = 0;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const Tile U = half_view<MODE>(T, h);
          if (T.n[h] > 0) mask |= 1 << h;
#pragma unroll
          for (int hr = 0; hr < RPL; ++hr) {
            int64_t qrow = -1;
            if (T.n[h] == 0 || !q_row_of<MODE>(a, U, tl + hr * kLoaderThreads, qrow)) qrow = -1;
            qr[h][hr] = (int32_t)qrow;
          }
        }
        return mask;
      };
      int t = next_unit(blockIdx.x);
      int32_t qr[2][RPL];
      int mask = t < n_tiles ? fetch_rows(t, qr) : 0;
      while (ok && t < n_tiles) {
        for (int h = 0; h < 2; ++h) {
          if (!(mask >> h & 1)) continue;
          const uint32_t qb = qs % kQBufs;
          if (qs >= (uint32_t)kQBufs) {
            ok = mbar_wait(&sh.q_empty[qb], (qs / kQBufs - 1) & 1, abort, status);
            if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
          }
#pragma unroll
          for (int hr = 0; hr < RPL; ++hr) {
            const int rr = tl + hr * kLoaderThreads;
            const bool has = qr[h][hr] >= 0;
            const __nv_bfloat16* src = a.q + (has ? (int64_t)qr[h][hr] : 0) * (int64_t)D;
#pragma unroll
            for (int c16 = 0; c16 < 16; ++c16) {
              const uint32_t dst = sQ + qb * kTile + (c16 >> 3) * kHalf + rr * 128 +
                                   ((((uint32_t)c16 & 7u) ^ ((uint32_t)rr & 7u)) << 4);
              cp_async16(dst, src + c16 * 8, has ? 16u : 0u);
            }
          }
          cp_async_wait_all();
          fence_proxy_async_smem();
          mbar_arrive(&sh.q_full[qb]);
          MOBA_TRACE(40, h);
          ++qs;
        }
        if (!ok) break;
        // the next unit's row ids, while this unit computes
        t = next_unit(t + gridDim.x);
        mask = t < n_tiles ? fetch_rows(t, qr) : 0;
      }
      cp_async_wait_all();
    }
  } else {
    regs_inc();
    // ====== softmax + epilogue: warps 4..7 half 0, warps 8..11 half 1 ======
    const int hh = (warp - 4) >> 2;
    const int quarter = warp & 3;          // TMEM lanes this warp may access
    const int r = quarter * 32 + lane;     // query row of this thread
    const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t tS = tmem + hh * 128 + lane_addr;
    const uint32_t tO = tmem + kOCol + hh * 128 + lane_addr;
    const float sl2 = rsqrtf((float)D) * 1.4426950408889634f;  // softmax scale, base 2
    uint32_t kc = 0, uc = 0;
    int base[2] = {0, 0};  // KV tiles each half processed in earlier units
    volatile int* exp_cnt = sh.exp_cnt;
    bool ok = true;
    // the unit's description is read one unit ahead: its global loads (tile
    // table, list offsets, sequence bounds) resolve while this unit runs
    Tile Tnext = (int)blockIdx.x < n_tiles ? get_tile<MODE>(a, cuv, blockIdx.x) : Tile{};
    for (int t = blockIdx.x; ok && t < n_tiles; t += gridDim.x) {
      const Tile T0 = resolve<MODE>(a, cuv, Tnext);
      if (t + (int)gridDim.x < n_tiles) Tnext = get_tile<MODE>(a, cuv, t + gridDim.x);
      if (T0.skip) continue;
      const int b0 = base[0], b1 = base[1];
      base[0] += T0.n[0];
      base[1] += T0.n[1];
      if (T0.n[hh] == 0) continue;
      const Tile T = half_view<MODE>(T0, hh);
      const Row R = get_row<MODE>(a, T, r);
      float m_i = -INFINITY, l_i = 0.f;
      for (int j = 0; j < T.n_kv; ++j, ++kc) {
        ok = mbar_wait(&sh.s_full[hh], kc & 1, abort, status);
        if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
        MOBA_TRACE(50, j);
        fence_after_sync();
        float s[TN];
        {
          // issue all four loads, then one wait
          uint32_t r0[32], r1[32], r2[32], r3[32];
          tmem_ld32(tS, r0);
          tmem_ld32(tS + 32, r1);
          tmem_ld32(tS + 64, r2);
          tmem_ld32(tS + 96, r3);
          tmem_wait_ld();
          MOBA_TRACE(56, j);
#pragma unroll
          for (int x = 0; x < 32; ++x) {
            s[x] = __uint_as_float(r0[x]);
            s[32 + x] = __uint_as_float(r1[x]);
            s[64 + x] = __uint_as_float(r2[x]);
            s[96 + x] = __uint_as_float(r3[x]);
          }
        }
        // causal mask on the diagonal tile (CUR / DENSE): key > query
        if (MODE != HIST && T.kv0 + j * TN + TN - 1 > T.p0) {
          const int lim = R.p - (T.kv0 + j * TN);  // last visible column
#pragma unroll
          for (int x = 0; x < TN; ++x)
            if (x > lim) s[x] = -INFINITY;
        }
        // row maximum: 16 independent chains of three-input maxima (chain u
        // takes columns u, u + 16, ..., u + 112: four instructions deep),
        // then a three-input tree
        float mv[16];
#pragma unroll
        for (int u = 0; u < 16; ++u) {
          const float a = fmax3(s[u], s[u + 16], s[u + 32]);
          const float b = fmax3(a, s[u + 48], s[u + 64]);
          const float c = fmax3(b, s[u + 80], s[u + 96]);
          mv[u] = fmaxf(c, s[u + 112]);
        }
        float m6[6];
#pragma unroll
        for (int u = 0; u < 5; ++u) m6[u] = fmax3(mv[3 * u], mv[3 * u + 1], mv[3 * u + 2]);
        m6[5] = mv[15];
        const float mx = fmax3(fmax3(m6[0], m6[1], m6[2]), fmax3(m6[3], m6[4], m6[5]), m6[0]);
        const float mt = mx * sl2;
        MOBA_TRACE(51, j);
        const bool need = mt > m_i + kRescaleLog2;
        const float m_new = need ? mt : m_i;
        if (j > 0 && __any_sync(0xffffffffu, need)) {
          // O[h] holds PV of the earlier KV tiles: S(j) was committed after
          // the last of them, so it is complete. Rescale it in place.
          const float alpha = need ? ex2(m_i - m_new) : 1.f;
#pragma unroll 1
          for (int c = 0; c < D / 32; ++c) {
            uint32_t rr[32];
            tmem_ld32(tO + c * 32, rr);
            tmem_wait_ld();
#pragma unroll
            for (int x = 0; x < 32; ++x) rr[x] = __float_as_uint(__uint_as_float(rr[x]) * alpha);
            tmem_st32(tO + c * 32, rr);
          }
          tmem_wait_st();
        }
        if (need) {
          l_i *= ex2(m_i - m_new);
          m_i = m_new;
        }
        // The two halves take turns on the exponential unit: half 1
        // exponentiates KV tile j after half 0 has, half 0 tile j after half
        // 1 has done tile j - 1. In anti-phase, one half's PV and next QK^T
        // run while the other half exponentiates (measured: history 870 ->
        // 809 ms at the million-token shape, 0.80 -> 0.75 ms at 32K).
        // Counts only grow, so a half that runs ahead into its next unit
        // cannot be mistaken for the turn being waited for.
        if ((MODE == DENSE || kTurnsAll) &&
            (hh == 0 ? (j >= 1 && j - 1 < T0.n[1]) : (j < T0.n[0]))) {
          const int need_cnt = 4 * (hh == 0 ? b1 + j : b0 + j + 1);
          const long long t0 = clock64();
          while (exp_cnt[hh ^ 1] < need_cnt) {
            if (*abort) { ok = false; break; }
            if (clock64() - t0 > kWaitLimitCycles) {
              *abort = 1;
              set_status(status, kStTimeout);
              ok = false;
              break;
            }
          }
          if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
        }
        // P = exp2(s * scale - m) in bf16, two per column, into the S buffer,
        // on column pairs (f32x2): kPolyOf8 of every 8 pairs by ex2_poly2 on
        // the FMA pipes, the others on the exponential unit; the row sum is
        // kept in 4 independent pair sums. P goes to the MMA issuer in four
        // quarters of 32 keys: quarter c is stored once computed, and waited
        // for (tcgen05.wait::st covers every earlier store) only after quarter
        // c + 1 is computed, so only the last store's latency is exposed.
        const uint64_t sl2x2 = f2(sl2, sl2), negm2 = f2(-m_i, -m_i);
        uint64_t ps2[4] = {0ull, 0ull, 0ull, 0ull};  // +0.f pairs
        uint32_t pk[2][16];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
#pragma unroll
          for (int x = 0; x < 16; ++x) {
            const int col = c * 32 + 2 * x;
            const uint64_t a2 = ffma2(f2(s[col], s[col + 1]), sl2x2, negm2);
            uint64_t e2;
            if (x % 8 < kPolyOf8) {
              e2 = ex2_poly2(a2);
            } else {
              float a0, a1;
              f2split(a2, a0, a1);
              e2 = f2(ex2(a0), ex2(a1));
            }
            ps2[x & 3] = fadd2(ps2[x & 3], e2);
            float e0, e1;
            f2split(e2, e0, e1);
            pk[c & 1][x] = pack_bf16x2(e0, e1);
          }
          if (c > 0) {
            // quarter c - 1 is in TMEM: its PV may start
            tmem_wait_st();
            fence_before_sync();
            mbar_arrive(&sh.p_q[hh][c - 1]);
            if (c == 2) MOBA_TRACE(52, j);
          }
          tmem_st16(tS + c * 16, pk[c & 1]);
        }
        MOBA_TRACE(58, j);
        __syncwarp();
        if (lane == 0) atomicAdd(const_cast<int*>(&exp_cnt[hh]), 1);
        tmem_wait_st();
        {
          const uint64_t q2 = fadd2(fadd2(ps2[0], ps2[1]), fadd2(ps2[2], ps2[3]));
          float q0, q1;
          f2split(q2, q0, q1);
          l_i += q0 + q1;
        }
        fence_before_sync();
        mbar_arrive(&sh.p_q[hh][3]);
        MOBA_TRACE(53, j);
      }
      if (!ok) break;
      // ---- epilogue: wait for the half's last PV, normalise, write
      const float inv_l = 1.f / l_i;
      const float lse = (m_i + log2f(l_i)) * 0.6931471805599453f;
      // CUR: the merge weights need only the lse values, not the last PV:
      // they are read (and the weights formed) while the PV runs
      constexpr int kPreLse = 4;
      float wpre[kPreLse];
      float m_all = -INFINITY, L_all = 0.f, w_own = 0.f;
      if (MODE == CUR && R.valid) {
        const int64_t nr = (int64_t)a.ch.nq * dm.topk;
        float lj[kPreLse];
#pragma unroll
        for (int j = 0; j < kPreLse; ++j)
          lj[j] = j < R.nhist ? a.part_lse[part_lse_at(part_row(R.prow + j, nr))] : -INFINITY;
        m_all = R.own ? lse : -INFINITY;
#pragma unroll
        for (int j = 0; j < kPreLse; ++j) m_all = fmaxf(m_all, lj[j]);
        for (int j = kPreLse; j < R.nhist; ++j)
          m_all = fmaxf(m_all, a.part_lse[part_lse_at(part_row(R.prow + j, nr))]);
        w_own = R.own ? ex2((lse - m_all) * 1.4426950408889634f) : 0.f;
        L_all = w_own;
#pragma unroll
        for (int j = 0; j < kPreLse; ++j) {
          wpre[j] = j < R.nhist ? ex2((lj[j] - m_all) * 1.4426950408889634f) : 0.f;
          L_all += wpre[j];
        }
        for (int j = kPreLse; j < R.nhist; ++j)
          L_all += ex2((a.part_lse[part_lse_at(part_row(R.prow + j, nr))] - m_all) *
                       1.4426950408889634f);
      }
      ok = mbar_wait(&sh.o_full[hh], uc & 1, abort, status);
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      MOBA_TRACE(54, 0);
      fence_after_sync();
      if (MODE == CUR) {
        // Own block done: merge with this row's history partials right here
        // (eq. 7-8 written with lse: w_j = exp(lse_j - m), o = sum_j w_j o_j /
        // sum_j w_j) and write the output; the own result never leaves the
        // SM. Slots 0..slot-1 of the row hold the history partials. Each
        // thread merges its own row; the warp's 32 rows are 32 consecutive
        // tokens of one head, so in the interleaved partial layout every
        // 32-byte piece load of the warp is one contiguous 1 KB access. A
        // row whose own block lost the prefix-mean gate gives its own result
        // weight 0.
        const int slot = R.valid ? R.nhist : 0;
        const int64_t prow0 = R.valid ? R.prow : 0;
        const int64_t orow =
            R.valid && MOBA_CHECK(R.t * dm.Hq + R.h < (int64_t)dm.T * dm.Hq, status)
                ? R.t * dm.Hq + R.h
                : -1;
        float o[D];
        {
          // all four loads in flight, then one wait
          uint32_t r0[32], r1[32], r2[32], r3[32];
          tmem_ld32(tO, r0);
          tmem_ld32(tO + 32, r1);
          tmem_ld32(tO + 64, r2);
          tmem_ld32(tO + 96, r3);
          tmem_wait_ld();
#pragma unroll
          for (int x = 0; x < 32; ++x) {
            o[x] = __uint_as_float(r0[x]) * inv_l;
            o[32 + x] = __uint_as_float(r1[x]) * inv_l;
            o[64 + x] = __uint_as_float(r2[x]) * inv_l;
            o[96 + x] = __uint_as_float(r3[x]) * inv_l;
          }
        }
        // O[h] is in registers: the next unit's PV may overwrite it
        fence_before_sync();
        mbar_arrive(&sh.o_free[hh]);
        if (orow >= 0) {
          const int64_t nr = (int64_t)a.ch.nq * dm.topk;
          const float m = m_all, L = L_all;
#pragma unroll
          for (int x = 0; x < D; ++x) o[x] *= w_own;
          for (int j = 0; j < slot; ++j) {
            const PartRow pj = part_row(prow0 + j, nr);
            float wj = 0.f;
#pragma unroll
            for (int q = 0; q < kPreLse; ++q)
              if (q == j) wj = wpre[q];
            if (j >= kPreLse) wj = ex2((a.part_lse[part_lse_at(pj)] - m) * 1.4426950408889634f);
#pragma unroll
            for (int x16 = 0; x16 < D / 16; ++x16) {
              uint32_t v[8];  // 16 bf16 values
              ld_global_v8_b32(part_piece<__nv_bfloat16>(a.part_o, pj, D, x16), v);
#pragma unroll
              for (int u = 0; u < 8; ++u) {
                o[16 * x16 + 2 * u] = fmaf(wj, __uint_as_float(v[u] << 16), o[16 * x16 + 2 * u]);
                o[16 * x16 + 2 * u + 1] =
                    fmaf(wj, __uint_as_float(v[u] & 0xffff0000u), o[16 * x16 + 2 * u + 1]);
              }
            }
          }
          const float inv = 1.f / L;
#pragma unroll
          for (int x = 0; x < D; ++x) o[x] *= inv;
          if (a.lse_out) a.lse_out[orow] = m + logf(L);
        }
        // the bf16 row leaves straight from registers in 32-byte pieces
        if (orow >= 0) {
#pragma unroll
          for (int x16 = 0; x16 < D / 16; ++x16) {
            uint32_t w[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) w[u] = pack_bf16x2(o[16 * x16 + 2 * u], o[16 * x16 + 2 * u + 1]);
            st_global_v8_b32(a.out + orow * D + 16 * x16, w);
          }
        }
      } else {
        // Each thread writes its own row in 32-byte pieces (a warp store
        // covers 32 rows; every 32-byte sector is written whole).
        const int64_t orow =
            R.valid && MOBA_CHECK(MODE == DENSE ? R.t * dm.Hq + R.h < (int64_t)dm.T * dm.Hq
                                                : R.prow < (int64_t)dm.T * a.ch.nq * dm.topk,
                                  status)
                ? (MODE == DENSE ? R.t * dm.Hq + R.h : R.prow)
                : -1;
        const PartRow prt = part_row(R.valid && MODE != DENSE ? R.prow : 0,
                                     (int64_t)a.ch.nq * dm.topk);
        uint32_t ro[D];
        {
          // all four loads in flight, then one wait; O[h] is then in
          // registers and the next unit's PV may overwrite it
          uint32_t r0[32], r1[32], r2[32], r3[32];
          tmem_ld32(tO, r0);
          tmem_ld32(tO + 32, r1);
          tmem_ld32(tO + 64, r2);
          tmem_ld32(tO + 96, r3);
          tmem_wait_ld();
          fence_before_sync();
          mbar_arrive(&sh.o_free[hh]);
#pragma unroll
          for (int x = 0; x < 32; ++x) {
            ro[x] = r0[x];
            ro[32 + x] = r1[x];
            ro[64 + x] = r2[x];
            ro[96 + x] = r3[x];
          }
        }
        if (orow >= 0) {
          if (MODE == DENSE) {
#pragma unroll
            for (int x16 = 0; x16 < D / 16; ++x16) {
              uint32_t w[8];
#pragma unroll
              for (int u = 0; u < 8; ++u)
                w[u] = pack_bf16x2(__uint_as_float(ro[16 * x16 + 2 * u]) * inv_l,
                                   __uint_as_float(ro[16 * x16 + 2 * u + 1]) * inv_l);
              st_global_v8_b32(a.out + orow * D + 16 * x16, w);
            }
          } else {
            // the row's 32-byte pieces of 16 bf16 (the interleaved partial layout)
#pragma unroll
            for (int x16 = 0; x16 < D / 16; ++x16) {
              uint32_t w[8];
#pragma unroll
              for (int u = 0; u < 8; ++u)
                w[u] = pack_bf16x2(__uint_as_float(ro[16 * x16 + 2 * u]) * inv_l,
                                   __uint_as_float(ro[16 * x16 + 2 * u + 1]) * inv_l);
              st_global_v8_b32(part_piece<__nv_bfloat16>(a.part_o, prt, D, x16), w);
            }
          }
        }
        if (orow >= 0) {
          if (MODE == DENSE) {
            if (a.lse_out) a.lse_out[R.t * dm.Hq + R.h] = lse;
          } else {
            a.part_lse[part_lse_at(prt)] = lse;
          }
        }
      }
      MOBA_TRACE(55, 0);
      ++uc;
    }
  }
  MOBA_TRACE_END();

  fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    fence_after_sync();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ---- host side -----------------------------------------------------------------
template <int MODE>
cudaError_t launch(int64_t tiles, const Args& args, const void* k, const void* v,
                   cudaStream_t st) {
  if (tiles <= 0) return cudaSuccess;
  CUtensorMap mk, mv;
  cudaError_t e;
  if ((e = make_head_map(&mk, k, args.dm.T, args.dm.Hkv, TN))) return e;
  if ((e = make_head_map(&mv, v, args.dm.T, args.dm.Hkv, TN))) return e;
  // Once per device: allow the shared memory, and check that the launch
  // allocates the registers the setmaxnreg split needs (setmaxnreg moves
  // registers between the warp groups inside the block's allocation).
  static std::mutex mu;
  static int ready[kMaxDevices] = {};  // 0 unknown, 1 ready, -1 unusable
  int dev = 0;
  if ((e = cudaGetDevice(&dev))) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (ready[dev] == 0) {
      if ((e = cudaFuncSetAttribute(attn_tc_kernel<MODE>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes)))
        return e;
      cudaFuncAttributes fa;
      if ((e = cudaFuncGetAttributes(&fa, attn_tc_kernel<MODE>))) return e;
      ready[dev] = fa.numRegs * kThreads >= 128 * kRegsOther + 256 * kRegsSoftmax ? 1 : -1;
    }
  }
  if (ready[dev] < 0) return cudaErrorInvalidConfiguration;
  const int64_t grid = tiles < sm_count() ? tiles : sm_count();
  attn_tc_kernel<MODE><<<(unsigned)grid, kThreads, kSmemBytes, st>>>(mk, mv, args);
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

// Rows of one HIST work unit in the tile table: two query halves.
int tc_tile_m() { return 2 * TM; }

cudaError_t launch_history_tc(const Dims& dm, const Chunk& ch, const void* q, const void* k,
                              const void* v, const int32_t* cu, const Regroup& rg,
                              const Partials& pt, int* status, cudaStream_t st) {
  Args a = base_args(dm, ch, q, cu, status);
  a.list_off = rg.list_off;
  a.pairs = rg.pairs;
  a.tiles = rg.tiles;
  a.tile_count = rg.tile_off + ch.n_lists;
  a.part_o = pt.o;
  a.part_lse = pt.lse;
  return launch<HIST>(rg.max_tiles, a, k, v, st);
}

cudaError_t launch_current_tc(const Dims& dm, const Chunk& ch, const void* q, const void* k,
                              const void* v, const int32_t* cu, const int32_t* idx,
                              const Partials& pt, void* out, float* lse, int* status,
                              cudaStream_t st) {
  if (dm.batch == 0 || dm.max_seqlen == 0) return cudaSuccess;
  Args a = base_args(dm, ch, q, cu, status);
  a.idx = idx;
  a.part_o = pt.o;
  a.part_lse = pt.lse;
  a.out = static_cast<__nv_bfloat16*>(out);
  a.lse_out = lse;
  const int64_t tiles = (int64_t)((dm.B / TM + 1) / 2) * dm.nb * dm.batch * ch.nq;
  a.n_tiles = (int)tiles;
  return launch<CUR>(tiles, a, k, v, st);
}

cudaError_t launch_dense_tc(const Dims& dm, const void* q, const void* k, const void* v,
                            const int32_t* cu, void* out, float* lse, int* status,
                            cudaStream_t st) {
  if (dm.batch == 0 || dm.max_seqlen == 0) return cudaSuccess;
  Chunk ch{0, dm.Hkv, 0, dm.Hq, 0, TM};
  Args a = base_args(dm, ch, q, cu, status);
  a.out = static_cast<__nv_bfloat16*>(out);
  a.lse_out = lse;
  const int64_t tiles = (int64_t)(((dm.max_seqlen + TM - 1) / TM + 1) / 2) * dm.batch * dm.Hq;
  a.n_tiles = (int)tiles;
  return launch<DENSE>(tiles, a, k, v, st);
}

}  // namespace moba
