// Shared device helpers and the launch interface between the C ABI (api.cu)
// and the kernels. Nothing here is visible outside libmoba.so.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace moba {

constexpr int kBF16 = 0;
constexpr int kF32 = 1;

// Device status codes (same values as moba_status).
constexpr int kStInvalidArg = -1;
constexpr int kStTimeout = -4;
constexpr int kStBadIndices = -6;
constexpr int kStCheck = -7;

// Sizes of one call, validated on the host.
struct Dims {
  int batch;       // sequences
  int T;           // total tokens
  int max_seqlen;  // bound on every sequence length
  int Hq, Hkv;     // heads
  int d;           // head dim
  int B;           // block size
  int topk;        // k
  int nb;          // blocks reserved per sequence = ceil(max_seqlen / B)
  int dtype;       // kBF16 / kF32
  int shared;      // 1: a kv head's query heads share the blocks of their mean score
  int prefix;      // 1: the own block is scored by its prefix mean instead of forced
  int kv_hm;       // 1: k and v are head-major [Hkv][T][d] (decode caches), else [T][Hkv][d]
};

// Element offset of row t of kv head g in k or v.
__host__ __device__ __forceinline__ int64_t kv_row(const Dims& dm, int64_t t, int g) {
  return (dm.kv_hm ? (int64_t)g * dm.T + t : t * dm.Hkv + g) * dm.d;
}

// History slots an index row can hold: k - 1 beside the forced own block,
// all k when the own block competes for its slot.
__host__ __device__ inline int hist_slots(const Dims& dm) { return dm.prefix ? dm.topk : dm.topk - 1; }

// The prefix-mean own-block scores are built from per-chunk key sums: a
// block is split into chunks of kOwnChunkRows rows.
constexpr int kOwnChunkRows = 32;
__host__ __device__ inline int own_chunks_per_block(const Dims& dm) {
  return (dm.B + kOwnChunkRows - 1) / kOwnChunkRows;
}

// Whether query row `row` (k entries) reads its own block c: always when the
// own block is forced, else when the row names it.
__device__ __forceinline__ bool reads_own(const Dims& dm, const int32_t* row, int c) {
  if (!dm.prefix) return true;
  bool on = false;
  for (int r = 0; r < dm.topk; ++r) on |= row[r] == c;
  return on;
}

// Work of one pass over a group of kv heads [g0, g0 + ng): its q heads are
// [g0 * grp, (g0 + ng) * grp). Partial results are indexed by
// prow = ((t * nq) + h_local) * topk + slot, nq = ng * grp.
struct Chunk {
  int g0, ng;      // kv heads of this pass
  int h0, nq;      // q heads of this pass
  int n_lists;     // batch * ng * nb regroup lists
  int tile_m;      // query rows per history tile
};

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T>
__device__ __forceinline__ T from_f32(float x);
template <>
__device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

// 16-byte vector of elements widened to fp32.
template <typename T>
struct Vec16;
template <>
struct Vec16<float> {
  static constexpr int N = 4;
  __device__ __forceinline__ static void load(const float* p, float* out) {
    const float4 r = __ldg(reinterpret_cast<const float4*>(p));
    out[0] = r.x; out[1] = r.y; out[2] = r.z; out[3] = r.w;
  }
};
template <>
struct Vec16<__nv_bfloat16> {
  static constexpr int N = 8;
  __device__ __forceinline__ static void load(const __nv_bfloat16* p, float* out) {
    const uint4 r = __ldg(reinterpret_cast<const uint4*>(p));
    const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      out[2 * i] = __uint_as_float(w[i] << 16);
      out[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
  }
};

// First error wins.
__device__ __forceinline__ void set_status(int* status, int code) {
  if (status) atomicCAS(status, 0, code);
}

// Checked build (MOBA_CHECKED defined: libmoba_checked.so): index and
// bounds checks at the kernels' computed global accesses. A failed check
// records kStCheck in the status word and the access is skipped; nothing
// traps. In the ordinary build MOBA_CHECK(cond, status) is the constant
// true and costs nothing.
#ifdef MOBA_CHECKED
__device__ __forceinline__ bool check_or_flag(bool ok, int* status) {
  if (!ok) set_status(status, kStCheck);
  return ok;
}
#define MOBA_CHECK(cond, status) (::moba::check_or_flag((cond), (status)))
#else
#define MOBA_CHECK(cond, status) (true)
#endif

// Sequence bounds with a device-side check against max_seqlen.
__device__ __forceinline__ bool seq_bounds(const Dims& dm, const int32_t* cu, int b, int64_t& start,
                                           int& len, int* status) {
  start = cu[b];
  len = cu[b + 1] - cu[b];
  if (len < 0 || len > dm.max_seqlen) {
    set_status(status, kStInvalidArg);
    return false;
  }
  return true;
}

}  // namespace moba

// ---- launchers (host), one per kernel family -------------------------------
namespace moba {

cudaError_t launch_meanpool(const Dims& dm, const void* k, const int32_t* cu, float* kbar,
                            int* status, cudaStream_t st);
// Block means of only the blocks holding each sequence's last
// cu_new[b+1] - cu_new[b] positions (max_new: the largest such count).
cudaError_t launch_meanpool_update(const Dims& dm, const void* k, const int32_t* cu,
                                   const int32_t* cu_new, int max_new, float* kbar, int* status,
                                   cudaStream_t st);
// Decode step (decode.cu): gate into idx, split-K attention into partials
// [decode_partial_rows] x (d + 1) merged by the last split of each row into
// out / lse; arrivals: n_queries * Hq ints of scratch (zeroed by the gate).
size_t decode_partial_rows(const Dims& dm, int n_queries);
cudaError_t launch_decode(const Dims& dm, int n_queries, const void* q, const void* k,
                          const void* v, const int32_t* cu, const int32_t* cu_q, const float* kbar,
                          int32_t* idx, float* part_o, float* part_lse, int* arrivals, void* out,
                          float* lse, int* status, cudaStream_t st);
// Tensor-core gate (bf16, d = 128, at most 256 blocks per sequence).
bool gate_tc_supported(const Dims& dm);
// Its sorting-network form for 5 to 15 history slots and the forced own
// block (gate_net.cu); launch_gate_tc hands such calls to it.
bool gate_net_supported(const Dims& dm);
cudaError_t launch_gate_net(const Dims& dm, const void* q, const float* kbar, const int32_t* cu,
                            int32_t* idx, int* status, cudaStream_t st);
cudaError_t launch_gate_tc(const Dims& dm, const void* q, const float* kbar, const float* own,
                           const int32_t* cu, int32_t* idx, int* status, cudaStream_t st);
// own: with dm.prefix, the own-block scores [T][Hq] (launch_own_score); else unused.
cudaError_t launch_gate(const Dims& dm, const void* q, const float* kbar, const float* own,
                        const int32_t* cu, int32_t* idx, int* status, cudaStream_t st);
// Own-block scores by prefix mean: own[t][h] = q_{t,h} . mean(k_{cB..p}) (fp32).
// csum: scratch for the chunk key sums, batch * nb * own_chunks_per_block * Hkv * d floats.
cudaError_t launch_own_score(const Dims& dm, const void* q, const void* k, const int32_t* cu,
                             float* own, float* csum, int* status, cudaStream_t st);

// Regrouping of (query, head, slot) by the history block it chose.
struct Regroup {
  int32_t* counts;     // [n_lists]
  int32_t* cursor;     // [n_lists]
  int32_t* list_off;   // [n_lists + 1]
  int32_t* tile_off;   // [n_lists + 1]; tile_off[n_lists] = number of tiles
  int32_t* pairs;      // [max pairs] partial-row ids grouped by list
  int4* tiles;         // [max tiles] (list, first row in list, list size, list's first entry):
                       // a work unit's description in one 16-byte load
  int64_t max_tiles;
};
cudaError_t launch_regroup(const Dims& dm, const Chunk& ch, const int32_t* idx, const int32_t* cu,
                           const Regroup& rg, int* status, cudaStream_t st);

// Partial attention results of one pass.
struct Partials {
  void* o;     // part_rows(T, nq * topk) rows of d values in the input dtype (layout below)
  float* lse;  // part_rows(T, nq * topk)
};

// A partial result o_j = u_j / l_j (normalised, so |o_j| <= max |v|) is
// stored in the input dtype -- bf16 for bf16 inputs, as merge-state kernels
// commonly keep it -- and merged in fp32; its lse stays fp32.
//
// Partial results of a pass are stored interleaved over 32 consecutive
// tokens. For partial row prow = (t * nq + h_local) * k + slot (nr = nq * k
// rows per token) the 32-byte piece c of the row sits at piece
// (tile * npc + c) * 32 + t % 32 (npc = the row's 32-byte pieces) with
// tile = (t / 32) * nr + prow % nr, and its lse at tile * 32 + t % 32. A
// warp holding 32 consecutive tokens of one head -- the own-block kernel's
// merge -- then reads each piece of its rows' partials as one contiguous
// 1 KB access instead of 32 scattered ones.
struct PartRow {
  int64_t tile;
  int lane;
};
__host__ __device__ inline PartRow part_row(int64_t prow, int64_t nr) {
  const int64_t t = prow / nr;
  return {(t >> 5) * nr + (prow - t * nr), (int)(t & 31)};
}
template <typename P>
__host__ __device__ inline P* part_piece(void* o, const PartRow& r, int d, int c) {
  const int npc = d * (int)sizeof(P) / 32;
  return reinterpret_cast<P*>(static_cast<char*>(o) + ((r.tile * npc + c) * 32 + r.lane) * 32);
}
template <typename P>
__host__ __device__ inline const P* part_piece(const void* o, const PartRow& r, int d, int c) {
  const int npc = d * (int)sizeof(P) / 32;
  return reinterpret_cast<const P*>(static_cast<const char*>(o) + ((r.tile * npc + c) * 32 + r.lane) * 32);
}
__host__ __device__ inline int64_t part_lse_at(const PartRow& r) { return r.tile * 32 + r.lane; }
// Storage rows of a pass: T rounded up to whole 32-token tiles.
inline size_t part_rows(int64_t T, int64_t nr) { return (size_t)((T + 31) / 32) * 32 * (size_t)nr; }

// Portable SIMT kernels (fp32 or bf16 inputs, any block size).
cudaError_t launch_history_simt(const Dims& dm, const Chunk& ch, const void* q, const void* k,
                                const void* v, const int32_t* cu, const Regroup& rg,
                                const Partials& pt, cudaStream_t st);
cudaError_t launch_current_simt(const Dims& dm, const Chunk& ch, const void* q, const void* k,
                                const void* v, const int32_t* cu, const int32_t* idx,
                                const Partials& pt, cudaStream_t st);
cudaError_t launch_dense_simt(const Dims& dm, const void* q, const void* k, const void* v,
                              const int32_t* cu, void* out, float* lse, cudaStream_t st);
// Backward (bwd.cu): dq, dk, dv (fp32, zeroed by the caller) of the whole
// batch; `ch` covers every head in one pass; Dsum [T * Hq] is scratch.
cudaError_t launch_bwd_dot(const Dims& dm, const void* out, const void* dout, float* Dsum,
                           cudaStream_t st);
cudaError_t launch_backward(const Dims& dm, const Chunk& ch, const void* q, const void* k,
                            const void* v, const void* dout, const float* lse, const float* Dsum,
                            const int32_t* cu, const int32_t* idx, const Regroup& rg, float* dq,
                            float* dk, float* dv, int* status, cudaStream_t st);
// Tensor-core backward (bf16, d = 128, B % 128 == 0).
bool bwd_tc_supported(const Dims& dm);
cudaError_t launch_backward_tc(const Dims& dm, const Chunk& ch, const void* q, const void* k,
                               const void* v, const void* dout, const float* lse,
                               const float* Dsum, const int32_t* cu, const int32_t* idx,
                               const Regroup& rg, float* dq, float* dk, float* dv, int* status,
                               cudaStream_t st);
constexpr int kSimtTileM = 32;

cudaError_t launch_merge(const Dims& dm, const Chunk& ch, const int32_t* idx, const int32_t* cu,
                         const Partials& pt, void* out, float* lse, cudaStream_t st);

}  // namespace moba
