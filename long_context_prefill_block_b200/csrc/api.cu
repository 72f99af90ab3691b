// C ABI of libmoba.so (declared in include/moba.h): argument validation,
// workspace layout and the launch sequence of the MoBA prefill forward pass
// (PaperTrace "2.1.3 MoBA", section 3.1): mean-pool -> gate/top-k ->
// regroup by key block -> history attention + own-block attention -> merge.
#include <cstdint>
#include <cstring>

#include "host_api.cuh"

#ifdef MOBA_TRACE
#include <mutex>
#include <vector>

#include "moba_trace.h"
#include "trace.cuh"
#endif

namespace moba {
// Per-device status word; kernels get its address, never the symbol.
__device__ int g_status;

cudaError_t launch_history_tc(const Dims& dm, const Chunk& ch, const void* q, const void* k,
                              const void* v, const int32_t* cu, const Regroup& rg,
                              const Partials& pt, int* status, cudaStream_t st);
cudaError_t launch_current_tc(const Dims& dm, const Chunk& ch, const void* q, const void* k,
                              const void* v, const int32_t* cu, const int32_t* idx,
                              const Partials& pt, void* out, float* lse, int* status,
                              cudaStream_t st);
cudaError_t launch_dense_tc(const Dims& dm, const void* q, const void* k, const void* v,
                            const int32_t* cu, void* out, float* lse, int* status,
                            cudaStream_t st);
bool tc_supported(const Dims& dm);
cudaError_t launch_wait_selftest(int* status, int* done, cudaStream_t st);
int tc_tile_m();

moba_status validate(const moba_params* p, Dims& dm) {
  if (!p) return MOBA_ERR_INVALID_ARG;
  if (p->batch < 0 || p->total_tokens < 0 || p->max_seqlen < 0 || p->num_q_heads <= 0 ||
      p->num_kv_heads <= 0 || p->num_q_heads % p->num_kv_heads != 0 || p->block_size <= 0 ||
      p->topk <= 0)
    return MOBA_ERR_INVALID_ARG;
  if (p->routing != 0 && p->routing != 1) return MOBA_ERR_INVALID_ARG;
  if (p->own_block != 0 && p->own_block != 1) return MOBA_ERR_INVALID_ARG;
  if (p->kv_layout != 0 && p->kv_layout != 1) return MOBA_ERR_INVALID_ARG;
  if (p->dtype != MOBA_BF16 && p->dtype != MOBA_F32) return MOBA_ERR_UNSUPPORTED;
  if (p->head_dim != 64 && p->head_dim != 128) return MOBA_ERR_UNSUPPORTED;
  if (p->topk > 32) return MOBA_ERR_UNSUPPORTED;
  // int32 row ids: T * Hq * k must fit.
  if ((int64_t)p->total_tokens * p->num_q_heads * p->topk >= (int64_t(1) << 31))
    return MOBA_ERR_UNSUPPORTED;
  dm.batch = p->batch;
  dm.T = p->total_tokens;
  dm.max_seqlen = p->max_seqlen;
  dm.Hq = p->num_q_heads;
  dm.Hkv = p->num_kv_heads;
  dm.d = p->head_dim;
  dm.B = p->block_size;
  dm.topk = p->topk;
  dm.nb = (int)(((int64_t)p->max_seqlen + p->block_size - 1) / p->block_size);
  dm.dtype = p->dtype == MOBA_BF16 ? kBF16 : kF32;
  dm.shared = p->routing;
  dm.prefix = p->own_block;
  dm.kv_hm = p->kv_layout;
  return MOBA_OK;
}

int* status_word() {
  void* ptr = nullptr;
  if (cudaGetSymbolAddress(&ptr, g_status) != cudaSuccess) return nullptr;
  return static_cast<int*>(ptr);
}

}  // namespace moba

using namespace moba;

namespace {

// Partial results are kept for at most this many bytes per pass; larger
// problems are processed one group of kv heads at a time.
constexpr size_t kPartialCap = size_t(32) << 30;

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

bool aligned32(const void* x) { return (reinterpret_cast<uintptr_t>(x) & 31) == 0; }

struct Layout {
  size_t kbar, own, idx, counts, cursor, list_off, tile_off, pairs, tiles, part_o, part_lse, total;
  int ng;             // kv heads per pass
  int64_t max_tiles;  // tile-table capacity per pass
};

// Own-block scores of the prefix-mean gate, when the gate runs: fp32 [T][Hq],
// then the per-chunk key sums they are built from.
size_t own_scores_bytes(const Dims& dm) { return (sizeof(float) * (size_t)dm.T * dm.Hq + 255) & ~size_t(255); }
size_t own_score_bytes(const Dims& dm, bool gate_runs) {
  if (!dm.prefix || !gate_runs) return 0;
  return own_scores_bytes(dm) + sizeof(float) * (size_t)dm.batch * dm.nb *
                                    own_chunks_per_block(dm) * dm.Hkv * dm.d;
}
float* own_chunk_sums(float* own, const Dims& dm) {
  return reinterpret_cast<float*>(reinterpret_cast<char*>(own) + own_scores_bytes(dm));
}

// Runs the gate: block means, the own-block scores of the prefix-mean
// variant, then gate/top-k.
cudaError_t run_gate(const Dims& dm, const void* q, const void* k, const int32_t* cu, float* kbar,
                     float* own, int32_t* idx, int* status, cudaStream_t st) {
  cudaError_t e = launch_meanpool(dm, k, cu, kbar, status, st);
  if (e == cudaSuccess && dm.prefix)
    e = launch_own_score(dm, q, k, cu, own, own_chunk_sums(own, dm), status, st);
  if (e == cudaSuccess) e = launch_gate(dm, q, kbar, own, cu, idx, status, st);
  return e;
}

// Workspace plan. `own_idx` reserves room for the index rows (moba_forward).
Layout plan(const Dims& dm, bool own_idx) {
  Layout L{};
  const int grp = dm.Hq / dm.Hkv;
  const size_t per_kv = (size_t)dm.T * grp * dm.topk * (dm.d * 4 + 4);
  size_t ng = per_kv ? kPartialCap / per_kv : dm.Hkv;
  if (ng < 1) ng = 1;
  if (ng > (size_t)dm.Hkv) ng = dm.Hkv;
  L.ng = (int)ng;
  const int64_t n_lists = (int64_t)dm.batch * L.ng * dm.nb;
  const int64_t max_pairs = (int64_t)dm.T * L.ng * grp * hist_slots(dm);
  const int tile_m = kSimtTileM < tc_tile_m() ? kSimtTileM : tc_tile_m();
  L.max_tiles = (max_pairs + tile_m - 1) / tile_m + n_lists;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = align256(off + bytes);
    return at;
  };
  L.kbar = take(sizeof(float) * (size_t)dm.batch * dm.nb * dm.Hkv * dm.d);
  L.own = take(own_score_bytes(dm, own_idx));
  L.idx = take(own_idx ? sizeof(int32_t) * (size_t)dm.T * dm.Hq * dm.topk : 0);
  L.counts = take(sizeof(int32_t) * n_lists);
  L.cursor = take(sizeof(int32_t) * n_lists);
  L.list_off = take(sizeof(int32_t) * (n_lists + 1));
  L.tile_off = take(sizeof(int32_t) * (n_lists + 1));
  L.pairs = take(sizeof(int32_t) * max_pairs);
  L.tiles = take(sizeof(int4) * L.max_tiles);
  const size_t prows = part_rows(dm.T, (int64_t)L.ng * grp * dm.topk);
  L.part_o = take((dm.dtype == kBF16 ? 2 : 4) * prows * dm.d);
  L.part_lse = take(sizeof(float) * prows);
  L.total = off;
  return L;
}

moba_status cuda_status(cudaError_t e) { return e == cudaSuccess ? MOBA_OK : MOBA_ERR_CUDA; }

#define MOBA_TRY(x)                                  \
  do {                                               \
    const cudaError_t e_ = (x);                      \
    if (e_ != cudaSuccess) return MOBA_ERR_CUDA;     \
  } while (0)

int num_passes(const Dims& dm, const Layout& L) { return (dm.Hkv + L.ng - 1) / L.ng; }

// Shared body of moba_forward, moba_forward_with_indices and
// moba_forward_staged. With `events`, events[0] is recorded before the first
// launch, events[1] after the mean-pool, events[2] after the gate, and for
// pass j events[3+4j .. 6+4j] after regroup, history attention, own-block
// attention and merge.
moba_status forward_impl(const moba_params* p, const void* q, const void* k, const void* v,
                         const int32_t* cu, const int32_t* idx_in, void* out, float* lse,
                         void* ws, size_t ws_bytes, void* stream, void* const* events = nullptr,
                         int n_events = 0) {
  Dims dm;
  moba_status s = validate(p, dm);
  if (s != MOBA_OK) return s;
  if (dm.kv_hm) return MOBA_ERR_UNSUPPORTED;  // head-major k / v: decode caches only
  if (dm.T == 0 || dm.batch == 0) return MOBA_OK;
  if (!q || !k || !v || !cu || !out) return MOBA_ERR_INVALID_ARG;
  if (!aligned32(q) || !aligned32(k) || !aligned32(v) || !aligned32(out) ||
      (lse && !aligned32(lse)))
    return MOBA_ERR_INVALID_ARG;
  const Layout L = plan(dm, idx_in == nullptr);
  if (!ws || ws_bytes < L.total || !aligned32(ws)) return MOBA_ERR_WORKSPACE;
  if (events && n_events < 3 + 4 * num_passes(dm, L)) return MOBA_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int ev = 0;
  auto mark = [&]() -> cudaError_t {
    if (!events) return cudaSuccess;
    return cudaEventRecord(static_cast<cudaEvent_t>(events[ev++]), st);
  };
  MOBA_TRY(mark());
  int* status = status_word();
  if (!status) return MOBA_ERR_CUDA;
  char* base = static_cast<char*>(ws);
  float* kbar = reinterpret_cast<float*>(base + L.kbar);
  const int32_t* idx = idx_in;
  if (!idx_in) {
    int32_t* own = reinterpret_cast<int32_t*>(base + L.idx);
    MOBA_TRY(launch_meanpool(dm, k, cu, kbar, status, st));
    MOBA_TRY(mark());
    float* own_score = reinterpret_cast<float*>(base + L.own);
    if (dm.prefix)
      MOBA_TRY(launch_own_score(dm, q, k, cu, own_score, own_chunk_sums(own_score, dm), status, st));
    MOBA_TRY(launch_gate(dm, q, kbar, own_score, cu, own, status, st));
    MOBA_TRY(mark());
    idx = own;
  } else {
    MOBA_TRY(mark());
    MOBA_TRY(mark());
  }
  const bool tc = tc_supported(dm);
  const int grp = dm.Hq / dm.Hkv;
  Regroup rg;
  rg.counts = reinterpret_cast<int32_t*>(base + L.counts);
  rg.cursor = reinterpret_cast<int32_t*>(base + L.cursor);
  rg.list_off = reinterpret_cast<int32_t*>(base + L.list_off);
  rg.tile_off = reinterpret_cast<int32_t*>(base + L.tile_off);
  rg.pairs = reinterpret_cast<int32_t*>(base + L.pairs);
  rg.tiles = reinterpret_cast<int4*>(base + L.tiles);
  Partials pt{base + L.part_o, reinterpret_cast<float*>(base + L.part_lse)};
  for (int g0 = 0; g0 < dm.Hkv; g0 += L.ng) {
    Chunk ch;
    ch.g0 = g0;
    ch.ng = dm.Hkv - g0 < L.ng ? dm.Hkv - g0 : L.ng;
    ch.h0 = g0 * grp;
    ch.nq = ch.ng * grp;
    ch.n_lists = dm.batch * ch.ng * dm.nb;
    ch.tile_m = tc ? tc_tile_m() : kSimtTileM;
    const int64_t pairs = (int64_t)dm.T * ch.nq * hist_slots(dm);
    rg.max_tiles = (pairs + ch.tile_m - 1) / ch.tile_m + ch.n_lists;
    MOBA_TRY(launch_regroup(dm, ch, idx, cu, rg, status, st));
    MOBA_TRY(mark());
    if (tc) {
      // the own-block kernel merges the partials in its epilogue
      MOBA_TRY(launch_history_tc(dm, ch, q, k, v, cu, rg, pt, status, st));
      MOBA_TRY(mark());
      MOBA_TRY(launch_current_tc(dm, ch, q, k, v, cu, idx, pt, out, lse, status, st));
      MOBA_TRY(mark());
    } else {
      MOBA_TRY(launch_history_simt(dm, ch, q, k, v, cu, rg, pt, st));
      MOBA_TRY(mark());
      MOBA_TRY(launch_current_simt(dm, ch, q, k, v, cu, idx, pt, st));
      MOBA_TRY(mark());
      MOBA_TRY(launch_merge(dm, ch, idx, cu, pt, out, lse, st));
    }
    MOBA_TRY(mark());
  }
  return MOBA_OK;
}

// Backward workspace: block means and index rows when the gate runs again,
// the regroup lists of every kv head (one pass), and D = dO . O per row.
struct BwdLayout {
  size_t kbar, own, idx, counts, cursor, list_off, tile_off, pairs, tiles, dsum, total;
  int64_t max_tiles;
};

BwdLayout plan_bwd(const Dims& dm, bool own_idx) {
  BwdLayout L{};
  const int64_t n_lists = (int64_t)dm.batch * dm.Hkv * dm.nb;
  const int64_t max_pairs = (int64_t)dm.T * dm.Hq * hist_slots(dm);
  L.max_tiles = (max_pairs + kSimtTileM - 1) / kSimtTileM + n_lists;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = align256(off + bytes);
    return at;
  };
  L.kbar = take(own_idx ? sizeof(float) * (size_t)dm.batch * dm.nb * dm.Hkv * dm.d : 0);
  L.own = take(own_score_bytes(dm, own_idx));
  L.idx = take(own_idx ? sizeof(int32_t) * (size_t)dm.T * dm.Hq * dm.topk : 0);
  L.counts = take(sizeof(int32_t) * n_lists);
  L.cursor = take(sizeof(int32_t) * n_lists);
  L.list_off = take(sizeof(int32_t) * (n_lists + 1));
  L.tile_off = take(sizeof(int32_t) * (n_lists + 1));
  L.pairs = take(sizeof(int32_t) * max_pairs);
  L.tiles = take(sizeof(int4) * L.max_tiles);
  L.dsum = take(sizeof(float) * (size_t)dm.T * dm.Hq);
  L.total = off;
  return L;
}

moba_status backward_impl(const moba_params* p, const void* q, const void* k, const void* v,
                          const int32_t* cu, const void* out, const float* lse, const void* dout,
                          const int32_t* idx_in, float* dq, float* dk, float* dv, void* ws,
                          size_t ws_bytes, void* stream) {
  Dims dm;
  moba_status s = validate(p, dm);
  if (s != MOBA_OK) return s;
  if (dm.kv_hm) return MOBA_ERR_UNSUPPORTED;
  if (dm.T == 0 || dm.batch == 0) return MOBA_OK;
  if (!q || !k || !v || !cu || !out || !lse || !dout || !dq || !dk || !dv)
    return MOBA_ERR_INVALID_ARG;
  for (const void* x : {q, k, v, out, dout, static_cast<const void*>(dq),
                        static_cast<const void*>(dk), static_cast<const void*>(dv)})
    if (!aligned32(x)) return MOBA_ERR_INVALID_ARG;
  const BwdLayout L = plan_bwd(dm, idx_in == nullptr);
  if (!ws || ws_bytes < L.total || !aligned32(ws)) return MOBA_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int* status = status_word();
  if (!status) return MOBA_ERR_CUDA;
  char* base = static_cast<char*>(ws);
  MOBA_TRY(cudaMemsetAsync(dq, 0, sizeof(float) * (size_t)dm.T * dm.Hq * dm.d, st));
  MOBA_TRY(cudaMemsetAsync(dk, 0, sizeof(float) * (size_t)dm.T * dm.Hkv * dm.d, st));
  MOBA_TRY(cudaMemsetAsync(dv, 0, sizeof(float) * (size_t)dm.T * dm.Hkv * dm.d, st));
  const int32_t* idx = idx_in;
  if (!idx_in) {
    float* kbar = reinterpret_cast<float*>(base + L.kbar);
    int32_t* own = reinterpret_cast<int32_t*>(base + L.idx);
    MOBA_TRY(run_gate(dm, q, k, cu, kbar, reinterpret_cast<float*>(base + L.own), own, status, st));
    idx = own;
  }
  Regroup rg;
  rg.counts = reinterpret_cast<int32_t*>(base + L.counts);
  rg.cursor = reinterpret_cast<int32_t*>(base + L.cursor);
  rg.list_off = reinterpret_cast<int32_t*>(base + L.list_off);
  rg.tile_off = reinterpret_cast<int32_t*>(base + L.tile_off);
  rg.pairs = reinterpret_cast<int32_t*>(base + L.pairs);
  rg.tiles = reinterpret_cast<int4*>(base + L.tiles);
  rg.max_tiles = L.max_tiles;
  Chunk ch;
  ch.g0 = 0;
  ch.ng = dm.Hkv;
  ch.h0 = 0;
  ch.nq = dm.Hq;
  ch.n_lists = dm.batch * dm.Hkv * dm.nb;
  ch.tile_m = kSimtTileM;
  MOBA_TRY(launch_regroup(dm, ch, idx, cu, rg, status, st));
  float* dsum = reinterpret_cast<float*>(base + L.dsum);
  MOBA_TRY(launch_bwd_dot(dm, out, dout, dsum, st));
  if (bwd_tc_supported(dm))
    MOBA_TRY(launch_backward_tc(dm, ch, q, k, v, dout, lse, dsum, cu, idx, rg, dq, dk, dv, status,
                                st));
  else
    MOBA_TRY(launch_backward(dm, ch, q, k, v, dout, lse, dsum, cu, idx, rg, dq, dk, dv, status, st));
  return MOBA_OK;
}

// Decode workspace: index rows, the split partials (o, then lse), the
// per-row arrival counters.
struct DecLayout {
  size_t idx, part_o, part_lse, arrivals, total;
};

DecLayout plan_decode(const Dims& dm, int n_queries) {
  DecLayout L{};
  const size_t rows = decode_partial_rows(dm, n_queries);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = align256(off + bytes);
    return at;
  };
  L.idx = take(sizeof(int32_t) * (size_t)n_queries * dm.Hq * dm.topk);
  L.part_o = take(sizeof(float) * rows * dm.d);
  L.part_lse = take(sizeof(float) * rows);
  L.arrivals = take(sizeof(int) * (size_t)n_queries * dm.Hq);
  L.total = off;
  return L;
}

}  // namespace

extern "C" {

size_t moba_decode_workspace_size(const moba_params* p, int n_queries) {
  Dims dm;
  if (validate(p, dm) != MOBA_OK || n_queries < 0) return 0;
  return plan_decode(dm, n_queries).total;
}

moba_status moba_decode(const moba_params* p, const void* q, const void* k_cache,
                        const void* v_cache, const int32_t* cu_seqlens, const int32_t* cu_q,
                        int n_queries, const float* kbar, void* out, float* lse, int32_t* idx,
                        void* ws, size_t ws_bytes, void* stream) {
  Dims dm;
  moba_status s = validate(p, dm);
  if (s != MOBA_OK) return s;
  if (n_queries < 0) return MOBA_ERR_INVALID_ARG;
  if (dm.prefix) return MOBA_ERR_UNSUPPORTED;
  if (dm.batch == 0 || n_queries == 0) return MOBA_OK;
  if ((int64_t)n_queries * dm.Hq * dm.topk >= (int64_t(1) << 31)) return MOBA_ERR_UNSUPPORTED;
  if (!q || !k_cache || !v_cache || !cu_seqlens || !cu_q || !kbar || !out)
    return MOBA_ERR_INVALID_ARG;
  if (!aligned32(q) || !aligned32(k_cache) || !aligned32(v_cache) || !aligned32(kbar) ||
      !aligned32(out))
    return MOBA_ERR_INVALID_ARG;
  const DecLayout L = plan_decode(dm, n_queries);
  if (!ws || ws_bytes < L.total || !aligned32(ws)) return MOBA_ERR_WORKSPACE;
  int* status = status_word();
  if (!status) return MOBA_ERR_CUDA;
  char* base = static_cast<char*>(ws);
  int32_t* rows = idx ? idx : reinterpret_cast<int32_t*>(base + L.idx);
  return cuda_status(launch_decode(dm, n_queries, q, k_cache, v_cache, cu_seqlens, cu_q, kbar, rows,
                                   reinterpret_cast<float*>(base + L.part_o),
                                   reinterpret_cast<float*>(base + L.part_lse),
                                   reinterpret_cast<int*>(base + L.arrivals), out, lse, status,
                                   static_cast<cudaStream_t>(stream)));
}

moba_status moba_meanpool_update(const moba_params* p, const void* k_cache,
                                 const int32_t* cu_seqlens, const int32_t* cu_new, int max_new,
                                 float* kbar, void* stream) {
  Dims dm;
  moba_status s = validate(p, dm);
  if (s != MOBA_OK) return s;
  if (max_new < 0) return MOBA_ERR_INVALID_ARG;
  if (dm.batch == 0 || dm.nb == 0 || max_new == 0) return MOBA_OK;
  if (!k_cache || !cu_seqlens || !cu_new || !kbar || !aligned32(k_cache) || !aligned32(kbar))
    return MOBA_ERR_INVALID_ARG;
  int* status = status_word();
  if (!status) return MOBA_ERR_CUDA;
  return cuda_status(launch_meanpool_update(dm, k_cache, cu_seqlens, cu_new, max_new, kbar, status,
                                            static_cast<cudaStream_t>(stream)));
}

int moba_num_blocks(const moba_params* p) {
  Dims dm;
  if (validate(p, dm) != MOBA_OK) return 0;
  return dm.nb;
}

size_t moba_backward_workspace_size(const moba_params* p, int have_indices) {
  Dims dm;
  if (validate(p, dm) != MOBA_OK) return 0;
  return plan_bwd(dm, have_indices == 0).total;
}

moba_status moba_backward(const moba_params* p, const void* q, const void* k, const void* v,
                          const int32_t* cu_seqlens, const void* out, const float* lse,
                          const void* dout, const int32_t* idx, float* dq, float* dk, float* dv,
                          void* ws, size_t ws_bytes, void* stream) {
  return backward_impl(p, q, k, v, cu_seqlens, out, lse, dout, idx, dq, dk, dv, ws, ws_bytes,
                       stream);
}

size_t moba_workspace_size(const moba_params* p) {
  Dims dm;
  if (validate(p, dm) != MOBA_OK) return 0;
  return plan(dm, true).total;
}

moba_status moba_meanpool(const moba_params* p, const void* k, const int32_t* cu_seqlens,
                          float* kbar, void* stream) {
  Dims dm;
  moba_status s = validate(p, dm);
  if (s != MOBA_OK) return s;
  if (dm.batch == 0 || dm.nb == 0) return MOBA_OK;
  if (!k || !cu_seqlens || !kbar || !aligned32(k) || !aligned32(kbar)) return MOBA_ERR_INVALID_ARG;
  int* status = status_word();
  if (!status) return MOBA_ERR_CUDA;
  return cuda_status(launch_meanpool(dm, k, cu_seqlens, kbar, status,
                                     static_cast<cudaStream_t>(stream)));
}

moba_status moba_gate_topk(const moba_params* p, const void* q, const void* k,
                           const int32_t* cu_seqlens, int32_t* idx, void* ws, size_t ws_bytes,
                           void* stream) {
  Dims dm;
  moba_status s = validate(p, dm);
  if (s != MOBA_OK) return s;
  if (dm.kv_hm) return MOBA_ERR_UNSUPPORTED;
  if (dm.T == 0 || dm.batch == 0) return MOBA_OK;
  if (!q || !k || !cu_seqlens || !idx || !aligned32(q) || !aligned32(k)) return MOBA_ERR_INVALID_ARG;
  // the gate needs the block means and, for the prefix-mean variant, the
  // own-block scores: the head of the forward's workspace plan
  const Layout L = plan(dm, true);
  const size_t need = dm.prefix ? L.own + own_score_bytes(dm, true)
                                : L.kbar + sizeof(float) * (size_t)dm.batch * dm.nb * dm.Hkv * dm.d;
  if (!ws || ws_bytes < need || !aligned32(ws)) return MOBA_ERR_WORKSPACE;
  int* status = status_word();
  if (!status) return MOBA_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* base = static_cast<char*>(ws);
  MOBA_TRY(run_gate(dm, q, k, cu_seqlens, reinterpret_cast<float*>(base + L.kbar),
                    reinterpret_cast<float*>(base + L.own), idx, status, st));
  return MOBA_OK;
}

moba_status moba_forward(const moba_params* p, const void* q, const void* k, const void* v,
                         const int32_t* cu_seqlens, void* out, float* lse, void* ws,
                         size_t ws_bytes, void* stream) {
  return forward_impl(p, q, k, v, cu_seqlens, nullptr, out, lse, ws, ws_bytes, stream);
}

int moba_num_passes(const moba_params* p) {
  Dims dm;
  if (validate(p, dm) != MOBA_OK) return 0;
  return num_passes(dm, plan(dm, true));
}

moba_status moba_forward_staged(const moba_params* p, const void* q, const void* k, const void* v,
                                const int32_t* cu_seqlens, void* out, float* lse, void* ws,
                                size_t ws_bytes, void* const* events, int n_events,
                                void* stream) {
  if (!events) return MOBA_ERR_INVALID_ARG;
  return forward_impl(p, q, k, v, cu_seqlens, nullptr, out, lse, ws, ws_bytes, stream, events,
                      n_events);
}

moba_status moba_forward_with_indices(const moba_params* p, const void* q, const void* k,
                                      const void* v, const int32_t* cu_seqlens,
                                      const int32_t* idx, void* out, float* lse, void* ws,
                                      size_t ws_bytes, void* stream) {
  Dims dm;
  moba_status s = validate(p, dm);
  if (s != MOBA_OK) return s;
  if (dm.T > 0 && dm.batch > 0 && !idx) return MOBA_ERR_INVALID_ARG;
  return forward_impl(p, q, k, v, cu_seqlens, idx, out, lse, ws, ws_bytes, stream);
}

moba_status dense_causal_forward(const moba_params* p, const void* q, const void* k,
                                 const void* v, const int32_t* cu_seqlens, void* out, float* lse,
                                 void* stream) {
  Dims dm;
  moba_status s = validate(p, dm);
  if (s != MOBA_OK) return s;
  if (dm.kv_hm) return MOBA_ERR_UNSUPPORTED;
  if (dm.T == 0 || dm.batch == 0) return MOBA_OK;
  if (!q || !k || !v || !cu_seqlens || !out) return MOBA_ERR_INVALID_ARG;
  if (!aligned32(q) || !aligned32(k) || !aligned32(v) || !aligned32(out) ||
      (lse && !aligned32(lse)))
    return MOBA_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int* status = status_word();
  if (!status) return MOBA_ERR_CUDA;
  if (tc_supported(dm)) return cuda_status(launch_dense_tc(dm, q, k, v, cu_seqlens, out, lse, status, st));
  return cuda_status(launch_dense_simt(dm, q, k, v, cu_seqlens, out, lse, st));
}

moba_status moba_device_status(void* stream, int clear) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return MOBA_ERR_CUDA;
  int value = 0;
  if (cudaMemcpyFromSymbol(&value, g_status, sizeof(int)) != cudaSuccess) return MOBA_ERR_CUDA;
  if (clear) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_status, &zero, sizeof(int)) != cudaSuccess) return MOBA_ERR_CUDA;
  }
  return static_cast<moba_status>(value);
}

moba_status moba_selftest_bounded_wait(int* done, void* stream) {
  if (!done) return MOBA_ERR_INVALID_ARG;
  int* status = status_word();
  if (!status) return MOBA_ERR_CUDA;
  return cuda_status(launch_wait_selftest(status, done, static_cast<cudaStream_t>(stream)));
}

const char* moba_status_string(moba_status s) {
  switch (s) {
    case MOBA_OK: return "ok";
    case MOBA_ERR_INVALID_ARG: return "invalid argument";
    case MOBA_ERR_UNSUPPORTED: return "unsupported configuration";
    case MOBA_ERR_CUDA: return "CUDA error";
    case MOBA_ERR_TIMEOUT: return "bounded device wait expired";
    case MOBA_ERR_WORKSPACE: return "workspace missing or too small";
    case MOBA_ERR_BAD_INDICES: return "index row not in canonical form";
    case MOBA_ERR_CHECK: return "device bounds check failed (checked build)";
  }
  return "unknown status";
}

}  // extern "C"

#ifdef MOBA_TRACE
// ---- trace build only: the registry of the traced files' target setters
namespace moba {
namespace trace {
namespace {
std::mutex& registry_mu() {
  static std::mutex mu;
  return mu;
}
std::vector<cudaError_t (*)(const Target&)>& registry() {
  static std::vector<cudaError_t (*)(const Target&)> fns;
  return fns;
}
moba_status set_all(const Target& t) {
  std::lock_guard<std::mutex> lock(registry_mu());
  for (auto fn : registry())
    if (fn(t) != cudaSuccess) return MOBA_ERR_CUDA;
  return MOBA_OK;
}
}  // namespace
void add_setter(cudaError_t (*fn)(const Target&)) {
  std::lock_guard<std::mutex> lock(registry_mu());
  registry().push_back(fn);
}
}  // namespace trace
}  // namespace moba

extern "C" {
moba_status moba_trace_arm(int kernel, int cta, unsigned long long* buf, int* counts, int cap) {
  if (!buf || !counts || cap <= 0 || cta < 0) return MOBA_ERR_INVALID_ARG;
  if (cudaMemset(counts, 0, sizeof(int) * moba::trace::kMaxWarps) != cudaSuccess)
    return MOBA_ERR_CUDA;
  return moba::trace::set_all(moba::trace::Target{buf, counts, cap, cta, kernel});
}
moba_status moba_trace_disarm(void) {
  return moba::trace::set_all(moba::trace::Target{nullptr, nullptr, 0, -1, 0});
}
}  // extern "C"
#endif
