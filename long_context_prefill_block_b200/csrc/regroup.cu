// Regrouping of queries by the key block they chose (PaperTrace "2.1.3
// MoBA", section 3.1 steps 3 and 5, section 5.4): the query -> block choices
// are inverted into one list per (sequence, kv head, history block) of the
// (query, q head, slot) entries that read it, so that one contiguous K/V
// block serves a dense tile of queries -- the MoE token-dispatch pattern of
// histogram, exclusive scan and scatter.
//
// An entry is a partial-row id prow = ((t * nq) + h_local) * k + slot, where
// slot is the entry's position in the query's index row; the history kernel
// writes its partial result there and the merge reads it back in query
// order, which also restores the original order. Entries inside a list are
// in atomic-arrival order: each query's result depends only on its own row,
// so the order changes no output bit.
//
// The count pass also checks each index row's canonical form (strictly
// ascending earlier blocks, then the own block c, then -1 padding; with the
// prefix-mean gate c may be absent) and records kStBadIndices for a row that
// breaks it; such entries are skipped.
#include "common.cuh"

namespace moba {
namespace {

constexpr int kThreads = 128;
constexpr int kScanThreads = 1024;

// Walks one index row; calls f(slot, block) for every history entry and
// returns false if the row is not canonical (own_required: block c must be
// named).
template <typename F>
__device__ __forceinline__ bool walk_row(const int32_t* row, int topk, int c, bool own_required,
                                         F f) {
  int prev = -1;
  bool seen_c = false, seen_pad = false, ok = true;
  for (int r = 0; r < topk; ++r) {
    const int e = row[r];
    if (seen_c || seen_pad) {
      ok &= (e == -1);
    } else if (e == c) {
      seen_c = true;
    } else if (e == -1) {
      seen_pad = true;
    } else if (e >= 0 && e < c && e > prev) {
      prev = e;
      f(r, e);
    } else {
      ok = false;
    }
  }
  // a row without its own block must name at least one earlier block
  return ok && (seen_c || (!own_required && prev >= 0));
}

// walk_row over a row held in registers (k <= 32), unrolled so that every
// index is a compile-time constant and the row stays in registers.
template <typename F>
__device__ __forceinline__ bool walk_row(const int32_t (&row)[32], int topk, int c,
                                         bool own_required, F f) {
  int prev = -1;
  bool seen_c = false, seen_pad = false, ok = true;
#pragma unroll
  for (int r = 0; r < 32; ++r) {
    if (r >= topk) break;
    const int e = row[r];
    if (seen_c || seen_pad) {
      ok &= (e == -1);
    } else if (e == c) {
      seen_c = true;
    } else if (e == -1) {
      seen_pad = true;
    } else if (e >= 0 && e < c && e > prev) {
      prev = e;
      f(r, e);
    } else {
      ok = false;
    }
  }
  return ok && (seen_c || (!own_required && prev >= 0));
}

template <bool SCATTER>
__global__ void __launch_bounds__(kThreads) regroup_pass(Dims dm, Chunk ch,
                                                         const int32_t* __restrict__ idx,
                                                         const int32_t* __restrict__ cu,
                                                         int32_t* counts, int32_t* cursor,
                                                         const int32_t* __restrict__ list_off,
                                                         int32_t* pairs, int* status) {
  const int b = blockIdx.y, hl = blockIdx.z;
  const int h = ch.h0 + hl;
  const int grp = dm.Hq / dm.Hkv;
  const int gl = h / grp - ch.g0;
  int64_t start;
  int len;
  if (!seq_bounds(dm, cu, b, start, len, SCATTER ? nullptr : status)) return;
  const int p = blockIdx.x * kThreads + threadIdx.x;
  if (p >= len) return;
  const int64_t t = start + p;
  const int c = p / dm.B;
  const int32_t* row = idx + (t * dm.Hq + h) * (int64_t)dm.topk;
  const int list0 = (b * ch.ng + gl) * dm.nb;
  const int64_t prow0 = (t * ch.nq + hl) * (int64_t)dm.topk;
  const bool ok = walk_row(row, dm.topk, c, !dm.prefix, [&](int slot, int e) {
    if (SCATTER) {
      const int list = list0 + e;
      const int pos = atomicAdd(&cursor[list], 1);
      const int64_t at = (int64_t)list_off[list] + pos;
      if (MOBA_CHECK(at < (int64_t)dm.T * ch.nq * hist_slots(dm), status))
        pairs[at] = (int32_t)(prow0 + slot);
    } else {
      atomicAdd(&counts[list0 + e], 1);
    }
  });
  if (!SCATTER && !ok) set_status(status, kStBadIndices);
}

// Same two passes with the lists of one CTA (kRows positions of one q head,
// hence one sequence and kv head) counted in shared memory first, so each
// list sees one global atomic per CTA instead of one per entry. The scatter
// pass reserves a contiguous range per list and places the CTA's entries in
// it. Used when a sequence has at most kSmemLists blocks.
constexpr int kRows = 256;
constexpr int kSmemLists = 8192;

template <bool SCATTER>
__global__ void __launch_bounds__(kRows) regroup_pass_smem(Dims dm, Chunk ch,
                                                           const int32_t* __restrict__ idx,
                                                           const int32_t* __restrict__ cu,
                                                           int32_t* counts, int32_t* cursor,
                                                           const int32_t* __restrict__ list_off,
                                                           int32_t* pairs, int* status, int vec) {
  extern __shared__ int32_t lsm[];
  int32_t* hist = lsm;            // [nb] entries of this CTA per block
  int32_t* base = lsm + dm.nb;    // [nb] SCATTER: first list position reserved for the CTA
  const int b = blockIdx.y, hl = blockIdx.z;
  const int h = ch.h0 + hl;
  const int grp = dm.Hq / dm.Hkv;
  const int gl = h / grp - ch.g0;
  int64_t start;
  int len;
  if (!seq_bounds(dm, cu, b, start, len, SCATTER ? nullptr : status)) return;
  const int p0 = blockIdx.x * kRows;
  if (p0 >= len) return;
  const int cmax = (min(p0 + kRows, len) - 1) / dm.B + 1;  // blocks any row may name
  for (int e = threadIdx.x; e < cmax; e += kRows) hist[e] = 0;
  __syncthreads();
  const int p = p0 + threadIdx.x;
  const bool valid = p < len;
  const int64_t t = start + p;
  const int c = p / dm.B;
  const int32_t* row_g = idx + (t * dm.Hq + h) * (int64_t)dm.topk;
  // the row in registers, by 16-byte loads when its length allows
  int32_t row[32];
  if (valid) {
    if (vec) {
#pragma unroll
      for (int r = 0; r < 32; r += 4)
        if (r < dm.topk) *reinterpret_cast<int4*>(row + r) = *reinterpret_cast<const int4*>(row_g + r);
    } else {
#pragma unroll
      for (int r = 0; r < 32; ++r)
        if (r < dm.topk) row[r] = row_g[r];
    }
  }
  const int list0 = (b * ch.ng + gl) * dm.nb;
  const int64_t prow0 = (t * ch.nq + hl) * (int64_t)dm.topk;
  bool ok = true;
  if (valid) ok = walk_row(row, dm.topk, c, !dm.prefix, [&](int, int e) { atomicAdd(&hist[e], 1); });
  if (!SCATTER && !ok) set_status(status, kStBadIndices);
  __syncthreads();
  for (int e = threadIdx.x; e < cmax; e += kRows) {
    const int n = hist[e];
    if (SCATTER) {
      base[e] = n ? atomicAdd(&cursor[list0 + e], n) : 0;
      hist[e] = 0;
    } else if (n) {
      atomicAdd(&counts[list0 + e], n);
    }
  }
  if (!SCATTER) return;
  __syncthreads();
  if (valid)
    walk_row(row, dm.topk, c, !dm.prefix, [&](int slot, int e) {
      const int pos = base[e] + atomicAdd(&hist[e], 1);
      const int64_t at = (int64_t)list_off[list0 + e] + pos;
      if (MOBA_CHECK(at < (int64_t)dm.T * ch.nq * hist_slots(dm), status))
        pairs[at] = (int32_t)(prow0 + slot);
    });
}

// Exclusive scans of the list sizes and of their tile counts (one CTA); the
// scatter pass's cursors start at zero.
__global__ void __launch_bounds__(kScanThreads) regroup_scan(int n_lists, int tile_m,
                                                            const int32_t* __restrict__ counts,
                                                            int32_t* list_off, int32_t* tile_off,
                                                            int32_t* cursor) {
  __shared__ int warp_a[kScanThreads / 32], warp_b[kScanThreads / 32];
  __shared__ int carry_a, carry_b;
  if (threadIdx.x == 0) carry_a = carry_b = 0;
  __syncthreads();
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  for (int base = 0; base < n_lists; base += kScanThreads) {
    const int i = base + threadIdx.x;
    const int a = i < n_lists ? counts[i] : 0;
    const int bt = (a + tile_m - 1) / tile_m;
    int xa = a, xb = bt;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int ya = __shfl_up_sync(0xffffffffu, xa, off);
      const int yb = __shfl_up_sync(0xffffffffu, xb, off);
      if (lane >= off) {
        xa += ya;
        xb += yb;
      }
    }
    if (lane == 31) {
      warp_a[wid] = xa;
      warp_b[wid] = xb;
    }
    __syncthreads();
    if (wid == 0) {
      int va = warp_a[lane], vb = warp_b[lane];
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int ya = __shfl_up_sync(0xffffffffu, va, off);
        const int yb = __shfl_up_sync(0xffffffffu, vb, off);
        if (lane >= off) {
          va += ya;
          vb += yb;
        }
      }
      warp_a[lane] = va;
      warp_b[lane] = vb;
    }
    __syncthreads();
    const int pa = (wid ? warp_a[wid - 1] : 0) + xa - a + carry_a;
    const int pb = (wid ? warp_b[wid - 1] : 0) + xb - bt + carry_b;
    if (i < n_lists) {
      list_off[i] = pa;
      tile_off[i] = pb;
      cursor[i] = 0;
    }
    __syncthreads();
    if (threadIdx.x == kScanThreads - 1) {
      carry_a = pa + a;
      carry_b = pb + bt;
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    list_off[n_lists] = carry_a;
    tile_off[n_lists] = carry_b;
  }
}

// Tile table: tile j of list L covers list rows [j * tile_m, (j+1) * tile_m);
// each entry also carries the list's size and first entry, so a work unit's
// description is one 16-byte load with no dependent loads behind it.
// One CTA per list, its threads writing consecutive entries (a list of the
// million-token shape holds hundreds of tiles).
__global__ void regroup_tiles(int n_lists, int tile_m, const int32_t* __restrict__ counts,
                              const int32_t* __restrict__ list_off,
                              const int32_t* __restrict__ tile_off, int4* tiles) {
  const int L = blockIdx.x;
  if (L >= n_lists) return;
  const int count = counts[L];
  const int n = (count + tile_m - 1) / tile_m;
  const int o = tile_off[L], first = list_off[L];
  for (int j = threadIdx.x; j < n; j += blockDim.x)
    tiles[o + j] = make_int4(L, j * tile_m, count, first);
}

}  // namespace

cudaError_t launch_regroup(const Dims& dm, const Chunk& ch, const int32_t* idx, const int32_t* cu,
                           const Regroup& rg, int* status, cudaStream_t st) {
  cudaError_t e;
  if ((e = cudaMemsetAsync(rg.counts, 0, sizeof(int32_t) * ch.n_lists, st))) return e;
  if (dm.batch == 0 || dm.max_seqlen == 0) {
    return cudaMemsetAsync(rg.tile_off + ch.n_lists, 0, sizeof(int32_t), st);
  }
  const bool smem_lists = dm.nb <= kSmemLists;
  // index rows start on 16-byte boundaries when k % 4 == 0 and idx does
  const int vec = (dm.topk % 4 == 0 && (reinterpret_cast<uintptr_t>(idx) & 15) == 0) ? 1 : 0;
  dim3 grid((dm.max_seqlen + kThreads - 1) / kThreads, dm.batch, ch.nq);
  dim3 grid_s((dm.max_seqlen + kRows - 1) / kRows, dm.batch, ch.nq);
  const size_t lsm = 2 * sizeof(int32_t) * dm.nb;
  if (smem_lists) {
    if ((e = cudaFuncSetAttribute(regroup_pass_smem<false>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, (int)lsm)))
      return e;
    if ((e = cudaFuncSetAttribute(regroup_pass_smem<true>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, (int)lsm)))
      return e;
    regroup_pass_smem<false><<<grid_s, kRows, lsm, st>>>(dm, ch, idx, cu, rg.counts, rg.cursor,
                                                         nullptr, nullptr, status, vec);
  } else {
    regroup_pass<false><<<grid, kThreads, 0, st>>>(dm, ch, idx, cu, rg.counts, rg.cursor, nullptr,
                                                   nullptr, status);
  }
  if ((e = cudaGetLastError())) return e;
  // the scan also zeroes the scatter pass's cursors
  regroup_scan<<<1, kScanThreads, 0, st>>>(ch.n_lists, ch.tile_m, rg.counts, rg.list_off,
                                           rg.tile_off, rg.cursor);
  if ((e = cudaGetLastError())) return e;
  if (smem_lists) {
    regroup_pass_smem<true><<<grid_s, kRows, lsm, st>>>(dm, ch, idx, cu, rg.counts, rg.cursor,
                                                        rg.list_off, rg.pairs, status, vec);
  } else {
    regroup_pass<true><<<grid, kThreads, 0, st>>>(dm, ch, idx, cu, rg.counts, rg.cursor,
                                                  rg.list_off, rg.pairs, status);
  }
  if ((e = cudaGetLastError())) return e;
  regroup_tiles<<<ch.n_lists, 128, 0, st>>>(ch.n_lists, ch.tile_m, rg.counts, rg.list_off,
                                            rg.tile_off, rg.tiles);
  return cudaGetLastError();
}

}  // namespace moba
