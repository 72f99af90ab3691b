/*
 * moba.h -- C ABI of libmoba.so: the MoBA (Mixture of Block Attention)
 * prefill forward pass on NVIDIA B200 (sm_100a).
 *
 * The method (PaperTrace knowledge page "2.1.3 MoBA", sections 1-3.1):
 * keys are mean-pooled over contiguous blocks of B tokens (eq. 3); each
 * query scores the blocks that lie wholly before its own block, always keeps
 * its own block (which uses one of the k slots) and takes the k-1 best
 * earlier blocks (section 2, section 2.1); exact softmax attention then runs
 * over the raw keys and values of the chosen blocks, causal inside the own
 * block (eq. 4-6), as ONE softmax over the union of candidates (eq. 7-8).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Layout: packed THD, row-major, contiguous, like flash-attn varlen:
 *   q   [T, Hq,  d]     k, v [T, Hkv, d]     out [T, Hq, d]
 *   cu_seqlens int32 [batch + 1], cu_seqlens[0] = 0, non-decreasing,
 *   cu_seqlens[batch] = T; sequence b owns rows cu[b] .. cu[b+1]-1.
 *   Blocks restart at every sequence start (block i of sequence b covers its
 *   positions iB .. iB+B-1); no key crosses a sequence boundary.
 * Heads: q head h reads kv head h / (Hq / Hkv) (grouped-query attention);
 *   routing is done per q head (moba_params.routing, .own_block: variants).
 * Element type: bf16 or fp32 (moba_params.dtype) for q, k, v and out;
 *   arithmetic is fp32 (bf16 tensor-core products, fp32 accumulation).
 * Pointers: every data pointer is a DEVICE pointer owned by the caller,
 *   32-byte aligned (the kernels move rows in 32-byte pieces; every PyTorch
 *   allocation and any view of whole rows qualifies), and so is a workspace.
 *   cu_seqlens is a device pointer too. The library never allocates device
 *   memory, never frees, and never synchronises the stream; temporary
 *   storage comes from the caller's workspace.
 * Stream: `stream` is a cudaStream_t passed as void* (NULL = legacy default).
 * Errors: arguments are validated on the host before anything is launched;
 *   an invalid call returns a negative moba_status and launches nothing.
 *   Errors found on the device (an index row that is not in canonical form,
 *   a bounded wait that expired) are recorded in a per-device status word
 *   read by moba_device_status().
 */
#ifndef MOBA_H_
#define MOBA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MOBA_API __attribute__((visibility("default")))
#else
#define MOBA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOBA_OK = 0,
  MOBA_ERR_INVALID_ARG = -1,  /* bad size, null pointer, misaligned pointer */
  MOBA_ERR_UNSUPPORTED = -2,  /* valid but not implemented (d, dtype, k range) */
  MOBA_ERR_CUDA = -3,         /* a CUDA runtime call or launch failed */
  MOBA_ERR_TIMEOUT = -4,      /* a bounded device wait expired */
  MOBA_ERR_WORKSPACE = -5,    /* workspace null or smaller than moba_workspace_size() */
  MOBA_ERR_BAD_INDICES = -6,  /* an index row was not in canonical form */
  MOBA_ERR_CHECK = -7         /* checked build only (libmoba_checked.so, built with
                                 MOBA_CHECKED): a device index or bounds check failed;
                                 the access was skipped */
} moba_status;

typedef enum { MOBA_BF16 = 0, MOBA_F32 = 1 } moba_dtype;

typedef struct {
  int batch;         /* number of sequences (>= 0) */
  int total_tokens;  /* T = cu_seqlens[batch] */
  int max_seqlen;    /* an upper bound on every sequence length */
  int num_q_heads;   /* Hq */
  int num_kv_heads;  /* Hkv; Hq % Hkv == 0 */
  int head_dim;      /* d: 64 or 128 */
  int block_size;    /* B >= 1 */
  int topk;          /* k, 1 <= k <= 32; the current block uses one slot */
  moba_dtype dtype;
  int routing;       /* 0 (default): every query head chooses its own blocks.
                        1: the query heads of a kv head's group share one choice,
                        made on the group's mean score (1/grp) sum_h q_h . kbar_i
                        (PaperTrace "2.1.3 MoBA", section 5.5, multi-head
                        settings: a group sharing candidates must aggregate its
                        heads' scores; the mean is this library's reading). */
  int own_block;     /* 0 (default): the query's own block c is always chosen and
                        takes one of the k slots. 1: block c is scored by the
                        mean of its keys up to and including the query (the
                        prefix mean, PaperTrace "2.1.3 MoBA", section 5.2 on
                        causal blocks) and competes with blocks 0..c-1; the k
                        slots go to the best min(k, c+1) blocks, ties to the
                        lower index. A query whose own block loses reads no key
                        of it, itself included; its index row then lists only
                        earlier blocks. With routing 1 the group's mean of the
                        own-block scores is used. */
  int kv_layout;     /* 0 (default): k and v are packed [T][Hkv][d], as everywhere.
                        1: k and v are head-major [Hkv][T][d] (each kv head's keys
                        contiguous): a decode KV cache laid out so the split-K
                        reads of one head stream contiguous rows (section 5.4:
                        decoding is bound by the KV reads). Accepted by
                        moba_meanpool, moba_meanpool_update and moba_decode; the
                        prefill entry points return MOBA_ERR_UNSUPPORTED. */
} moba_params;

/* Number of key blocks reserved per sequence: ceil(max_seqlen / B). */
MOBA_API int moba_num_blocks(const moba_params* p);

/* Bytes of device workspace that moba_gate_topk, moba_forward and
 * moba_forward_with_indices need for these parameters; 0 if the parameters
 * are invalid. Partial results are kept for a group of kv heads at a time,
 * so the size stays bounded for million-token inputs. */
MOBA_API size_t moba_workspace_size(const moba_params* p);

/* Block means, eq. (3): kbar[b][i][g][:] = mean of the keys of block i of
 * sequence b and kv head g, over the positions present (a trailing partial
 * block averages what it has). kbar: fp32 [batch][moba_num_blocks][Hkv][d];
 * slots past a sequence's last block are written as 0. */
MOBA_API moba_status moba_meanpool(const moba_params* p, const void* k, const int32_t* cu_seqlens,
                          float* kbar, void* stream);

/* The parameter-free gate with top-k (eq. 3 and section 2): for every token
 * t and q head h, idx[t][h][:] = the chosen blocks of that query in
 * ascending order -- the chosen earlier blocks first, then the query's own
 * block c -- padded with -1 to k entries. Only blocks i < c are scored
 * (s_i = q . kbar_i, fp32); blocks after c are never chosen; ties go to the
 * lower block index. idx: int32 [T][Hq][k]. With own_block = 1 the own
 * block is a scored candidate (prefix mean) and appears only if chosen.
 * Ranking resolution: scores are compared as fp32, except on the tensor-core
 * path for 6 <= k <= 16 with the forced own block (bf16, d = 128, at most
 * 256 blocks per sequence), which ranks 32-bit keys holding a score's top 24
 * order bits: two scores within 2^-15 of each other (relative) rank by block
 * index there, inside the 1e-4 relative near-tie band of the method.
 * Uses the workspace for kbar (and, with own_block = 1, for the own-block
 * scores: T * Hq floats). */
MOBA_API moba_status moba_gate_topk(const moba_params* p, const void* q, const void* k,
                           const int32_t* cu_seqlens, int32_t* idx, void* ws, size_t ws_bytes,
                           void* stream);

/* moba_gate_topk for callers that cannot allocate device memory (code
 * running inside a runtime that owns all device memory and forbids
 * cudaMalloc, or a latency-critical path that cannot afford cudaMalloc's
 * device-wide synchronisation). The paper has no counterpart: this is a
 * deployment variant of the same gate, with identical results.
 * It needs no workspace: the block means live in a 4 MiB array compiled into
 * the library, which every GPU that loads the library holds until the
 * process exits. It calls no allocating routine.
 * Limit: batch * moba_num_blocks(p) * Hkv * d * 4 bytes must not exceed
 * 4 MiB, else MOBA_ERR_WORKSPACE is returned and nothing is launched; this
 * check comes before the pointer checks, so it does not depend on them.
 * The first call on a device looks up the array's device address (with that
 * device current); make that first call before any stream capture.
 * All calls share the one array and it keeps the last call's contents
 * (nothing in it has to start at zero); calls that overlap on the GPU --
 * on different streams, or from different host threads -- race on it.
 * A sequence longer than max_seqlen is skipped and recorded in the status
 * word (moba_device_status), as moba_gate_topk does.
 * own_block = 1 needs workspace for its scores: MOBA_ERR_UNSUPPORTED. */
MOBA_API moba_status moba_gate_topk_noalloc(const moba_params* p, const void* q, const void* k,
                                            const int32_t* cu_seqlens, int32_t* idx,
                                            void* stream);

/* The full forward pass: gate, regrouping of queries by the block they
 * chose, exact attention over the chosen history blocks (non-causal, eq. 6)
 * and the own block (causal, eq. 5), merged by online softmax (eq. 7-8)
 * into out [T][Hq][d] (input dtype). lse, if not NULL, receives the natural
 * log-sum-exp of the scaled logits per (t, h), fp32 [T][Hq]. */
MOBA_API moba_status moba_forward(const moba_params* p, const void* q, const void* k, const void* v,
                         const int32_t* cu_seqlens, void* out, float* lse, void* ws,
                         size_t ws_bytes, void* stream);

/* Number of passes over groups of kv heads that moba_forward makes. */
MOBA_API int moba_num_passes(const moba_params* p);

/* moba_forward with per-stage timing, the fair per-stage report of section
 * 5.4 (gate, top-k, work-list build, sparse attention): `events` holds
 * n_events >= 3 + 4 * moba_num_passes(p) cudaEvent_t handles (created by the
 * caller, passed as void*). events[0] is recorded before the first launch,
 * events[1] after the mean-pool, events[2] after the gate/top-k, and for pass
 * j events[3+4j], [4+4j], [5+4j], [6+4j] after the regrouping, the history
 * attention, the own-block attention and the merge (on the tensor-core path
 * the own-block kernel performs the merge, so the last interval is empty).
 * Results are identical to moba_forward. */
MOBA_API moba_status moba_forward_staged(const moba_params* p, const void* q, const void* k,
                                         const void* v, const int32_t* cu_seqlens, void* out,
                                         float* lse, void* ws, size_t ws_bytes,
                                         void* const* events, int n_events, void* stream);

/* As moba_forward, with the chosen blocks supplied by the caller instead of
 * the gate (forced candidates; a sliding-window or sink pattern is a special
 * gate, section 3). idx: int32 [T][Hq][k] in the canonical form that
 * moba_gate_topk writes: strictly ascending earlier blocks (each < c), then
 * c, then -1 (with own_block = 1, c may be absent: the row then reads no
 * key of the own block). A row not in that form records MOBA_ERR_BAD_INDICES in the
 * device status word; its output is then unspecified, but every access stays
 * in bounds. */
MOBA_API moba_status moba_forward_with_indices(const moba_params* p, const void* q, const void* k,
                                      const void* v, const int32_t* cu_seqlens,
                                      const int32_t* idx, void* out, float* lse, void* ws,
                                      size_t ws_bytes, void* stream);

/* Backward pass (PaperTrace "2.1.3 MoBA", section 5.3: the hard top-k
 * indices only build the mask and pass no gradient to the routing scores;
 * the loss flows back through the Q/K/V that were read). Gradients of
 * L = sum(dout * out) with respect to q, k and v over the same candidate keys
 * as the forward: per query row, P_j = exp(q.k_j / sqrt(d) - lse),
 * dS_j = P_j (dout.v_j - dout.out), dq = sum_j dS_j k_j / sqrt(d),
 * dk_j += dS_j q / sqrt(d), dv_j += P_j dout (every q head of a group adds
 * into its kv head's dk, dv).
 *   q, k, v, cu_seqlens: as for moba_forward; out [T][Hq][d] and lse [T][Hq]
 *   (fp32, natural log): the forward's results for these inputs; dout:
 *   [T][Hq][d], q's dtype.
 *   idx: the forward's index rows [T][Hq][k] (canonical form), or NULL to
 *   run the gate again (p->routing as in the forward).
 *   dq [T][Hq][d], dk and dv [T][Hkv][d]: fp32, caller-owned, overwritten.
 *   ws: moba_backward_workspace_size(p, idx != NULL) bytes, 32-byte aligned.
 * Errors as moba_forward (MOBA_ERR_BAD_INDICES via the status word). */
MOBA_API size_t moba_backward_workspace_size(const moba_params* p, int have_indices);
MOBA_API moba_status moba_backward(const moba_params* p, const void* q, const void* k,
                                   const void* v, const int32_t* cu_seqlens, const void* out,
                                   const float* lse, const void* dout, const int32_t* idx,
                                   float* dq, float* dk, float* dv, void* ws, size_t ws_bytes,
                                   void* stream);

/* Decode step (PaperTrace "2.1.3 MoBA", section 5.1 on long outputs:
 * incremental block means and logical block numbers; section 5.4: a decode
 * step asks few queries and is bound by the KV reads and the launches).
 * The KV cache holds, per request r, keys and values packed as in a prefill
 * batch: tokens cu_seqlens[r] .. cu_seqlens[r+1]-1, cache length L_r (the new
 * tokens' keys and values already appended). Request r asks
 * n_r = cu_q[r+1] - cu_q[r] queries (1 for plain decoding, more for a
 * speculative draft): the queries of its last positions L_r - n_r .. L_r - 1,
 * in order. Every query gets exactly the prefill forward's result for its
 * position (gate over the complete earlier blocks, own block forced, top-k,
 * one softmax over the chosen keys, causal in the own block). Block ids are
 * logical: block i of a request is its positions iB .. iB+B-1.
 *   p: batch = requests, total_tokens = cache tokens, max_seqlen = the
 *      longest cache; routing as in the prefill; own_block must be 0
 *      (MOBA_ERR_UNSUPPORTED otherwise).
 *   q: [n_queries][Hq][d] (p->dtype); k_cache, v_cache: [total_tokens][Hkv][d];
 *   cu_seqlens, cu_q: device int32 [batch + 1]; cu_q[batch] = n_queries and
 *      0 <= n_r <= L_r (else MOBA_ERR_INVALID_ARG in the status word).
 *   kbar: fp32 [batch][moba_num_blocks(p)][Hkv][d], the cache's block means
 *      (moba_meanpool once, then moba_meanpool_update after each append);
 *      only complete blocks before each query's own block are read.
 *   out: [n_queries][Hq][d] (p->dtype); lse: fp32 [n_queries][Hq] or NULL;
 *   idx: int32 [n_queries][Hq][k] receives the chosen blocks (canonical
 *      form), or NULL.
 *   ws: moba_decode_workspace_size(p, n_queries) bytes, 32-byte aligned. */
MOBA_API size_t moba_decode_workspace_size(const moba_params* p, int n_queries);
MOBA_API moba_status moba_decode(const moba_params* p, const void* q, const void* k_cache,
                                 const void* v_cache, const int32_t* cu_seqlens,
                                 const int32_t* cu_q, int n_queries, const float* kbar, void* out,
                                 float* lse, int32_t* idx, void* ws, size_t ws_bytes,
                                 void* stream);

/* Incremental block means (section 5.1): after n_r = cu_new[r+1] - cu_new[r]
 * tokens were appended to request r's cache (cu_seqlens describing the cache
 * after the append), recomputes, exactly as moba_meanpool would, the entries
 * of kbar for the blocks that hold positions L_r - n_r .. L_r - 1, and leaves
 * every other entry untouched. max_new >= max_r n_r bounds the launch.
 * cu_new: device int32 [batch + 1]. */
MOBA_API moba_status moba_meanpool_update(const moba_params* p, const void* k_cache,
                                          const int32_t* cu_seqlens, const int32_t* cu_new,
                                          int max_new, float* kbar, void* stream);

/* Dense causal softmax attention, eq. (1) with a causal mask (every key
 * j <= p of the query's own sequence), for comparison and for the full
 * budget limit (section 4). block_size and topk in p must be valid but do
 * not change the result. Needs no workspace. */
MOBA_API moba_status dense_causal_forward(const moba_params* p, const void* q, const void* k,
                                 const void* v, const int32_t* cu_seqlens, void* out, float* lse,
                                 void* stream);

/* Synchronises `stream`, returns the device status word of the current
 * device (MOBA_OK, MOBA_ERR_TIMEOUT, MOBA_ERR_BAD_INDICES, MOBA_ERR_INVALID_ARG
 * for a sequence longer than max_seqlen, or in the checked build
 * MOBA_ERR_CHECK) and clears it if `clear` is non-zero. The first error
 * recorded wins. */
MOBA_API moba_status moba_device_status(void* stream, int clear);

/* Self-test of the bounded waits used by the tensor-core kernels (no paper
 * counterpart; failure detection): launches one CTA that waits on a barrier
 * nothing arrives on. After about 2e9 SM cycles (about a second) the wait
 * gives up, the kernel writes 2 to *done (device int) and records
 * MOBA_ERR_TIMEOUT in the status word, which moba_device_status() then
 * returns; the context stays usable. Nothing faults or hangs. */
MOBA_API moba_status moba_selftest_bounded_wait(int* done, void* stream);

/* Static description of a status code. */
MOBA_API const char* moba_status_string(moba_status s);

#ifdef __cplusplus
}
#endif

#endif /* MOBA_H_ */
