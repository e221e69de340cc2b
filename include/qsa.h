/*
 * qsa.h -- C ABI of libqsa.so: the forward pass of Qwen Sparse Attention (QSA)
 * on NVIDIA B200 (sm_100a).
 *
 * The method (web pages on Qwen3.8-Flash-Next):
 *   - design report summary "Qwen3.8-Next architecture design report"
 *     (macin.top, on "On the Design of Qwen3.8-Next Architecture"), section
 *     "Four architecture components", item 2 "Qwen Sparse Attention (QSA)":
 *     the indexer works on micro-blocks of r=4 tokens; the keys of a block are
 *     averaged and then position-encoded; scoring costs O(n^2/r); the indexer
 *     has 4 query heads sharing one key (MQA); each query keeps K=2048 tokens.
 *   - Miles docs "Qwen3.8-Flash-Next", section 1 "Model Introduction": each
 *     QSA layer derives its own indexer queries and compressed keys, scores
 *     them and keeps a budget of key tokens per query; attention then reads
 *     only those tokens; selection rows are built outside the attention kernel
 *     so that it needs no causal or segment logic; 24 heads, 2 query groups,
 *     kv-channels 256, rotary base 1e7 at rotary percent 0.25.
 *   - tahou.com article on the Qwen3.8-Flash-Next release, section "GDN+QSA":
 *     a lightweight indexer groups the sequence into micro-blocks, scores
 *     their importance, and attention runs on the most relevant regions only.
 *
 * Readings fixed here where the pages are silent:
 *   score       s(t,b) = sum_h w[t,h] * max(0, q~[t,h] . k^[b]) over the
 *               idx_heads indexer heads (the DeepSeek-DSA form), no extra scale;
 *   block key   k^[b] = RoPE_{r*b}( (1/r) sum_{j<r} k_idx[r*b+j] ), computed in
 *               fp32 in that order and stored in the I/O dtype (bf16 RNE);
 *   query       q~[t,h] = RoPE_t(q_idx[t,h]) stored in the I/O dtype;
 *   RoPE        partial: the first rope_dims = floor(idx_dim*rope_fraction)
 *               (even) dims rotate in rotate-half pairs (i, i+rope_dims/2),
 *               theta_i = rope_base^(-2i/rope_dims), angle formed in fp64;
 *   candidates  blocks b < b_t = floor(t/r) (all complete);
 *   selection   if b_t+1 <= S = budget_tokens/r, blocks 0..b_t; otherwise the
 *               own block b_t plus the S-1 best candidates under the order
 *               (score descending, block index ascending; -0 equals +0);
 *   attention   token j is attended iff floor(j/r) is selected and j <= t;
 *               head h reads KV group floor(h / (n_q_heads/n_kv_groups));
 *               softmax scale 1/sqrt(head_dim) unless given.
 *
 * Conventions shared by every call:
 *   - The caller owns every buffer.  The library never allocates, never
 *     synchronises the stream and keeps no pointer after a call returns.
 *   - "device" pointers are CUDA global memory of the current device,
 *     16-byte aligned, densely packed in the layouts given (innermost last).
 *     "host" pointers are read during the call only.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default).
 *     All work is enqueued on it in order; a call returns before it runs.
 *   - Host-checkable errors return QSA_ERR_INVALID_ARG / QSA_ERR_UNSUPPORTED /
 *     QSA_ERR_WORKSPACE before anything is enqueued.  A failed launch returns
 *     QSA_ERR_CUDA.  Device-side faults of bounded waits, and selection
 *     entries outside [0, n_cap/r) that an attention kernel skipped, are
 *     reported by qsa_device_status().  A call with no query tokens is a
 *     no-op (QSA_OK).
 *   - Supported shapes: r == 4, head_dim == 256, n_q_heads/n_kv_groups <= 16,
 *     idx_heads == 4, idx_dim in {64, 128}, budget_tokens a multiple of r with
 *     budget_tokens/r <= 512.
 *
 * Token batch.  A call processes T query tokens given as segments: segment i
 * holds q_len consecutive positions pos0 .. pos0+q_len-1 of the sequence in
 * cache slot `slot`, stored at token rows q_offset .. q_offset+q_len-1 of
 * every token-major array (q, q_idx, w, o, lse, sel, nsel, score rows).
 * Prefill, a prefill chunk over a cached prefix, and decode (q_len = 1) are
 * all segments.  The cache must already hold every token <= pos0+q_len-1.
 */
#ifndef QSA_H
#define QSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  QSA_OK = 0,
  QSA_ERR_INVALID_ARG = 1,  /* bad pointer, size, layout or segment; nothing enqueued */
  QSA_ERR_UNSUPPORTED = 2,  /* valid configuration the kernels do not implement      */
  QSA_ERR_WORKSPACE = 3,    /* workspace NULL or smaller than qsa_workspace_size()     */
  QSA_ERR_CUDA = 4,         /* a CUDA runtime call or kernel launch failed             */
  QSA_ERR_TIMEOUT = 5,      /* a bounded device-side wait gave up (qsa_device_status)  */
  QSA_ERR_BAD_INDEX = 6     /* a caller-supplied sel entry was out of range and skipped
                               (qsa_device_status)                                     */
} qsa_status_t;

typedef enum { QSA_DTYPE_F32 = 0, QSA_DTYPE_BF16 = 1 } qsa_dtype_t;

/* Per-layer constants (Miles docs section 1; design report QSA item). */
typedef struct {
  int32_t r;              /* tokens per micro-block: 4                               */
  int32_t budget_tokens;  /* kept tokens per query: 2048 (multiple of r)             */
  int32_t n_q_heads;      /* attention query heads: 24                               */
  int32_t n_kv_groups;    /* KV groups: 2                                            */
  int32_t head_dim;       /* 256                                                     */
  int32_t idx_heads;      /* indexer query heads: 4                                  */
  int32_t idx_dim;        /* indexer head dim: 64 or 128                             */
  float rope_fraction;    /* rotated share of idx_dim: 0.25                          */
  double rope_base;       /* 1e7                                                     */
  float softmax_scale;    /* <= 0 selects 1/sqrt(head_dim)                           */
  qsa_dtype_t dtype;      /* I/O dtype of q, q_idx, k_idx, k^, K, V and o            */
} qsa_config_t;

/* One run of consecutive query tokens of one cached sequence. */
typedef struct {
  int32_t q_offset;       /* first token row in the token-major arrays               */
  int32_t q_len;          /* number of query tokens (>= 0)                           */
  int32_t pos0;           /* absolute position of the first query token (>= 0)       */
  int32_t slot;           /* cache slot of the sequence, in [0, n_slots)             */
} qsa_segment_t;

/* Per-sequence caches (device memory, caller-owned).  n_cap tokens per slot. */
typedef struct {
  const void* k_idx;      /* [n_slots][n_cap][idx_dim]            indexer keys        */
  void* khat;             /* [n_slots][n_cap/r][idx_dim]          pooled block keys   */
  const void* k;          /* [n_slots][n_kv_groups][n_cap][head_dim]  main keys       */
  const void* v;          /* [n_slots][n_kv_groups][n_cap][head_dim]  main values     */
  int32_t n_slots;
  int64_t n_cap;          /* multiple of r                                          */
} qsa_cache_t;

typedef enum {
  QSA_OP_COMPRESS = 0,
  QSA_OP_INDEX = 1,
  QSA_OP_SELECT = 2,
  QSA_OP_ATTN = 3,
  QSA_OP_FORWARD = 4,
  QSA_OP_FORWARD_LOWMEM = 5,
  QSA_OP_ATTN_UNION = 6,
  QSA_OP_FORWARD_PREFIXED = 7
} qsa_op_t;

/* A cached prefix that a segment's sequence shares with other sequences:
 * its first `blocks` micro-blocks (blocks*r tokens) live in cache slot
 * `slot` (k_idx, khat, K, V), once for all the sequences that use it; the
 * rest of the sequence lives in the segment's own slot, at the same absolute
 * positions (positions below blocks*r of the own slot are never read).
 * blocks == 0: the segment shares nothing. */
typedef struct {
  int32_t slot;
  int32_t blocks;
} qsa_prefix_t;

/*
 * Key pooling + block position encoding (design report, QSA item: keys are
 * averaged per micro-block, then position-encoded).  For each i < n_ranges,
 * writes k^ of blocks [blk_begin[i], blk_end[i]) of cache slot slots[i]:
 *   cache->khat[slot][b][:] = RoPE_{r*b}(mean of cache->k_idx[slot][r*b .. r*b+r-1][:]).
 * slots, blk_begin, blk_end: host arrays [n_ranges].  Requires
 * 0 <= blk_begin <= blk_end <= n_cap/r.  Reads k_idx, writes khat only.
 */
qsa_status_t qsa_compress_keys(const qsa_config_t* cfg, const qsa_cache_t* cache,
                               const int32_t* slots, const int64_t* blk_begin,
                               const int64_t* blk_end, int32_t n_ranges, void* stream);

/*
 * Indexer scores (design report, QSA item: 4-head MQA indexer scoring
 * micro-blocks; Miles docs section 1: each layer scores its own compressed
 * keys).  For every query token i at position t (segments, host array):
 *   scores[i][b] = sum_h w[i][h] * max(0, RoPE_t(q_idx[i][h]) . khat[slot][b]),
 *   b in [0, floor(t/r)).
 * q_idx: device [T][idx_heads][idx_dim] (I/O dtype); w: device [T][idx_heads]
 * fp32; cache->khat must hold blocks [0, floor(t/r)) for every query.
 * scores: device fp32 [T][ld_scores]; entries b >= floor(t/r) of a row are not
 * written.  ld_scores >= max floor(t/r) over all queries, and >= 1.
 * n_tokens: T, the row count of the token-major arrays.
 */
qsa_status_t qsa_index_scores(const qsa_config_t* cfg, const qsa_cache_t* cache,
                              const qsa_segment_t* segs, int32_t n_segs, int32_t n_tokens,
                              const void* q_idx, const float* w, float* scores,
                              int64_t ld_scores, void* stream);

/*
 * Top-k block selection (pages: budget 2048 tokens per query; the own block
 * rule and the tie order are this library's readings, see top of file).
 * For every query token i at position t: sel[i][0..nsel[i]) = the kept blocks
 * in ascending order (the own block floor(t/r) last), sel[i][nsel[i]..S) = -1,
 * nsel[i] = min(S, floor(t/r)+1), S = budget_tokens/r.
 * scores: device fp32 [T][ld_scores] as written by qsa_index_scores.
 * sel: device int32 [T][S]; nsel: device int32 [T].
 * workspace: device, >= qsa_workspace_size(..., QSA_OP_SELECT) bytes (may be
 * NULL when that size is 0).  Contents on entry are ignored.
 */
qsa_status_t qsa_select_topk(const qsa_config_t* cfg, const qsa_segment_t* segs,
                             int32_t n_segs, int32_t n_tokens, const float* scores,
                             int64_t ld_scores, int32_t* sel, int32_t* nsel, void* workspace,
                             size_t ws_bytes, void* stream);

/*
 * Sparse GQA softmax attention over the kept tokens (Miles docs section 1:
 * attention reads only the kept key tokens; 24 heads, 2 query groups, head
 * dim 256).  For every query token i at position t and head h (group
 * g = h / (n_q_heads/n_kv_groups)):
 *   J = { j : floor(j/r) in sel[i][0..nsel[i]), j <= t },
 *   o[i][h][:]  = sum_{j in J} softmax_j(scale * q[i][h] . K[slot][g][j]) V[slot][g][j][:],
 *   lse[i][h]   = log sum_{j in J} exp(scale * q[i][h] . K[slot][g][j])   (natural log).
 * q, o: device [T][n_q_heads][head_dim] (I/O dtype).  lse: device fp32
 * [T][n_q_heads] or NULL.  sel/nsel as produced by qsa_select_topk (entries
 * must lie in [0, n_cap/r)).  workspace >= qsa_workspace_size(..., QSA_OP_ATTN).
 */
qsa_status_t qsa_sparse_attn_fwd(const qsa_config_t* cfg, const qsa_cache_t* cache,
                                 const qsa_segment_t* segs, int32_t n_segs, int32_t n_tokens,
                                 const void* q, const int32_t* sel, const int32_t* nsel, void* o,
                                 float* lse, void* workspace, size_t ws_bytes, void* stream);

/*
 * qsa_sparse_attn_fwd computed on tiles of neighbouring queries (the same o
 * and lse, up to the rounding of P to bf16 against a different reference
 * maximum).  Miles docs section 1: each query attends only its kept tokens;
 * neighbouring tokens whose indexer queries are close keep mostly the same
 * blocks.  Each segment is cut into tiles of mq = min(32, 128 / heads per
 * group) consecutive query tokens; a tile gathers the ascending union of its
 * members' kept blocks once per KV group, and a per-block member mask plus
 * each member's causal limit give every query exactly its own key set J.
 * Gathered K/V bytes per query fall by the tile's sharing factor (mq x 512
 * blocks / union length); with no sharing they equal the per-query path's.
 * Arguments, layouts and errors as qsa_sparse_attn_fwd; in addition every
 * sel row must hold distinct blocks (qsa_select_topk writes them so).
 * bf16 only (QSA_ERR_UNSUPPORTED otherwise).  workspace >=
 * qsa_workspace_size(..., QSA_OP_ATTN_UNION) bytes (the union lists and
 * masks: about 8 * mq * budget_tokens / r bytes per tile); contents on entry
 * are ignored.
 */
qsa_status_t qsa_sparse_attn_fwd_union(const qsa_config_t* cfg, const qsa_cache_t* cache,
                                       const qsa_segment_t* segs, int32_t n_segs, int32_t n_tokens,
                                       const void* q, const int32_t* sel, const int32_t* nsel, void* o,
                                       float* lse, void* workspace, size_t ws_bytes, void* stream);

/*
 * Backward of qsa_sparse_attn_fwd (Miles docs section 1: the QSA attention
 * kernel has a forward and a backward pass over the same kept tokens).  For
 * the loss sum over tokens and heads of dout . o, with the forward's
 * probabilities P_hj = exp(scale q_h . k_j - lse_h) over the kept tokens:
 *   dq_h  = scale sum_j P_hj (dout_h . v_j - dout_h . o_h) k_j
 *   dk_j += scale sum_{t,h} P_hj (dout_h . v_j - dout_h . o_h) q_h
 *   dv_j += sum_{t,h} P_hj dout_h
 * q, o, dout: device [T][H][D] in the I/O dtype (o and lse as qsa_sparse_attn_fwd
 * or qsa_forward wrote them); lse: device fp32 [T][H]; sel/nsel as the forward
 * used them.  dq: device fp32 [T][H][D], written.  dk, dv: device fp32 arrays
 * laid out like cache->k / cache->v ([n_slots][n_kv_groups][n_cap][head_dim]),
 * ACCUMULATED into (fp32 atomic adds, so the order of additions and the last
 * bits vary from run to run): zero them before the first call of a step.
 * The indexer and the selection have no gradient here.  bf16 runs on the
 * tensor cores with P and the probability gradients rounded to bf16 for the
 * products (as the forward rounds P); fp32 runs on CUDA cores in fp32.
 */
qsa_status_t qsa_sparse_attn_bwd(const qsa_config_t* cfg, const qsa_cache_t* cache,
                                 const qsa_segment_t* segs, int32_t n_segs, int32_t n_tokens,
                                 const void* q, const void* o, const float* lse, const void* dout,
                                 const int32_t* sel, const int32_t* nsel, float* dq, float* dk,
                                 float* dv, void* stream);

/*
 * The whole QSA forward pass for a token batch (prefill, chunked prefill over
 * a cached prefix, decode, or a mix), enqueued on one stream with no host
 * synchronisation:
 *   1. qsa_compress_keys for the blocks each segment completes:
 *      [floor(pos0/r), floor((pos0+q_len)/r));
 *   2. qsa_index_scores; 3. qsa_select_topk; 4. qsa_sparse_attn_fwd.
 * (When no query of the batch scores a block this call completes, as in
 * decode, step 1 runs alongside step 2; the results are the same.)
 * Blocks before floor(pos0/r) must already be pooled in cache->khat.
 * sel/nsel: device outputs as in qsa_select_topk, or both NULL to keep them in
 * the workspace.  workspace >= qsa_workspace_size(..., QSA_OP_FORWARD).
 */
qsa_status_t qsa_forward(const qsa_config_t* cfg, const qsa_cache_t* cache,
                         const qsa_segment_t* segs, int32_t n_segs, int32_t n_tokens,
                         const void* q, const void* q_idx, const float* w, void* o, float* lse,
                         int32_t* sel, int32_t* nsel, void* workspace, size_t ws_bytes,
                         void* stream);

/*
 * qsa_forward for sequences that share cached prefixes (the release article's
 * section "GDN+QSA" quotes its 1M-context throughput at a 90 % prefix-cache
 * hit: many requests on one cached prefix).  prefix: host array [n_segs];
 * segment i's sequence is prefix[i] followed by its own slot (see
 * qsa_prefix_t).  Results are those of qsa_forward on each sequence's whole
 * cache.  The queries of all segments with the same (slot, blocks) are
 * scored over the prefix's blocks together, up to 16 queries per pass over
 * the prefix's pooled keys (in qsa_forward every decode query streams its
 * own); each segment's own blocks are scored from its slot; the attention
 * reads kept prefix blocks from the prefix's slot.
 * Requires bf16 I/O, and segments with blocks > 0 of fewer than 16 queries
 * (decode and speculative decode; QSA_ERR_UNSUPPORTED otherwise), and for
 * every segment with blocks > 0: 0 <= slot < n_slots and blocks*r <= pos0
 * (all of its queries past the prefix; QSA_ERR_INVALID_ARG otherwise).  The prefix's blocks must
 * already be pooled in its slot's khat.  workspace >= qsa_workspace_size(...,
 * QSA_OP_FORWARD_PREFIXED).
 */
qsa_status_t qsa_forward_prefixed(const qsa_config_t* cfg, const qsa_cache_t* cache,
                                  const qsa_segment_t* segs, const qsa_prefix_t* prefix, int32_t n_segs,
                                  int32_t n_tokens, const void* q, const void* q_idx, const float* w,
                                  void* o, float* lse, int32_t* sel, int32_t* nsel, void* workspace,
                                  size_t ws_bytes, void* stream);

/*
 * qsa_forward without the score matrix, for callers short of device memory.
 * The design report's QSA item defines the indexer scores and the top-k;
 * fusing them is this library's choice, not the pages'.  Same
 * arguments, results and errors; workspace >= qsa_workspace_size(...,
 * QSA_OP_FORWARD_LOWMEM).  For bf16 segments of 16 or more queries steps 2-3
 * run fused: the indexer scores every 16th pooled block; a threshold per
 * query is taken from that sample (about 1536 of the query's blocks are
 * expected at or above it); a second indexer pass keeps only the (score,
 * block) pairs at or above it, at most 4096 per query; the selection runs
 * exactly on those.  A query whose list holds fewer than S-1 or more than
 * 4096 pairs is selected exactly over all of its blocks, scores recomputed
 * on CUDA cores (qsa_select_fallbacks counts these).  Selections equal
 * qsa_forward's up to the rounding order of the scores.  Other segments run
 * as in qsa_forward.
 *
 * Memory: 4*ceil(n_blocks/16) + 32 KiB per query instead of 4*n_blocks bytes
 * (128K-token prefill: 5.6 GB instead of 17.2 GB).  Time: slower than
 * qsa_forward on B200 (the filtering costs the indexer's epilogue more
 * instructions than the score writes it saves).
 */
qsa_status_t qsa_forward_lowmem(const qsa_config_t* cfg, const qsa_cache_t* cache,
                                const qsa_segment_t* segs, int32_t n_segs, int32_t n_tokens,
                                const void* q, const void* q_idx, const float* w, void* o, float* lse,
                                int32_t* sel, int32_t* nsel, void* workspace, size_t ws_bytes,
                                void* stream);

/*
 * qsa_select_topk without a caller workspace, for callers that cannot call
 * cudaMalloc: code running where the allocator is off limits (a custom
 * allocator or memory pool owns all device memory, an embedding that forbids
 * allocation after start-up, or a section whose memory use must be fixed in
 * advance).  The pages have no counterpart to this call; it is an interface
 * convenience, not part of the method.
 *
 * Same arguments, results and errors as qsa_select_topk, minus the
 * workspace.  Rows beyond 32K candidate blocks, in a batch of few rows,
 * keep their row histograms, counters and candidate lists (48 KiB per token
 * row) in a device array built into the library,
 * QSA_NOALLOC_SCRATCH_BYTES (16 MiB) per device, held by every GPU that
 * loads the library until the process exits; each call clears the part it
 * uses with cudaMemsetAsync on `stream`.  A batch whose selection needs more
 * than that (see qsa_workspace_size(..., QSA_OP_SELECT)) returns
 * QSA_ERR_WORKSPACE and enqueues nothing.  Nothing is allocated or freed.
 *
 * The first call on a device looks up the array's device address (a CUDA
 * runtime query, once per device, with that device current); make that first
 * call before any stream capture on the device.  After a device reset the
 * first call in the new context looks it up again, so the same rule applies
 * to it.  All calls on a device share
 * the one array and it keeps the last call's contents: calls that can
 * overlap on the GPU (other streams without ordering between them) race on
 * it; calls ordered on one stream do not.
 */
#define QSA_NOALLOC_SCRATCH_BYTES (16u << 20)
qsa_status_t qsa_select_topk_noalloc(const qsa_config_t* cfg, const qsa_segment_t* segs,
                                     int32_t n_segs, int32_t n_tokens, const float* scores,
                                     int64_t ld_scores, int32_t* sel, int32_t* nsel,
                                     void* stream);

/* Workspace bytes an operation needs for this batch (0 if none; SIZE_MAX on an
 * invalid argument).  Host-only; no CUDA call. */
size_t qsa_workspace_size(const qsa_config_t* cfg, const qsa_segment_t* segs, int32_t n_segs,
                          int32_t n_tokens, qsa_op_t op);

/* Reads and clears the current device's error word; synchronises `stream`.
 * QSA_OK if nothing was recorded; QSA_ERR_TIMEOUT if a bounded device-side
 * wait gave up; QSA_ERR_BAD_INDEX if an attention kernel (forward, union or
 * backward) met a sel entry other than the -1 padding outside
 * [0, n_cap/r): such an entry is skipped (it contributes no key) and the
 * rest of the row is attended as usual.  The first error recorded since the
 * last call wins. */
qsa_status_t qsa_device_status(void* stream);

/* Reads into *count and clears the number of query rows whose selection took
 * an exact fallback since the last call: the sampled threshold admitted too
 * few or too many candidates (a diagnostic of the selection's speed, not an
 * error; the result is exact either way).  Synchronises `stream`.
 * QSA_ERR_INVALID_ARG if count is NULL. */
qsa_status_t qsa_select_fallbacks(void* stream, int64_t* count);

/* Diagnostic for the failure path (the pages have no counterpart): enqueues
 * one kernel whose thread waits, through the same bounded wait the
 * tensor-core kernels use but with a ~0.1 s limit, on an mbarrier phase that
 * nothing completes.  The wait gives up and records QSA_ERR_TIMEOUT in the
 * device error word; no fault, no trap, the context stays usable.  A
 * following qsa_device_status() returns QSA_ERR_TIMEOUT and clears it. */
qsa_status_t qsa_selftest_wait_timeout(void* stream);

/* Static description of a status code. */
const char* qsa_status_string(qsa_status_t status);

/* Library version as major*10000 + minor*100 + patch. */
int32_t qsa_version(void);

/* Number of CUDA kernels this library has enqueued since it was loaded, in
 * this process (all devices, all streams).  Host counter; no CUDA call. */
int64_t qsa_launch_count(void);

#ifdef __cplusplus
}
#endif
#endif /* QSA_H */
