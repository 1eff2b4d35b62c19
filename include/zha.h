/*
 * zha.h -- C-ABI of libzha: the Zyphra Hierarchical Attention (ZHA) hot path
 * on NVIDIA B200 (sm_100a).
 *
 * The method (lefilia.fr page "Zyphra presente Zyphra Hierarchical Attention
 * (ZHA), une voie vers une attention vraiment sous-quadratique", paragraph 1):
 * the KV cache stays complete and a tree over it only decides which keys each
 * query reads. Keys are cut into contiguous blocks of b tokens; each block gets
 * one summary key derived from 16 learned reference queries; each higher level
 * summarises groups of b nodes of the level below (a level-l node covers b^l
 * tokens). A query scores the top nodes, keeps the fewest nodes whose
 * estimated attention mass reaches the fraction p, descends only into the
 * kept branches until it reaches individual keys, and always keeps token 0.
 * Paragraph 2 gives the operating point p = 0.95 and the two geometries
 * (b = 4, L = 6) and (b = 256, L = 1).
 *
 * Formulas the pages leave open are fixed by this library as:
 *   summary   s = (1/16) sum_r sum_c softmax_c(R_r . x_c / sqrt(d)) x_c over the
 *             node's children x_c (raw keys at level 1, stored summaries above);
 *             R is 16 x d, shared by all KV heads;
 *   node mass exp(q . s / sqrt(d) + ln b^l);
 *   causal tail: tokens of [b^L T_top(t), t] with T_top(t) = floor((t+1)/b^L)
 *             are always attended (they are not yet in a complete top node);
 *   GQA:      q head h reads KV head h / (Hq / Hkv) and selects on its own.
 * Selection uses a canonical fp32 arithmetic (sequential fmaf dot products, a
 * Cody-Waite/Taylor exponential, fixed-point masses: M = trunc(e^(z-zmax) 2^40),
 * need = ceil(T p_q / 2^32), p_q = floor(p 2^32 + 0.5), ties to the lower node
 * index), so selected index sets are reproducible bit for bit.
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers owned by the caller (for example
 *     PyTorch tensors), contiguous, 16-byte aligned. The library never
 *     allocates device memory and never synchronises the device. The only
 *     state it keeps between calls is, per device, the streams and events
 *     zha_decode forks its unit groups onto (created on its first call there)
 *     and zha_decode_noalloc's static array. Every entry point is re-entrant
 *     except zha_decode_noalloc (one array per device).
 *   - `stream` is a cudaStream_t passed as void*; every call is asynchronous on
 *     it.
 *   - Argument errors return synchronously before any launch
 *     (ZHA_ERR_INVALID_ARG / ZHA_ERR_UNSUPPORTED / ZHA_ERR_WORKSPACE).
 *     Launch failures return ZHA_ERR_CUDA. Data-dependent conditions found by a
 *     kernel (an index list longer than its capacity, a candidate list longer
 *     than the workspace) are OR-ed as zha_status bits into *dev_status (a
 *     device int32 the caller zeroes and reads after its own synchronisation);
 *     outputs are then truncated safely. No kernel traps or asserts.
 *   - dtype ZHA_BF16: K, V, Q, outputs and stored summaries are bf16.
 *     dtype ZHA_F32: all of them are fp32. R is always fp32.
 *   - Layouts (row-major):
 *       K, V       [batch][n_kv_heads][capacity][head_dim]
 *       summaries  level l (1..L) starts at element level_offsets[l-1] of
 *                  `tree` and is [batch][n_kv_heads][capacity / b^l][head_dim];
 *                  node (l, j) covers tokens [j b^l, (j+1) b^l)
 *       decode Q   [batch][n_q_heads][head_dim], query position seq_len[s]-1
 *       outputs    same shape as their queries
 *       level_counts [query][q head][L], kept node counts, top level first
 */
#ifndef ZHA_H
#define ZHA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum zha_status {
  ZHA_OK = 0,
  ZHA_ERR_INVALID_ARG = 1,   /* null pointer, bad size or geometry, p out of range */
  ZHA_ERR_UNSUPPORTED = 2,   /* valid but not implemented (e.g. head_dim not 64/128) */
  ZHA_ERR_CUDA = 4,          /* a launch or runtime call failed */
  ZHA_ERR_CAPACITY = 8,      /* device status bit: an index list hit idx_cap */
  ZHA_ERR_WORKSPACE = 16,    /* workspace smaller than zha_workspace_bytes() */
  ZHA_ERR_TIMEOUT = 32,      /* device status bit: a bounded wait gave up */
  ZHA_ERR_INTERNAL = 64      /* device status bit: an internal consistency check failed */
} zha_status;

typedef enum zha_dtype { ZHA_F32 = 0, ZHA_BF16 = 1 } zha_dtype;

typedef enum zha_op {
  ZHA_OP_SELECT = 0,
  ZHA_OP_ATTEND = 1,
  ZHA_OP_DECODE = 2,
  ZHA_OP_PREFILL = 3,
  ZHA_OP_DENSE = 4
} zha_op;

/* Geometry and shapes. b (block) >= 2 and either divides 32 or is a multiple
 * of 32 up to 1024; 1 <= levels <= 8; head_dim 64 or 128; n_q_heads a multiple
 * of n_kv_heads with at most 8 query heads per KV head. */
typedef struct zha_config {
  int32_t head_dim;   /* d */
  int32_t block;      /* b */
  int32_t levels;     /* L */
  int32_t n_q_heads;  /* Hq */
  int32_t n_kv_heads; /* Hkv */
  int32_t batch;      /* B */
  int64_t capacity;   /* rows per (sequence, KV head) in K and V */
  int32_t dtype;      /* zha_dtype */
  int32_t reserved;   /* must be 0 */
} zha_config;

/* The cache a call works on. k, v, r are read-only; tree is written by the
 * build/extend calls and read by the others; seq_len[b] (device int32) is the
 * number of valid tokens of sequence b. */
typedef struct zha_cache {
  const void* k;
  const void* v;
  const float* r;          /* [16][head_dim] learned reference queries */
  void* tree;              /* summaries, see layout above */
  const int32_t* seq_len;  /* [batch], device */
} zha_cache;

/* Human-readable name of a status value (or of the lowest set bit). */
const char* zha_status_string(int32_t status);

/* Host-only query: bytes of the summary tree and the element offset of each
 * level (level_offsets[l-1] for l = 1..L; may be NULL). */
zha_status zha_tree_layout(const zha_config* cfg, size_t* tree_bytes, int64_t* level_offsets);

/* Host-only query: workspace bytes the given operation needs for up to
 * max_queries query tokens (decode/dense: ignored, the batch is used; prefill:
 * the chunk length T). */
zha_status zha_workspace_bytes(const zha_config* cfg, int32_t op, int64_t max_queries,
                               size_t* bytes);

/* Build every complete node of every level for the first seq_len[b] tokens of
 * each sequence (lefilia.fr page, par. 1: blocks are summarised, then each
 * higher level summarises groups of b nodes below). Nodes that are not
 * complete are left untouched. */
zha_status zha_build_tree(const zha_config* cfg, const zha_cache* cache, void* stream);

/* Build exactly the nodes that became complete when sequence b grew from
 * old_len[b] (device int32) to seq_len[b] tokens (lefilia.fr page, par. 1:
 * the tree covers the whole cache, so a node is summarised as soon as its b
 * children exist; the summary formula above is the same one the build uses).
 * max_new_tokens is a host
 * upper bound on seq_len[b] - old_len[b] over all b (it sizes the launch);
 * growth beyond it is left unbuilt. */
zha_status zha_extend_tree(const zha_config* cfg, const zha_cache* cache, const int32_t* old_len,
                           int64_t max_new_tokens, void* stream);

/* Top-p traversal (lefilia.fr page, par. 1) for nq query tokens with all Hq
 * heads each: q [nq][Hq][d]; token i belongs to sequence q_seq[i] at position
 * q_pos[i] (device int32 arrays, q_pos[i] < seq_len[q_seq[i]]). For query
 * (i, h) the ascending selected token list
 *   S = tokens of kept level-1 nodes U {0} U [b^L T_top, t]
 * is written to idx + (i*Hq + h)*idx_cap, its length to n_idx[i*Hq + h] and
 * the kept node counts per level to level_counts (nullable). p in (0, 1];
 * p >= 1 keeps every candidate. Lists longer than idx_cap are truncated and
 * set ZHA_ERR_CAPACITY in *dev_status. ws/ws_bytes: ZHA_OP_SELECT workspace. */
zha_status zha_select(const zha_config* cfg, const zha_cache* cache, const void* q,
                      const int32_t* q_seq, const int32_t* q_pos, int64_t nq, double p,
                      int32_t* idx, int64_t idx_cap, int32_t* n_idx, int32_t* level_counts,
                      void* ws, size_t ws_bytes, int32_t* dev_status, void* stream);

/* Exact softmax attention of each query (i, h) over its list idx/n_idx (as
 * written by zha_select, ascending token positions of sequence q_seq[i])
 * (lefilia.fr page, par. 1: after the descent the query attends exactly over
 * the raw K/V entries it selected; the cache itself is never pruned):
 * out[i][h] = sum_j softmax_j(q . k_j / sqrt(d)) v_j. fp32 accumulation.
 * ws/ws_bytes: ZHA_OP_ATTEND workspace for nq queries. */
zha_status zha_attend(const zha_config* cfg, const zha_cache* cache, const void* q,
                      const int32_t* q_seq, int64_t nq, const int32_t* idx, int64_t idx_cap,
                      const int32_t* n_idx, void* out, void* ws, size_t ws_bytes,
                      int32_t* dev_status, void* stream);

/* One decode step for every sequence (lefilia.fr page, par. 1 and 2: the
 * top-p descent at p = 0.95 followed by exact attention over the selected raw
 * keys, token 0 and the causal tail): selection at position seq_len[b] - 1
 * followed by attention over the selected keys, q [B][Hq][d] -> out [B][Hq][d].
 * The query heads sharing a KV head share every read: each summary row is
 * scored for all of them in one pass (every row under the complete top nodes,
 * while that prefix is at most 1.5 GB; above it the cluster traversal of
 * zha_select scores the union of their frontiers), each head then cuts its own
 * frontier, and the K/V rows of their kept nodes are read once with per-head
 * masks. level_counts is
 * nullable. The tree must already contain every node complete at seq_len
 * (call zha_extend_tree after appending tokens). ws: ZHA_OP_DECODE workspace.
 * Streams: the (sequence, KV head) units are split into up to 4 groups whose
 * kernels run on streams of decreasing priority that the library creates
 * once per device (forked from `stream` by an event and joined back into it
 * before the call returns), so that one group's cut overlaps the other
 * groups' scoring and attention. Work queued on `stream` after the call
 * waits for all of it, and the call can be captured into a CUDA graph; the
 * streams are created by the first call on a device that is not being
 * captured (until then the call runs on `stream` alone). Outputs equal those
 * of zha_decode_select followed by zha_decode_attend bit for bit. */
zha_status zha_decode(const zha_config* cfg, const zha_cache* cache, const void* q, double p,
                      void* out, int32_t* level_counts, void* ws, size_t ws_bytes,
                      int32_t* dev_status, void* stream);

/* The two halves of zha_decode on `stream` alone, for callers that schedule
 * or time them separately. zha_decode_select runs the selection for every
 * sequence and leaves the kept level-1 nodes (union over the query heads of
 * each KV head, with per-head masks) in ws; zha_decode_attend then attends
 * over them. Both must get the same cfg, cache, q and ws; nothing may touch
 * ws in between. */
zha_status zha_decode_select(const zha_config* cfg, const zha_cache* cache, const void* q,
                             double p, int32_t* level_counts, void* ws, size_t ws_bytes,
                             int32_t* dev_status, void* stream);
zha_status zha_decode_attend(const zha_config* cfg, const zha_cache* cache, const void* q,
                             void* out, void* ws, size_t ws_bytes, void* stream);

/* Work counters of the last zha_decode / zha_decode_select on ws, written to
 * the device int32 array stats[B * Hkv][L + 1]: for each (sequence, KV head),
 * the number of distinct nodes scored at levels L..1 (union over its query
 * heads; each costs one summary-row read) followed by the number of distinct
 * kept level-1 nodes (each costs b K rows and b V rows). Asynchronous. */
zha_status zha_decode_stats(const zha_config* cfg, const void* ws, size_t ws_bytes,
                            int32_t* stats, void* stream);

/* Chunked prefill of sequence `seq` (lefilia.fr page, par. 1: every query of
 * the chunk descends the tree on its own and attends its selected keys,
 * restricted causally to keys at or before its position): the caller has
 * written the chunk's K and V rows [chunk_start, chunk_start + T) and set
 * seq_len[seq] = chunk_start + T.
 * Extends the tree over the chunk, then for every token i of the chunk
 * (position chunk_start + i) and head h selects causally and attends:
 * q [T][Hq][d] -> out [T][Hq][d]. level_counts ([T][Hq][L]) is nullable.
 * ws: ZHA_OP_PREFILL workspace for max_queries = T.
 * The top level of every (token, head) is first scored on the tensor cores
 * (zha_prefill_top_scores) when the geometry allows it; a (token, KV head)
 * whose tensor-core selection is certified skips the top level's canonical
 * scoring. Certified or not, every selection equals the canonical one. If
 * the tensor-core completion wait runs out (bounded at 1 s), dev_status gets
 * ZHA_ERR_TIMEOUT, no unit is certified and the top level is scored
 * canonically: the results stay exact. */
zha_status zha_prefill_chunk(const zha_config* cfg, const zha_cache* cache, const void* q,
                             int32_t seq, int64_t chunk_start, int64_t T, double p, void* out,
                             int32_t* level_counts, void* ws, size_t ws_bytes,
                             int32_t* dev_status, void* stream);

/* Tensor-core top-level scores of a prefill chunk and their certificates
 * (lefilia page, par. 1: a query scores the top nodes first; in a chunk all
 * (token, head) queries of a KV head score the same top summaries, so this is
 * one bf16 GEMM per KV head on tcgen05 with fp32 accumulation in TMEM).
 *   - Input: the tree must already cover the chunk (zha_prefill_chunk extends
 *     it; or zha_build_tree / zha_extend_tree); q [T][Hq][d] as in
 *     zha_prefill_chunk, 16-byte aligned; positions chunk_start + i.
 *   - z_top (nullable, device): [T][Hq][capacity / b^L] fp32; entry [i][h][n]
 *     is the tensor-core score fl(fl(acc * 1/sqrt(d)) + L ln b) of top node n
 *     for n < T_top(i) = (chunk_start + i + 1) / b^L; later entries untouched.
 *     It differs from the canonical score by at most a bound derived from
 *     |q| |s_n| (no rounding-order guarantee).
 *   - certified (nullable, device): [T][Hq] int32, 1 when the canonical cut
 *     over the top level is proven equal to the cut taken on z_top (the proof
 *     is the same one zha_prefill_chunk relies on), else 0. All 0 after a
 *     ZHA_ERR_TIMEOUT, when z_top is not written.
 *   - ws: ZHA_OP_PREFILL workspace for max_queries >= T (not preserved).
 *   - Errors: ZHA_ERR_UNSUPPORTED unless dtype is bf16, head_dim 128, L >= 2,
 *     G <= 8 and capacity / b^L <= 1024; ZHA_ERR_INVALID_ARG for a bad chunk,
 *     p or a misaligned q; ZHA_ERR_TIMEOUT in dev_status if the tensor-core
 *     completion wait ran out. Asynchronous on `stream`. */
zha_status zha_prefill_top_scores(const zha_config* cfg, const zha_cache* cache, const void* q,
                                  int32_t seq, int64_t chunk_start, int64_t T, double p,
                                  float* z_top, int32_t* certified, void* ws, size_t ws_bytes,
                                  int32_t* dev_status, void* stream);

/* Dense flash-decoding over every key [0, seq_len[b] - 1] (the baseline the
 * sparse path is measured against; lefilia.fr page, par. 2 and 4 compare the
 * method with dense attention): q [B][Hq][d] -> out [B][Hq][d].
 * ws: ZHA_OP_DENSE workspace. */
zha_status zha_dense_decode(const zha_config* cfg, const zha_cache* cache, const void* q,
                            void* out, void* ws, size_t ws_bytes, void* stream);

/* The token list each query head of the last zha_decode / zha_decode_select
 * on ws attends (lefilia.fr page, par. 1: the raw keys under the kept
 * level-1 nodes, plus the first token; the causal tail is the task's rule):
 * for sequence s and head h, idx + (s*Hq + h)*idx_cap receives, ascending,
 *   {0} U tokens of the level-1 nodes kept by h U [b^L T_top, seq_len[s] - 1]
 * -- exactly the K/V rows zha_decode_attend reads for that head -- and
 * n_idx[s*Hq + h] its length. It reads the kept level-1 node union and the
 * per-head masks the traversal left in ws, so it must get the same cfg and
 * cache (seq_len) and run after that selection with nothing touching ws in
 * between. Lists longer than idx_cap are truncated and set ZHA_ERR_CAPACITY
 * in *dev_status (nullable). idx, n_idx device int32. Asynchronous. */
zha_status zha_decode_kept_lists(const zha_config* cfg, const zha_cache* cache, const void* ws,
                                 size_t ws_bytes, int32_t* idx, int64_t idx_cap, int32_t* n_idx,
                                 int32_t* dev_status, void* stream);

/* ---- FP4 router variant (lefilia.fr page, par. 4: a 4-bit variant of the
 * router was tried; the page gives no format) ----------------------------
 * A block-scaled 4-bit copy of the summary tree, scored in place of the
 * tree's rows by the decode selection; everything else of the step (cut,
 * union, attention over the raw K/V) is unchanged. Format: every block of
 * 32 consecutive elements of a stored summary row becomes 4-bit codes --
 * bit 3 the sign, bits 0-2 the index k of the magnitude in
 * {0, 0.5, 1, 1.5, 2, 3, 4, 6} (the e2m1 encoding) -- and one exponent e:
 * value = sign * mag[k] * 2^e, with e the smallest integer such that the
 * block's largest magnitude is at most 6 * 2^e (0 for an all-zero block),
 * each |x| / 2^e rounded to the nearest magnitude, an exact tie to the even
 * k, zeros stored with sign 0. A 256-byte bf16 row (d = 128) becomes 64
 * bytes of codes and 8 bytes of exponents. The selection this gives is a
 * labelled variant of the canonical one (it scores rounded summaries);
 * scoring itself is the canonical fp32 chain over the exact 4-bit values.
 * Layout of the copy: the code of tree element i (element order and
 * level_off as zha_tree_layout) in byte i/2, the low nibble for even i; the
 * int16 exponent of block i/32 at byte codes_bytes + 2*(i/32), codes_bytes =
 * tree_elems/2 rounded up to a multiple of 256. */

/* Bytes of the FP4 copy of a tree of this configuration. */
zha_status zha_fp4_tree_bytes(const zha_config* cfg, size_t* bytes);

/* Writes the FP4 copy (device buffer of zha_fp4_tree_bytes) of the rows of
 * every node complete at seq_len, or, with old_len (device int32 [B],
 * nullable), of the nodes completed in (old_len[b], seq_len[b]] -- call it
 * after zha_build_tree / zha_extend_tree with the same old_len. The tree
 * itself is read only. Asynchronous on stream. */
zha_status zha_fp4_quantize_tree(const zha_config* cfg, const zha_cache* cache, void* fp4_tree,
                                 const int32_t* old_len, void* stream);

/* zha_decode with the selection scored on the FP4 copy fp4_tree (kept up to
 * date with zha_fp4_quantize_tree): same arguments, workspace
 * (ZHA_OP_DECODE), streams, outputs and errors as zha_decode, plus
 * ZHA_ERR_UNSUPPORTED unless head_dim is 128 and the step takes the dense
 * decode selection (the tree prefix under the complete top nodes is at
 * most 1.5 GB and a head's cut state fits shared memory). zha_decode_stats
 * and zha_decode_kept_lists read its workspace as after zha_decode. */
zha_status zha_decode_fp4(const zha_config* cfg, const zha_cache* cache, const void* fp4_tree,
                          const void* q, double p, void* out, int32_t* level_counts, void* ws,
                          size_t ws_bytes, int32_t* dev_status, void* stream);

/* zha_decode without a caller workspace. The pages describe no counterpart of
 * this call; it exists for callers that cannot hand the library a workspace --
 * plugins loaded by a host that owns the device allocator and exposes none of
 * it, and hot paths where an allocation is not allowed (cudaMalloc and
 * cudaFree synchronise the device). It computes exactly what zha_decode
 * computes, using as its workspace a 64 MiB array in the library's static
 * device memory instead of ws; nothing is allocated by the call.
 *   - Limit: geometries whose ZHA_OP_DECODE workspace (zha_workspace_bytes)
 *     exceeds 64 MiB are rejected with ZHA_ERR_WORKSPACE before any launch
 *     (for example B = 1, Hkv = 2, G = 8, b = 4, L = 6 fits up to about 2.19M
 *     tokens).
 *   - Set-up: the first call on each device looks up the array's device
 *     address (this loads its module on that device); make that first call
 *     with the device current and outside any stream capture. The address is
 *     kept for the process, so the device must not be reset (cudaDeviceReset,
 *     or its primary context destroyed) between calls.
 *   - Memory: the 64 MiB are held on each device until the process exits.
 *     Under the default lazy module loading only devices this entry point
 *     ran on hold them; with CUDA_MODULE_LOADING=EAGER every process that
 *     loads libzha holds them on every device it uses.
 *   - The scratch needs no clearing: every word is written before it is read.
 *   - Every launch runs on `stream` itself: unlike zha_decode, this call uses
 *     no streams or events of the library's own.
 *   - Unlike the other entry points this one is NOT re-entrant: every call on
 *     a device shares the one array, so two calls whose executions overlap
 *     (different streams, or different host threads, without ordering between
 *     them) race and corrupt each other's results. Order them on one stream or
 *     with events.
 * Arguments, layouts, dev_status and errors are those of zha_decode. */
zha_status zha_decode_noalloc(const zha_config* cfg, const zha_cache* cache, const void* q,
                              double p, void* out, int32_t* level_counts, int32_t* dev_status,
                              void* stream);

#ifdef __cplusplus
}
#endif

#endif /* ZHA_H */
