// Host-side internal interfaces of libzha (not part of the public C-ABI).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/zha.h"

namespace zha {

constexpr int kMaxLevelsHost = 8;
constexpr int kMaxClusterHost = 16;  // upper bound of traverse_cluster_size()

// Geometry derived once per call from a zha_config.
struct Geometry {
  int d, b, L, Hq, Hkv, B, G;
  int64_t ncap;
  int dtype;               // zha_dtype
  int64_t span[kMaxLevelsHost + 1];        // b^l, l = 0..L
  int64_t level_rows[kMaxLevelsHost];      // rows per unit of level l at index l-1
  int64_t level_off[kMaxLevelsHost];       // element offset of level l at index l-1
  int64_t tree_elems;
  float inv_sqrt_d;
  float lnsize[kMaxLevelsHost];            // fp32(l ln b) at index l-1
  int elem_bytes;
};

zha_status make_geometry(const zha_config* cfg, Geometry* g);

// ---- tree build -----------------------------------------------------------
// old_len == nullptr builds every complete node; otherwise nodes completed in
// (old_len, seq_len]. max_new_tokens < 0 means "whole sequence".
cudaError_t launch_tree(const Geometry& g, const void* k, void* tree, const float* r,
                        const int32_t* seq_len, const int32_t* old_len, int64_t max_new_tokens,
                        cudaStream_t stream);

// ---- traversal ------------------------------------------------------------
struct TraverseOut {
  // decode mode: per unit, the union of kept level-1 nodes with per-head masks,
  // as C ordered segments (C = traverse_cluster_size) of traverse_kept_stride
  uint32_t* kept;          // [units][C][stride] packed (mask << 24) | node
  int32_t* n_kept;         // [units][C]
  // list mode: per query head, the selected token list
  int32_t* idx;            // [nq][Hq][idx_cap]
  int64_t idx_cap;
  int32_t* n_idx;          // [nq][Hq]
  int32_t* level_counts;   // [nq][Hq][L] (nullable)
  int32_t* stats;          // [units][L] union candidates per level (nullable)
};

// Certified top-level selections (prefill, tensor-core scoring) of `units`
// (query token, KV head) units, indexed like the traversal's units. When
// ok[u] != 0 the canonical cut of every head of unit u at the top level is
// known: mask[u][i] bit h says head h keeps top node i, cnt[u][h] counts them.
struct TopSeeds {
  const int32_t* ok;    // [units]
  const uint8_t* mask;  // [units][stride]
  const int32_t* cnt;   // [units][G]
  int64_t stride;
};

// CTAs per traversal cluster for `units` (query token, KV head) units.
int traverse_cluster_size(const Geometry& g, int64_t units, int num_sms);
// Scratch bytes of the traversal (candidate segments, scores, keep bits).
size_t traverse_ws_bytes(const Geometry& g, int64_t units, int num_sms);
// Bytes of the decode-mode kept list and its per-segment stride (entries).
size_t traverse_kept_bytes(const Geometry& g, int64_t units, int num_sms);
int64_t traverse_kept_stride(const Geometry& g);

// Decode mode (q_pos == nullptr): query token = sequence s at position
// seq_len[s]-1, q [B][Hq][d]. Otherwise query token i at (q_seq[i], q_pos[i]),
// q [nq][Hq][d]. list_mode selects the per-head index-list output.
cudaError_t launch_traverse(const Geometry& g, const void* tree, const void* q,
                            const int32_t* seq_len, const int32_t* q_seq, const int32_t* q_pos,
                            int64_t nq, uint64_t p_q, int list_mode, const TraverseOut& out,
                            void* ws, size_t ws_bytes, int32_t* status, int num_sms,
                            cudaStream_t stream, const TopSeeds* seeds = nullptr);

// ---- decode selection with every summary row scored up front ---------------
// True when a decode step of `units` (sequence, KV head) units takes this path
// (its shared-memory state fits and the tree prefix it reads is bounded).
bool decode_dense_ok(const Geometry& g, int64_t units);
size_t decode_dense_ws_bytes(const Geometry& g, int64_t units);
// Decode mode only (query of sequence s at seq_len[s] - 1): writes the kept
// level-1 union with per-head masks in `segs` ordered segments per unit, the
// per-head level counts (nullable) and the rows scored per level (stats).
// Units [unit0, unit0 + n_units) only when n_units > 0. fp4_tree (nullable,
// d = 128): score the FP4 router variant's 4-bit rows instead of the tree's.
cudaError_t launch_decode_dense(const Geometry& g, const void* tree, const void* q,
                                const int32_t* seq_len, uint64_t p_q, void* ws,
                                int32_t* level_counts, int32_t* stats, uint32_t* kept,
                                int32_t* n_kept, int64_t kept_stride, int segs, int32_t* status,
                                int num_sms, cudaStream_t stream, int64_t unit0 = 0,
                                int64_t n_units = 0, const void* fp4_tree = nullptr);

// ---- FP4 router variant: block-scaled 4-bit copy of the tree ------------------
// Layout: codes of tree element i in byte i / 2 (low nibble for even i), then
// at fp4_codes_bytes the int16 exponent of block i / 32 (32 elements).
size_t fp4_codes_bytes(const Geometry& g);
size_t fp4_tree_bytes(const Geometry& g);
// Quantizes the rows of every node complete at seq_len (old_len null) or
// completed in (old_len, seq_len].
cudaError_t launch_fp4_quantize(const Geometry& g, const void* tree, void* fp4,
                                const int32_t* seq_len, const int32_t* old_len, int num_sms,
                                cudaStream_t stream);

// ---- prefill top level on the tensor cores ----------------------------------
// Top nodes per (sequence, KV head): ncap / b^L.
int64_t top_cap(const Geometry& g);
// bf16, head_dim 128, L >= 2, at most 8 query heads per KV head and 1024 top nodes.
bool top_tc_supported(const Geometry& g);
// Scratch of launch_top_select for n_tok query tokens (0 when unsupported).
size_t top_tc_ws_bytes(const Geometry& g, int64_t n_tok);
// Scores the top level of n_tok consecutive query tokens of sequence `seq`
// (positions pos0 .., q [n_tok][Hq][d]) on the tensor cores and certifies each
// (token, KV head) unit; *seeds points into ws afterwards. z_out ([n_tok][Hq]
// [top_cap]) and cert_out ([n_tok][Hq]) are optional diagnostics.
cudaError_t launch_top_select(const Geometry& g, const void* tree, const int32_t* seq_len,
                              int seq, const void* q, int64_t pos0, int64_t n_tok, uint64_t p_q,
                              void* ws, size_t ws_bytes, TopSeeds* seeds, float* z_out,
                              int32_t* cert_out, int32_t* status, cudaStream_t stream);

// ---- attention ------------------------------------------------------------
enum StreamKind { kStreamTree = 0, kStreamDense = 1, kStreamList = 2 };

struct AttendArgs {
  int kind;                      // StreamKind
  const void* k;
  const void* v;
  const void* q;                 // tree/dense: [B][Hq][d]; list: [nq][Hq][d]
  void* out;                     // same shape as q
  const int32_t* seq_len;        // [B]
  const int32_t* q_seq;          // list mode / explicit positions: [nq]
  const int32_t* q_pos;          // tree stream with explicit positions (prefill), else null
  int64_t nq;                    // query tokens (decode/dense: B)
  // tree stream: kept level-1 nodes as kept_segs ordered segments per unit
  const uint32_t* kept;          // [units][kept_segs][kept_stride]
  const int32_t* n_kept;         // [units][kept_segs]
  int64_t kept_stride;
  int kept_segs;
  // list stream
  const int32_t* idx;
  int64_t idx_cap;
  const int32_t* n_idx;
  // units [unit0, unit0 + n_units) only (n_units 0: all); the split count
  // stays that of the whole launch, so a range's outputs equal the whole's
  int64_t unit0;
  int64_t n_units;
};

size_t attend_ws_bytes(const Geometry& g, int kind, int64_t nq, int num_sms);

cudaError_t launch_attend(const Geometry& g, const AttendArgs& a, void* ws, size_t ws_bytes,
                          int num_sms, cudaStream_t stream);

// Prefill attention of a tile of n consecutive query tokens of sequence `seq`
// (positions pos0 ..): all tokens' rows of a KV head share each K/V block on
// tensor cores, masked by the traversal's kept level-1 lists (decode-mode
// output of launch_traverse for the same tile).
bool tile_attend_supported(const Geometry& g);
int64_t tile_map_stride(const Geometry& g);
size_t tile_attend_ws_bytes(const Geometry& g, int64_t n, int num_sms);
cudaError_t launch_attend_tile(const Geometry& g, const void* k, const void* v,
                               const int32_t* seq_len, int seq, int64_t pos0, int64_t n,
                               const void* q, void* out, const uint32_t* kept,
                               const int32_t* n_kept, int64_t kept_stride, int kept_segs,
                               void* ws, size_t ws_bytes, int num_sms, cudaStream_t stream);

// Decode mode: each query head's token list (token 0, the tokens of the kept
// level-1 nodes whose mask has the head's bit, the causal tail) from the
// traversal's kept segments; idx [B][Hq][idx_cap], n_idx [B][Hq].
cudaError_t launch_kept_lists(const Geometry& g, const uint32_t* kept, const int32_t* n_kept,
                              int64_t stride, int segs, const int32_t* seq_len, int32_t* idx,
                              int64_t idx_cap, int32_t* n_idx, int32_t* status,
                              cudaStream_t stream);

int device_sm_count();

// zha_decode with every launch on the caller's stream (no streams or events of
// the library's own); the same outputs as zha_decode.
zha_status decode_one_stream(const zha_config* cfg, const zha_cache* cache, const void* q,
                             double p, void* out, int32_t* level_counts, void* ws,
                             size_t ws_bytes, int32_t* dev_status, void* stream);

}  // namespace zha
