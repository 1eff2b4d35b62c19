// libzha C-ABI entry points: argument validation, workspace layout, dispatch.
// Every declaration lives in include/zha.h, which documents meaning, layout,
// ownership and error behaviour of each argument.
#include <cuda_runtime.h>
#include <math.h>
#include <string.h>

#include <mutex>

#include "zha_internal.h"

namespace zha {

static bool pow2_le8(int g) { return g == 1 || g == 2 || g == 4 || g == 8; }

zha_status make_geometry(const zha_config* cfg, Geometry* g) {
  if (!cfg || !g) return ZHA_ERR_INVALID_ARG;
  memset(g, 0, sizeof(*g));
  if (cfg->reserved != 0) return ZHA_ERR_INVALID_ARG;
  if (cfg->dtype != ZHA_F32 && cfg->dtype != ZHA_BF16) return ZHA_ERR_INVALID_ARG;
  if (cfg->head_dim != 64 && cfg->head_dim != 128) return ZHA_ERR_UNSUPPORTED;
  const int b = cfg->block;
  const bool small_b = b >= 2 && b <= 32 && (32 % b) == 0;
  const bool large_b = b >= 64 && b <= 1024 && (b % 32) == 0;
  if (!small_b && !large_b) return ZHA_ERR_UNSUPPORTED;
  if (cfg->levels < 1 || cfg->levels > kMaxLevelsHost) return ZHA_ERR_INVALID_ARG;
  if (cfg->n_kv_heads < 1 || cfg->n_q_heads < 1 || cfg->n_q_heads % cfg->n_kv_heads)
    return ZHA_ERR_INVALID_ARG;
  if (!pow2_le8(cfg->n_q_heads / cfg->n_kv_heads)) return ZHA_ERR_UNSUPPORTED;
  if (cfg->batch < 1 || cfg->capacity < 1) return ZHA_ERR_INVALID_ARG;
  g->d = cfg->head_dim;
  g->b = b;
  g->L = cfg->levels;
  g->Hq = cfg->n_q_heads;
  g->Hkv = cfg->n_kv_heads;
  g->B = cfg->batch;
  g->G = cfg->n_q_heads / cfg->n_kv_heads;
  g->ncap = cfg->capacity;
  g->dtype = cfg->dtype;
  g->elem_bytes = cfg->dtype == ZHA_BF16 ? 2 : 4;
  g->span[0] = 1;
  for (int l = 1; l <= g->L; ++l) {
    g->span[l] = g->span[l - 1] * b;
    if (g->span[l] > ((int64_t)1 << 40)) return ZHA_ERR_INVALID_ARG;
  }
  // node ids travel in 24 bits next to an 8-bit head mask
  if (g->ncap / b + 1 >= ((int64_t)1 << 24)) return ZHA_ERR_UNSUPPORTED;
  int64_t off = 0;
  for (int l = 1; l <= g->L; ++l) {
    g->level_rows[l - 1] = g->ncap / g->span[l];
    g->level_off[l - 1] = off;
    off += (int64_t)g->B * g->Hkv * g->level_rows[l - 1] * g->d;
    g->lnsize[l - 1] = (float)((double)l * log((double)b));
  }
  g->tree_elems = off;
  g->inv_sqrt_d = (float)(1.0 / sqrt((double)g->d));
  return ZHA_OK;
}

int device_sm_count() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return 148;
  }
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
    cudaGetLastError();
    return 148;
  }
  return n;
}

static size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

static int check_p(double p, uint64_t* p_q) {
  if (!(p > 0.0)) return 0;  // also rejects NaN
  const double pc = p >= 1.0 ? 1.0 : p;
  *p_q = (uint64_t)floor(pc * 4294967296.0 + 0.5);
  return *p_q >= 1;
}

static zha_status cuda_status(cudaError_t e) { return e == cudaSuccess ? ZHA_OK : ZHA_ERR_CUDA; }

// ---- workspace layouts ----------------------------------------------------

struct DecodeLayout {
  size_t trav, kept, n_kept, stats, part, total;
  int64_t units;
  bool dense;  // selection by decode_dense (decode steps), else the frontier traversal
  int groups;  // unit groups of a decode step
};

// Unit groups of a decode step on the dense path (see run_decode_step).
#ifndef ZHA_DECODE_GROUPS
#define ZHA_DECODE_GROUPS 4
#endif
constexpr int kDecodeGroups = ZHA_DECODE_GROUPS;
constexpr int kMinUnitsPerGroup = 2;

static int decode_groups(bool dense, int64_t units) {
  if (!dense) return 1;
  int64_t k = units / kMinUnitsPerGroup;
  if (k > kDecodeGroups) k = kDecodeGroups;
  return k < 1 ? 1 : (int)k;
}

// dense: the caller is a decode step (one query per sequence at seq_len - 1)
static DecodeLayout decode_layout(const Geometry& g, int64_t nq, int kind, int sms,
                                  bool decode = false) {
  DecodeLayout L{};
  L.units = nq * g.Hkv;
  L.dense = decode && decode_dense_ok(g, L.units);
  L.groups = decode_groups(L.dense, L.units);
  size_t off = 0;
  L.trav = off;
  off = align256(off + (L.dense ? decode_dense_ws_bytes(g, L.units)
                                : traverse_ws_bytes(g, L.units, sms)));
  L.kept = off;
  off = align256(off + traverse_kept_bytes(g, L.units, sms));
  L.n_kept = off;
  off = align256(off + sizeof(int32_t) * (size_t)L.units * kMaxClusterHost);
  L.stats = off;
  off = align256(off + sizeof(int32_t) * (size_t)L.units * g.L);
  L.part = off;
  off = align256(off + attend_ws_bytes(g, kind, nq, sms));
  L.total = off;
  return L;
}

// Prefill processes the chunk in tiles of query tokens sized to fill the GPU.
static int64_t prefill_tile(const Geometry& g, int64_t T, int sms) {
  int64_t t = (2 * (int64_t)sms) / g.Hkv;
  if (t < 1) t = 1;
  if (t > T) t = T;
  return t;
}

struct PrefillLayout {
  size_t old_len, q_seq, q_pos, dec, top, top_bytes, tatt, tatt_bytes, total;
  int64_t tile;
  DecodeLayout d;
};

static PrefillLayout prefill_layout(const Geometry& g, int64_t T, int sms) {
  PrefillLayout P{};
  P.tile = prefill_tile(g, T, sms);
  size_t off = 0;
  P.old_len = off;
  off = align256(off + sizeof(int32_t) * (size_t)g.B);
  P.q_seq = off;
  off = align256(off + sizeof(int32_t) * (size_t)P.tile);
  P.q_pos = off;
  off = align256(off + sizeof(int32_t) * (size_t)P.tile);
  P.dec = off;
  P.d = decode_layout(g, P.tile, kStreamTree, sms);
  off = align256(off + P.d.total);
  // tensor-core top level of the whole chunk (scores, certificates, seeds)
  P.top = off;
  P.top_bytes = top_tc_ws_bytes(g, T);
  off = align256(off + P.top_bytes);
  // tile attention (keep map and split partials of one query tile)
  P.tatt = off;
  P.tatt_bytes = tile_attend_ws_bytes(g, P.tile, sms);
  off = align256(off + P.tatt_bytes);
  P.total = off;
  return P;
}

__global__ void fill_prefill_kernel(int32_t* old_len, const int32_t* seq_len, int B, int seq,
                                    int64_t chunk_start) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < B) old_len[i] = (i == seq) ? (int32_t)chunk_start : seq_len[i];
}

__global__ void fill_positions_kernel(int32_t* q_seq, int32_t* q_pos, int seq, int64_t start,
                                      int64_t count) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i < count) {
    q_seq[i] = seq;
    q_pos[i] = (int32_t)(start + i);
  }
}

}  // namespace zha

using namespace zha;

extern "C" {

const char* zha_status_string(int32_t status) {
  if (status == ZHA_OK) return "ok";
  if (status & ZHA_ERR_INVALID_ARG) return "invalid argument";
  if (status & ZHA_ERR_UNSUPPORTED) return "unsupported configuration";
  if (status & ZHA_ERR_CUDA) return "CUDA error";
  if (status & ZHA_ERR_CAPACITY) return "index list capacity exceeded";
  if (status & ZHA_ERR_WORKSPACE) return "workspace too small";
  if (status & ZHA_ERR_TIMEOUT) return "bounded wait timed out";
  if (status & ZHA_ERR_INTERNAL) return "internal consistency check failed";
  return "unknown status";
}

zha_status zha_tree_layout(const zha_config* cfg, size_t* tree_bytes, int64_t* level_offsets) {
  Geometry g;
  zha_status st = make_geometry(cfg, &g);
  if (st != ZHA_OK) return st;
  if (tree_bytes) *tree_bytes = (size_t)g.tree_elems * g.elem_bytes;
  if (level_offsets)
    for (int l = 0; l < g.L; ++l) level_offsets[l] = g.level_off[l];
  return ZHA_OK;
}

zha_status zha_workspace_bytes(const zha_config* cfg, int32_t op, int64_t max_queries,
                               size_t* bytes) {
  Geometry g;
  zha_status st = make_geometry(cfg, &g);
  if (st != ZHA_OK) return st;
  if (!bytes) return ZHA_ERR_INVALID_ARG;
  const int sms = device_sm_count();
  switch (op) {
    case ZHA_OP_SELECT:
      if (max_queries < 1) return ZHA_ERR_INVALID_ARG;
      *bytes = align256(traverse_ws_bytes(g, max_queries * g.Hkv, sms));
      return ZHA_OK;
    case ZHA_OP_ATTEND:
      if (max_queries < 1) return ZHA_ERR_INVALID_ARG;
      *bytes = align256(attend_ws_bytes(g, kStreamList, max_queries, sms));
      return ZHA_OK;
    case ZHA_OP_DECODE:
      *bytes = decode_layout(g, g.B, kStreamTree, sms, true).total;
      return ZHA_OK;
    case ZHA_OP_DENSE:
      *bytes = align256(attend_ws_bytes(g, kStreamDense, g.B, sms));
      return ZHA_OK;
    case ZHA_OP_PREFILL:
      if (max_queries < 1) return ZHA_ERR_INVALID_ARG;
      *bytes = prefill_layout(g, max_queries, sms).total;
      return ZHA_OK;
    default:
      return ZHA_ERR_INVALID_ARG;
  }
}

static zha_status check_cache(const zha_cache* c, bool need_kv) {
  if (!c || !c->tree || !c->seq_len || !c->r) return ZHA_ERR_INVALID_ARG;
  if (need_kv && (!c->k || !c->v)) return ZHA_ERR_INVALID_ARG;
  if (!c->k) return ZHA_ERR_INVALID_ARG;
  return ZHA_OK;
}

zha_status zha_build_tree(const zha_config* cfg, const zha_cache* cache, void* stream) {
  Geometry g;
  zha_status st = make_geometry(cfg, &g);
  if (st != ZHA_OK) return st;
  if ((st = check_cache(cache, false)) != ZHA_OK) return st;
  return cuda_status(launch_tree(g, cache->k, cache->tree, cache->r, cache->seq_len, nullptr, -1,
                                 (cudaStream_t)stream));
}

zha_status zha_extend_tree(const zha_config* cfg, const zha_cache* cache, const int32_t* old_len,
                           int64_t max_new_tokens, void* stream) {
  Geometry g;
  zha_status st = make_geometry(cfg, &g);
  if (st != ZHA_OK) return st;
  if ((st = check_cache(cache, false)) != ZHA_OK) return st;
  if (!old_len || max_new_tokens < 0) return ZHA_ERR_INVALID_ARG;
  if (max_new_tokens == 0) return ZHA_OK;
  return cuda_status(launch_tree(g, cache->k, cache->tree, cache->r, cache->seq_len, old_len,
                                 max_new_tokens, (cudaStream_t)stream));
}

zha_status zha_select(const zha_config* cfg, const zha_cache* cache, const void* q,
                      const int32_t* q_seq, const int32_t* q_pos, int64_t nq, double p,
                      int32_t* idx, int64_t idx_cap, int32_t* n_idx, int32_t* level_counts,
                      void* ws, size_t ws_bytes, int32_t* dev_status, void* stream) {
  Geometry g;
  zha_status st = make_geometry(cfg, &g);
  if (st != ZHA_OK) return st;
  if ((st = check_cache(cache, false)) != ZHA_OK) return st;
  uint64_t p_q;
  if (!q || !q_seq || !q_pos || nq < 1 || !idx || idx_cap < 1 || !n_idx || !ws || !check_p(p, &p_q))
    return ZHA_ERR_INVALID_ARG;
  const int sms = device_sm_count();
  if (ws_bytes < traverse_ws_bytes(g, nq * g.Hkv, sms)) return ZHA_ERR_WORKSPACE;
  TraverseOut out{};
  out.idx = idx;
  out.idx_cap = idx_cap;
  out.n_idx = n_idx;
  out.level_counts = level_counts;
  return cuda_status(launch_traverse(g, cache->tree, q, cache->seq_len, q_seq, q_pos, nq, p_q, 1,
                                     out, ws, ws_bytes, dev_status, sms, (cudaStream_t)stream));
}

zha_status zha_attend(const zha_config* cfg, const zha_cache* cache, const void* q,
                      const int32_t* q_seq, int64_t nq, const int32_t* idx, int64_t idx_cap,
                      const int32_t* n_idx, void* out, void* ws, size_t ws_bytes,
                      int32_t* dev_status, void* stream) {
  (void)dev_status;
  Geometry g;
  zha_status st = make_geometry(cfg, &g);
  if (st != ZHA_OK) return st;
  if ((st = check_cache(cache, true)) != ZHA_OK) return st;
  if (!q || !q_seq || nq < 1 || !idx || idx_cap < 1 || !n_idx || !out || !ws)
    return ZHA_ERR_INVALID_ARG;
  const int sms = device_sm_count();
  if (ws_bytes < attend_ws_bytes(g, kStreamList, nq, sms)) return ZHA_ERR_WORKSPACE;
  AttendArgs a{};
  a.kind = kStreamList;
  a.k = cache->k;
  a.v = cache->v;
  a.q = q;
  a.out = out;
  a.seq_len = cache->seq_len;
  a.q_seq = q_seq;
  a.nq = nq;
  a.idx = idx;
  a.idx_cap = idx_cap;
  a.n_idx = n_idx;
  return cuda_status(launch_attend(g, a, ws, ws_bytes, sms, (cudaStream_t)stream));
}

static zha_status run_tree_select(const Geometry& g, const zha_cache* cache, const void* q,
                                  const int32_t* q_seq, const int32_t* q_pos, int64_t nq,
                                  uint64_t p_q, int32_t* level_counts, unsigned char* ws,
                                  const DecodeLayout& L, int32_t* dev_status, int sms,
                                  cudaStream_t s, const TopSeeds* seeds = nullptr,
                                  const void* fp4 = nullptr) {
  if (L.dense && !q_pos && !seeds)
    return cuda_status(launch_decode_dense(
        g, cache->tree, q, cache->seq_len, p_q, ws + L.trav, level_counts,
        reinterpret_cast<int32_t*>(ws + L.stats), reinterpret_cast<uint32_t*>(ws + L.kept),
        reinterpret_cast<int32_t*>(ws + L.n_kept), traverse_kept_stride(g),
        traverse_cluster_size(g, L.units, sms), dev_status, sms, s, 0, 0, fp4));
  if (fp4) return ZHA_ERR_UNSUPPORTED;  // the FP4 rows are read by the dense decode path only
  TraverseOut to{};
  to.kept = reinterpret_cast<uint32_t*>(ws + L.kept);
  to.n_kept = reinterpret_cast<int32_t*>(ws + L.n_kept);
  to.stats = reinterpret_cast<int32_t*>(ws + L.stats);
  to.level_counts = level_counts;
  return cuda_status(launch_traverse(g, cache->tree, q, cache->seq_len, q_seq, q_pos, nq, p_q, 0,
                                     to, ws + L.trav, L.kept - L.trav, dev_status, sms, s, seeds));
}

static zha_status run_tree_attend(const Geometry& g, const zha_cache* cache, const void* q,
                                  const int32_t* q_seq, const int32_t* q_pos, int64_t nq,
                                  void* out, unsigned char* ws, const DecodeLayout& L, int sms,
                                  cudaStream_t s) {
  AttendArgs a{};
  a.kind = kStreamTree;
  a.k = cache->k;
  a.v = cache->v;
  a.q = q;
  a.out = out;
  a.seq_len = cache->seq_len;
  a.q_seq = q_seq;
  a.q_pos = q_pos;
  a.nq = nq;
  a.kept = reinterpret_cast<const uint32_t*>(ws + L.kept);
  a.n_kept = reinterpret_cast<const int32_t*>(ws + L.n_kept);
  a.kept_stride = traverse_kept_stride(g);
  a.kept_segs = traverse_cluster_size(g, L.units, sms);
  return cuda_status(launch_attend(g, a, ws + L.part, L.total - L.part, sms, s));
}

static zha_status run_tree_decode(const Geometry& g, const zha_cache* cache, const void* q,
                                  const int32_t* q_seq, const int32_t* q_pos, int64_t nq,
                                  uint64_t p_q, void* out, int32_t* level_counts,
                                  unsigned char* ws, const DecodeLayout& L, int32_t* dev_status,
                                  int sms, cudaStream_t s, const TopSeeds* seeds = nullptr,
                                  const void* fp4 = nullptr) {
  zha_status st = run_tree_select(g, cache, q, q_seq, q_pos, nq, p_q, level_counts, ws, L,
                                  dev_status, sms, s, seeds, fp4);
  if (st != ZHA_OK) return st;
  return run_tree_attend(g, cache, q, q_seq, q_pos, nq, out, ws, L, sms, s);
}

// ---- decode step over groups of units on concurrent streams -----------------
//
// A decode step's cut runs one CTA per query head and is bound by its chain of
// dependent passes, not by the SM count; the scoring and the attention around
// it are bound by HBM. So the units of a step are cut into groups, each with a
// stream of its own, at decreasing priorities (group 0 highest): a group
// scores, cuts, merges and attends, and the block scheduler serves the
// earlier groups first, so one group's cut overlaps the later groups' scoring
// and the earlier groups' attention. Every kernel computes per unit exactly
// what the single-stream order computes (the attention keeps the split count
// of the whole step), so the outputs are the same bit for bit.
constexpr int kPipeDevices = 64;

struct DecodePipe {
  bool ready;
  cudaStream_t s[kDecodeGroups];
  cudaEvent_t fork, done[kDecodeGroups];
};
static std::mutex g_pipe_mutex;  // held while a step's launches are enqueued
static DecodePipe g_pipe[kPipeDevices];

// Streams and events of the current device, created on first use and kept for
// the life of the process (nullptr when they cannot be had, or when they would
// have to be created while `s` is being captured into a graph).
static DecodePipe* decode_pipe(cudaStream_t s) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kPipeDevices) {
    cudaGetLastError();
    return nullptr;
  }
  DecodePipe& P = g_pipe[dev];
  if (P.ready) return &P;
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(s, &cs) != cudaSuccess || cs != cudaStreamCaptureStatusNone) {
    cudaGetLastError();
    return nullptr;
  }
  int least = 0, greatest = 0;
  if (cudaDeviceGetStreamPriorityRange(&least, &greatest) != cudaSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  bool ok = cudaEventCreateWithFlags(&P.fork, cudaEventDisableTiming) == cudaSuccess;
  for (int k = 0; ok && k < kDecodeGroups; ++k) {
    const int prio = greatest + k < least ? greatest + k : least;
    ok = cudaStreamCreateWithPriority(&P.s[k], cudaStreamNonBlocking, prio) == cudaSuccess &&
         cudaEventCreateWithFlags(&P.done[k], cudaEventDisableTiming) == cudaSuccess;
  }
  if (!ok) {  // what was created stays (a few handles); the step runs on one stream
    cudaGetLastError();
    return nullptr;
  }
  P.ready = true;
  return &P;
}

static zha_status run_dense_decode_grouped(const Geometry& g, const zha_cache* cache,
                                           const void* q, uint64_t p_q, void* out,
                                           int32_t* level_counts, unsigned char* ws,
                                           const DecodeLayout& L, int32_t* dev_status, int sms,
                                           cudaStream_t s, int K, DecodePipe& P, const void* fp4) {
  AttendArgs a{};
  a.kind = kStreamTree;
  a.k = cache->k;
  a.v = cache->v;
  a.q = q;
  a.out = out;
  a.seq_len = cache->seq_len;
  a.nq = g.B;
  a.kept = reinterpret_cast<const uint32_t*>(ws + L.kept);
  a.n_kept = reinterpret_cast<const int32_t*>(ws + L.n_kept);
  a.kept_stride = traverse_kept_stride(g);
  a.kept_segs = traverse_cluster_size(g, L.units, sms);
  cudaError_t err = cudaEventRecord(P.fork, s);
  int launched = 0;  // groups whose stream joined the step
  for (int k = 0; k < K && err == cudaSuccess; ++k) {
    const int64_t u0 = L.units * k / K, u1 = L.units * (k + 1) / K;
    cudaStream_t sk = P.s[k];
    err = cudaStreamWaitEvent(sk, P.fork, 0);
    if (err != cudaSuccess) break;
    launched = k + 1;
    err = launch_decode_dense(g, cache->tree, q, cache->seq_len, p_q, ws + L.trav, level_counts,
                              reinterpret_cast<int32_t*>(ws + L.stats),
                              reinterpret_cast<uint32_t*>(ws + L.kept),
                              reinterpret_cast<int32_t*>(ws + L.n_kept), a.kept_stride,
                              a.kept_segs, dev_status, sms, sk, u0, u1 - u0, fp4);
    if (err != cudaSuccess) break;
    a.unit0 = u0;
    a.n_units = u1 - u0;
    err = launch_attend(g, a, ws + L.part, L.total - L.part, sms, sk);
  }
  // join every stream that took part, also after a failed launch
  for (int k = 0; k < launched; ++k) {
    const cudaError_t e1 = cudaEventRecord(P.done[k], P.s[k]);
    const cudaError_t e2 = e1 == cudaSuccess ? cudaStreamWaitEvent(s, P.done[k], 0) : e1;
    if (err == cudaSuccess) err = e2;
  }
  return cuda_status(err);
}

// A decode step: the grouped form when the selection takes the dense path and
// the streams can be had, else select then attend on the caller's stream.
static zha_status run_decode_step(const Geometry& g, const zha_cache* cache, const void* q,
                                  uint64_t p_q, void* out, int32_t* level_counts,
                                  unsigned char* ws, const DecodeLayout& L, int32_t* dev_status,
                                  int sms, cudaStream_t s, bool concurrent,
                                  const void* fp4 = nullptr) {
  const int K = concurrent ? L.groups : 1;
  if (K > 1) {
    std::lock_guard<std::mutex> lock(g_pipe_mutex);
    DecodePipe* P = decode_pipe(s);
    if (P) return run_dense_decode_grouped(g, cache, q, p_q, out, level_counts, ws, L, dev_status,
                                           sms, s, K, *P, fp4);
  }
  return run_tree_decode(g, cache, q, nullptr, nullptr, g.B, p_q, out, level_counts, ws, L,
                         dev_status, sms, s, nullptr, fp4);
}

__global__ void decode_stats_kernel(const int32_t* stats, const int32_t* n_kept, int units, int L,
                                    int segs, int32_t* out) {
  const int u = blockIdx.x * blockDim.x + threadIdx.x;
  if (u >= units) return;
  int kept = 0;
  for (int r = 0; r < segs; ++r) kept += n_kept[(int64_t)u * segs + r];
  for (int l = 0; l < L; ++l) out[(int64_t)u * (L + 1) + l] = stats[(int64_t)u * L + l];
  out[(int64_t)u * (L + 1) + L] = kept;
}

static zha_status decode_impl(const zha_config* cfg, const zha_cache* cache, const void* q,
                              double p, void* out, int32_t* level_counts, void* ws,
                              size_t ws_bytes, int32_t* dev_status, void* stream, bool concurrent,
                              const void* fp4 = nullptr) {
  Geometry g;
  zha_status st = make_geometry(cfg, &g);
  if (st != ZHA_OK) return st;
  if ((st = check_cache(cache, true)) != ZHA_OK) return st;
  uint64_t p_q;
  if (!q || !out || !ws || !check_p(p, &p_q)) return ZHA_ERR_INVALID_ARG;
  const int sms = device_sm_count();
  const DecodeLayout L = decode_layout(g, g.B, kStreamTree, sms, true);
  if (fp4 && (!L.dense || g.d != 128)) return ZHA_ERR_UNSUPPORTED;
  if (ws_bytes < L.total) return ZHA_ERR_WORKSPACE;
  return run_decode_step(g, cache, q, p_q, out, level_counts, static_cast<unsigned char*>(ws), L,
                         dev_status, sms, (cudaStream_t)stream, concurrent, fp4);
}

zha_status zha_decode(const zha_config* cfg, const zha_cache* cache, const void* q, double p,
                      void* out, int32_t* level_counts, void* ws, size_t ws_bytes,
                      int32_t* dev_status, void* stream) {
  return decode_impl(cfg, cache, q, p, out, level_counts, ws, ws_bytes, dev_status, stream, true);
}

zha_status zha_fp4_tree_bytes(const zha_config* cfg, size_t* bytes) {
  Geometry g;
  zha_status st = make_geometry(cfg, &g);
  if (st != ZHA_OK) return st;
  if (!bytes) return ZHA_ERR_INVALID_ARG;
  *bytes = fp4_tree_bytes(g);
  return ZHA_OK;
}

zha_status zha_fp4_quantize_tree(const zha_config* cfg, const zha_cache* cache, void* fp4_tree,
                                 const int32_t* old_len, void* stream) {
  Geometry g;
  zha_status st = make_geometry(cfg, &g);
  if (st != ZHA_OK) return st;
  if (!cache || !cache->tree || !cache->seq_len || !fp4_tree) return ZHA_ERR_INVALID_ARG;
  return cuda_status(launch_fp4_quantize(g, cache->tree, fp4_tree, cache->seq_len, old_len,
                                         device_sm_count(), (cudaStream_t)stream));
}

zha_status zha_decode_fp4(const zha_config* cfg, const zha_cache* cache, const void* fp4_tree,
                          const void* q, double p, void* out, int32_t* level_counts, void* ws,
                          size_t ws_bytes, int32_t* dev_status, void* stream) {
  if (!fp4_tree) return ZHA_ERR_INVALID_ARG;
  return decode_impl(cfg, cache, q, p, out, level_counts, ws, ws_bytes, dev_status, stream, true,
                     fp4_tree);
}

zha_status zha_decode_select(const zha_config* cfg, const zha_cache* cache, const void* q,
                             double p, int32_t* level_counts, void* ws, size_t ws_bytes,
                             int32_t* dev_status, void* stream) {
  Geometry g;
  zha_status st = make_geometry(cfg, &g);
  if (st != ZHA_OK) return st;
  if ((st = check_cache(cache, false)) != ZHA_OK) return st;
  uint64_t p_q;
  if (!q || !ws || !check_p(p, &p_q)) return ZHA_ERR_INVALID_ARG;
  const int sms = device_sm_count();
  const DecodeLayout L = decode_layout(g, g.B, kStreamTree, sms, true);
  if (ws_bytes < L.total) return ZHA_ERR_WORKSPACE;
  return run_tree_select(g, cache, q, nullptr, nullptr, g.B, p_q, level_counts,
                         static_cast<unsigned char*>(ws), L, dev_status, sms,
                         (cudaStream_t)stream);
}

zha_status zha_decode_attend(const zha_config* cfg, const zha_cache* cache, const void* q,
                             void* out, void* ws, size_t ws_bytes, void* stream) {
  Geometry g;
  zha_status st = make_geometry(cfg, &g);
  if (st != ZHA_OK) return st;
  if ((st = check_cache(cache, true)) != ZHA_OK) return st;
  if (!q || !out || !ws) return ZHA_ERR_INVALID_ARG;
  const int sms = device_sm_count();
  const DecodeLayout L = decode_layout(g, g.B, kStreamTree, sms, true);
  if (ws_bytes < L.total) return ZHA_ERR_WORKSPACE;
  return run_tree_attend(g, cache, q, nullptr, nullptr, g.B, out,
                         static_cast<unsigned char*>(ws), L, sms, (cudaStream_t)stream);
}

zha_status zha_decode_stats(const zha_config* cfg, const void* ws, size_t ws_bytes,
                            int32_t* stats, void* stream) {
  Geometry g;
  zha_status st = make_geometry(cfg, &g);
  if (st != ZHA_OK) return st;
  if (!ws || !stats) return ZHA_ERR_INVALID_ARG;
  const int sms = device_sm_count();
  const DecodeLayout L = decode_layout(g, g.B, kStreamTree, sms, true);
  if (ws_bytes < L.total) return ZHA_ERR_WORKSPACE;
  const unsigned char* w = static_cast<const unsigned char*>(ws);
  const int units = (int)L.units;
  decode_stats_kernel<<<(units + 127) / 128, 128, 0, (cudaStream_t)stream>>>(
      reinterpret_cast<const int32_t*>(w + L.stats), reinterpret_cast<const int32_t*>(w + L.n_kept),
      units, g.L, traverse_cluster_size(g, L.units, sms), stats);
  return cuda_status(cudaGetLastError());
}

zha_status zha_decode_kept_lists(const zha_config* cfg, const zha_cache* cache, const void* ws,
                                 size_t ws_bytes, int32_t* idx, int64_t idx_cap, int32_t* n_idx,
                                 int32_t* dev_status, void* stream) {
  Geometry g;
  zha_status st = make_geometry(cfg, &g);
  if (st != ZHA_OK) return st;
  if (!cache || !cache->seq_len || !ws || !idx || idx_cap < 1 || !n_idx)
    return ZHA_ERR_INVALID_ARG;
  const int sms = device_sm_count();
  const DecodeLayout L = decode_layout(g, g.B, kStreamTree, sms, true);
  if (ws_bytes < L.total) return ZHA_ERR_WORKSPACE;
  const unsigned char* w = static_cast<const unsigned char*>(ws);
  return cuda_status(launch_kept_lists(
      g, reinterpret_cast<const uint32_t*>(w + L.kept), reinterpret_cast<const int32_t*>(w + L.n_kept),
      traverse_kept_stride(g), traverse_cluster_size(g, L.units, sms), cache->seq_len, idx, idx_cap,
      n_idx, dev_status, (cudaStream_t)stream));
}

zha_status zha_prefill_chunk(const zha_config* cfg, const zha_cache* cache, const void* q,
                             int32_t seq, int64_t chunk_start, int64_t T, double p, void* out,
                             int32_t* level_counts, void* ws, size_t ws_bytes,
                             int32_t* dev_status, void* stream) {
  Geometry g;
  zha_status st = make_geometry(cfg, &g);
  if (st != ZHA_OK) return st;
  if ((st = check_cache(cache, true)) != ZHA_OK) return st;
  uint64_t p_q;
  if (!q || !out || !ws || T < 1 || seq < 0 || seq >= g.B || chunk_start < 0 ||
      chunk_start + T > g.ncap || !check_p(p, &p_q))
    return ZHA_ERR_INVALID_ARG;
  const int sms = device_sm_count();
  const PrefillLayout P = prefill_layout(g, T, sms);
  if (ws_bytes < P.total) return ZHA_ERR_WORKSPACE;
  cudaStream_t s = (cudaStream_t)stream;
  unsigned char* w = static_cast<unsigned char*>(ws);
  int32_t* old_len = reinterpret_cast<int32_t*>(w + P.old_len);
  int32_t* q_seq = reinterpret_cast<int32_t*>(w + P.q_seq);
  int32_t* q_pos = reinterpret_cast<int32_t*>(w + P.q_pos);
  fill_prefill_kernel<<<(g.B + 127) / 128, 128, 0, s>>>(old_len, cache->seq_len, g.B, seq,
                                                       chunk_start);
  if (cudaGetLastError() != cudaSuccess) return ZHA_ERR_CUDA;
  cudaError_t e = launch_tree(g, cache->k, cache->tree, cache->r, cache->seq_len, old_len, T, s);
  if (e != cudaSuccess) return ZHA_ERR_CUDA;
  // the top level of every (token, KV head) of the chunk on the tensor cores;
  // certified units skip it in the traversal, the rest score it canonically
  TopSeeds seeds{};
  const bool tc = P.top_bytes > 0 && (reinterpret_cast<uintptr_t>(q) & 15) == 0;
  if (tc) {
    e = launch_top_select(g, cache->tree, cache->seq_len, seq, q, chunk_start, T, p_q, w + P.top,
                          P.top_bytes, &seeds, nullptr, nullptr, dev_status, s);
    if (e != cudaSuccess) return ZHA_ERR_CUDA;
  }
  const size_t row_bytes = (size_t)g.Hq * g.d * g.elem_bytes;
  for (int64_t i0 = 0; i0 < T; i0 += P.tile) {
    const int64_t n = (T - i0) < P.tile ? (T - i0) : P.tile;
    fill_positions_kernel<<<(unsigned)((n + 127) / 128), 128, 0, s>>>(q_seq, q_pos, seq,
                                                                      chunk_start + i0, n);
    if (cudaGetLastError() != cudaSuccess) return ZHA_ERR_CUDA;
    const DecodeLayout L = decode_layout(g, n, kStreamTree, sms);
    TopSeeds ts{};
    if (tc) {
      ts.ok = seeds.ok + i0 * g.Hkv;
      ts.mask = seeds.mask + i0 * g.Hkv * seeds.stride;
      ts.cnt = seeds.cnt + i0 * g.Hkv * g.G;
      ts.stride = seeds.stride;
    }
    const unsigned char* q_tile = static_cast<const unsigned char*>(q) + i0 * row_bytes;
    unsigned char* out_tile = static_cast<unsigned char*>(out) + i0 * row_bytes;
    st = run_tree_select(g, cache, q_tile, q_seq, q_pos, n, p_q,
                         level_counts ? level_counts + i0 * g.Hq * g.L : nullptr, w + P.dec, L,
                         dev_status, sms, s, tc ? &ts : nullptr);
    if (st != ZHA_OK) return st;
    if (P.tatt_bytes > 0) {  // the tile's tokens share K/V blocks on tensor cores
      st = cuda_status(launch_attend_tile(
          g, cache->k, cache->v, cache->seq_len, seq, chunk_start + i0, n, q_tile, out_tile,
          reinterpret_cast<const uint32_t*>(w + P.dec + L.kept),
          reinterpret_cast<const int32_t*>(w + P.dec + L.n_kept), traverse_kept_stride(g),
          traverse_cluster_size(g, L.units, sms), w + P.tatt, P.tatt_bytes, sms, s));
    } else {
      st = run_tree_attend(g, cache, q_tile, q_seq, q_pos, n, out_tile, w + P.dec, L, sms, s);
    }
    if (st != ZHA_OK) return st;
  }
  return ZHA_OK;
}

zha_status zha_prefill_top_scores(const zha_config* cfg, const zha_cache* cache, const void* q,
                                  int32_t seq, int64_t chunk_start, int64_t T, double p,
                                  float* z_top, int32_t* certified, void* ws, size_t ws_bytes,
                                  int32_t* dev_status, void* stream) {
  Geometry g;
  zha_status st = make_geometry(cfg, &g);
  if (st != ZHA_OK) return st;
  if ((st = check_cache(cache, false)) != ZHA_OK) return st;
  uint64_t p_q;
  if (!q || !ws || T < 1 || seq < 0 || seq >= g.B || chunk_start < 0 ||
      chunk_start + T > g.ncap || !check_p(p, &p_q) || (reinterpret_cast<uintptr_t>(q) & 15))
    return ZHA_ERR_INVALID_ARG;
  if (!top_tc_supported(g)) return ZHA_ERR_UNSUPPORTED;
  const int sms = device_sm_count();
  const PrefillLayout P = prefill_layout(g, T, sms);
  if (ws_bytes < P.total) return ZHA_ERR_WORKSPACE;
  TopSeeds seeds{};
  return cuda_status(launch_top_select(g, cache->tree, cache->seq_len, seq, q, chunk_start, T,
                                       p_q, static_cast<unsigned char*>(ws) + P.top, P.top_bytes,
                                       &seeds, z_top, certified, dev_status,
                                       (cudaStream_t)stream));
}

zha_status zha_dense_decode(const zha_config* cfg, const zha_cache* cache, const void* q,
                            void* out, void* ws, size_t ws_bytes, void* stream) {
  Geometry g;
  zha_status st = make_geometry(cfg, &g);
  if (st != ZHA_OK) return st;
  if (!cache || !cache->k || !cache->v || !cache->seq_len || !q || !out || !ws)
    return ZHA_ERR_INVALID_ARG;
  const int sms = device_sm_count();
  if (ws_bytes < attend_ws_bytes(g, kStreamDense, g.B, sms)) return ZHA_ERR_WORKSPACE;
  AttendArgs a{};
  a.kind = kStreamDense;
  a.k = cache->k;
  a.v = cache->v;
  a.q = q;
  a.out = out;
  a.seq_len = cache->seq_len;
  a.nq = g.B;
  return cuda_status(launch_attend(g, a, ws, ws_bytes, sms, (cudaStream_t)stream));
}

}  // extern "C"

namespace zha {

zha_status decode_one_stream(const zha_config* cfg, const zha_cache* cache, const void* q,
                             double p, void* out, int32_t* level_counts, void* ws,
                             size_t ws_bytes, int32_t* dev_status, void* stream) {
  return decode_impl(cfg, cache, q, p, out, level_counts, ws, ws_bytes, dev_status, stream, false);
}

}  // namespace zha
