// Top-down top-p traversal of the summary tree, all query heads of a KV head
// together.
//
// lefilia.fr page "Zyphra presente Zyphra Hierarchical Attention (ZHA) ...",
// paragraph 1: a query scores the top nodes, keeps the smallest set covering a
// fraction p of the estimated attention mass, expands only the kept branches
// down to the raw KV entries, and always keeps the first token.
//
// Unit of work: one query token and one KV head, i.e. the G = Hq/Hkv query
// heads that read the same tree. At every level the unit's candidate list is
// the UNION of the heads' frontiers; each entry carries an 8-bit mask of the
// heads whose frontier contains it, so every summary row is read once per unit
// and scored against all G queries.
//
// A thread-block cluster of C CTAs cooperates on a unit. CTA r owns an ordered
// SEGMENT of the frontier: the top nodes are split into C contiguous ranges and
// each CTA keeps the children of its own kept nodes, so the concatenation of
// the segments in rank order is always sorted by node index and no global
// compaction is needed. Per level:
//   1. score   -- each CTA scores its segment for all heads (canonical fp32
//                 chains; 4 candidates x G heads per thread).      cluster sync
//   2. cut     -- the CTA owning head h (h mod C) runs the exact cut for h over
//                 every segment: radix select on the order-preserving bits of z
//                 with fixed-point mass sums per bucket (11-bit digits), then
//                 writes h's keep bits.                            cluster sync
//   3. expand  -- each CTA turns its segment's keep bits into the next level's
//                 candidates (children of nodes kept by any head).
// Canonical arithmetic (identical to the CPU oracle):
//   z = (dot(q, s) * inv_sqrt_d) + fp32(l ln b),  M = trunc(exp(z - zmax) 2^40),
//   need = ceil(T p_q / 2^32); keep the shortest prefix of (z desc, node asc)
//   whose mass reaches need (every candidate when p_q >= 2^32).
#include <cooperative_groups.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "zha_device.cuh"
#include "zha_internal.h"

namespace cg = cooperative_groups;

namespace zha {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kBuckets = 2048;
constexpr int kDigit = 11;
constexpr int kCandPerThread = 4;
constexpr uint32_t kNodeMask = 0x00ffffffu;
constexpr int kChunk = 8 * kThreads;  // candidates per streamed chunk (8 per thread)
constexpr int kStages = 3;            // cp.async ring depth of the cut passes
constexpr int kListCap = 2048;        // crossing-bucket members finished in shared memory
constexpr int kRankCap = 256;         // per-head frontiers this small are cut by explicit ranks

struct TravParams {
  const void* tree;
  int64_t level_off[kMaxLevels];
  int64_t level_rows[kMaxLevels];
  int64_t span[kMaxLevels + 1];
  float lnsize[kMaxLevels];
  float inv_sqrt_d;
  const void* q;
  const int32_t* seq_len;
  const int32_t* q_seq;
  const int32_t* q_pos;
  int Hq, Hkv, b, L, B;
  int64_t ncap;
  uint64_t p_q;
  int keep_all;
  int list_mode;
  int64_t seg;           // capacity of one segment (candidates), multiple of 32
  uint32_t* cand;        // [units][2][C][seg]   (head mask << 24) | node
  float* zbuf;           // [units][G][C][seg]
  uint32_t* kbits;       // [units][G][C][seg/32]
  uint32_t* kept;        // [units][C][seg]     decode mode: union-kept level-1 nodes
  int32_t* n_kept;       // [units][C]
  int32_t* idx;          // [nq][Hq][idx_cap]   list mode
  int64_t idx_cap;
  int32_t* n_idx;
  int32_t* level_counts;
  int32_t* stats;        // [units][L]: union candidates scored per level (nullable)
  int32_t* status;
};

// Per-CTA values read by the other CTAs of the cluster through DSMEM.
struct Xch {
  unsigned int count;            // candidates in my segment at this level
  float zmax[kMaxGroup];
  float zmin[kMaxGroup];
};

// Every member read or written with 8/16-byte vector accesses is 16-aligned.
struct Smem {
  alignas(16) unsigned int hlo[kBuckets];
  alignas(16) unsigned int hhi[kBuckets];
  alignas(16) unsigned int hcnt[kBuckets];
  alignas(16) float ring_z[kStages][kChunk];
  alignas(16) uint32_t ring_c[kStages][kChunk];
  alignas(16) float list_z[kListCap];
  alignas(16) uint32_t list_pos[kListCap];   // (segment << 24) | index: ascending = node order
  alignas(16) float q[kMaxGroup * 128];      // [i][8] fp32, i < D (float4 reads)
  unsigned int list_n;
  unsigned int seg_n[kMaxCluster];
  unsigned int chunk_start[kMaxCluster + 1];
  unsigned int res_base[kMaxCluster];   // resident copy: segment r at ring[res_base[r]]
  float g_zmax[kMaxCluster][kMaxGroup];  // every rank's segment extremes, gathered once
  float g_zmin[kMaxCluster][kMaxGroup];
  float red_f[kWarps][kMaxGroup][2];
  unsigned long long red_u64[kWarps];
  unsigned int red_u32[kWarps];
  unsigned long long bc_u64[4];
  unsigned int bc_u32[8];
  Xch xch;
};

// Exclusive scan of v over the CTA in thread order; *total receives the sum.
__device__ __forceinline__ unsigned int block_excl_scan(unsigned int v, unsigned int* total,
                                                        Smem& S) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  unsigned int x = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const unsigned int y = __shfl_up_sync(0xffffffffu, x, off);
    if (lane >= off) x += y;
  }
  if (lane == 31) S.red_u32[warp] = x;
  __syncthreads();
  unsigned int wbase = 0, tot = 0;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) {
    const unsigned int s = S.red_u32[w];
    if (w < warp) wbase += s;
    tot += s;
  }
  __syncthreads();
  *total = tot;
  return wbase + x - v;
}

__device__ __forceinline__ unsigned long long block_sum_u64(unsigned long long v, Smem& S) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  if (lane == 0) S.red_u64[warp] = v;
  __syncthreads();
  unsigned long long t = 0;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) t += S.red_u64[w];
  __syncthreads();
  return t;
}

// Exclusive scan of a u64 over the CTA in thread order.
__device__ __forceinline__ unsigned long long block_excl_scan_u64(unsigned long long v, Smem& S) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  unsigned long long x = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const unsigned long long y = __shfl_up_sync(0xffffffffu, x, off);
    if (lane >= off) x += y;
  }
  if (lane == 31) S.red_u64[warp] = x;
  __syncthreads();
  unsigned long long wbase = 0;
#pragma unroll
  for (int w = 0; w < kWarps; ++w)
    if (w < warp) wbase += S.red_u64[w];
  __syncthreads();
  return wbase + x - v;
}

// Exact 64-bit accumulation into a (lo, hi) pair of 32-bit shared counters.
__device__ __forceinline__ void hist_add(Smem& S, int b, unsigned long long m, unsigned int n) {
  const unsigned int lo = (unsigned int)m;
  const unsigned int old = atomicAdd(&S.hlo[b], lo);
  const unsigned int hi = (unsigned int)(m >> 32) + ((old + lo < old) ? 1u : 0u);
  if (hi) atomicAdd(&S.hhi[b], hi);
  atomicAdd(&S.hcnt[b], n);
}

__device__ __forceinline__ unsigned long long ceil_mul_shift32(unsigned long long T,
                                                               unsigned long long pq) {
  const unsigned long long lo = T * pq;
  const unsigned long long hi = __umul64hi(T, pq);
  unsigned long long r = (hi << 32) | (lo >> 32);
  if (lo & 0xffffffffull) r += 1;
  return r;
}


// Streams head h's (score, candidate) pairs of every segment, in ascending node
// order, through a cp.async ring; f(z[8], c[8], nvalid, pos0) sees the 8
// consecutive candidates of this thread (pos0 = (segment << 24) | first index).
constexpr int kResidentCap = kStages * kChunk;  // candidates kept resident per head

// Copies head h's scores and candidate entries of every segment into the ring
// (segment r at res_base[r], 32-aligned); returns false if they do not fit.
__device__ __forceinline__ bool load_resident(Smem& S, int C, const uint32_t* cbase,
                                              const float* zbase, int64_t seg) {
  float* rz = &S.ring_z[0][0];
  uint32_t* rc = &S.ring_c[0][0];
  unsigned int acc = 0;
  for (int r = 0; r < C; ++r) acc += (S.seg_n[r] + 31u) & ~31u;
  if (acc > (unsigned)kResidentCap) return false;
  if (threadIdx.x == 0) {
    unsigned int b = 0;
    for (int r = 0; r < C; ++r) {
      S.res_base[r] = b;
      b += (S.seg_n[r] + 31u) & ~31u;
    }
  }
  __syncthreads();
  for (int r = 0; r < C; ++r) {
    const int pieces = (int)((S.seg_n[r] + 3u) >> 2);
    for (int e = threadIdx.x; e < pieces; e += kThreads) {
      cp_async16(rz + S.res_base[r] + e * 4, zbase + r * seg + e * 4);
      cp_async16(rc + S.res_base[r] + e * 4, cbase + r * seg + e * 4);
    }
  }
  cp_async_commit();
  cp_async_wait<0>();
  __syncthreads();
  return true;
}

// Visits head h's (score, candidate) pairs of every segment, in ascending node
// order; f(z[8], c[8], nvalid, pos0, idx0, r) sees 8 consecutive candidates of
// segment r starting at index idx0 (pos0 = (r << 24) | idx0). Chunks come from
// the resident copy, or are streamed through the cp.async ring.
template <typename F>
__device__ __forceinline__ void stream_head(Smem& S, int C, const uint32_t* cbase,
                                            const float* zbase, int64_t seg, bool resident,
                                            F&& f) {
  const int tid = threadIdx.x;
  const int nchunks = (int)S.chunk_start[C];
  auto locate = [&](int k, int& r, int64_t& off) {
    r = 0;
    while ((int)S.chunk_start[r + 1] <= k) ++r;
    off = (int64_t)(k - (int)S.chunk_start[r]) * kChunk;
  };
  auto issue = [&](int k, int st) {
    if (k < nchunks) {
      int r;
      int64_t off;
      locate(k, r, off);
      const int64_t n = S.seg_n[r];
      const int len = (int)((n - off) < kChunk ? (n - off) : kChunk);
      const int pieces = (len + 3) >> 2;  // 16-byte pieces (segments are 128-byte aligned)
      for (int e = tid; e < pieces; e += kThreads) {
        cp_async16(&S.ring_z[st][e * 4], zbase + r * seg + off + e * 4);
        cp_async16(&S.ring_c[st][e * 4], cbase + r * seg + off + e * 4);
      }
    }
    cp_async_commit();
  };
  if (!resident) {
#pragma unroll
    for (int st = 0; st < kStages - 1; ++st) issue(st, st);
  }
  for (int k = 0; k < nchunks; ++k) {
    const float* zsrc;
    const uint32_t* csrc;
    int r;
    int64_t off;
    locate(k, r, off);
    if (!resident) {
      issue(k + kStages - 1, (k + kStages - 1) % kStages);
      cp_async_wait<kStages - 1>();
      __syncthreads();
      zsrc = &S.ring_z[k % kStages][0];
      csrc = &S.ring_c[k % kStages][0];
    } else {
      zsrc = &S.ring_z[0][0] + S.res_base[r] + off;
      csrc = &S.ring_c[0][0] + S.res_base[r] + off;
    }
    const int64_t n = S.seg_n[r];
    const int len = (int)((n - off) < kChunk ? (n - off) : kChunk);
    const int first = tid * 8;
    const int nvalid = len - first < 0 ? 0 : (len - first > 8 ? 8 : len - first);
    float z[8];
    uint32_t c[8];
    if (nvalid > 0) {
      const float4 z0 = *reinterpret_cast<const float4*>(zsrc + first);
      const float4 z1 = *reinterpret_cast<const float4*>(zsrc + first + 4);
      const uint4 c0 = *reinterpret_cast<const uint4*>(csrc + first);
      const uint4 c1 = *reinterpret_cast<const uint4*>(csrc + first + 4);
      z[0] = z0.x; z[1] = z0.y; z[2] = z0.z; z[3] = z0.w;
      z[4] = z1.x; z[5] = z1.y; z[6] = z1.z; z[7] = z1.w;
      c[0] = c0.x; c[1] = c0.y; c[2] = c0.z; c[3] = c0.w;
      c[4] = c1.x; c[5] = c1.y; c[6] = c1.z; c[7] = c1.w;
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        z[j] = 0.0f;
        c[j] = 0u;
      }
    }
    f(z, c, nvalid, ((uint32_t)r << 24) | (uint32_t)(off + first), off + first, r);
    if (!resident) __syncthreads();
  }
  if (!resident) cp_async_wait<0>();
}

// Adds (mass m, count n) to bucket d, aggregating across the warp when every
// participating lane hits the same bucket.
__device__ __forceinline__ void hist_add_warp(Smem& S, bool valid, uint32_t d,
                                              unsigned long long m, unsigned int n) {
  const int lane = threadIdx.x & 31;
  const unsigned vmask = __ballot_sync(0xffffffffu, valid);
  if (vmask == 0u) return;
  const int leader = __ffs(vmask) - 1;
  const uint32_t d0 = __shfl_sync(0xffffffffu, d, leader);
  if (__all_sync(0xffffffffu, !valid || d == d0)) {
    unsigned long long s = valid ? m : 0ull;
    unsigned int c = valid ? n : 0u;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      s += __shfl_xor_sync(0xffffffffu, s, off);
      c += __shfl_xor_sync(0xffffffffu, c, off);
    }
    if (lane == leader) hist_add(S, (int)d0, s, c);
  } else if (valid) {
    hist_add(S, (int)d, m, n);
  }
}

// Crossing digit of the current histogram: above + mass(digits > d) < need <=
// above + mass(digits >= d). Returns false if none exists (never for exact sums).
__device__ __forceinline__ bool find_crossing(Smem& S, int nb, unsigned long long above,
                                              unsigned long long need, uint32_t* beta,
                                              unsigned long long* above_out,
                                              unsigned long long* bmass, unsigned int* bcnt) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  constexpr int kPerT = kBuckets / kThreads;
  unsigned long long mloc[kPerT];
  unsigned long long tsum = 0;
#pragma unroll
  for (int j = 0; j < kPerT; ++j) {
    const int d = tid * kPerT + j;  // buckets >= nb were not cleared this pass
    mloc[j] = d < nb ? ((unsigned long long)S.hhi[d] << 32) | S.hlo[d] : 0ull;
    tsum += mloc[j];
  }
  unsigned long long x = tsum;  // suffix over lanes (higher lanes = higher digits)
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const unsigned long long y = __shfl_down_sync(0xffffffffu, x, off);
    if (lane + off < 32) x += y;
  }
  if (lane == 0) S.red_u64[warp] = x;
  if (tid == 0) S.bc_u32[2] = 0xffffffffu;
  __syncthreads();
  unsigned long long run = above + (x - tsum);
#pragma unroll
  for (int w2 = 0; w2 < kWarps; ++w2)
    if (w2 > warp) run += S.red_u64[w2];
#pragma unroll
  for (int j = kPerT - 1; j >= 0; --j) {
    const int d = tid * kPerT + j;
    if (run < need && run + mloc[j] >= need) {
      S.bc_u32[2] = (unsigned)d;
      S.bc_u64[0] = run;
      S.bc_u64[1] = mloc[j];
      S.bc_u32[3] = S.hcnt[d];
    }
    run += mloc[j];
  }
  __syncthreads();
  const bool ok = S.bc_u32[2] != 0xffffffffu;
  *beta = S.bc_u32[2];
  *above_out = S.bc_u64[0];
  *bmass = S.bc_u64[1];
  *bcnt = S.bc_u32[3];
  __syncthreads();
  return ok;
}

__device__ __forceinline__ void clear_hist(Smem& S, int nb) {
  for (int e = threadIdx.x; e < nb; e += kThreads) {
    S.hlo[e] = 0u;
    S.hhi[e] = 0u;
    S.hcnt[e] = 0u;
  }
  __syncthreads();
}

// Score candidates [0, n) of a segment against G queries; 4 candidates per
// thread so that each broadcast of q[i][0..G) feeds 4*G chains. zseg points at
// head 0's array; head h's array is zstride further.
template <typename T, int D, int G>
__device__ __forceinline__ void score_segment(const TravParams& p, Smem& S, const T* lvl,
                                              const uint32_t* cand, float* zseg, int64_t zstride,
                                              int64_t n, float lns, float* lmax, float* lmin,
                                              bool top, int64_t top_base) {
  constexpr int kPer = Elem<T>::kPerChunk;
  constexpr int kNch = D * (int)sizeof(T) / 16;
  const int tid = threadIdx.x;
  for (int64_t base = 0; base < n; base += kThreads * kCandPerThread) {
    const uint4* rows[kCandPerThread];
    uint32_t pm[kCandPerThread];
    bool ok[kCandPerThread];
#pragma unroll
    for (int k = 0; k < kCandPerThread; ++k) {
      const int64_t i = base + k * kThreads + tid;
      ok[k] = i < n;
      const uint32_t cv = ok[k] ? (top ? ((((1u << G) - 1u) << 24) | (uint32_t)(top_base + i))
                                       : cand[i])
                                : 0u;
      pm[k] = cv >> 24;
      rows[k] = reinterpret_cast<const uint4*>(lvl + (int64_t)(cv & kNodeMask) * D);
    }
    float2 acc[kCandPerThread][(G + 1) / 2];
    float acc1[kCandPerThread];
#pragma unroll
    for (int k = 0; k < kCandPerThread; ++k) {
      acc1[k] = 0.0f;
#pragma unroll
      for (int j = 0; j < (G + 1) / 2; ++j) acc[k][j] = make_float2(0.0f, 0.0f);
    }
    uint4 cur[kCandPerThread], nxt[kCandPerThread];
#pragma unroll
    for (int k = 0; k < kCandPerThread; ++k) {
      cur[k] = ok[k] ? rows[k][0] : make_uint4(0, 0, 0, 0);
      nxt[k] = cur[k];
    }
#pragma unroll 1
    for (int ch = 0; ch < kNch; ++ch) {
      if (ch + 1 < kNch) {
#pragma unroll
        for (int k = 0; k < kCandPerThread; ++k)
          nxt[k] = ok[k] ? rows[k][ch + 1] : make_uint4(0, 0, 0, 0);
      }
      float x[kCandPerThread][kPer];
#pragma unroll
      for (int k = 0; k < kCandPerThread; ++k) Elem<T>::unpack(cur[k], x[k]);
#pragma unroll
      for (int e = 0; e < kPer; ++e) {
        const float* qv = S.q + (ch * kPer + e) * kMaxGroup;
        if constexpr (G == 1) {
#pragma unroll
          for (int k = 0; k < kCandPerThread; ++k) acc1[k] = __fmaf_rn(qv[0], x[k][e], acc1[k]);
        } else if constexpr (G == 2) {
          const float2 q2 = *reinterpret_cast<const float2*>(qv);
#pragma unroll
          for (int k = 0; k < kCandPerThread; ++k)
            acc[k][0] = ffma2(q2, make_float2(x[k][e], x[k][e]), acc[k][0]);
        } else {
          float4 q4[G / 4];
#pragma unroll
          for (int j = 0; j < G / 4; ++j) q4[j] = *reinterpret_cast<const float4*>(qv + 4 * j);
#pragma unroll
          for (int k = 0; k < kCandPerThread; ++k) {
            const float2 xx = make_float2(x[k][e], x[k][e]);
#pragma unroll
            for (int j = 0; j < G / 4; ++j) {
              acc[k][2 * j] = ffma2(make_float2(q4[j].x, q4[j].y), xx, acc[k][2 * j]);
              acc[k][2 * j + 1] = ffma2(make_float2(q4[j].z, q4[j].w), xx, acc[k][2 * j + 1]);
            }
          }
        }
      }
#pragma unroll
      for (int k = 0; k < kCandPerThread; ++k) cur[k] = nxt[k];
    }
#pragma unroll
    for (int k = 0; k < kCandPerThread; ++k) {
      if (!ok[k]) continue;
      const int64_t i = base + k * kThreads + tid;
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float raw = (G == 1) ? acc1[k] : ((h & 1) ? acc[k][h / 2].y : acc[k][h / 2].x);
        const float z = __fadd_rn(__fmul_rn(raw, p.inv_sqrt_d), lns);
        zseg[(int64_t)h * zstride + i] = z;
        if ((pm[k] >> h) & 1u) {
          lmax[h] = fmaxf(lmax[h], z);
          lmin[h] = fminf(lmin[h], z);
        }
      }
    }
  }
}

template <typename T, int D, int G>
__global__ void __launch_bounds__(kThreads, 2) traverse_kernel(TravParams p) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  Smem& S = *reinterpret_cast<Smem*>(smem_raw);
  cg::cluster_group cluster = cg::this_cluster();
  const int C = (int)cluster.num_blocks();
  const int rank = (int)cluster.block_rank();
  const int unit = blockIdx.x / C;
  const int tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  const int Hkv = p.Hkv;
  const int qi = unit / Hkv, kvh = unit % Hkv;
  int seq;
  int64_t t;
  if (p.q_pos) {
    seq = p.q_seq[qi];
    t = p.q_pos[qi];
  } else {
    seq = qi;
    t = (int64_t)p.seq_len[qi] - 1;
  }
  // never read beyond the sequence's valid rows or the cache capacity
  if (seq < 0 || seq >= p.B) {
    seq = 0;
    t = -1;
  } else {
    int64_t n = p.seq_len[seq];
    if (n > p.ncap) n = p.ncap;
    if (t > n - 1) t = n - 1;
  }
  const int64_t n_vis = t + 1;
  const int64_t T_top = n_vis / p.span[p.L];
  const int tree_unit = seq * Hkv + kvh;
  const int b = p.b;
  const int64_t seg = p.seg;

  for (int e = tid; e < D * kMaxGroup; e += kThreads) {
    const int i = e / kMaxGroup, h = e % kMaxGroup;
    const T* qrow = static_cast<const T*>(p.q) + ((int64_t)qi * p.Hq + (int64_t)kvh * G + h) * D;
    S.q[e] = (h < G) ? Elem<T>::to_f(qrow[i]) : 0.0f;
  }
  if (p.stats && rank == 0 && tid < p.L) p.stats[(int64_t)unit * p.L + tid] = 0;
  __syncthreads();

  uint32_t* cand_u = p.cand + (int64_t)unit * 2 * C * seg;
  float* z_u = p.zbuf + (int64_t)unit * G * C * seg;
  uint32_t* kb_u = p.kbits + (int64_t)unit * G * C * (seg / 32);
  auto cptr = [&](int buf, int r) { return cand_u + ((int64_t)buf * C + r) * seg; };
  auto zptr = [&](int h, int r) { return z_u + ((int64_t)h * C + r) * seg; };
  auto kptr = [&](int h, int r) { return kb_u + ((int64_t)h * C + r) * (seg / 32); };
  int32_t* lc_base = p.level_counts ? p.level_counts + ((int64_t)qi * p.Hq + (int64_t)kvh * G) * p.L
                                    : nullptr;

  // ---- no complete top node: every visible token is attended (dense) ----
  if (T_top == 0) {
    if (p.list_mode) {
      for (int h = rank; h < G; h += C) {
        const int64_t qh = (int64_t)qi * p.Hq + (int64_t)kvh * G + h;
        int32_t* out = p.idx + qh * p.idx_cap;
        for (int64_t j = tid; j < n_vis && j < p.idx_cap; j += kThreads) out[j] = (int32_t)j;
        if (tid == 0) {
          p.n_idx[qh] = (int32_t)n_vis;
          if (n_vis > p.idx_cap) raise_status(p.status, ZHA_ERR_CAPACITY);
        }
      }
    } else if (tid == 0) {
      p.n_kept[(int64_t)unit * C + rank] = 0;
    }
    if (lc_base)
      for (int h = rank; h < G; h += C)
        for (int e = tid; e < p.L; e += kThreads) lc_base[(int64_t)h * p.L + e] = 0;
    return;  // uniform across the cluster: no barrier is pending
  }

  // my segment at the top level: a contiguous range of the complete top nodes
  const int64_t top_lo = T_top * rank / C;
  int64_t my_n = T_top * (rank + 1) / C - top_lo;
  int cur = 0;
  for (int level = p.L; level >= 1; --level) {
    const bool top = level == p.L;
    const T* lvl = static_cast<const T*>(p.tree) + p.level_off[level - 1] +
                   (int64_t)tree_unit * p.level_rows[level - 1] * D;
    // ------------------------------------------------------------------
    // 1. score my segment
    // ------------------------------------------------------------------
    float lmax[G], lmin[G];
#pragma unroll
    for (int h = 0; h < G; ++h) {
      lmax[h] = -INFINITY;
      lmin[h] = INFINITY;
    }
    score_segment<T, D, G>(p, S, lvl, cptr(cur, rank), zptr(0, rank), (int64_t)C * seg, my_n,
                           p.lnsize[level - 1], lmax, lmin, top, top_lo);
    if (top) {  // materialise the top candidates (all heads)
      uint32_t* cc = cptr(cur, rank);
      for (int64_t i = tid; i < my_n; i += kThreads)
        cc[i] = (((1u << G) - 1u) << 24) | (uint32_t)(top_lo + i);
    }
#pragma unroll
    for (int h = 0; h < G; ++h) {
      float mx = lmax[h], mn = lmin[h];
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
        mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, off));
      }
      if (lane == 0) {
        S.red_f[warp][h][0] = mx;
        S.red_f[warp][h][1] = mn;
      }
    }
    __syncthreads();
    if (tid < G) {
      float mx = -INFINITY, mn = INFINITY;
      for (int w = 0; w < kWarps; ++w) {
        mx = fmaxf(mx, S.red_f[w][tid][0]);
        mn = fminf(mn, S.red_f[w][tid][1]);
      }
      S.xch.zmax[tid] = mx;
      S.xch.zmin[tid] = mn;
    }
    if (tid == 0) S.xch.count = (unsigned int)my_n;
    __syncthreads();
    cluster.sync();  // S1: every segment scored
    if (p.stats && tid == 0) atomicAdd(&p.stats[(int64_t)unit * p.L + (p.L - level)], (int)my_n);

    // ------------------------------------------------------------------
    // 2. exact cut for the heads this CTA owns
    // ------------------------------------------------------------------
    for (int e = tid; e < C * (2 * G + 1); e += kThreads) {  // one parallel DSMEM gather
      const int r = e / (2 * G + 1), k = e % (2 * G + 1);
      const Xch* rx = cluster.map_shared_rank(&S.xch, r);
      if (k == 0) S.seg_n[r] = rx->count;
      else if (k <= G) S.g_zmax[r][k - 1] = rx->zmax[k - 1];
      else S.g_zmin[r][k - 1 - G] = rx->zmin[k - 1 - G];
    }
    __syncthreads();
    if (tid == 0) {
      unsigned int acc = 0;
      for (int r = 0; r < C; ++r) {
        S.chunk_start[r] = acc;
        acc += (S.seg_n[r] + kChunk - 1) / kChunk;
      }
      S.chunk_start[C] = acc;
    }
    __syncthreads();
    for (int h = rank; h < G; h += C) {
      const uint32_t* cseg = cptr(cur, 0);  // segment r at cseg + r * seg
      const float* zseg = zptr(h, 0);
      if (tid == 0) {
        float mx = -INFINITY, mn = INFINITY;
        for (int r = 0; r < C; ++r) {
          mx = fmaxf(mx, S.g_zmax[r][h]);
          mn = fminf(mn, S.g_zmin[r][h]);
        }
        S.bc_u32[0] = __float_as_uint(mx);
        S.bc_u32[1] = __float_as_uint(mn);
        S.list_n = 0u;
      }
      __syncthreads();
      const float zmax = __uint_as_float(S.bc_u32[0]);
      // small frontiers: one copy into shared memory serves every pass
      const bool resident = load_resident(S, C, cseg, zseg, seg);
      if (resident) {
        // gather head h's candidates (score, position); tiny frontiers are cut by
        // explicit ranks instead of digit passes
        if (tid == 0) S.list_n = 0u;
        __syncthreads();
        stream_head(S, C, cseg, zseg, seg, true,
                    [&](const float* z, const uint32_t* c, int nvalid, uint32_t pos0, int64_t,
                        int) {
#pragma unroll
          for (int j = 0; j < 8; ++j)
            if (j < nvalid && ((c[j] >> (24 + h)) & 1u)) {
              const unsigned slot = atomicAdd(&S.list_n, 1u);
              if (slot < (unsigned)kListCap) {
                S.list_z[slot] = z[j];
                S.list_pos[slot] = pos0 + (uint32_t)j;
              }
            }
        });
        __syncthreads();
      }
      const int n_h = resident ? (int)S.list_n : kRankCap + 1;
      __syncthreads();  // every warp has read list_n before the radix path resets it
      if (n_h <= kRankCap) {
        // rank_i = #{j : z_j > z_i, or z_j == z_i and pos_j < pos_i}; mass M_i is
        // scattered to its rank; the cut is the shortest rank prefix reaching need
        unsigned long long tloc = 0;
        for (int i = tid; i < n_h; i += kThreads) {
          const float zi = S.list_z[i];
          const uint32_t pi = S.list_pos[i];
          unsigned int rk = 0;
          for (int j = 0; j < n_h; ++j) {
            const float zj = S.list_z[j];
            rk += (zj > zi || (zj == zi && S.list_pos[j] < pi)) ? 1u : 0u;
          }
          const unsigned long long m = mass_fixed(zi, zmax);
          tloc += m;
          S.hcnt[i] = rk;
          S.hlo[rk] = (unsigned int)m;
          S.hhi[rk] = (unsigned int)(m >> 32);
        }
        const unsigned long long Tm = block_sum_u64(tloc, S);
        const unsigned long long need_r = ceil_mul_shift32(Tm, p.p_q);
        // thread t owns ranks [4t, 4t + 4)
        unsigned long long part[4];
        unsigned long long tsum = 0;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int rk = tid * 4 + j;
          part[j] = rk < n_h ? (((unsigned long long)S.hhi[rk] << 32) | S.hlo[rk]) : 0ull;
          tsum += part[j];
        }
        unsigned long long run = block_excl_scan_u64(tsum, S);
        if (tid == 0) S.bc_u32[5] = (unsigned)n_h;
        __syncthreads();
        if (!p.keep_all) {
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int rk = tid * 4 + j;
            if (rk < n_h && run < need_r && run + part[j] >= need_r) S.bc_u32[5] = (unsigned)rk + 1u;
            run += part[j];
          }
        }
        __syncthreads();
        const unsigned int k = S.bc_u32[5];
        // keep bits: clear head h's words, then set the kept ranks
        for (int r = 0; r < C; ++r) {
          uint32_t* kb = kptr(h, r);
          for (int wd = tid; wd < (int)((S.seg_n[r] + 31u) >> 5); wd += kThreads) kb[wd] = 0u;
        }
        __syncthreads();
        for (int i = tid; i < n_h; i += kThreads)
          if (S.hcnt[i] < k) {
            const uint32_t pi = S.list_pos[i];
            atomicOr(&kptr(h, (int)(pi >> 24))[(pi & kNodeMask) >> 5], 1u << (pi & 31u));
          }
        if (lc_base && tid == 0) lc_base[(int64_t)h * p.L + (p.L - level)] = (int32_t)k;
        __syncthreads();
      }
      if (n_h > kRankCap) {  // radix-select cut
      if (tid == 0) S.list_n = 0u;
      __syncthreads();
      const uint32_t kmax = order_key(zmax), kmin = order_key(__uint_as_float(S.bc_u32[1]));
      const uint32_t diff = kmax ^ kmin;
      int shift = diff ? 32 - __clz(diff) : 0;
      uint32_t prefix = (uint32_t)((uint64_t)kmax >> shift);
      unsigned long long above = 0, need = 0, bmass = 1;
      unsigned int bcnt = 1;
      bool done = p.keep_all != 0;
      bool listed = false;    // the current group lives in S.list_*
      bool first = true;
      for (int pass = 0; !done && pass < 4; ++pass) {  // <= ceil(32/11) digit passes
        const int w = shift < kDigit ? shift : kDigit;
        const int sh = shift - w;
        clear_hist(S, 1 << w);
        unsigned long long tloc = 0;
        if (!listed) {
          // full streaming pass over every candidate of head h
          stream_head(S, C, cseg, zseg, seg, resident,
                      [&](const float* z, const uint32_t* c, int nvalid, uint32_t, int64_t, int) {
            // the 8 masses first (independent chains), then per-thread run-length
            // aggregation of equal digits
            bool ok[8];
            uint32_t dg[8];
            unsigned long long ms[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const uint32_t key = order_key(z[j]);
              ok[j] = j < nvalid && ((c[j] >> (24 + h)) & 1u) &&
                      (uint32_t)((uint64_t)key >> shift) == prefix;
              dg[j] = (key >> sh) & ((1u << w) - 1u);
              ms[j] = ok[j] ? mass_fixed(z[j], zmax) : 0ull;
            }
            bool have = false;
            uint32_t rd = 0;
            unsigned long long rm = 0;
            unsigned int rc = 0;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              if (ok[j]) {
                tloc += ms[j];
                if (have && dg[j] != rd) {
                  hist_add(S, (int)rd, rm, rc);
                  rm = 0;
                  rc = 0;
                }
                have = true;
                rd = dg[j];
                rm += ms[j];
                rc += 1;
              }
            }
            hist_add_warp(S, have, rd, rm, rc);
          });
        } else {
          const int nl = (int)S.list_n;
          for (int base = 0; base < nl; base += kThreads) {
            const int i = base + tid;
            bool valid = false;
            uint32_t d = 0;
            unsigned long long m = 0;
            if (i < nl) {
              const uint32_t key = order_key(S.list_z[i]);
              if ((uint32_t)((uint64_t)key >> shift) == prefix) {
                valid = true;
                d = (key >> sh) & ((1u << w) - 1u);
                m = mass_fixed(S.list_z[i], zmax);
              }
            }
            hist_add_warp(S, valid, d, m, 1u);
          }
        }
        if (first) {
          const unsigned long long Tm = block_sum_u64(tloc, S);
          need = ceil_mul_shift32(Tm, p.p_q);
          first = false;
        }
        __syncthreads();
        uint32_t beta;
        if (!find_crossing(S, 1 << w, above, need, &beta, &above, &bmass, &bcnt)) {
          if (tid == 0) raise_status(p.status, ZHA_ERR_INTERNAL);  // never loop forever
          done = true;
          break;
        }
        prefix = (prefix << w) | beta;
        shift = sh;
        done = (bcnt == 1u) || (shift == 0);
        if (!done && !listed && bcnt <= (unsigned)kListCap) {
          // gather the crossing bucket's members once; later digits run in smem
          stream_head(S, C, cseg, zseg, seg, resident,
                      [&](const float* z, const uint32_t* c, int nvalid, uint32_t pos0, int64_t,
                          int) {
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              if (j < nvalid && ((c[j] >> (24 + h)) & 1u) &&
                  (uint32_t)((uint64_t)order_key(z[j]) >> shift) == prefix) {
                const unsigned slot = atomicAdd(&S.list_n, 1u);
                if (slot < (unsigned)kListCap) {
                  S.list_z[slot] = z[j];
                  S.list_pos[slot] = pos0 + (uint32_t)j;
                }
              }
            }
          });
          listed = true;
        }
      }
      // keep = (key >> shift) > prefix, plus the first tie_need members of the
      // boundary group (key >> shift) == prefix in ascending node order
      unsigned long long tie_need = 0;
      if (!p.keep_all) {
        const unsigned long long mt = bmass / bcnt;
        tie_need = (need - above + mt - 1) / mt;
      }
      const bool rank_ties = !p.keep_all && tie_need < bcnt;
      // with the boundary group listed, the kept ties are those whose position is
      // at most the tie_need-th smallest position of the group
      uint32_t pos_thr = 0xffffffffu;
      const bool thr_mode = rank_ties && listed;
      if (thr_mode) {
        if (tid == 0) S.bc_u32[4] = 0u;
        __syncthreads();
        const int nl = (int)S.list_n;
        for (int i = tid; i < nl; i += kThreads) {
          if ((uint32_t)((uint64_t)order_key(S.list_z[i]) >> shift) != prefix) continue;
          unsigned int rk = 0;  // members of the group with a smaller position
          for (int j = 0; j < nl; ++j)
            if ((uint32_t)((uint64_t)order_key(S.list_z[j]) >> shift) == prefix &&
                S.list_pos[j] < S.list_pos[i])
              ++rk;
          if (rk + 1 == tie_need) S.bc_u32[4] = S.list_pos[i];
        }
        __syncthreads();
        pos_thr = S.bc_u32[4];
      }
      unsigned int kept_loc = 0, tie_run = 0;
      stream_head(S, C, cseg, zseg, seg, resident,
                  [&](const float* z, const uint32_t* c, int nvalid, uint32_t pos0,
                      int64_t idx0, int r) {
        uint32_t bits = 0, ties = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (j < nvalid && ((c[j] >> (24 + h)) & 1u)) {
            bool keep = true, tie = false;
            if (!p.keep_all) {
              const uint32_t pre = (uint32_t)((uint64_t)order_key(z[j]) >> shift);
              keep = pre > prefix;
              tie = pre == prefix;
            }
            if (tie) {
              if (!rank_ties || (thr_mode && pos0 + (uint32_t)j <= pos_thr)) keep = true;
              else if (!thr_mode) ties |= 1u << j;
            }
            if (keep) bits |= 1u << j;
          }
        }
        if (rank_ties && !thr_mode) {  // ordered ranks of unlisted ties (rare)
          unsigned int tot;
          unsigned int rk = block_excl_scan(__popc(ties), &tot, S);
#pragma unroll
          for (int j = 0; j < 8; ++j)
            if ((ties >> j) & 1u) {
              if (tie_run + rk < tie_need) bits |= 1u << j;
              ++rk;
            }
          tie_run += tot;
        }
        kept_loc += __popc(bits);
        // 4 consecutive threads own the 32 candidates of one keep word
        uint32_t word = bits << (8 * (threadIdx.x & 3));
        word |= __shfl_xor_sync(0xffffffffu, word, 1);
        word |= __shfl_xor_sync(0xffffffffu, word, 2);
        if ((threadIdx.x & 3) == 0 && nvalid > 0) kptr(h, r)[(idx0 >> 5)] = word;
      });
      unsigned int ktot;
      block_excl_scan(kept_loc, &ktot, S);
      if (lc_base && tid == 0) lc_base[(int64_t)h * p.L + (p.L - level)] = (int32_t)ktot;
      }  // radix-select cut

      if (level == 1 && p.list_mode) {
        // ascending token list of head h: {0} (unless node 0 is kept) +
        // tokens of the kept level-1 nodes + causal tail
        __syncthreads();
        const int64_t qh = (int64_t)qi * p.Hq + (int64_t)kvh * G + h;
        int32_t* out = p.idx + qh * p.idx_cap;
        int r0 = 0;
        while (r0 < C && S.seg_n[r0] == 0) ++r0;
        const bool node0 =
            r0 < C && (cptr(cur, r0)[0] & kNodeMask) == 0u && (kptr(h, r0)[0] & 1u);
        const int64_t off0 = node0 ? 0 : 1;
        if (!node0 && tid == 0 && p.idx_cap > 0) out[0] = 0;
        unsigned int pos_run = 0;
        for (int r = 0; r < C; ++r) {
          const uint32_t* cc = cptr(cur, r);
          const uint32_t* kb = kptr(h, r);
          const int64_t n = S.seg_n[r];
          for (int64_t base = 0; base < n; base += kThreads) {
            const int64_t i = base + tid;
            const bool kh = i < n && ((kb[i >> 5] >> (i & 31)) & 1u);
            unsigned int tot;
            const unsigned int rk = block_excl_scan(kh ? 1u : 0u, &tot, S);
            if (kh) {
              const int64_t pos = off0 + (int64_t)b * (pos_run + rk);
              const int64_t node = cc[i] & kNodeMask;
              for (int c = 0; c < b; ++c)
                if (pos + c < p.idx_cap) out[pos + c] = (int32_t)(node * b + c);
            }
            pos_run += tot;
          }
        }
        const int64_t tail_start = p.span[p.L] * T_top;
        const int64_t tail_len = n_vis - tail_start;
        const int64_t tail_pos = off0 + (int64_t)b * pos_run;
        for (int64_t j = tid; j < tail_len; j += kThreads)
          if (tail_pos + j < p.idx_cap) out[tail_pos + j] = (int32_t)(tail_start + j);
        if (tid == 0) {
          const int64_t n = tail_pos + tail_len;
          p.n_idx[qh] = (int32_t)n;
          if (n > p.idx_cap) raise_status(p.status, ZHA_ERR_CAPACITY);
        }
      }
      __syncthreads();
    }
    cluster.sync();  // S2: keep bits of every head written

    // ------------------------------------------------------------------
    // 3. expand my segment into the next level's candidates
    // ------------------------------------------------------------------
    {
      const uint32_t* cc = cptr(cur, rank);
      uint32_t* cn = cptr(cur ^ 1, rank);
      unsigned int run = 0;
      for (int64_t base = 0; base < my_n; base += kThreads) {
        const int64_t i = base + tid;
        uint32_t km = 0u, cv = 0u;
        if (i < my_n) {
          cv = cc[i];
#pragma unroll
          for (int h = 0; h < G; ++h) km |= ((kptr(h, rank)[i >> 5] >> (i & 31)) & 1u) << h;
        }
        unsigned int tot;
        const unsigned int rk = block_excl_scan(km ? 1u : 0u, &tot, S);
        if (km) {
          const int64_t pos = (int64_t)run + rk;
          const uint32_t node = cv & kNodeMask;
          if (level > 1) {
            for (int c = 0; c < b; ++c)
              cn[pos * b + c] = (km << 24) | (node * (uint32_t)b + (uint32_t)c);
          } else if (!p.list_mode) {
            p.kept[((int64_t)unit * C + rank) * seg + pos] = (km << 24) | node;
          }
        }
        run += tot;
      }
      if (level == 1 && !p.list_mode && tid == 0)
        p.n_kept[(int64_t)unit * C + rank] = (int32_t)run;
      my_n = (int64_t)run * b;
      if (level > 1 && my_n > seg) {  // cannot happen: a segment holds every level-1 node
        raise_status(p.status, ZHA_ERR_WORKSPACE);
        my_n = seg;
      }
    }
    cur ^= 1;
    __syncthreads();
  }
  // no DSMEM access follows the last cluster barrier, so CTAs may exit freely
}

template <typename T, int D, int G>
cudaError_t launch_t(const TravParams& p, int64_t units, int C, cudaStream_t stream) {
  const size_t smem = sizeof(Smem);
  auto kern = traverse_kernel<T, D, G>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  if (C > 8) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(units * C), 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, p);
}

template <typename T, int D>
cudaError_t launch_g(int G, const TravParams& p, int64_t units, int C, cudaStream_t s) {
  switch (G) {
    case 1: return launch_t<T, D, 1>(p, units, C, s);
    case 2: return launch_t<T, D, 2>(p, units, C, s);
    case 4: return launch_t<T, D, 4>(p, units, C, s);
    case 8: return launch_t<T, D, 8>(p, units, C, s);
    default: return cudaErrorInvalidValue;
  }
}

int64_t seg_capacity(const Geometry& g) {
  // one segment can hold every level-1 node (an unbalanced frontier's worst case)
  return ((g.level_rows[0] + 1 + 31) / 32) * 32;
}

// Clusters of C CTAs that can be resident at once for this geometry.
template <typename T, int D, int G>
int max_clusters_t(int C) {
  auto kern = traverse_kernel<T, D, G>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)sizeof(Smem)) != cudaSuccess)
    return (cudaGetLastError(), 0);
  if (C > 8 && cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) !=
                   cudaSuccess)
    return (cudaGetLastError(), 0);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)C, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = sizeof(Smem);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) return (cudaGetLastError(), 0);
  return n;
}

template <typename T, int D>
int max_clusters_g(int G, int C) {
  switch (G) {
    case 1: return max_clusters_t<T, D, 1>(C);
    case 2: return max_clusters_t<T, D, 2>(C);
    case 4: return max_clusters_t<T, D, 4>(C);
    default: return max_clusters_t<T, D, 8>(C);
  }
}

int max_clusters(const Geometry& g, int C) {
  static int cache[2][2][4][5];  // dtype, d, G, log2 C (0 = not queried)
  const int i0 = g.dtype == ZHA_BF16, i1 = g.d == 128;
  const int i2 = g.G == 1 ? 0 : g.G == 2 ? 1 : g.G == 4 ? 2 : 3;
  const int i3 = C == 1 ? 0 : C == 2 ? 1 : C == 4 ? 2 : C == 8 ? 3 : 4;
  int& v = cache[i0][i1][i2][i3];
  if (v == 0) {
    int n;
    if (g.dtype == ZHA_BF16)
      n = g.d == 128 ? max_clusters_g<__nv_bfloat16, 128>(g.G, C)
                     : max_clusters_g<__nv_bfloat16, 64>(g.G, C);
    else
      n = g.d == 128 ? max_clusters_g<float, 128>(g.G, C) : max_clusters_g<float, 64>(g.G, C);
    v = n > 0 ? n : -1;
  }
  return v;
}

}  // namespace

// The largest power-of-two cluster (<= 16 CTAs) that keeps every unit resident
// in one wave and at most two CTAs per SM.
int traverse_cluster_size(const Geometry& g, int64_t units, int num_sms) {
  int best = 1;
  for (int C = 2; C <= kMaxCluster; C *= 2) {
    if (units * C > 2 * (int64_t)num_sms) break;
    const int n = max_clusters(g, C);
    if (n > 0 && n >= units) best = C;
  }
  return best;
}

size_t traverse_ws_bytes(const Geometry& g, int64_t units, int num_sms) {
  const int C = traverse_cluster_size(g, units, num_sms);
  const size_t seg = (size_t)seg_capacity(g);
  const size_t per = (size_t)C * seg * (2 * sizeof(uint32_t) + (size_t)g.G * sizeof(float)) +
                     (size_t)g.G * C * (seg / 32) * sizeof(uint32_t);
  return per * (size_t)units + 256;
}

size_t traverse_kept_bytes(const Geometry& g, int64_t units, int num_sms) {
  return (size_t)units * traverse_cluster_size(g, units, num_sms) * (size_t)seg_capacity(g) *
         sizeof(uint32_t);
}

int64_t traverse_kept_stride(const Geometry& g) { return seg_capacity(g); }

cudaError_t launch_traverse(const Geometry& g, const void* tree, const void* q,
                            const int32_t* seq_len, const int32_t* q_seq, const int32_t* q_pos,
                            int64_t nq, uint64_t p_q, int list_mode, const TraverseOut& out,
                            void* ws, size_t ws_bytes, int32_t* status, int num_sms,
                            cudaStream_t stream) {
  const int64_t units = nq * g.Hkv;
  if (units <= 0) return cudaSuccess;
  if (ws_bytes < traverse_ws_bytes(g, units, num_sms)) return cudaErrorInvalidValue;
  TravParams p{};
  p.tree = tree;
  for (int l = 0; l < g.L; ++l) {
    p.level_off[l] = g.level_off[l];
    p.level_rows[l] = g.level_rows[l];
    p.lnsize[l] = g.lnsize[l];
  }
  for (int l = 0; l <= g.L; ++l) p.span[l] = g.span[l];
  p.inv_sqrt_d = g.inv_sqrt_d;
  p.q = q;
  p.seq_len = seq_len;
  p.q_seq = q_seq;
  p.q_pos = q_pos;
  p.Hq = g.Hq;
  p.Hkv = g.Hkv;
  p.b = g.b;
  p.L = g.L;
  p.B = g.B;
  p.ncap = g.ncap;
  p.p_q = p_q;
  p.keep_all = p_q >= (1ull << 32);
  p.list_mode = list_mode;
  p.seg = seg_capacity(g);
  const int C = traverse_cluster_size(g, units, num_sms);
  unsigned char* w = static_cast<unsigned char*>(ws);
  p.cand = reinterpret_cast<uint32_t*>(w);
  w += sizeof(uint32_t) * (size_t)units * 2 * C * p.seg;
  p.zbuf = reinterpret_cast<float*>(w);
  w += sizeof(float) * (size_t)units * g.G * C * p.seg;
  p.kbits = reinterpret_cast<uint32_t*>(w);
  if (!list_mode) {
    if (!out.kept || !out.n_kept) return cudaErrorInvalidValue;
    p.kept = out.kept;
    p.n_kept = out.n_kept;
  }
  p.idx = out.idx;
  p.idx_cap = out.idx_cap;
  p.n_idx = out.n_idx;
  p.level_counts = out.level_counts;
  p.stats = out.stats;
  p.status = status;
  if (g.dtype == ZHA_BF16) {
    if (g.d == 128) return launch_g<__nv_bfloat16, 128>(g.G, p, units, C, stream);
    return launch_g<__nv_bfloat16, 64>(g.G, p, units, C, stream);
  }
  if (g.d == 128) return launch_g<float, 128>(g.G, p, units, C, stream);
  return launch_g<float, 64>(g.G, p, units, C, stream);
}

}  // namespace zha
