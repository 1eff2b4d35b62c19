// Top-down top-p traversal of the summary tree, all query heads of a KV head
// together.
//
// lefilia.fr page "Zyphra presente Zyphra Hierarchical Attention (ZHA) ...",
// paragraph 1: a query scores the top nodes, keeps the fewest nodes whose
// estimated attention mass reaches the fraction p, descends only into the kept
// branches until it reaches individual keys, and always keeps token 0.
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
// the segments in rank order is always sorted by node index. Per level:
//   1. score  -- each CTA scores its segment for all heads (canonical fp32
//                chains, 4 candidates x G heads per thread); the segment's
//                score extremes go to distributed shared memory.  cluster sync
//   2. cut    -- a distributed select per head. Every CTA histograms its own
//                segment for all heads at once into 256 buckets holding the
//                exact fixed-point mass and the count of their members; the
//                CTA owning head h sums the C histograms of h
//                through DSMEM, finds the bucket where the mass taken in
//                descending score order reaches the target, and publishes the
//                narrowed group.                      two cluster syncs a pass
//                The first pass buckets z linearly over the head's score
//                range, so the crossing group is small; later passes resolve
//                the group's order-preserving key 8 bits at a time. The
//                result is a rule per head: keep iff key > kthr, or key ==
//                kthr and the candidate is among the first quota[r] such
//                candidates of segment r (exact ties, node order).
//   3. expand -- each CTA applies the rules to its own segment and writes the
//                children of the nodes kept by any head, or, at level 1, the
//                kept list.
// No candidate, score or keep bit crosses CTAs through global memory.
// Canonical arithmetic (identical to the CPU oracle):
//   z = (dot(q, s) * inv_sqrt_d) + fp32(l ln b),  M = trunc(exp(z - zmax) 2^40),
//   need = ceil(T p_q / 2^32); keep the shortest prefix of (z desc, node asc)
//   whose mass reaches need (every candidate when p_q >= 2^32).
#include <atomic>

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
constexpr int kDigit = 8;                 // key bits resolved per radix pass
constexpr int kBuckets = 1 << kDigit;     // == kThreads: one bucket per thread
constexpr int kCandPerThread = 4;
constexpr uint32_t kNodeMask = 0x00ffffffu;
constexpr int kGather = 512;  // groups this small are finished by the head's owner alone
constexpr int kSingleMax = 512;  // frontiers this small are traversed by rank 0 alone
static_assert(kBuckets == kThreads, "one histogram bucket per thread");

enum HeadMode : int {
  kModeRadix = 0,     // group being narrowed by key digits
  kModeAll = 1,       // keep every candidate of the head
  kModeThr = 2,       // keep iff key >= kthr
  kModeTie = 3,       // keep iff key > kthr, or key == kthr within the segment's quota
  kModeQuant = 4,     // first pass pending: buckets are a linear map of z
  kModeGathered = 5,  // keep iff first-pass bucket > qbeta, or == qbeta and either
                      // key > kgmax or key in [kgmin, kgmax] and the owner marked
                      // the candidate kept
};

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
  float* zbuf;           // [units][C][seg][G]   scores, candidate-major
  uint8_t* qbuf;         // [units][C][seg][G]   first-pass bucket of each score
  uint8_t* mkbuf;        // [units][C][seg][G]   kModeGathered: owner's keep mark
  uint32_t* kept;        // [units][C][seg]     decode mode: union-kept level-1 nodes
  int32_t* n_kept;       // [units][C]
  int32_t* idx;          // [nq][Hq][idx_cap]   list mode
  int64_t idx_cap;
  int32_t* n_idx;
  int32_t* level_counts;
  int32_t* stats;        // [units][L]: union candidates scored per level (nullable)
  int32_t* status;
  // certified top-level selections (nullable): a unit with seed_ok != 0
  // starts one level below the top
  const int32_t* seed_ok;    // [units]
  const uint8_t* seed_mask;  // [units][seed_stride] bit h: head h keeps top node i
  const int32_t* seed_cnt;   // [units][G]
  int64_t seed_stride;
  // one CTA per unit (C = 1): shipped-member lists of kGather entries per
  // head in global memory (shared memory holds two CTAs per SM only with
  // kWarpGather-entry lists)
  float* glist_z;            // [units][G][kGather]
  uint32_t* glist_pos;       // [units][G][kGather]
};

// Cut state of one head. After every publish step it is identical on all CTAs
// of the cluster (each copies it from the head's owner).
struct HeadState {
  unsigned long long above;  // mass of the candidates ranked above the current group
  unsigned long long need;   // coverage target
  unsigned long long bmass;  // mass of the current group
  unsigned int prefix;       // kModeRadix: key prefix shared by the current group
  int shift;                 // kModeRadix: key bits below the prefix
  unsigned int kgmin, kgmax; // key range of the group (its members are exactly the
                             // head's candidates with a key in this range)
  float zlo, zscale;         // kModeQuant: bucket = clamp(floor((z - zlo) zscale))
  unsigned int cabove;       // candidates ranked above the current group
  unsigned int bcnt;         // candidates in the current group
  int mode;                  // HeadMode
  unsigned int kthr;         // threshold key of the final rule
  unsigned int count;        // kept candidates (the level count)
  unsigned int qbeta;        // first-pass bucket of the group (0xffffffff: none)
  int zfree;                 // the final rule was set while the group was still the
                             // whole first-pass bucket: every candidate's fate follows
                             // from its bucket (and, kModeGathered, its mark) alone
  unsigned int quota[kMaxCluster];  // kModeTie: kept members of each segment
};

// Per-CTA values read by the other CTAs through DSMEM after the score sync;
// double-buffered by level parity so a fast CTA never overwrites a value a
// slow one is still reading.
struct Xch {
  unsigned int count;             // candidates in my segment
  unsigned int hcount[kMaxGroup]; // ... of which in head h's frontier
  float zmax[kMaxGroup];
  float zmin[kMaxGroup];
};

struct Smem {
  alignas(16) unsigned int hist_lo[kMaxGroup][kBuckets];       // bucket masses, low and
  alignas(16) unsigned int hist_hi[kMaxGroup][kBuckets];       // high 32 bits
  alignas(16) unsigned int hist_c[kMaxGroup][kBuckets];        // bucket counts
  alignas(16) float q[kMaxGroup * 128];                        // [i][8] fp32, i < D
  HeadState pub[kMaxGroup];   // owner's result of the last pass
  HeadState st[kMaxGroup];    // this CTA's copy of every head's state
  Xch xch[2];
  unsigned int seg_n[kMaxCluster];     // every rank's segment size at this level
  float zmax[kMaxGroup];               // cluster-wide score maximum per head
  unsigned long long red_u64[kWarps][2];
  unsigned int red_u32[kWarps][2];
  unsigned int found[6];
  unsigned long long found_u64[2];
  unsigned int kc[kMaxGroup];          // kept candidates of my segment per head
  unsigned int node0;                  // list mode: heads keeping node 0 (bit mask)
  unsigned int tie_run[kMaxGroup];     // kModeTie: members seen so far (expand)
  float red_f[kWarps][kMaxGroup][2];
  float g_zmax[kMaxCluster][kMaxGroup];          // gathered per-rank extremes and counts
  float g_zmin[kMaxCluster][kMaxGroup];
  unsigned int g_hcnt[kMaxCluster][kMaxGroup];
  unsigned int nh[kMaxGroup];                    // candidates of head h at this level
  unsigned int tie_cnt[kMaxCluster];             // crossing-bucket members per rank
  unsigned int my_hcnt[kMaxGroup];               // my segment's candidates in head h's frontier
  // score_segment: each thread's next summary-row chunks in flight (cp.async)
  alignas(16) uint4 ring[3][kCandPerThread][kThreads];
  // groups of at most kGather members are shipped to the head's owner: one
  // list per owned head (slot h / C), filled by every rank through DSMEM;
  // the lists follow the struct in dynamic shared memory (list_z, list_pos)
  unsigned int mlist_n[kMaxGroup];
  alignas(16) unsigned long long mrank_m[kGather];   // member sort keys
  unsigned long long red_scan[kWarps];
  unsigned int lm_n;                    // members staged in S.mrank_m before shipping
  // rank 0's hand-over of a grown frontier to the whole cluster
  int sw_level;                         // level the cluster resumes at (0: finished)
  int sw_cur;                           // candidate buffer holding the frontier
  unsigned int sw_n;                    // frontier size
};

// Shipped-member lists after the struct: z[slots][cap], then
// position[slots][cap] with position = (rank << 24) | segment index. The area
// holds list_slots(G, C) * kGather entries of each; while rank 0 works alone
// it owns every head and splits the area into G slots of fewer entries.
__device__ __forceinline__ float* list_z(Smem& S) {
  return reinterpret_cast<float*>(reinterpret_cast<unsigned char*>(&S) + sizeof(Smem));
}
__device__ __forceinline__ uint32_t* list_pos(Smem& S, int slots, int cap) {
  return reinterpret_cast<uint32_t*>(list_z(S) + slots * cap);
}
// owned heads per CTA (lists needed)
__host__ __device__ __forceinline__ int list_slots(int G, int C) { return (G + C - 1) / C; }

// Exclusive scan of v over the CTA in thread order; *total receives the sum.
__device__ __forceinline__ unsigned int block_excl_scan(unsigned int v, unsigned int* total,
                                                        Smem& S, int slot = 0) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  unsigned int x = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const unsigned int y = __shfl_up_sync(0xffffffffu, x, off);
    if (lane >= off) x += y;
  }
  if (lane == 31) S.red_u32[warp][slot] = x;
  __syncthreads();
  unsigned int wbase = 0, tot = 0;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) {
    const unsigned int s = S.red_u32[w][slot];
    if (w < warp) wbase += s;
    tot += s;
  }
  __syncthreads();
  *total = tot;
  return wbase + x - v;
}

// L2 eviction policy of the per-candidate scores, which every pass of the cut
// re-reads (evict last).
__device__ __forceinline__ uint64_t policy_evict_last() {
  uint64_t pol;
  asm("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}
__device__ __forceinline__ void st_policy(float4* ptr, float4 v, uint64_t pol) {
  asm volatile("st.global.L2::cache_hint.v4.f32 [%0], {%1, %2, %3, %4}, %5;" ::"l"(ptr), "f"(v.x),
               "f"(v.y), "f"(v.z), "f"(v.w), "l"(pol)
               : "memory");
}

// The G scores of candidate i (candidate-major rows of G floats).
template <int G>
__device__ __forceinline__ void load_scores(const float* zown, int64_t i, float* z) {
  if constexpr (G >= 4) {
#pragma unroll
    for (int j = 0; j < G / 4; ++j) {
      const float4 v = *reinterpret_cast<const float4*>(zown + i * G + 4 * j);
      z[4 * j] = v.x;
      z[4 * j + 1] = v.y;
      z[4 * j + 2] = v.z;
      z[4 * j + 3] = v.w;
    }
  } else if constexpr (G == 2) {
    const float2 v = *reinterpret_cast<const float2*>(zown + i * 2);
    z[0] = v.x;
    z[1] = v.y;
  } else {
    z[0] = zown[i];
  }
}

// The G first-pass bucket bytes of candidate i, packed (byte h = head h).
template <int G>
__device__ __forceinline__ uint64_t load_qrow(const uint8_t* q, int64_t i) {
  if constexpr (G == 8) return __ldcg(reinterpret_cast<const unsigned long long*>(q) + i);
  else if constexpr (G == 4) return __ldcg(reinterpret_cast<const unsigned int*>(q) + i);
  else if constexpr (G == 2) return __ldcg(reinterpret_cast<const unsigned short*>(q) + i);
  else return __ldcg(q + i);
}
template <int G>
__device__ __forceinline__ void store_qrow(uint8_t* q, int64_t i, uint64_t v) {
  if constexpr (G == 8) reinterpret_cast<unsigned long long*>(q)[i] = v;
  else if constexpr (G == 4) reinterpret_cast<unsigned int*>(q)[i] = (unsigned int)v;
  else if constexpr (G == 2) reinterpret_cast<unsigned short*>(q)[i] = (unsigned short)v;
  else q[i] = (uint8_t)v;
}

// Bit h set where byte h of a is greater than / equal to byte h of b, or
// where byte h of a is nonzero (SIMD byte compares, then the top bit of each
// 0x00/0xff byte gathered into one byte by a multiply).
__device__ __forceinline__ uint32_t gather_bits(uint64_t m) {
  return (uint32_t)(((m & 0x8080808080808080ull) * 0x0002040810204081ull) >> 56);
}
__device__ __forceinline__ uint32_t bytes_gt(uint64_t a, uint64_t b) {
  return gather_bits(((uint64_t)__vcmpgtu4((unsigned)(a >> 32), (unsigned)(b >> 32)) << 32) |
                     __vcmpgtu4((unsigned)a, (unsigned)b));
}
__device__ __forceinline__ uint32_t bytes_eq(uint64_t a, uint64_t b) {
  return gather_bits(((uint64_t)__vcmpeq4((unsigned)(a >> 32), (unsigned)(b >> 32)) << 32) |
                     __vcmpeq4((unsigned)a, (unsigned)b));
}
__device__ __forceinline__ uint32_t bytes_nz(uint64_t a) {
  return gather_bits(((uint64_t)__vcmpne4((unsigned)(a >> 32), 0u) << 32) |
                     __vcmpne4((unsigned)a, 0u));
}

// The canonical dot products of this thread's rows (up to K of them) with the
// G queries, the rows' 16-byte chunks streamed through this thread's slots of
// S.ring with DEPTH chunks per row (K * DEPTH <= 12): chunk ch of row k sits
// in slot (ch % DEPTH) * K + k. Only this thread writes and reads its slots,
// so waiting on its own cp.async groups suffices.
template <typename T, int D, int G, int K, int DEPTH>
__device__ __forceinline__ void stream_rows(Smem& S, const uint4* const* rows, const bool* ok,
                                            float2 (*acc)[(G + 1) / 2], float* acc1) {
  static_assert(K * DEPTH <= 3 * kCandPerThread, "ring slots per thread");
  constexpr int kPer = Elem<T>::kPerChunk;
  constexpr int kNch = D * (int)sizeof(T) / 16;
  const int tid = threadIdx.x;
  uint4* slots = &S.ring[0][0][0];  // slot s of this thread at slots[s * kThreads + tid]
#pragma unroll
  for (int st = 0; st < DEPTH - 1; ++st) {
#pragma unroll
    for (int k = 0; k < K; ++k)
      if (ok[k] && st < kNch) cp_async16(&slots[(st * K + k) * kThreads + tid], rows[k] + st);
    cp_async_commit();
  }
#pragma unroll 1
  for (int ch = 0; ch < kNch; ++ch) {
    if (ch + DEPTH - 1 < kNch) {
      const int st = (ch + DEPTH - 1) % DEPTH;
#pragma unroll
      for (int k = 0; k < K; ++k)
        if (ok[k]) cp_async16(&slots[(st * K + k) * kThreads + tid], rows[k] + ch + DEPTH - 1);
    }
    cp_async_commit();
    cp_async_wait<DEPTH - 1>();  // this thread's copies of chunk ch have landed
    float x[K][kPer];
#pragma unroll
    for (int k = 0; k < K; ++k) {
      const uint4 c = ok[k] ? slots[((ch % DEPTH) * K + k) * kThreads + tid] : make_uint4(0, 0, 0, 0);
      Elem<T>::unpack(c, x[k]);
    }
#pragma unroll
    for (int e = 0; e < kPer; ++e) {
      const float* qv = S.q + (ch * kPer + e) * kMaxGroup;
      if constexpr (G == 1) {
#pragma unroll
        for (int k = 0; k < K; ++k) acc1[k] = __fmaf_rn(qv[0], x[k][e], acc1[k]);
      } else if constexpr (G == 2) {
        const float2 q2 = *reinterpret_cast<const float2*>(qv);
#pragma unroll
        for (int k = 0; k < K; ++k) acc[k][0] = ffma2(q2, make_float2(x[k][e], x[k][e]), acc[k][0]);
      } else {
        float4 q4[G / 4];
#pragma unroll
        for (int j = 0; j < G / 4; ++j) q4[j] = *reinterpret_cast<const float4*>(qv + 4 * j);
#pragma unroll
        for (int k = 0; k < K; ++k) {
          const float2 xx = make_float2(x[k][e], x[k][e]);
#pragma unroll
          for (int j = 0; j < G / 4; ++j) {
            acc[k][2 * j] = ffma2(make_float2(q4[j].x, q4[j].y), xx, acc[k][2 * j]);
            acc[k][2 * j + 1] = ffma2(make_float2(q4[j].z, q4[j].w), xx, acc[k][2 * j + 1]);
          }
        }
      }
    }
  }
}

// Score candidates [0, n) of a segment against G queries; up to 4 candidates
// per thread so that each broadcast of q[i][0..G) feeds 4*G chains. The G scores
// of candidate i go to zseg[i*G .. i*G+G). lmax/lmin accumulate the extremes
// over the candidates in each head's frontier.
template <typename T, int D, int G>
__device__ __forceinline__ void score_segment(const TravParams& p, Smem& S, const T* lvl,
                                              const uint32_t* cand, float* zseg, int64_t n,
                                              float lns, float* lmax, float* lmin, bool top,
                                              int64_t top_base) {
  const int tid = threadIdx.x;
  const uint64_t pol_z = policy_evict_last();
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
    // each thread streams its rows' 16-byte chunks through its own 12 slots of
    // a shared-memory ring: 11 chunks in flight with one row, 5 per row with
    // two rows, 2 per row with three or four
    const int kr = ok[3] ? 4 : ok[2] ? 3 : ok[1] ? 2 : ok[0] ? 1 : 0;
    if (kr == 1) {
      stream_rows<T, D, G, 1, 12>(S, rows, ok, acc, acc1);
    } else if (kr == 2) {
      stream_rows<T, D, G, 2, 6>(S, rows, ok, acc, acc1);
    } else if (kr > 2) {
      stream_rows<T, D, G, 4, 3>(S, rows, ok, acc, acc1);
    }
#pragma unroll
    for (int k = 0; k < kCandPerThread; ++k) {
      if (!ok[k]) continue;
      const int64_t i = base + k * kThreads + tid;
      float z[G];
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float raw = (G == 1) ? acc1[k] : ((h & 1) ? acc[k][h / 2].y : acc[k][h / 2].x);
        z[h] = __fadd_rn(__fmul_rn(raw, p.inv_sqrt_d), lns);
        if ((pm[k] >> h) & 1u) {
          lmax[h] = fmaxf(lmax[h], z[h]);
          lmin[h] = fminf(lmin[h], z[h]);
        }
      }
      if constexpr (G >= 4) {
#pragma unroll
        for (int j = 0; j < G / 4; ++j)
          st_policy(reinterpret_cast<float4*>(zseg + i * G + 4 * j),
                    make_float4(z[4 * j], z[4 * j + 1], z[4 * j + 2], z[4 * j + 3]), pol_z);
      } else if constexpr (G == 2) {
        *reinterpret_cast<float2*>(zseg + i * 2) = make_float2(z[0], z[1]);
      } else {
        zseg[i] = z[0];
      }
    }
  }
}

// Adds (mass m, count 1) to bucket d of head h. The 64-bit mass goes into two
// 32-bit counters with an explicit carry (a 64-bit shared-memory add is far
// slower under contention).
__device__ __forceinline__ void hist_add(Smem& S, int h, uint32_t d, unsigned long long m) {
  const unsigned lo = (unsigned)m;
  const unsigned old = atomicAdd(&S.hist_lo[h][d], lo);
  const unsigned hi = (unsigned)(m >> 32) + ((old + lo < old) ? 1u : 0u);
  if (hi) atomicAdd(&S.hist_hi[h][d], hi);
  atomicAdd(&S.hist_c[h][d], 1u);
}

// hist_add for all G heads of one candidate at once, without branches: head
// h adds (m[h], c[h]) to bucket d[h] (c[h] = 0 and m[h] = 0 for a head that
// does not count this candidate). The G low-word atomics are issued back to
// back before any carry is resolved.
template <int G>
__device__ __forceinline__ void hist_add_heads(Smem& S, const uint32_t* d,
                                               const unsigned long long* m, const uint32_t* c) {
  unsigned old[G];
#pragma unroll
  for (int h = 0; h < G; ++h) old[h] = c[h] ? atomicAdd(&S.hist_lo[h][d[h]], (unsigned)m[h]) : 0u;
#pragma unroll
  for (int h = 0; h < G; ++h) {
    const unsigned lo = (unsigned)m[h];
    const unsigned hi = (unsigned)(m[h] >> 32) + ((old[h] + lo < old[h]) ? 1u : 0u);
    if (hi) atomicAdd(&S.hist_hi[h][d[h]], hi);
    if (c[h]) atomicAdd(&S.hist_c[h][d[h]], c[h]);
  }
}

// The state of a head after a pass found its crossing bucket beta (ok):
// above / cabove are the mass and count ranked above the bucket, bcnt / bmass
// the bucket's, [gmin, gmax] its key interval and tie_cnt[r] its members in
// segment r.
__device__ __forceinline__ HeadState narrow_state(const TravParams& p, const HeadState& s0,
                                                  bool quant, bool ok, unsigned long long need,
                                                  unsigned beta, unsigned long long above,
                                                  unsigned cabove, unsigned bcnt,
                                                  unsigned long long bmass, uint32_t gmin,
                                                  uint32_t gmax, const unsigned* tie_cnt, int C,
                                                  unsigned nh) {
  HeadState ns = s0;
  ns.need = need;
  if (!ok) {  // cannot happen with exact sums; keep everything rather than loop
    raise_status(p.status, ZHA_ERR_INTERNAL);
    ns.mode = kModeAll;
    ns.count = nh;
    return ns;
  }
  ns.above = above;
  ns.cabove = cabove;
  ns.bmass = bmass;
  ns.bcnt = bcnt;
  ns.kgmin = gmin;
  ns.kgmax = gmax;
  if (quant) ns.qbeta = beta;
  ns.zfree = quant ? 1 : 0;  // a final rule set now needs no scores in the expand
  ns.mode = kModeRadix;
  if (bcnt == 1u) {
    ns.mode = kModeThr;  // the group's only member is the last kept candidate;
    ns.kthr = ns.kgmin;  // no other candidate has a key in the group's interval
    ns.count = ns.cabove + 1u;
  } else if (ns.kgmin == ns.kgmax) {
    // bcnt members share one key, hence one z and one mass: keep the first
    // tie_need of them in node order
    const unsigned long long mt = ns.bmass / bcnt;
    const unsigned long long rem = need - ns.above;
    const unsigned long long tn = mt ? (rem + mt - 1) / mt : bcnt;
    ns.kthr = ns.kgmin;
    if (tn >= bcnt) {
      ns.mode = kModeThr;
      ns.count = ns.cabove + bcnt;
    } else {
      ns.mode = kModeTie;
      ns.count = ns.cabove + (unsigned)tn;
      unsigned long long run = 0;
      for (int r = 0; r < C; ++r) {
        const unsigned long long cr = tie_cnt[r];
        ns.quota[r] = (unsigned)(run >= tn ? 0ull : (tn - run < cr ? tn - run : cr));
        run += cr;
      }
    }
  }
  return ns;
}

// Owner step of one pass for head h (every thread of the owner CTA calls it):
// sums the C per-rank histograms of h through DSMEM, finds the bucket where
// the mass in descending score order reaches the target, narrows the head's
// state to that bucket's group and leaves it in S.pub[h].
template <int G>
__device__ __noinline__ void owner_pass(const TravParams& p, Smem& S, cg::cluster_group& cluster,
                                        int C, int h) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const HeadState s0 = S.st[h];
  const bool quant = s0.mode == kModeQuant;
  int nb = kBuckets;
  if (!quant) {
    int sh, w;
    radix_digit(s0.kgmin, s0.kgmax, &sh, &w);
    nb = 1 << w;
  }
  unsigned long long m = 0;
  unsigned int c = 0;
  if (tid < nb) {
#pragma unroll
    for (int r = 0; r < kMaxCluster; ++r) {
      if (r < C) {
        const Smem* R = cluster.map_shared_rank(&S, r);
        m += ((unsigned long long)R->hist_hi[h][tid] << 32) | R->hist_lo[h][tid];
        c += R->hist_c[h][tid];
      }
    }
  }
  // suffix sums over buckets (thread t = bucket t; higher buckets rank first)
  unsigned long long xs = m;
  unsigned int xc = c;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const unsigned long long ym = __shfl_down_sync(0xffffffffu, xs, off);
    const unsigned int yc = __shfl_down_sync(0xffffffffu, xc, off);
    if (lane + off < 32) {
      xs += ym;
      xc += yc;
    }
  }
  if (lane == 0) {
    S.red_u64[warp][0] = xs;
    S.red_u32[warp][0] = xc;
  }
  if (tid == 0) S.found[0] = 0xffffffffu;
  __syncthreads();
  unsigned long long hm = 0, total = 0;
  unsigned int hc = 0;
#pragma unroll
  for (int w2 = 0; w2 < kWarps; ++w2) {
    total += S.red_u64[w2][0];
    if (w2 > warp) {
      hm += S.red_u64[w2][0];
      hc += S.red_u32[w2][0];
    }
  }
  // the first pass sees every candidate of the head: its total fixes the target
  const unsigned long long need = quant ? ceil_mul_shift32(total, p.p_q) : s0.need;
  const unsigned long long above = s0.above + hm + (xs - m);  // mass of buckets > tid
  if (tid < nb && above < need && above + m >= need) {
    S.found[0] = (unsigned)tid;
    S.found[1] = s0.cabove + hc + (xc - c);
    S.found[2] = c;
    S.found_u64[0] = above;
    S.found_u64[1] = m;
  }
  __syncthreads();
  const unsigned beta = S.found[0];
  const bool ok = beta != 0xffffffffu;
  const unsigned bcnt = ok ? S.found[2] : 0u;
  // the group's key interval: the bucket's interval on the first pass, the
  // digit's sub-interval of the previous group on later passes
  uint32_t gmin = 0, gmax = 0;
  if (ok) {
    if (quant && s0.zscale == 0.0f) {  // every score equals zlo
      gmin = gmax = order_key(s0.zlo);
    } else if (quant) {
      if (tid == 0) quant_interval(s0.zlo, s0.zscale, beta, &S.found[3], &S.found[4]);
      __syncthreads();
      gmin = S.found[3];
      gmax = S.found[4];
    } else {
      int sh, w;
      radix_digit(s0.kgmin, s0.kgmax, &sh, &w);
      const uint32_t top = (uint32_t)(((unsigned long long)s0.kgmin >> (sh + w)) << (sh + w));
      const uint32_t dlo = top | (beta << sh);
      const uint32_t dhi = dlo | (uint32_t)((1ull << sh) - 1ull);
      gmin = dlo > s0.kgmin ? dlo : s0.kgmin;
      gmax = dhi < s0.kgmax ? dhi : s0.kgmax;
    }
  }
  const bool tie = ok && bcnt > 1u && gmin == gmax;
  if (tie && tid < C) {  // members of the tie group in each segment
    const Smem* R = cluster.map_shared_rank(&S, tid);
    S.tie_cnt[tid] = R->hist_c[h][beta];
  }
  if (tie) __syncthreads();
  if (tid == 0)
    S.pub[h] = narrow_state(p, s0, quant, ok, need, beta, S.found_u64[0], S.found[1], bcnt,
                            S.found_u64[1], gmin, gmax, S.tie_cnt, C, S.nh[h]);
  __syncthreads();
}

// Owner step for a head whose group (at most kGather members) has been
// shipped to the lists mz/mpos (listed entries): sorts the members by
// (z desc, position asc) (bitonic network on (key << 32 | ~position)), finds
// the shortest prefix whose mass reaches what the group must still cover,
// marks every member's fate in mkbuf (the keep byte of (segment, index, head))
// and publishes kModeGathered in S.pub[h].
template <int G>
__device__ __noinline__ void owner_finish(const TravParams& p, Smem& S, int h, const float* mz,
                                          const uint32_t* mpos, unsigned listed, int cap,
                                          uint8_t* mk_u, int64_t seg) {
  static_assert(kGather == 2 * kThreads, "two sort slots per thread");
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const HeadState s0 = S.st[h];
  const int n = (int)(listed < (unsigned)cap ? listed : cap);
  int np2 = 2;
  while (np2 < n) np2 <<= 1;
  unsigned long long* key = S.mrank_m;  // sort keys, descending
  for (int i = tid; i < np2; i += kThreads)
    key[i] = i < n ? ((unsigned long long)order_key(mz[i]) << 32) | (0xffffffffu - mpos[i])
                   : 0ull;
  __syncthreads();
  for (int k = 2; k <= np2; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int i = tid; i < np2; i += kThreads) {
        const int l = i ^ j;
        if (l > i) {
          const unsigned long long a = key[i], b = key[l];
          const bool desc = (i & k) == 0;
          if (desc ? a < b : a > b) {
            key[i] = b;
            key[l] = a;
          }
        }
      }
      __syncthreads();
    }
  }
  // masses in rank order; thread t owns ranks 2t and 2t + 1
  const float zmax = S.zmax[h];
  const int r0 = 2 * tid;
  const unsigned long long m0 =
      r0 < n ? mass_fixed(key_float((uint32_t)(key[r0] >> 32)), zmax) : 0ull;
  const unsigned long long m1 =
      r0 + 1 < n ? mass_fixed(key_float((uint32_t)(key[r0 + 1] >> 32)), zmax) : 0ull;
  unsigned long long x = m0 + m1;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const unsigned long long y = __shfl_up_sync(0xffffffffu, x, off);
    if (lane >= off) x += y;
  }
  if (lane == 31) S.red_scan[warp] = x;
  if (tid == 0) S.found[5] = 0xffffffffu;
  __syncthreads();
  unsigned long long run = 0;
#pragma unroll
  for (int w = 0; w < kWarps; ++w)
    if (w < warp) run += S.red_scan[w];
  run += x - (m0 + m1);  // mass of ranks < r0
  const unsigned long long rem = s0.need - s0.above;  // > 0: the group holds the crossing
  if (r0 < n && run < rem && run + m0 >= rem) S.found[5] = (unsigned)r0;
  if (r0 + 1 < n && run + m0 < rem && run + m0 + m1 >= rem) S.found[5] = (unsigned)r0 + 1u;
  __syncthreads();
  unsigned int k = S.found[5];
  const bool ok = k != 0xffffffffu && n == (int)s0.bcnt;
  if (!ok) k = (unsigned)n - 1u;  // cannot happen with exact sums: keep the whole group
  for (int r = tid; r < n; r += kThreads) {
    const uint32_t pi = 0xffffffffu - (uint32_t)key[r];
    const int64_t rr = pi >> 24, idx = pi & kNodeMask;
    mk_u[(rr * seg + idx) * G + h] = (unsigned)r <= k ? 1 : 0;
  }
  if (tid == 0) {
    if (!ok) raise_status(p.status, ZHA_ERR_INTERNAL);
    HeadState ns = s0;
    ns.mode = kModeGathered;
    ns.count = s0.cabove + k + 1u;
    S.pub[h] = ns;
  }
  __syncthreads();
}

// Single-CTA versions of the owner steps (rank 0 alone owns every head): warp
// h handles head h, so the G heads are narrowed concurrently. Same results as
// owner_pass / owner_finish with C = 1.
constexpr int kWarpGather = kGather / kMaxGroup;  // members per head, single-CTA gathers

template <int G>
__device__ __noinline__ void owner_pass_warp(const TravParams& p, Smem& S, int h) {
  const int lane = threadIdx.x & 31;
  const HeadState s0 = S.st[h];
  const bool quant = s0.mode == kModeQuant;
  int nb = kBuckets;
  if (!quant) {
    int sh, w;
    radix_digit(s0.kgmin, s0.kgmax, &sh, &w);
    nb = 1 << w;
  }
  constexpr int kPer = kBuckets / 32;  // buckets per lane, lane-major
  unsigned long long m[kPer];
  unsigned int c[kPer];
  unsigned long long tm = 0;
  unsigned int tc = 0;
#pragma unroll
  for (int j = 0; j < kPer; ++j) {
    const int d = lane * kPer + j;
    m[j] = d < nb ? ((unsigned long long)S.hist_hi[h][d] << 32) | S.hist_lo[h][d] : 0ull;
    c[j] = d < nb ? S.hist_c[h][d] : 0u;
    tm += m[j];
    tc += c[j];
  }
  unsigned long long xs = tm;  // inclusive suffix over lanes (higher lanes rank first)
  unsigned int xc = tc;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const unsigned long long ym = __shfl_down_sync(0xffffffffu, xs, off);
    const unsigned int yc = __shfl_down_sync(0xffffffffu, xc, off);
    if (lane + off < 32) {
      xs += ym;
      xc += yc;
    }
  }
  const unsigned long long total = __shfl_sync(0xffffffffu, xs, 0);
  const unsigned long long need = quant ? ceil_mul_shift32(total, p.p_q) : s0.need;
  unsigned long long run = s0.above + (xs - tm);
  unsigned int runc = s0.cabove + (xc - tc);
  int fbeta = -1;
  unsigned long long fabove = 0, fbmass = 0;
  unsigned int fcab = 0, fbcnt = 0;
#pragma unroll
  for (int j = kPer - 1; j >= 0; --j) {
    const int d = lane * kPer + j;
    if (d < nb && run < need && run + m[j] >= need) {
      fbeta = d;
      fabove = run;
      fbmass = m[j];
      fcab = runc;
      fbcnt = c[j];
    }
    run += m[j];
    runc += c[j];
  }
  const unsigned fmask = __ballot_sync(0xffffffffu, fbeta >= 0);
  const bool ok = fmask != 0u;
  const int src = ok ? __ffs(fmask) - 1 : 0;
  const unsigned beta = (unsigned)__shfl_sync(0xffffffffu, fbeta, src);
  const unsigned long long above = __shfl_sync(0xffffffffu, fabove, src);
  const unsigned long long bmass = __shfl_sync(0xffffffffu, fbmass, src);
  const unsigned cabove = __shfl_sync(0xffffffffu, fcab, src);
  const unsigned bcnt = __shfl_sync(0xffffffffu, fbcnt, src);
  if (lane == 0) {
    uint32_t gmin = 0, gmax = 0;
    if (ok) {
      if (quant && s0.zscale == 0.0f) {
        gmin = gmax = order_key(s0.zlo);
      } else if (quant) {
        quant_interval(s0.zlo, s0.zscale, beta, &gmin, &gmax);
      } else {
        int sh, w;
        radix_digit(s0.kgmin, s0.kgmax, &sh, &w);
        const uint32_t top = (uint32_t)(((unsigned long long)s0.kgmin >> (sh + w)) << (sh + w));
        const uint32_t dlo = top | (beta << sh);
        const uint32_t dhi = dlo | (uint32_t)((1ull << sh) - 1ull);
        gmin = dlo > s0.kgmin ? dlo : s0.kgmin;
        gmax = dhi < s0.kgmax ? dhi : s0.kgmax;
      }
    }
    const unsigned tie_cnt[1] = {bcnt};
    S.pub[h] = narrow_state(p, s0, quant, ok, need, beta, above, cabove, bcnt, bmass, gmin, gmax,
                            tie_cnt, 1, S.nh[h]);
  }
  __syncwarp();
}

template <int G>
__device__ __noinline__ void owner_finish_warp(const TravParams& p, Smem& S, int h, int slots,
                                               int cap, uint8_t* mk_u, int64_t seg) {
  const int lane = threadIdx.x & 31;
  const HeadState s0 = S.st[h];
  const int n = (int)(S.mlist_n[h] < (unsigned)cap ? S.mlist_n[h] : cap);
  const float* mz = list_z(S) + h * cap;
  const uint32_t* mpos = list_pos(S, slots, cap) + h * cap;
  unsigned long long* mass = S.mrank_m + h * kWarpGather;  // by rank
  const float zmax = S.zmax[h];
  constexpr int kPerLane = kWarpGather / 32;
  unsigned rk[kPerLane];
#pragma unroll
  for (int t = 0; t < kPerLane; ++t) {
    const int i = lane + 32 * t;
    rk[t] = 0u;
    if (i < n) {
      const float zi = mz[i];
      const uint32_t pi = mpos[i];
      for (int j = 0; j < n; ++j) {
        const float zj = mz[j];
        rk[t] += (zj > zi || (zj == zi && mpos[j] < pi)) ? 1u : 0u;
      }
      mass[rk[t]] = mass_fixed(zi, zmax);
    }
  }
  __syncwarp();
  // lane l owns ranks kPerLane*l .. kPerLane*l + kPerLane - 1
  unsigned long long mr[kPerLane], tsum = 0;
#pragma unroll
  for (int t = 0; t < kPerLane; ++t) {
    const int r = kPerLane * lane + t;
    mr[t] = r < n ? mass[r] : 0ull;
    tsum += mr[t];
  }
  unsigned long long x = tsum;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const unsigned long long y = __shfl_up_sync(0xffffffffu, x, off);
    if (lane >= off) x += y;
  }
  unsigned long long run = x - tsum;  // mass of lower ranks
  const unsigned long long rem = s0.need - s0.above;
  int kf = -1;
#pragma unroll
  for (int t = 0; t < kPerLane; ++t) {
    const int r = kPerLane * lane + t;
    if (r < n && run < rem && run + mr[t] >= rem) kf = r;
    run += mr[t];
  }
  const unsigned kmask = __ballot_sync(0xffffffffu, kf >= 0);
  const bool ok = kmask != 0u && n == (int)s0.bcnt;
  unsigned k = kmask ? (unsigned)__shfl_sync(0xffffffffu, kf, __ffs(kmask) - 1) : 0u;
  if (!ok) k = (unsigned)n - 1u;  // cannot happen with exact sums: keep the whole group
#pragma unroll
  for (int t = 0; t < kPerLane; ++t) {
    const int i = lane + 32 * t;
    if (i < n) {
      const uint32_t pi = mpos[i];
      mk_u[((int64_t)(pi >> 24) * seg + (pi & kNodeMask)) * G + h] = rk[t] <= k ? 1 : 0;
    }
  }
  if (lane == 0) {
    if (!ok) raise_status(p.status, ZHA_ERR_INTERNAL);
    HeadState ns = s0;
    ns.mode = kModeGathered;
    ns.count = s0.cabove + k + 1u;
    S.pub[h] = ns;
  }
  __syncwarp();
}

// After the hand-over barrier: reads where rank 0 left its frontier and copies
// this rank's equal slice of it (rank 0's segment of buffer *cur) into this
// rank's segment of the same buffer. Returns the slice length; *level = 0
// when rank 0 finished alone.
__device__ __noinline__ int64_t join_frontier(Smem& S, cg::cluster_group& cluster, int C,
                                              int rank, uint32_t* cand_u, int64_t seg,
                                              int* level, int* cur) {
  const Smem* R0 = cluster.map_shared_rank(&S, 0);
  *level = R0->sw_level;
  *cur = R0->sw_cur;
  const int64_t n = R0->sw_n;
  int64_t len = 0;
  if (*level > 0) {
    const int64_t lo = n * rank / C, hi = n * (rank + 1) / C;
    const uint32_t* src = cand_u + (int64_t)*cur * C * seg;  // rank 0's segment
    uint32_t* dst = cand_u + ((int64_t)*cur * C + rank) * seg;
    for (int64_t g = lo + threadIdx.x; g < hi; g += kThreads) dst[g - lo] = __ldcg(src + g);
    len = hi - lo;
    if (threadIdx.x < kMaxGroup) S.my_hcnt[threadIdx.x] = 0u;  // rank 0 carries the totals
  }
  __syncthreads();
  return len;
}

// A certified top-level selection (prefill on the tensor cores) expanded into
// the frontier of the level below, as the expand step would write it: the b
// children of every top node some head keeps, in node order, each carrying the
// mask of the heads that keep its parent. Records the top level's per-head
// counts and candidates. Returns the frontier size.
template <int G>
__device__ __noinline__ int64_t seed_frontier(const TravParams& p, Smem& S, int unit,
                                              int64_t T_top, uint32_t* cn, int32_t* lc_base) {
  const uint8_t* sm = p.seed_mask + (int64_t)unit * p.seed_stride;
  const int b = p.b;
  unsigned int run = 0;
  for (int64_t base = 0; base < T_top; base += kThreads) {
    const int64_t i = base + threadIdx.x;
    const uint32_t m = i < T_top ? (uint32_t)sm[i] & ((1u << G) - 1u) : 0u;
    unsigned int tot;
    const unsigned int rk = block_excl_scan(m ? 1u : 0u, &tot, S);
    if (m)
      for (int c = 0; c < b; ++c)
        cn[(int64_t)(run + rk) * b + c] = (m << 24) | ((uint32_t)i * (uint32_t)b + (uint32_t)c);
    run += tot;
  }
  if (threadIdx.x < G) {
    const int32_t k = p.seed_cnt[(int64_t)unit * G + threadIdx.x];
    S.my_hcnt[threadIdx.x] = (unsigned int)k * (unsigned int)b;
    if (lc_base) lc_base[(int64_t)threadIdx.x * p.L] = k;
  }
  if (p.stats && threadIdx.x == 0) atomicAdd(&p.stats[(int64_t)unit * p.L], (int)T_top);
  __syncthreads();
  return (int64_t)run * b;
}

// Final keep rule of one head for a candidate with order key `key`; *member
// reports a kModeTie candidate whose keep depends on its rank among the ties.
__device__ __forceinline__ bool keep_rule(int mode, unsigned kthr, uint32_t key, bool* member) {
  *member = false;
  if (mode == kModeAll) return true;
  if (mode == kModeThr) return key >= kthr;
  if (key > kthr) return true;
  *member = key == kthr;
  return false;
}

template <typename T, int D, int G>
__global__ void __launch_bounds__(kThreads, 2) traverse_kernel(const __grid_constant__ TravParams p) {
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
  float* zown = p.zbuf + ((int64_t)unit * C + rank) * seg * G;  // [seg][G]
  uint8_t* qown = p.qbuf + ((int64_t)unit * C + rank) * seg * G;  // [seg][G]
  uint8_t* mk_u = p.mkbuf + (int64_t)unit * C * seg * G;           // [C][seg][G]
  const uint8_t* mkown = mk_u + (int64_t)rank * seg * G;
  auto cptr = [&](int buf) { return cand_u + ((int64_t)buf * C + rank) * seg; };
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
    return;  // uniform across the cluster and before any DSMEM access
  }

  // Small frontiers are traversed by rank 0 alone (Ce = 1, CTA barriers
  // only); when a frontier outgrows kSingleMax rank 0 hands it over and the
  // whole cluster (Ce = C) takes equal slices of it. Every rank passes the
  // hand-over barrier exactly once.
  const bool single = C > 1 && T_top <= kSingleMax;
  int Ce = single ? 1 : C;
  int level = p.L;
  int cur = 0;
  // my segment at the top level: a contiguous range of the complete top nodes
  int64_t top_lo = single ? 0 : T_top * rank / C;
  int64_t my_n = single ? T_top : T_top * (rank + 1) / C - top_lo;
  bool joined = !single;  // passed the hand-over barrier
  // certified top level: its selection is given, rank 0 starts one level lower
  // (uniform across the cluster: it depends on the unit only)
  const bool seeded = p.seed_ok && p.L >= 2 && (C == 1 || single) && p.seed_ok[unit] != 0;
  if (seeded && rank == 0) {
    my_n = seed_frontier<G>(p, S, unit, T_top, cptr(0), lc_base);
    level = p.L - 1;
  }
  if (single && rank != 0) {
    cluster.sync();  // hand-over: rank 0's frontier (or its finish) is published
    joined = true;
    my_n = join_frontier(S, cluster, C, rank, cand_u, seg, &level, &cur);
    if (level > 0) Ce = C;
    else if (!p.list_mode && tid == 0)
      p.n_kept[(int64_t)unit * C + rank] = 0;  // rank 0 produced every kept node
  }
  for (; level >= 1; --level) {
    if (Ce == 1 && single && level < p.L && my_n > kSingleMax) {  // rank 0 hands over
      if (tid == 0) {
        S.sw_level = level;
        S.sw_cur = cur;
        S.sw_n = (unsigned int)my_n;
      }
      cluster.sync();   // hand-over
      joined = true;
      my_n = my_n / C;  // rank 0's slice is the prefix of its own segment
      Ce = C;
    }
    const bool top = level == p.L;
    const T* lvl = static_cast<const T*>(p.tree) + p.level_off[level - 1] +
                   (int64_t)tree_unit * p.level_rows[level - 1] * D;
    uint32_t* cc = cptr(cur);
    // ------------------------------------------------------------------
    // 1. score my segment
    // ------------------------------------------------------------------
    {
      float lmax[G], lmin[G];
#pragma unroll
      for (int h = 0; h < G; ++h) {
        lmax[h] = -INFINITY;
        lmin[h] = INFINITY;
      }
      score_segment<T, D, G>(p, S, lvl, cc, zown, my_n, p.lnsize[level - 1], lmax, lmin, top,
                             top_lo);
      if (top)  // materialise the top candidates (all heads)
        for (int64_t i = tid; i < my_n; i += kThreads)
          cc[i] = (((1u << G) - 1u) << 24) | (uint32_t)(top_lo + i);
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
      Xch& X = S.xch[level & 1];
      if (tid < G) {
        float mx = -INFINITY, mn = INFINITY;
        for (int w = 0; w < kWarps; ++w) {
          mx = fmaxf(mx, S.red_f[w][tid][0]);
          mn = fminf(mn, S.red_f[w][tid][1]);
        }
        X.zmax[tid] = mx;
        X.zmin[tid] = mn;
        X.hcount[tid] = top ? (unsigned int)my_n : S.my_hcnt[tid];
      }
      if (tid == 0) X.count = (unsigned int)my_n;
    }
    if (Ce > 1) cluster.sync();  // S1: every segment scored
    else __syncthreads();
    if (p.stats && tid == 0) atomicAdd(&p.stats[(int64_t)unit * p.L + (p.L - level)], (int)my_n);

    // ------------------------------------------------------------------
    // 2. distributed cut
    // ------------------------------------------------------------------
    for (int e = tid; e < Ce * (3 * G + 1); e += kThreads) {  // one parallel DSMEM gather
      const int r = e / (3 * G + 1), k = e % (3 * G + 1);
      const Xch* rx = &cluster.map_shared_rank(&S, r)->xch[level & 1];
      if (k == 0) S.seg_n[r] = rx->count;
      else if (k <= G) S.g_zmax[r][k - 1] = rx->zmax[k - 1];
      else if (k <= 2 * G) S.g_zmin[r][k - 1 - G] = rx->zmin[k - 1 - G];
      else S.g_hcnt[r][k - 1 - 2 * G] = rx->hcount[k - 1 - 2 * G];
    }
    __syncthreads();
    if (tid < G) {
      float mx = -INFINITY, mn = INFINITY;
      unsigned int n = 0;
      for (int r = 0; r < Ce; ++r) {
        mx = fmaxf(mx, S.g_zmax[r][tid]);
        mn = fminf(mn, S.g_zmin[r][tid]);
        n += S.g_hcnt[r][tid];
      }
      S.zmax[tid] = mx;
      S.nh[tid] = n;
      HeadState s{};
      s.count = n;
      if (p.keep_all || n == 0u) {
        s.mode = kModeAll;
      } else {
        // the first pass spreads the head's scores over 256 linear buckets;
        // scores more than 32 below the maximum carry zero mass and share
        // bucket 0
        s.mode = kModeQuant;
        const float lo = fmaxf(mn, __fsub_rn(mx, 32.0f));
        s.zlo = lo;
        s.zscale = mx > lo ? __fdiv_rn(256.0f, __fsub_rn(mx, lo)) : 0.0f;
      }
      s.qbeta = 0xffffffffu;
      S.st[tid] = s;
      S.mlist_n[tid] = 0u;  // my gather lists (slots of the heads I own)
    }
    __syncthreads();
    // entries per shipped-member list (rank 0 alone: one list per head, each
    // finished by one warp)
    // one CTA per unit keeps kGather-entry lists in global memory; rank 0
    // alone in a cluster keeps kWarpGather-entry lists in shared memory
    const bool glob = C == 1 && p.glist_z != nullptr;
    const int cap = (Ce > 1 || glob) ? kGather : kWarpGather;
    auto list_zh = [&](Smem* O, int h) -> float* {
      return glob ? p.glist_z + ((int64_t)unit * G + h) * kGather : list_z(*O) + (h / Ce) * cap;
    };
    auto list_ph = [&](Smem* O, int h) -> uint32_t* {
      return glob ? p.glist_pos + ((int64_t)unit * G + h) * kGather
                  : list_pos(*O, list_slots(G, Ce), cap) + (h / Ce) * cap;
    };
    for (int pass = 0; pass < 40; ++pass) {  // every pass strictly narrows each group
      // heads whose group is still open: histogram pass, or (small group)
      // shipped to the owner who finishes the cut alone
      unsigned hist_heads = 0, gather_heads = 0;
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const int m = S.st[h].mode;
        if (m == kModeQuant) hist_heads |= 1u << h;
        else if (m == kModeRadix)
          (S.st[h].bcnt <= (unsigned)cap ? gather_heads : hist_heads) |= 1u << h;
      }
      const unsigned open_heads = hist_heads | gather_heads;
      if (!open_heads) break;  // uniform: every CTA holds the same states
      const bool first = pass == 0;  // every open head is in kModeQuant
      if (tid == 0) S.lm_n = 0u;
      if (hist_heads)
        for (int e = tid; e < G * kBuckets; e += kThreads) {
          (&S.hist_lo[0][0])[e] = 0u;
          (&S.hist_hi[0][0])[e] = 0u;
          (&S.hist_c[0][0])[e] = 0u;
        }
      __syncthreads();
      // consecutive candidates per thread, loaded up front (fewer with 8 heads
      // to stay within the register budget)
      if (first) {
        constexpr int kHU = G >= 8 ? 1 : 4;
        // every open head is in kModeQuant: bucket every score, histogram it,
        // and keep the bucket bytes for the later passes and the expand
        // software-pipelined: the next candidates' scores are in flight while
        // the current ones are bucketed
        uint32_t hm[kHU];
        float z[kHU][G];
        auto fetch = [&](int64_t i0, uint32_t* hmo, float (*zo)[G]) {
#pragma unroll
          for (int u = 0; u < kHU; ++u) {
            const bool in = i0 + u < my_n;
            hmo[u] = in ? (cc[i0 + u] >> 24) & open_heads : 0u;
            if (in) load_scores<G>(zown, i0 + u, zo[u]);
          }
        };
        fetch(kHU * tid, hm, z);
        for (int64_t base = 0; base < my_n; base += kHU * kThreads) {
          const int64_t i0 = base + kHU * tid;
          uint32_t hm_c[kHU];
          float z_c[kHU][G];
#pragma unroll
          for (int u = 0; u < kHU; ++u) {
            hm_c[u] = hm[u];
#pragma unroll
            for (int h = 0; h < G; ++h) z_c[u][h] = z[u][h];
          }
          if (base + kHU * kThreads < my_n) fetch(i0 + kHU * kThreads, hm, z);
          uint64_t qrow[kHU];
#pragma unroll
          for (int u = 0; u < kHU; ++u) qrow[u] = 0;
#pragma unroll
          for (int u = 0; u < kHU; ++u) {
            uint32_t d[G], c[G];
            unsigned long long m[G];
#pragma unroll
            for (int h = 0; h < G; ++h) {
              const bool v = (hm_c[u] >> h) & 1u;
              const uint32_t b = quant_bucket(z_c[u][h], S.st[h].zlo, S.st[h].zscale);
              qrow[u] |= (uint64_t)b << (8 * h);
              d[h] = v ? b : (uint32_t)lane;  // spread the zero adds of absent heads
              // computed for every head (independent chains), kept for present ones
              m[h] = mass_fixed(z_c[u][h], S.zmax[h]) & (0ull - (unsigned long long)v);
              c[h] = v ? 1u : 0u;
            }
            hist_add_heads<G>(S, d, m, c);
          }
#pragma unroll
          for (int u = 0; u < kHU; ++u)
            if (i0 + u < my_n) store_qrow<G>(qown, i0 + u, qrow[u]);
        }
      } else {
        // later passes touch only the members of the open groups: candidates
        // whose first-pass bucket is the group's, and whose key lies in the
        // group's interval
        constexpr int kHU = G >= 8 ? 2 : 4;
        uint64_t qb_pack = 0;
#pragma unroll
        for (int h = 0; h < G; ++h) qb_pack |= (uint64_t)(S.st[h].qbeta & 0xffu) << (8 * h);
        // the next candidates' masks and bucket bytes are in flight while the
        // current members' scores are loaded and shipped
        uint32_t mem[kHU];
        auto fetch = [&](int64_t i0, uint32_t* memo) {
#pragma unroll
          for (int u = 0; u < kHU; ++u) {
            const bool in = i0 + u < my_n;
            const uint32_t hm = in ? (cc[i0 + u] >> 24) & open_heads : 0u;
            memo[u] = hm ? hm & bytes_eq(load_qrow<G>(qown, i0 + u), qb_pack) : 0u;
          }
        };
        fetch(kHU * tid, mem);
        for (int64_t base = 0; base < my_n; base += kHU * kThreads) {
          const int64_t i0 = base + kHU * tid;
          uint32_t mem_c[kHU];
          float z_c[kHU][G];
#pragma unroll
          for (int u = 0; u < kHU; ++u) mem_c[u] = mem[u];
          if (base + kHU * kThreads < my_n) fetch(i0 + kHU * kThreads, mem);
#pragma unroll
          for (int u = 0; u < kHU; ++u)  // scores of this thread's group members only
            if (mem_c[u]) load_scores<G>(zown, i0 + u, z_c[u]);
          // members in the group's key interval, per candidate (bit h = head h)
          uint32_t vm[kHU];
#pragma unroll
          for (int u = 0; u < kHU; ++u) {
            vm[u] = 0u;
#pragma unroll
            for (int h = 0; h < G; ++h) {
              if (!((mem_c[u] >> h) & 1u)) continue;
              const uint32_t key = order_key(z_c[u][h]);
              if (key >= S.st[h].kgmin && key <= S.st[h].kgmax) vm[u] |= 1u << h;
            }
          }
#pragma unroll
          for (int h = 0; h < G; ++h) {  // heads narrowed by another histogram pass
            if (!((hist_heads >> h) & 1u)) continue;
            int sh, w;
            radix_digit(S.st[h].kgmin, S.st[h].kgmax, &sh, &w);
#pragma unroll
            for (int u = 0; u < kHU; ++u)
              if ((vm[u] >> h) & 1u)
                hist_add(S, h, (order_key(z_c[u][h]) >> sh) & ((1u << w) - 1u),
                         mass_fixed(z_c[u][h], S.zmax[h]));
          }
          if (gather_heads) {
            // stage the members locally: entry = z (low word) and
            // (head << 28) | (rank << 24) | index (high word); a full stage
            // ships the rest directly
#pragma unroll
            for (int u = 0; u < kHU; ++u) {
              const uint32_t gv = vm[u] & gather_heads;
              const unsigned nb = __popc(gv);
              unsigned excl = nb;
#pragma unroll
              for (int off = 1; off < 32; off <<= 1) {
                const unsigned y = __shfl_up_sync(0xffffffffu, excl, off);
                if (lane >= off) excl += y;
              }
              const unsigned wtot = __shfl_sync(0xffffffffu, excl, 31);
              excl -= nb;
              unsigned wbase = 0;
              if (lane == 0 && wtot) wbase = atomicAdd(&S.lm_n, wtot);
              wbase = __shfl_sync(0xffffffffu, wbase, 0);
              uint32_t rest = gv;
              unsigned k = wbase + excl;
              while (rest) {
                const int h = __ffs(rest) - 1;
                rest &= rest - 1;
                const uint32_t tag = ((uint32_t)h << 28) | ((uint32_t)rank << 24) | (uint32_t)(i0 + u);
                if (k < (unsigned)kGather) {
                  S.mrank_m[k] = ((unsigned long long)tag << 32) | __float_as_uint(z_c[u][h]);
                } else {  // stage full: reserve one owner slot directly
                  Smem* O = cluster.map_shared_rank(&S, h % Ce);
                  const unsigned ko = atomicAdd(&O->mlist_n[h / Ce], 1u);
                  if (ko < (unsigned)cap) {
                    list_zh(O, h)[ko] = z_c[u][h];
                    list_ph(O, h)[ko] = tag & 0x0fffffffu;
                  }
                }
                ++k;
              }
            }
          }
        }
        if (gather_heads) {
          // ship the staged members: warp h reserves the owner's slots for head
          // h with one DSMEM atomic and copies its members over
          __syncthreads();
          const unsigned n_st = S.lm_n < (unsigned)kGather ? S.lm_n : (unsigned)kGather;
          for (int h = warp; h < G; h += kWarps) {
            if (!((gather_heads >> h) & 1u)) continue;
            unsigned cnt = 0;
            for (unsigned e = lane; e < n_st; e += 32) cnt += (unsigned)(S.mrank_m[e] >> 60) == (unsigned)h;
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, off);
            if (!cnt) continue;
            Smem* O = cluster.map_shared_rank(&S, h % Ce);
            unsigned base = 0;
            if (lane == 0) base = atomicAdd(&O->mlist_n[h / Ce], cnt);
            base = __shfl_sync(0xffffffffu, base, 0);
            float* oz = list_zh(O, h);
            uint32_t* op = list_ph(O, h);
            for (unsigned e0 = 0; e0 < n_st; e0 += 32) {
              const unsigned e = e0 + lane;
              const unsigned long long v = e < n_st ? S.mrank_m[e] : 0ull;
              const bool mine = e < n_st && (unsigned)(v >> 60) == (unsigned)h;
              const unsigned mb = __ballot_sync(0xffffffffu, mine);
              if (mine) {
                const unsigned k = base + __popc(mb & ((1u << lane) - 1u));
                if (k < (unsigned)cap) {
                  oz[k] = __uint_as_float((uint32_t)v);
                  op[k] = (uint32_t)(v >> 32) & 0x0fffffffu;
                }
              }
              base += __popc(mb);
            }
          }
        }
      }
      if (Ce > 1) cluster.sync();  // every rank's histograms and shipped members complete
      else __syncthreads();
      if (Ce > 1) {
        for (int h = rank; h < G; h += Ce) {
          if ((hist_heads >> h) & 1u) owner_pass<G>(p, S, cluster, Ce, h);
          else if ((gather_heads >> h) & 1u)
            owner_finish<G>(p, S, h, list_zh(&S, h), list_ph(&S, h), S.mlist_n[h / Ce], cap,
                            mk_u, seg);
        }
      } else if (glob) {
        // the whole CTA sorts each gathered head's group in turn; one warp
        // per head narrows the others
        for (int h = 0; h < G; ++h)
          if ((gather_heads >> h) & 1u)
            owner_finish<G>(p, S, h, list_zh(&S, h), list_ph(&S, h), S.mlist_n[h], cap, mk_u, seg);
        if (warp < G && ((hist_heads >> warp) & 1u)) owner_pass_warp<G>(p, S, warp);
      } else if (warp < G) {  // one warp per head
        if ((hist_heads >> warp) & 1u) owner_pass_warp<G>(p, S, warp);
        else if ((gather_heads >> warp) & 1u)
          owner_finish_warp<G>(p, S, warp, list_slots(G, Ce), cap, mk_u, seg);
      }
      if (Ce > 1) cluster.sync();  // every owner published
      else __syncthreads();
      {  // copy the new states of the open heads from their owners
        constexpr int kWords = (int)(sizeof(HeadState) / 4);
        for (int e = tid; e < G * kWords; e += kThreads) {
          const int h = e / kWords, k = e % kWords;
          if (!((open_heads >> h) & 1u)) continue;
          const Smem* R = cluster.map_shared_rank(&S, h % Ce);
          reinterpret_cast<unsigned int*>(&S.st[h])[k] =
              reinterpret_cast<const unsigned int*>(&R->pub[h])[k];
        }
      }
      __syncthreads();
    }
    if (tid < G) {
      const int m = S.st[tid].mode;
      if (m == kModeRadix || m == kModeQuant) {  // unreachable: passes always finish
        if (rank == 0) raise_status(p.status, ZHA_ERR_INTERNAL);
        S.st[tid].mode = kModeAll;
        S.st[tid].count = S.nh[tid];
      }
    }
    if (lc_base && rank == 0 && tid < G)
      lc_base[(int64_t)tid * p.L + (p.L - level)] = (int32_t)S.st[tid].count;

    // ------------------------------------------------------------------
    // 3. expand my segment with the final rules
    // ------------------------------------------------------------------
    if (tid < G) {
      S.kc[tid] = 0u;
      S.tie_run[tid] = 0u;
    }
    __syncthreads();
    // the rules as byte-parallel masks (bit h = head h)
    // A gathered group narrowed by radix passes (gathn) is a key sub-interval
    // of its first-pass bucket: bucket members above it are kept, below it
    // dropped, and only members inside it carry the owner's mark.
    uint32_t allm = 0, gathz = 0, gathn = 0, thrz = 0, tiez = 0, needz = 0;
    uint64_t qb_pack = 0;
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const HeadState& st = S.st[h];
      const uint32_t bit = 1u << h;
      if (st.mode == kModeAll) allm |= bit;
      else if (st.mode == kModeGathered) (st.zfree ? gathz : gathn) |= bit;
      else if (st.mode == kModeThr) (st.zfree ? thrz : needz) |= bit;
      else if (st.mode == kModeTie) (st.zfree ? tiez : needz) |= bit;
      qb_pack |= (uint64_t)(st.qbeta & 0xffu) << (8 * h);
    }
    bool any_tie = false;
#pragma unroll
    for (int h = 0; h < G; ++h) any_tie |= S.st[h].mode == kModeTie;
    {
      uint32_t* cn = cptr(cur ^ 1);  // next level's candidates, or (list mode) keep masks
      unsigned int run = 0;
      constexpr int kEU = 4;  // consecutive candidates per thread
      for (int64_t base = 0; base < my_n; base += kEU * kThreads) {
        const int64_t i0 = base + kEU * tid;
        uint32_t km[kEU], cv[kEU], ties[kEU], eqm[kEU];
        uint64_t qrow[kEU], mrow[kEU];
#pragma unroll
        for (int u = 0; u < kEU; ++u) {
          km[u] = ties[u] = 0u;
          const bool in = i0 + u < my_n;
          cv[u] = in ? cc[i0 + u] : 0u;
          qrow[u] = in ? load_qrow<G>(qown, i0 + u) : 0ull;
          mrow[u] = in ? load_qrow<G>(mkown, i0 + u) : 0ull;
        }
        // the fate of a candidate follows from its first-pass bucket: above the
        // group's bucket it is kept, below it dropped; members of the bucket
        // carry the owner's mark (kModeGathered), are all kept (kModeThr set on
        // the first pass) or are exact ties ranked in node order (kModeTie)
#pragma unroll
        for (int u = 0; u < kEU; ++u) {
          const uint32_t hm = cv[u] >> 24;
          const uint32_t gt = bytes_gt(qrow[u], qb_pack), eq = bytes_eq(qrow[u], qb_pack);
          km[u] = hm & (allm | (gt & ~allm) | (eq & gathz & bytes_nz(mrow[u])) | (eq & thrz));
          ties[u] = hm & eq & tiez;
          eqm[u] = hm & eq & (needz | gathn);
        }
        if (needz | gathn) {  // rules narrowed below the first-pass bucket: compare scores
#pragma unroll
          for (int u = 0; u < kEU; ++u) {
            if (!eqm[u]) continue;  // (also every candidate past the segment's end)
            float z[G];
            load_scores<G>(zown, i0 + u, z);
#pragma unroll
            for (int h = 0; h < G; ++h) {
              const HeadState& st = S.st[h];
              if (!((eqm[u] >> h) & 1u)) continue;
              const uint32_t key = order_key(z[h]);
              if ((gathn >> h) & 1u) {
                if (key > st.kgmax || (key >= st.kgmin && ((mrow[u] >> (8 * h)) & 0xffu)))
                  km[u] |= 1u << h;
                continue;
              }
              bool member;
              if (keep_rule(st.mode, st.kthr, key, &member)) km[u] |= 1u << h;
              if (member) ties[u] |= 1u << h;
            }
          }
        }
        if (any_tie) {  // exact ties: the segment keeps its first quota members in node order
#pragma unroll
          for (int h = 0; h < G; ++h) {
            if (S.st[h].mode != kModeTie) continue;
            unsigned f = 0;
#pragma unroll
            for (int u = 0; u < kEU; ++u) f += (ties[u] >> h) & 1u;
            unsigned int tot;
            const unsigned int run_h = S.tie_run[h];
            unsigned int rk = run_h + block_excl_scan(f, &tot, S);  // syncs: run_h read by all
            const unsigned int quota = S.st[h].quota[rank];
#pragma unroll
            for (int u = 0; u < kEU; ++u)
              if ((ties[u] >> h) & 1u) {
                if (rk < quota) km[u] |= 1u << h;
                ++rk;
              }
            if (tid == 0) S.tie_run[h] = run_h + tot;
          }
        }
        unsigned int nk = 0;
#pragma unroll
        for (int u = 0; u < kEU; ++u) nk += km[u] ? 1u : 0u;
#pragma unroll
        for (int h = 0; h < G; ++h) {
          unsigned int f = 0;
#pragma unroll
          for (int u = 0; u < kEU; ++u) f += (km[u] >> h) & 1u;
#pragma unroll
          for (int off = 16; off > 0; off >>= 1) f += __shfl_xor_sync(0xffffffffu, f, off);
          if (lane == 0 && f) atomicAdd(&S.kc[h], f);
        }
        unsigned int tot;
        int64_t pos = (int64_t)run + block_excl_scan(nk, &tot, S);
#pragma unroll
        for (int u = 0; u < kEU; ++u) {
          if (km[u]) {
            const uint32_t node = cv[u] & kNodeMask;
            if (level > 1) {
              for (int c = 0; c < b; ++c)
                cn[pos * b + c] = (km[u] << 24) | (node * (uint32_t)b + (uint32_t)c);
            } else if (!p.list_mode) {
              p.kept[((int64_t)unit * C + rank) * seg + pos] = (km[u] << 24) | node;
            }
            ++pos;
          }
          if (level == 1 && p.list_mode && i0 + u < my_n) cn[i0 + u] = km[u];  // for the emission
        }
        run += tot;
      }
      if (level == 1 && !p.list_mode && tid == 0)
        p.n_kept[(int64_t)unit * C + rank] = (int32_t)run;
      // per-head kept counts of my segment (S.kc): the next level's head
      // frontiers hold b children of each
      __syncthreads();
      if (tid < G) S.my_hcnt[tid] = S.kc[tid] * (unsigned int)b;
      my_n = (int64_t)run * b;
      if (level > 1 && my_n > seg) {  // cannot happen: a segment holds every level-1 node
        if (tid == 0) raise_status(p.status, ZHA_ERR_WORKSPACE);
        my_n = seg;
      }
    }
    if (level > 1) cur ^= 1;  // the expanded segment is the next frontier

    if (level == 1 && p.list_mode) {
      // per-head ascending token lists: {0} (unless node 0 is kept) + tokens of
      // the kept level-1 nodes in node order + causal tail
      const uint32_t* km_seg = cptr(cur ^ 1);
      const int64_t n1 = S.seg_n[rank];  // candidates of my segment at level 1
      if (tid == 0)
        S.node0 = (n1 > 0 && (cc[0] & kNodeMask) == 0u) ? km_seg[0] : 0u;
      if (Ce > 1) cluster.sync();  // every rank's kept counts published
      else __syncthreads();
      unsigned int base[G], total[G];
      uint32_t node0 = 0;
#pragma unroll
      for (int h = 0; h < G; ++h) base[h] = total[h] = 0u;
      for (int r = 0; r < Ce; ++r) {
        const Smem* R = cluster.map_shared_rank(&S, r);
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const unsigned int v = R->kc[h];
          if (r < rank) base[h] += v;
          total[h] += v;
        }
        node0 |= R->node0;
      }
      const int64_t tail_start = p.span[p.L] * T_top;
      const int64_t tail_len = n_vis - tail_start;
#pragma unroll 1
      for (int h = 0; h < G; ++h) {
        const int64_t qh = (int64_t)qi * p.Hq + (int64_t)kvh * G + h;
        int32_t* out = p.idx + qh * p.idx_cap;
        const int64_t off0 = ((node0 >> h) & 1u) ? 0 : 1;
        unsigned int prun = base[h];
        for (int64_t b0 = 0; b0 < n1; b0 += kThreads) {
          const int64_t i = b0 + tid;
          const unsigned f = i < n1 ? (km_seg[i] >> h) & 1u : 0u;
          unsigned int tot;
          const unsigned int rk = block_excl_scan(f, &tot, S);
          if (f) {
            const int64_t pos = off0 + (int64_t)b * (prun + rk);
            const int64_t node = cc[i] & kNodeMask;
            for (int c = 0; c < b; ++c)
              if (pos + c < p.idx_cap) out[pos + c] = (int32_t)(node * b + c);
          }
          prun += tot;
        }
        if (rank == 0 && tid == 0 && off0 == 1 && p.idx_cap > 0) out[0] = 0;
        if (rank == Ce - 1) {
          const int64_t tail_pos = off0 + (int64_t)b * total[h];
          for (int64_t j = tid; j < tail_len; j += kThreads)
            if (tail_pos + j < p.idx_cap) out[tail_pos + j] = (int32_t)(tail_start + j);
          if (tid == 0) {
            const int64_t n = tail_pos + tail_len;
            p.n_idx[qh] = (int32_t)n;
            if (n > p.idx_cap) raise_status(p.status, ZHA_ERR_CAPACITY);
          }
        }
      }
    }
    __syncthreads();
  }
  if (!joined) {  // rank 0 finished alone: release the waiting ranks
    if (tid == 0) S.sw_level = 0;
    cluster.sync();  // hand-over
  }
  // no CTA may leave while another can still read its shared memory
  cluster.sync();
}

// Dynamic shared memory of a CTA: the struct plus its shipped-member lists.
// A cluster's owners gather up to kGather members per owned head; a CTA
// working alone (C = 1, or rank 0 on the small top levels) owns every head
// with up to kWarpGather members each. Sizing C = 1 for the latter keeps two
// CTAs per SM.
size_t smem_bytes(int G, int C) {
  const size_t entries = C > 1 ? (size_t)list_slots(G, C) * kGather : 0;
  const size_t alone = (size_t)list_slots(G, 1) * kWarpGather;
  return sizeof(Smem) + (entries > alone ? entries : alone) * (sizeof(float) + sizeof(uint32_t));
}

template <typename T, int D, int G>
cudaError_t launch_t(const TravParams& p, int64_t units, int C, cudaStream_t stream) {
  const size_t smem = smem_bytes(G, C);
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
                           (int)smem_bytes(G, C)) != cudaSuccess)
    return (cudaGetLastError(), 0);
  if (C > 8 && cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) !=
                   cudaSuccess)
    return (cudaGetLastError(), 0);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)C, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem_bytes(G, C);
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

// Cached per (dtype, d, G, C) for the process; every device is assumed to be
// the same part. Calls from several host threads may query concurrently and
// store the same value, so the cache entries are relaxed atomics.
int max_clusters(const Geometry& g, int C) {
  static std::atomic<int> cache[2][2][4][kMaxCluster + 1];  // 0 = not queried
  const int i0 = g.dtype == ZHA_BF16, i1 = g.d == 128;
  const int i2 = g.G == 1 ? 0 : g.G == 2 ? 1 : g.G == 4 ? 2 : 3;
  std::atomic<int>& v = cache[i0][i1][i2][C];
  int n = v.load(std::memory_order_relaxed);
  if (n == 0) {
    if (g.dtype == ZHA_BF16)
      n = g.d == 128 ? max_clusters_g<__nv_bfloat16, 128>(g.G, C)
                     : max_clusters_g<__nv_bfloat16, 64>(g.G, C);
    else
      n = g.d == 128 ? max_clusters_g<float, 128>(g.G, C) : max_clusters_g<float, 64>(g.G, C);
    if (n <= 0) n = -1;
    v.store(n, std::memory_order_relaxed);
  }
  return n;
}

}  // namespace

// The largest cluster (<= 16 CTAs) that keeps every unit resident in one wave
// with at most two CTAs per SM.
int traverse_cluster_size(const Geometry& g, int64_t units, int num_sms) {
  for (int C = kMaxCluster; C >= 2; --C) {
    if (units * C > 2 * (int64_t)num_sms) continue;
    const int n = max_clusters(g, C);
    if (n > 0 && n >= units) return C;
  }
  return 1;
}

size_t traverse_ws_bytes(const Geometry& g, int64_t units, int num_sms) {
  const int C = traverse_cluster_size(g, units, num_sms);
  const size_t seg = (size_t)seg_capacity(g);
  // candidates (two buffers), scores, first-pass buckets and owner marks,
  // plus the global member lists of one-CTA units
  const size_t per = (size_t)C * seg * (2 * sizeof(uint32_t) + (size_t)g.G * (sizeof(float) + 2));
  const size_t lists = C == 1 ? (size_t)g.G * kGather * (sizeof(float) + sizeof(uint32_t)) : 0;
  return (per + lists) * (size_t)units + 512;
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
                            cudaStream_t stream, const TopSeeds* seeds) {
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
  w += sizeof(float) * (size_t)units * C * p.seg * g.G;
  p.qbuf = reinterpret_cast<uint8_t*>(w);
  w += (size_t)units * C * p.seg * g.G;
  p.mkbuf = reinterpret_cast<uint8_t*>(w);
  w += (size_t)units * C * p.seg * g.G;
  if (C == 1) {
    w = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(w) + 255) & ~(uintptr_t)255);
    p.glist_z = reinterpret_cast<float*>(w);
    w += sizeof(float) * (size_t)units * g.G * kGather;
    p.glist_pos = reinterpret_cast<uint32_t*>(w);
  }
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
  if (seeds && seeds->ok && g.L >= 2) {
    p.seed_ok = seeds->ok;
    p.seed_mask = seeds->mask;
    p.seed_cnt = seeds->cnt;
    p.seed_stride = seeds->stride;
  }
  if (g.dtype == ZHA_BF16) {
    if (g.d == 128) return launch_g<__nv_bfloat16, 128>(g.G, p, units, C, stream);
    return launch_g<__nv_bfloat16, 64>(g.G, p, units, C, stream);
  }
  if (g.d == 128) return launch_g<float, 128>(g.G, p, units, C, stream);
  return launch_g<float, 64>(g.G, p, units, C, stream);
}

}  // namespace zha
