// Top-down top-p traversal of the summary tree, all query heads of a KV head
// together.
//
// lefilia.fr page "Zyphra presente Zyphra Hierarchical Attention (ZHA) ...",
// paragraph 1: a query scores the top nodes, keeps the smallest set covering a
// fraction p of the estimated attention mass, expands only the kept branches
// down to the raw KV entries, and always keeps the first token.
//
// Unit of work: one query token and one KV head, i.e. the G = Hq/Hkv query
// heads that read the same tree. The unit's candidate list at each level is
// the UNION of the heads' candidate lists; each entry carries an 8-bit mask of
// the heads whose frontier contains it, so every summary row is read from HBM
// once per unit and scored against all G queries (8 dot products per row).
// A thread-block cluster of C CTAs cooperates on a unit: candidates are split
// into C contiguous slices, and the per-head cut is agreed through distributed
// shared memory.
//
// Per level and per head (canonical fp32, identical to the CPU oracle):
//   z     = (dot(q, s) * inv_sqrt_d) + fp32(l ln b)
//   M     = trunc(exp(z - zmax) * 2^40)                (uint64, exact sums)
//   need  = ceil(T * p_q / 2^32),  T = sum M
//   keep the smallest prefix of (z desc, node asc) whose mass reaches need.
// The cut is found by a radix select on the order-preserving bits of z with
// per-bucket mass sums (8-bit digits starting at the highest bit where the
// unit's z values differ), stopping as soon as the crossing bucket holds one
// candidate or one exact value; equal scores are kept in ascending node order.
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
constexpr int kBuckets = 256;
constexpr uint32_t kNodeMask = 0x00ffffffu;

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
  uint32_t* cand;      // [units][2][max_cand]
  float* zbuf;         // [units][G][max_cand]
  int64_t max_cand;
  uint32_t* kept;      // [units][max_cand]   (decode mode)
  int32_t* n_kept;     // [units]
  int32_t* idx;        // [nq][Hq][idx_cap]    (list mode)
  int64_t idx_cap;
  int32_t* n_idx;
  int32_t* level_counts;
  int32_t* status;
};

// Per-CTA state that other CTAs of the cluster read through DSMEM.
struct Xch {
  unsigned long long hmass[kMaxGroup][kBuckets];
  unsigned int hcnt[kMaxGroup][kBuckets];
  unsigned long long T[kMaxGroup];
  float zmax[kMaxGroup];
  float zmin[kMaxGroup];
  // results published by the owner CTA of each head
  unsigned long long r_above[kMaxGroup];
  unsigned long long r_need[kMaxGroup];
  unsigned long long r_bmass[kMaxGroup];
  unsigned int r_prefix[kMaxGroup];
  unsigned int r_bcnt[kMaxGroup];
  int r_shift[kMaxGroup];
  int r_done[kMaxGroup];
  // emit phase
  unsigned int tie_local[kMaxGroup];
  unsigned int kept_cnt[kMaxGroup];
  unsigned int nk;
  unsigned int node0_mask;
};

constexpr int kMaxCluster = 16;

struct Scratch {
  unsigned long long warp_u64[kWarps];
  unsigned int warp_u32[kWarps];
  unsigned int bcast_u32[4];
  unsigned long long bcast_u64[4];
  float warp_f[kWarps][kMaxGroup][2];
  unsigned int kcnt[kMaxGroup];
  unsigned int tcnt[kMaxGroup];
  // local copies of cluster-wide values (gathered once through DSMEM)
  float g_zmax[kMaxCluster][kMaxGroup];
  float g_zmin[kMaxCluster][kMaxGroup];
  unsigned int g_u32[kMaxCluster][kMaxGroup + 1];
  unsigned long long l_above[kMaxGroup], l_need[kMaxGroup], l_bmass[kMaxGroup];
  unsigned int l_bcnt[kMaxGroup], l_prefix[kMaxGroup];
  int l_shift[kMaxGroup], l_done[kMaxGroup];
  unsigned int node0;
};

// Exclusive scan of v over the CTA in thread order; *total receives the sum.
__device__ __forceinline__ unsigned int block_excl_scan(unsigned int v, unsigned int* total,
                                                        Scratch& sc) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  unsigned int x = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const unsigned int y = __shfl_up_sync(0xffffffffu, x, off);
    if (lane >= off) x += y;
  }
  if (lane == 31) sc.warp_u32[warp] = x;
  __syncthreads();
  unsigned int wbase = 0, tot = 0;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) {
    const unsigned int s = sc.warp_u32[w];
    if (w < warp) wbase += s;
    tot += s;
  }
  __syncthreads();
  *total = tot;
  return wbase + x - v;
}

// Inclusive suffix sum (from the highest thread index down) of a u64 per thread.
__device__ __forceinline__ unsigned long long block_suffix_u64(unsigned long long v, Scratch& sc) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  unsigned long long x = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const unsigned long long y = __shfl_down_sync(0xffffffffu, x, off);
    if (lane + off < 32) x += y;
  }
  if (lane == 0) sc.warp_u64[warp] = x;
  __syncthreads();
  unsigned long long above = 0;
#pragma unroll
  for (int w = 0; w < kWarps; ++w)
    if (w > warp) above += sc.warp_u64[w];
  __syncthreads();
  return x + above;
}

__device__ __forceinline__ unsigned long long ceil_mul_shift32(unsigned long long T,
                                                               unsigned long long pq) {
  // ceil(T * pq / 2^32) with a 128-bit product
  const unsigned long long lo = T * pq;
  const unsigned long long hi = __umul64hi(T, pq);
  unsigned long long r = (hi << 32) | (lo >> 32);
  if (lo & 0xffffffffull) r += 1;
  return r;
}

template <typename T, int D, int G>
__global__ void __launch_bounds__(kThreads, 1) traverse_kernel(TravParams p) {
  constexpr int kRowBytes = D * (int)sizeof(T);
  constexpr int kNch = kRowBytes / 16;
  constexpr int kPer = Elem<T>::kPerChunk;
  constexpr int kTile = (kRowBytes <= 256) ? 256 : 128;
  static_assert(kNch >= 8, "swizzle needs at least 8 chunks per row");

  extern __shared__ __align__(128) unsigned char smem[];
  unsigned char* tiles = smem;                                       // 2 * kTile * kRowBytes
  float* qs = reinterpret_cast<float*>(tiles + 2 * kTile * kRowBytes);  // [D][8]
  Xch* xch = reinterpret_cast<Xch*>(qs + D * kMaxGroup);
  Scratch* scp = reinterpret_cast<Scratch*>(xch + 1);
  Scratch& sc = *scp;

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
  const uint32_t full_mask = (1u << G) - 1u;

  // queries of the G heads, widened to fp32, interleaved [i][h]
  {
    const T* qrow = static_cast<const T*>(p.q) + ((int64_t)qi * p.Hq + (int64_t)kvh * G) * D;
    for (int e = tid; e < D * kMaxGroup; e += kThreads) {
      const int i = e / kMaxGroup, h = e % kMaxGroup;
      qs[e] = (h < G) ? Elem<T>::to_f(qrow[(int64_t)h * D + i]) : 0.0f;
    }
  }
  __syncthreads();

  uint32_t* cbuf0 = p.cand + (int64_t)unit * 2 * p.max_cand;
  uint32_t* cbuf1 = cbuf0 + p.max_cand;
  float* zb = p.zbuf + (int64_t)unit * G * p.max_cand;

  int32_t* lc_base = p.level_counts ? p.level_counts + ((int64_t)qi * p.Hq + (int64_t)kvh * G) * p.L
                                    : nullptr;

  // ---- no complete top node: every visible token is attended (dense) ----
  if (T_top == 0) {
    if (p.list_mode) {
      for (int h = 0; h < G; ++h) {
        const int64_t qh = (int64_t)qi * p.Hq + (int64_t)kvh * G + h;
        int32_t* out = p.idx + qh * p.idx_cap;
        for (int64_t j = (int64_t)rank * kThreads + tid; j < n_vis; j += (int64_t)C * kThreads)
          if (j < p.idx_cap) out[j] = (int32_t)j;
        if (rank == 0 && tid == 0) {
          p.n_idx[qh] = (int32_t)n_vis;
          if (n_vis > p.idx_cap) raise_status(p.status, ZHA_ERR_CAPACITY);
        }
      }
    } else if (rank == 0 && tid == 0) {
      p.n_kept[unit] = 0;
    }
    if (lc_base && rank == 0)
      for (int e = tid; e < G * p.L; e += kThreads) lc_base[e] = 0;
    return;  // uniform across the cluster: no cluster barrier is pending
  }

  int64_t n_cand = T_top;
  int cur = 0;
  for (int level = p.L; level >= 1; --level) {
    uint32_t* cin = cur ? cbuf1 : cbuf0;
    uint32_t* cnext = cur ? cbuf0 : cbuf1;
    const bool top = (level == p.L);
    const int64_t lo = n_cand * rank / C;
    const int64_t hi = n_cand * (rank + 1) / C;
    const T* lvl = static_cast<const T*>(p.tree) + p.level_off[level - 1] +
                   (int64_t)tree_unit * p.level_rows[level - 1] * D;
    const float lns = p.lnsize[level - 1];

    if (n_cand > p.max_cand) {  // cannot happen with a correctly sized workspace
      raise_status(p.status, ZHA_ERR_WORKSPACE);
      n_cand = p.max_cand;
    }

    // ------------------------------------------------------------------
    // 1. score the slice: z[h][i] for every candidate and head
    // ------------------------------------------------------------------
    float lmax[G], lmin[G];
#pragma unroll
    for (int h = 0; h < G; ++h) {
      lmax[h] = -INFINITY;
      lmin[h] = INFINITY;
    }
    const int64_t n_tiles = (hi - lo + kTile - 1) / kTile;
    auto issue_tile = [&](int64_t tl, int buf) {
      unsigned char* dst = tiles + buf * kTile * kRowBytes;
      const int64_t rows = (hi - tl) < kTile ? (hi - tl) : kTile;
      for (int e = tid; e < kTile * kNch; e += kThreads) {
        const int r = e / kNch, c = e % kNch;
        if (r < rows) {
          const int64_t ci = tl + r;
          const uint32_t node = top ? (uint32_t)ci : (cin[ci] & kNodeMask);
          const unsigned char* src =
              reinterpret_cast<const unsigned char*>(lvl + (int64_t)node * D) + c * 16;
          cp_async16(dst + r * kRowBytes + swz(c, r) * 16, src);
        }
      }
      cp_async_commit();
    };
    if (n_tiles > 0) issue_tile(lo, 0);
    for (int64_t k = 0; k < n_tiles; ++k) {
      const int64_t tl = lo + k * kTile;
      if (k + 1 < n_tiles) {
        issue_tile(tl + kTile, (int)((k + 1) & 1));
        cp_async_wait<1>();
      } else {
        cp_async_wait<0>();
      }
      __syncthreads();
      const unsigned char* buf = tiles + (k & 1) * kTile * kRowBytes;
      const int64_t ci = tl + tid;
      if (tid < kTile && ci < hi) {
        const uint32_t pm = top ? full_mask : (cin[ci] >> 24);
        float acc[G];
        float2 acc2[(G + 1) / 2];
#pragma unroll
        for (int h = 0; h < G; ++h) acc[h] = 0.0f;
#pragma unroll
        for (int j = 0; j < (G + 1) / 2; ++j) acc2[j] = make_float2(0.0f, 0.0f);
        const unsigned char* row = buf + tid * kRowBytes;
#pragma unroll 2
        for (int ch = 0; ch < kNch; ++ch) {
          const uint4 raw = lds128(row + swz(ch, tid) * 16);
          float x[kPer];
          Elem<T>::unpack(raw, x);
#pragma unroll
          for (int e = 0; e < kPer; ++e) {
            const float* qi_ = qs + (ch * kPer + e) * kMaxGroup;
            if constexpr (G == 1) {
              acc[0] = __fmaf_rn(qi_[0], x[e], acc[0]);
            } else {
              const float2 xx = make_float2(x[e], x[e]);
#pragma unroll
              for (int j = 0; j < G / 4; ++j) {
                const float4 qv = *reinterpret_cast<const float4*>(qi_ + 4 * j);
                acc2[2 * j] = ffma2(make_float2(qv.x, qv.y), xx, acc2[2 * j]);
                acc2[2 * j + 1] = ffma2(make_float2(qv.z, qv.w), xx, acc2[2 * j + 1]);
              }
              if constexpr (G == 2) {
                const float2 qv = *reinterpret_cast<const float2*>(qi_);
                acc2[0] = ffma2(qv, xx, acc2[0]);
              }
            }
          }
        }
        if constexpr (G > 1) {
#pragma unroll
          for (int j = 0; j < G / 2; ++j) {
            acc[2 * j] = acc2[j].x;
            acc[2 * j + 1] = acc2[j].y;
          }
        }
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const float z = __fadd_rn(__fmul_rn(acc[h], p.inv_sqrt_d), lns);
          zb[(int64_t)h * p.max_cand + ci] = z;
          if ((pm >> h) & 1u) {
            lmax[h] = fmaxf(lmax[h], z);
            lmin[h] = fminf(lmin[h], z);
          }
        }
        if (top) cin[ci] = (full_mask << 24) | (uint32_t)ci;
      }
      __syncthreads();
    }
    // CTA reduce of max/min per head
#pragma unroll
    for (int h = 0; h < G; ++h) {
      float mx = lmax[h], mn = lmin[h];
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
        mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, off));
      }
      if (lane == 0) {
        sc.warp_f[warp][h][0] = mx;
        sc.warp_f[warp][h][1] = mn;
      }
    }
    __syncthreads();
    if (tid < G) {
      float mx = -INFINITY, mn = INFINITY;
      for (int w = 0; w < kWarps; ++w) {
        mx = fmaxf(mx, sc.warp_f[w][tid][0]);
        mn = fminf(mn, sc.warp_f[w][tid][1]);
      }
      xch->zmax[tid] = mx;
      xch->zmin[tid] = mn;
    }
    cluster.sync();  // S1: slices scored, candidate list materialised

    // per-head state (identical in every thread of every CTA of the cluster)
    if (tid < C * G) {  // gather every rank's extremes once, then read locally
      const Xch* rx = cluster.map_shared_rank(xch, tid / G);
      sc.g_zmax[tid / G][tid % G] = rx->zmax[tid % G];
      sc.g_zmin[tid / G][tid % G] = rx->zmin[tid % G];
    }
    __syncthreads();
    float zmax[G];
    uint32_t prefix[G];
    int shift[G];
    unsigned long long above[G], need[G], bmass[G];
    uint32_t bcnt[G];
    bool done[G];
    bool any_open = false;
#pragma unroll
    for (int h = 0; h < G; ++h) {
      float mx = -INFINITY, mn = INFINITY;
      for (int r = 0; r < C; ++r) {
        mx = fmaxf(mx, sc.g_zmax[r][h]);
        mn = fminf(mn, sc.g_zmin[r][h]);
      }
      zmax[h] = mx;
      const uint32_t kmax = order_key(mx), kmin = order_key(mn);
      const uint32_t diff = kmax ^ kmin;
      const int hb = diff ? 32 - __clz(diff) : 0;
      shift[h] = hb;
      prefix[h] = (uint32_t)((uint64_t)kmax >> hb);
      above[h] = 0;
      need[h] = 0;
      bmass[h] = 0;
      bcnt[h] = 0;
      done[h] = p.keep_all != 0;
      any_open |= !done[h];
    }

    // ------------------------------------------------------------------
    // 2. radix passes: per-bucket mass sums, owner CTA finds the crossing
    // ------------------------------------------------------------------
    bool first = true;
    // at most ceil(32 / 8) digit passes; the bound also guards the loop
    for (int pass = 0; any_open && pass < 5; ++pass) {
      for (int e = tid; e < kMaxGroup * kBuckets; e += kThreads) {
        (&xch->hmass[0][0])[e] = 0ull;
        (&xch->hcnt[0][0])[e] = 0u;
      }
      __syncthreads();
      unsigned long long tloc[G];
#pragma unroll
      for (int h = 0; h < G; ++h) tloc[h] = 0ull;
      for (int64_t base = lo; base < hi; base += kThreads) {
        const int64_t ci = base + tid;
        const bool in = ci < hi;
        const uint32_t pm = in ? (cin[ci] >> 24) : 0u;
#pragma unroll
        for (int h = 0; h < G; ++h) {
          if (done[h]) continue;  // uniform
          const int w = shift[h] < 8 ? shift[h] : 8;
          const int sh = shift[h] - w;
          bool valid = false;
          uint32_t digit = 0;
          unsigned long long m = 0ull;
          if (in && ((pm >> h) & 1u)) {
            const float z = zb[(int64_t)h * p.max_cand + ci];
            const uint32_t key = order_key(z);
            if ((uint32_t)((uint64_t)key >> shift[h]) == prefix[h]) {
              valid = true;
              digit = (uint32_t)((key >> sh) & ((1u << w) - 1u));
              m = mass_fixed(z, zmax[h]);
              tloc[h] += m;
            }
          }
          const unsigned vmask = __ballot_sync(0xffffffffu, valid);
          if (vmask == 0u) continue;
          const int leader = __ffs(vmask) - 1;
          const uint32_t d0 = __shfl_sync(0xffffffffu, digit, leader);
          if (__all_sync(0xffffffffu, !valid || digit == d0)) {
            unsigned long long s = m;
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
            if (lane == leader) {
              atomicAdd(&xch->hmass[h][d0], s);
              atomicAdd(&xch->hcnt[h][d0], (unsigned)__popc(vmask));
            }
          } else if (valid) {
            atomicAdd(&xch->hmass[h][digit], m);
            atomicAdd(&xch->hcnt[h][digit], 1u);
          }
        }
      }
      if (first) {
#pragma unroll
        for (int h = 0; h < G; ++h) {
          unsigned long long s = tloc[h];
#pragma unroll
          for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
          if (lane == 0) sc.warp_u64[warp] = s;
          __syncthreads();
          if (tid == 0) {
            unsigned long long tot = 0;
            for (int w2 = 0; w2 < kWarps; ++w2) tot += sc.warp_u64[w2];
            xch->T[h] = tot;
          }
          __syncthreads();
        }
      }
      __syncthreads();
      cluster.sync();  // S2: local histograms published

      for (int h = 0; h < G; ++h) {
        if (done[h] || (h % C) != rank) continue;  // uniform per CTA
        if (first && tid == 0) {
          unsigned long long tot = 0;
          for (int r = 0; r < C; ++r) tot += cluster.map_shared_rank(xch, r)->T[h];
          sc.bcast_u64[0] = ceil_mul_shift32(tot, p.p_q);
        }
        __syncthreads();
        const unsigned long long nd = first ? sc.bcast_u64[0] : need[h];
        const int w = shift[h] < 8 ? shift[h] : 8;
        const int nb = 1 << w;
        unsigned long long bm = 0ull;
        unsigned int bc = 0u;
        if (tid < nb) {
          for (int r = 0; r < C; ++r) {
            const Xch* rx = cluster.map_shared_rank(xch, r);
            bm += rx->hmass[h][tid];
            bc += rx->hcnt[h][tid];
          }
        }
        // suffix sums from the highest digit: the crossing digit d has
        // above + suffix_excl(d) < need <= above + suffix_incl(d)
        if (tid == 0) {  // fallback if no crossing exists (impossible for exact sums)
          xch->r_above[h] = above[h];
          xch->r_need[h] = nd;
          xch->r_bmass[h] = 1ull;
          xch->r_bcnt[h] = 1u;
          xch->r_prefix[h] = prefix[h] << w;
          xch->r_shift[h] = shift[h] - w;
          xch->r_done[h] = 2;
        }
        const unsigned long long suf = block_suffix_u64(tid < nb ? bm : 0ull, sc);
        const unsigned long long ab = above[h];
        if (tid < nb && ab + suf >= nd && ab + (suf - bm) < nd) {
          xch->r_above[h] = ab + (suf - bm);
          xch->r_need[h] = nd;
          xch->r_bmass[h] = bm;
          xch->r_bcnt[h] = bc;
          xch->r_prefix[h] = (prefix[h] << w) | (uint32_t)tid;
          xch->r_shift[h] = shift[h] - w;
          xch->r_done[h] = (bc == 1u) || (shift[h] - w == 0);
        }
        __syncthreads();
        if (tid == 0 && xch->r_done[h] == 2) raise_status(p.status, ZHA_ERR_INTERNAL);
      }
      cluster.sync();  // S3: results published
      if (tid < G && !done[tid]) {
        const Xch* ox = cluster.map_shared_rank(xch, tid % C);
        sc.l_above[tid] = ox->r_above[tid];
        sc.l_need[tid] = ox->r_need[tid];
        sc.l_bmass[tid] = ox->r_bmass[tid];
        sc.l_bcnt[tid] = ox->r_bcnt[tid];
        sc.l_prefix[tid] = ox->r_prefix[tid];
        sc.l_shift[tid] = ox->r_shift[tid];
        sc.l_done[tid] = ox->r_done[tid];
      }
      __syncthreads();

      any_open = false;
#pragma unroll
      for (int h = 0; h < G; ++h) {
        if (done[h]) continue;
        above[h] = sc.l_above[h];
        need[h] = sc.l_need[h];
        bmass[h] = sc.l_bmass[h];
        bcnt[h] = sc.l_bcnt[h];
        const uint32_t np = sc.l_prefix[h];
        const int nsh = sc.l_shift[h];
        done[h] = sc.l_done[h] != 0;
        if (done[h] && tid == 0) {
          // this CTA's share of the boundary group, for tie ranks later
          const uint32_t d = np & ((1u << (shift[h] - nsh)) - 1u);
          xch->tie_local[h] = xch->hcnt[h][d];
        }
        prefix[h] = np;
        shift[h] = nsh;
        any_open |= !done[h];
      }
      first = false;
      __syncthreads();
    }
    cluster.sync();  // S4: tie_local visible; histograms no longer read

    // ------------------------------------------------------------------
    // 3. emit: kept mask per candidate, counts, tie ranks where needed
    // ------------------------------------------------------------------
    unsigned long long tie_need[G];
    bool need_rank[G];
    unsigned int tie_base[G];
#pragma unroll
    for (int h = 0; h < G; ++h) {
      need_rank[h] = false;
      tie_need[h] = 0;
      tie_base[h] = 0;
      if (!p.keep_all) {
        const unsigned long long mt = bmass[h] / bcnt[h];
        tie_need[h] = (need[h] - above[h] + mt - 1) / mt;
        need_rank[h] = tie_need[h] < bcnt[h];
      }
    }
    if (tid < C * G) sc.g_u32[tid / G][tid % G] = cluster.map_shared_rank(xch, tid / G)->tie_local[tid % G];
    __syncthreads();
#pragma unroll
    for (int h = 0; h < G; ++h)
      if (need_rank[h])
        for (int r = 0; r < rank; ++r) tie_base[h] += sc.g_u32[r][h];
    __syncthreads();
    if (tid < kMaxGroup) {
      sc.kcnt[tid] = 0u;
      sc.tcnt[tid] = 0u;
    }
    if (tid == 0) xch->node0_mask = 0u;
    __syncthreads();
    unsigned int nk_loc = 0;
    for (int64_t base = lo; base < hi; base += kThreads) {
      const int64_t ci = base + tid;
      const bool in = ci < hi;
      const uint32_t cv = in ? cin[ci] : 0u;
      const uint32_t pm = cv >> 24;
      uint32_t km = 0u;
#pragma unroll
      for (int h = 0; h < G; ++h) {
        bool inc = in && ((pm >> h) & 1u);
        bool keep = false, tie = false;
        if (inc) {
          if (p.keep_all) {
            keep = true;
          } else {
            const uint32_t key = order_key(zb[(int64_t)h * p.max_cand + ci]);
            const uint32_t pre = (uint32_t)((uint64_t)key >> shift[h]);
            keep = pre > prefix[h];
            tie = pre == prefix[h];
          }
        }
        if (need_rank[h]) {  // uniform: ordered rank among the boundary group
          unsigned int tot;
          const unsigned int r = block_excl_scan(tie ? 1u : 0u, &tot, sc);
          if (tie && tie_base[h] + sc.tcnt[h] + r < tie_need[h]) keep = true;
          __syncthreads();
          if (tid == 0) sc.tcnt[h] += tot;
          __syncthreads();
        } else if (tie) {
          keep = true;
        }
        if (keep) km |= 1u << h;
      }
      if (in) cin[ci] = (km << 24) | (cv & kNodeMask);
      nk_loc += (km != 0u);
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const unsigned cnt = __popc(__ballot_sync(0xffffffffu, (km >> h) & 1u));
        if (lane == 0 && cnt) atomicAdd(&sc.kcnt[h], cnt);
      }
      if (level == 1 && in && (cv & kNodeMask) == 0u) xch->node0_mask = km;
    }
    {
      unsigned int tot;
      block_excl_scan(nk_loc, &tot, sc);
      if (tid == 0) xch->nk = tot;
      if (tid < G) xch->kept_cnt[tid] = sc.kcnt[tid];
    }
    __syncthreads();
    cluster.sync();  // S5: union / per-head counts published
    if (tid < C * (G + 1)) {
      const int r = tid / (G + 1), h = tid % (G + 1);
      const Xch* rx = cluster.map_shared_rank(xch, r);
      sc.g_u32[r][h] = (h < G) ? rx->kept_cnt[h] : rx->nk;
    }
    if (tid == 0) {
      int r0 = 0;  // rank holding global candidate 0 (node 0 is always first if present)
      while (n_cand * (r0 + 1) / C < 1) ++r0;
      sc.node0 = cluster.map_shared_rank(xch, r0)->node0_mask;
    }
    __syncthreads();

    unsigned int ubase = 0, utotal = 0;
    for (int r = 0; r < C; ++r) {
      const unsigned int v = sc.g_u32[r][G];
      if (r < rank) ubase += v;
      utotal += v;
    }
    // per-level kept counts (top level first)
    if (lc_base && rank == 0 && tid < G) {
      unsigned int tot = 0;
      for (int r = 0; r < C; ++r) tot += sc.g_u32[r][tid];
      lc_base[(int64_t)tid * p.L + (p.L - level)] = (int32_t)tot;
    }

    // ordered compaction of the union-kept candidates of this slice
    unsigned int run = 0;
    for (int64_t base = lo; base < hi; base += kThreads) {
      const int64_t ci = base + tid;
      const uint32_t cv = ci < hi ? cin[ci] : 0u;
      const uint32_t km = cv >> 24;
      unsigned int tot;
      const unsigned int r = block_excl_scan(km ? 1u : 0u, &tot, sc);
      if (km) {
        const int64_t pos = (int64_t)ubase + run + r;
        const uint32_t node = cv & kNodeMask;
        if (level > 1) {
          for (int c = 0; c < b; ++c)
            cnext[pos * b + c] = (km << 24) | (node * (uint32_t)b + (uint32_t)c);
        } else if (!p.list_mode) {
          p.kept[(int64_t)unit * p.max_cand + pos] = cv;
        }
      }
      run += tot;
    }

    if (level == 1) {
      if (!p.list_mode) {
        if (rank == 0 && tid == 0) p.n_kept[unit] = (int32_t)utotal;
      } else {
        // per-head ascending token lists: {0} (unless node 0 kept) + kept
        // level-1 nodes' tokens + causal tail
        const int64_t tail_start = p.span[p.L] * T_top;
        const int64_t tail_len = n_vis - tail_start;
        const uint32_t node0 = sc.node0;
        for (int h = 0; h < G; ++h) {
          const int64_t qh = (int64_t)qi * p.Hq + (int64_t)kvh * G + h;
          int32_t* out = p.idx + qh * p.idx_cap;
          unsigned int hb = 0, htot = 0;
          for (int r = 0; r < C; ++r) {
            const unsigned int v = sc.g_u32[r][h];
            if (r < rank) hb += v;
            htot += v;
          }
          const int64_t off0 = ((node0 >> h) & 1u) ? 0 : 1;
          unsigned int hrun = 0;
          for (int64_t base = lo; base < hi; base += kThreads) {
            const int64_t ci = base + tid;
            const uint32_t cv = ci < hi ? cin[ci] : 0u;
            const bool kh = ((cv >> 24) >> h) & 1u;
            unsigned int tot;
            const unsigned int r = block_excl_scan(kh ? 1u : 0u, &tot, sc);
            if (kh) {
              const int64_t pos = off0 + (int64_t)b * (hb + hrun + r);
              const int64_t node = cv & kNodeMask;
              for (int c = 0; c < b; ++c)
                if (pos + c < p.idx_cap) out[pos + c] = (int32_t)(node * b + c);
            }
            hrun += tot;
          }
          const int64_t tail_pos = off0 + (int64_t)b * htot;
          if (rank == 0) {
            if (off0 == 1 && tid == 0 && p.idx_cap > 0) out[0] = 0;
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
    }
    n_cand = (int64_t)utotal * b;
    cur ^= 1;
    __syncthreads();
    cluster.sync();  // S6: next candidate list complete
  }
}

template <typename T, int D, int G>
cudaError_t launch_t(const TravParams& p, int64_t units, int C, cudaStream_t stream) {
  constexpr int kRowBytes = D * (int)sizeof(T);
  constexpr int kTile = (kRowBytes <= 256) ? 256 : 128;
  const size_t smem = 2 * (size_t)kTile * kRowBytes + sizeof(float) * D * kMaxGroup +
                      sizeof(Xch) + sizeof(Scratch);
  auto kern = traverse_kernel<T, D, G>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
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

}  // namespace

size_t traverse_ws_bytes(const Geometry& g, int64_t units) {
  const int64_t max_cand = g.level_rows[0] + 1;
  const size_t per = (size_t)max_cand * (2 * sizeof(uint32_t) + (size_t)g.G * sizeof(float));
  return per * (size_t)units + 256;
}

cudaError_t launch_traverse(const Geometry& g, const void* tree, const void* q,
                            const int32_t* seq_len, const int32_t* q_seq, const int32_t* q_pos,
                            int64_t nq, uint64_t p_q, int list_mode, const TraverseOut& out,
                            void* ws, size_t ws_bytes, int32_t* status, int num_sms,
                            cudaStream_t stream) {
  const int64_t units = nq * g.Hkv;
  if (units <= 0) return cudaSuccess;
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
  const int64_t max_cand = g.level_rows[0] + 1;
  p.max_cand = max_cand;
  unsigned char* w = static_cast<unsigned char*>(ws);
  p.cand = reinterpret_cast<uint32_t*>(w);
  w += sizeof(uint32_t) * 2 * max_cand * units;
  p.zbuf = reinterpret_cast<float*>(w);
  if (!list_mode) {
    if (!out.kept || !out.n_kept) return cudaErrorInvalidValue;
    p.kept = out.kept;
    p.n_kept = out.n_kept;
  }
  p.idx = out.idx;
  p.idx_cap = out.idx_cap;
  p.n_idx = out.n_idx;
  p.level_counts = out.level_counts;
  p.status = status;
  (void)ws_bytes;
  int C = 1;
  while (C < 8 && units * (C * 2) <= num_sms) C *= 2;
  if (g.dtype == ZHA_BF16) {
    if (g.d == 128) return launch_g<__nv_bfloat16, 128>(g.G, p, units, C, stream);
    return launch_g<__nv_bfloat16, 64>(g.G, p, units, C, stream);
  }
  if (g.d == 128) return launch_g<float, 128>(g.G, p, units, C, stream);
  return launch_g<float, 64>(g.G, p, units, C, stream);
}

}  // namespace zha
