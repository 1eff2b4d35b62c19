// Split-K flash-decoding attention over a stream of selected KV rows.
//
// lefilia.fr page "Zyphra presente Zyphra Hierarchical Attention (ZHA) ...",
// paragraph 1: the KV cache stays complete and the tree only decides which
// keys each query reads; attention then runs over the selected raw entries:
//     o = sum_{j in S} softmax_j(q . k_j / sqrt(d)) v_j .
//
// One kernel serves three row streams:
//   tree  -- one unit = (sequence, KV head) with its G query heads: token 0,
//            the union of the heads' kept level-1 nodes (b rows each, with an
//            8-bit head mask from the traversal) and the causal tail. Each K/V
//            row is read from HBM once and serves every head whose mask bit is
//            set (masked heads see -inf).
//   dense -- every row [0, t] for every head (the dense baseline).
//   list  -- one unit = one query head with an explicit ascending index list.
// A unit's rows are split over S CTAs (split-K); each CTA keeps an online
// softmax per head and writes (m, l, acc[d]); a combine kernel merges splits.
//
// Inside a CTA every warp runs its own two-stage cp.async pipeline over 32-row
// blocks (lane = row): 16-byte chunks land XOR-swizzled so that a lane reading
// its own row and all lanes reading one row are both bank-conflict free.
// QK: lane = row, G heads, fp32x2 FMAs over head pairs. PV: lane = a slice of
// the head dimension, fp32x2 FMAs over dimension pairs. Scores use exp2 with
// q pre-scaled by log2(e)/sqrt(d).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "zha_device.cuh"
#include "zha_internal.h"

namespace zha {
namespace {

constexpr float kLog2e = 1.4426950408889634f;

struct AttParams {
  int kind;
  const void* k;
  const void* v;
  const void* q;
  const int32_t* seq_len;
  const int32_t* q_seq;
  const int32_t* q_pos;    // tree stream with explicit positions (prefill)
  int64_t ncap;
  int Hq, Hkv, G, b, L, B;
  int b_shift;             // log2(b) when b is a power of two, else -1
  int64_t span_L;
  float qscale;            // log2(e) / sqrt(d)
  // tree stream
  const uint32_t* kept;
  const int32_t* n_kept;
  int64_t kept_stride;
  int kept_segs;
  // list stream
  const int32_t* idx;
  int64_t idx_cap;
  const int32_t* n_idx;
  int S;                   // splits per unit
  int unit0;               // first unit of this launch (grid: its units x S)
  float* part;             // [units][S][G][D + 2]
};

template <typename T, int D>
struct Cfg {
  static constexpr int kRowBytes = D * (int)sizeof(T);
  static constexpr int kNch = kRowBytes / 16;
  static constexpr int kStageBytes = 32 * kRowBytes * 2;  // K and V of 32 rows
  static constexpr int kWarpBytes = 2 * kStageBytes + 32 * kMaxGroup * 8;
  static constexpr int kWarps = (200 * 1024) / kWarpBytes < 6 ? (200 * 1024) / kWarpBytes : 6;
  static constexpr int kThreads = 32 * kWarps;
  static constexpr int kDimsPerLane = D / 32;
};

// Describes the rows of one CTA's share of a unit.
struct Span {
  int64_t kv_unit;      // (sequence, KV head) row block
  int tok0;             // 1 if token 0 is a separate leading row
  int64_t n0, n1;       // node range in the kept list (tree)
  int64_t t0, t1;       // tail rows (tree) / dense rows / list positions
  int64_t tail_start;
  int64_t rows;
  const uint32_t* kept;        // segment 0 of the unit
  const uint32_t* kept_local;  // this CTA's node range [n0, n1) in shared memory, or null
  const unsigned int* segbase; // [segs + 1] prefix of segment sizes (shared memory)
  int64_t stride;
  const int32_t* list;
};

// Exclusive prefix of the unit's kept-segment sizes into segbase[0 .. segs]
// (called by one full warp): every lane loads one size at once, so the CTA
// does not wait for the sizes one after another.
__device__ __forceinline__ void seg_prefix(const AttParams& p, int unit, int64_t T_top,
                                           unsigned int* segbase) {
  const int lane = threadIdx.x & 31;
  unsigned int v = (lane < p.kept_segs && T_top > 0)
                       ? (unsigned int)p.n_kept[(int64_t)unit * p.kept_segs + lane]
                       : 0u;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const unsigned int y = __shfl_up_sync(0xffffffffu, v, off);
    if (lane >= off) v += y;
  }
  if (lane < p.kept_segs) segbase[lane + 1] = v;
  if (lane == 0) segbase[0] = 0u;
}

// Row of virtual index v in the CTA share, with its head mask (0 = skip).
__device__ __forceinline__ void row_of(const AttParams& p, const Span& s, int64_t v,
                                       int64_t* row, uint32_t* mask, uint32_t all) {
  if (p.kind == kStreamTree) {
    if (v < s.tok0) {
      *row = 0;
      *mask = all;
      return;
    }
    v -= s.tok0;
    const int64_t nrows = (s.n1 - s.n0) * p.b;
    if (v < nrows) {
      // node slot and offset within the node (v < 2^31: a CTA's share of a unit)
      const uint32_t vv = (uint32_t)v;
      const uint32_t q = p.b_shift >= 0 ? vv >> p.b_shift : vv / (uint32_t)p.b;
      const int off = (int)(vv - q * (uint32_t)p.b);
      const int64_t j = s.n0 + q;
      uint32_t e;
      if (s.kept_local) {
        e = s.kept_local[j - s.n0];
      } else {
        int r = 0;
        while ((int64_t)s.segbase[r + 1] <= j) ++r;
        e = s.kept[r * s.stride + (j - s.segbase[r])];
      }
      const int64_t node = e & 0x00ffffffu;
      *row = node * p.b + off;
      *mask = (node == 0 && off == 0) ? 0u : (e >> 24);
      return;
    }
    *row = s.tail_start + s.t0 + (v - nrows);
    *mask = all;
    return;
  }
  if (p.kind == kStreamDense) {
    *row = s.t0 + v;
    *mask = all;
    return;
  }
  *row = s.list[s.t0 + v];
  *mask = 1u;
}

template <typename T, int D, int G>
__global__ void __launch_bounds__(Cfg<T, D>::kThreads, 1) attend_kernel(AttParams p) {
  using C = Cfg<T, D>;
  constexpr int kNch = C::kNch;
  constexpr int kPer = Elem<T>::kPerChunk;
  constexpr int kDL = C::kDimsPerLane;
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ unsigned int s_segbase[kMaxCluster + 1];
  float* qs = reinterpret_cast<float*>(smem);                       // [D][8]
  unsigned char* wbase = smem + D * kMaxGroup * sizeof(float);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  unsigned char* my = wbase + warp * C::kWarpBytes;
  float2* pbuf = reinterpret_cast<float2*>(my + 2 * C::kStageBytes);  // [32][8]

  const int unit = p.unit0 + (int)(blockIdx.x / p.S);
  const int split = blockIdx.x % p.S;
  const uint32_t all = (1u << G) - 1u;

  // ---- this CTA's share of the unit's row stream ----
  Span s{};
  const T* qrow;
  if (p.kind == kStreamList) {
    const int64_t qi = unit / p.Hq;
    const int h = unit % p.Hq;
    int seq = p.q_seq[qi];
    int64_t n = p.n_idx[unit] < p.idx_cap ? p.n_idx[unit] : p.idx_cap;
    if (seq < 0 || seq >= p.B) {
      seq = 0;
      n = 0;
    }
    s.kv_unit = (int64_t)seq * p.Hkv + h / (p.Hq / p.Hkv);
    s.t0 = n * split / p.S;
    s.t1 = n * (split + 1) / p.S;
    s.rows = s.t1 - s.t0;
    s.list = p.idx + (int64_t)unit * p.idx_cap;
    qrow = static_cast<const T*>(p.q) + (int64_t)unit * D;
  } else {
    const int qi = unit / p.Hkv, kvh = unit % p.Hkv;
    int seq = p.q_pos ? p.q_seq[qi] : qi;
    int64_t t = p.q_pos ? (int64_t)p.q_pos[qi] : (int64_t)p.seq_len[seq] - 1;
    if (seq < 0 || seq >= p.B) {
      seq = 0;
      t = -1;
    } else {
      int64_t n = p.seq_len[seq];
      if (n > p.ncap) n = p.ncap;
      if (t > n - 1) t = n - 1;
    }
    s.kv_unit = (int64_t)seq * p.Hkv + kvh;
    qrow = static_cast<const T*>(p.q) + ((int64_t)qi * p.Hq + (int64_t)kvh * G) * D;
    if (p.kind == kStreamDense) {
      s.t0 = (t + 1) * split / p.S;
      s.t1 = (t + 1) * (split + 1) / p.S;
      s.rows = s.t1 - s.t0;
    } else {
      const int64_t T_top = (t + 1) / p.span_L;
      s.tail_start = p.span_L * T_top;
      const int64_t tail_len = t + 1 - s.tail_start;
      if (tid < 32) seg_prefix(p, unit, T_top, s_segbase);
      __syncthreads();
      const int64_t nk = s_segbase[p.kept_segs];
      s.kept = p.kept + (int64_t)unit * p.kept_segs * p.kept_stride;
      s.segbase = s_segbase;
      s.stride = p.kept_stride;
      s.tok0 = (T_top > 0 && split == 0) ? 1 : 0;
      s.n0 = nk * split / p.S;
      s.n1 = nk * (split + 1) / p.S;
      s.t0 = tail_len * split / p.S;
      s.t1 = tail_len * (split + 1) / p.S;
      s.rows = s.tok0 + (s.n1 - s.n0) * p.b + (s.t1 - s.t0);
    }
  }
  for (int e = tid; e < D * kMaxGroup; e += blockDim.x) {
    const int i = e / kMaxGroup, h = e % kMaxGroup;
    qs[e] = (h < G) ? Elem<T>::to_f(qrow[(int64_t)h * D + i]) * p.qscale : 0.0f;
  }
  __syncthreads();

  const T* kbase = static_cast<const T*>(p.k) + s.kv_unit * p.ncap * D;
  const T* vbase = static_cast<const T*>(p.v) + s.kv_unit * p.ncap * D;

  // per-warp online softmax state
  float m_run[G];
  float l_lane[G];
  float2 acc[G][kDL / 2 > 0 ? kDL / 2 : 1];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    m_run[h] = -INFINITY;
    l_lane[h] = 0.0f;
#pragma unroll
    for (int j = 0; j < (kDL / 2 > 0 ? kDL / 2 : 1); ++j) acc[h][j] = make_float2(0.f, 0.f);
  }

  const int64_t nblk = (s.rows + 31) / 32;
  const int nw = blockDim.x / 32;
  uint32_t mask_cur = 0, mask_next = 0;

  auto issue = [&](int64_t blk, int stage) -> uint32_t {
    const int64_t v = blk * 32 + lane;
    uint32_t m = 0;
    if (v < s.rows) {
      int64_t row;
      row_of(p, s, v, &row, &m, all);
      if (row < 0 || row >= p.ncap) m = 0u;  // caller-provided lists are bounds-checked
      if (m) {
        unsigned char* kd = my + stage * C::kStageBytes + lane * C::kRowBytes;
        unsigned char* vd = kd + 32 * C::kRowBytes;
        const unsigned char* ks = reinterpret_cast<const unsigned char*>(kbase + row * D);
        const unsigned char* vs = reinterpret_cast<const unsigned char*>(vbase + row * D);
#pragma unroll
        for (int c = 0; c < kNch; ++c) {
          cp_async16(kd + swz(c, lane) * 16, ks + c * 16);
          cp_async16(vd + swz(c, lane) * 16, vs + c * 16);
        }
      }
    }
    cp_async_commit();
    return m;
  };

  int64_t blk = warp;
  if (blk < nblk) mask_cur = issue(blk, 0);
  int stage = 0;
  for (; blk < nblk; blk += nw) {
    const int64_t nb = blk + nw;
    if (nb < nblk) {
      mask_next = issue(nb, stage ^ 1);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncwarp();
    const unsigned char* kst = my + stage * C::kStageBytes;
    const unsigned char* vst = kst + 32 * C::kRowBytes;
    // ---- QK: lane = row, all G heads ----
    float sc[G];
    {
      float2 a2[(G + 1) / 2];
#pragma unroll
      for (int j = 0; j < (G + 1) / 2; ++j) a2[j] = make_float2(0.f, 0.f);
      float a1 = 0.0f;
      if (mask_cur) {
        const unsigned char* row = kst + lane * C::kRowBytes;
#pragma unroll 4
        for (int ch = 0; ch < kNch; ++ch) {
          const uint4 raw = lds128(row + swz(ch, lane) * 16);
          float x[kPer];
          Elem<T>::unpack(raw, x);
#pragma unroll
          for (int e = 0; e < kPer; ++e) {
            const float* qv = qs + (ch * kPer + e) * kMaxGroup;
            if constexpr (G == 1) {
              a1 = fmaf(qv[0], x[e], a1);
            } else {
              const float2 xx = make_float2(x[e], x[e]);
#pragma unroll
              for (int j = 0; j < G / 4; ++j) {
                const float4 q4 = *reinterpret_cast<const float4*>(qv + 4 * j);
                a2[2 * j] = ffma2(make_float2(q4.x, q4.y), xx, a2[2 * j]);
                a2[2 * j + 1] = ffma2(make_float2(q4.z, q4.w), xx, a2[2 * j + 1]);
              }
              if constexpr (G == 2) a2[0] = ffma2(*reinterpret_cast<const float2*>(qv), xx, a2[0]);
            }
          }
        }
      }
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float raw = (G == 1) ? a1 : ((h & 1) ? a2[h / 2].y : a2[h / 2].x);
        sc[h] = ((mask_cur >> h) & 1u) ? raw : -INFINITY;
      }
    }
    // ---- online softmax (warp) ----
#pragma unroll
    for (int h = 0; h < G; ++h) {
      float mb = sc[h];
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) mb = fmaxf(mb, __shfl_xor_sync(0xffffffffu, mb, off));
      const float mn = fmaxf(m_run[h], mb);
      float alpha, pr;
      if (mn == -INFINITY) {
        alpha = 1.0f;
        pr = 0.0f;
      } else {
        alpha = exp2f(m_run[h] - mn);
        pr = exp2f(sc[h] - mn);
      }
      m_run[h] = mn;
      l_lane[h] = l_lane[h] * alpha + pr;
      const float2 aa = make_float2(alpha, alpha);
#pragma unroll
      for (int j = 0; j < (kDL / 2 > 0 ? kDL / 2 : 1); ++j) acc[h][j] = fmul2(acc[h][j], aa);
      pbuf[lane * kMaxGroup + h] = make_float2(pr, pr);
    }
    __syncwarp();
    // ---- PV: lane = dims [lane*kDL, lane*kDL + kDL) ----
    unsigned live = __ballot_sync(0xffffffffu, mask_cur != 0u);
    while (live) {
      const int r = __ffs(live) - 1;
      live &= live - 1;
      const unsigned char* vrow = vst + r * C::kRowBytes;
      const int byte0 = lane * kDL * (int)sizeof(T);
      const unsigned char* src = vrow + swz(byte0 >> 4, r) * 16 + (byte0 & 15);
      float vv[kDL > 0 ? kDL : 1];
      if constexpr (sizeof(T) == 2) {
        if constexpr (kDL == 4) {
          const uint2 w = *reinterpret_cast<const uint2*>(src);
          const float2 a = bf16x2_to_f2(w.x), b2 = bf16x2_to_f2(w.y);
          vv[0] = a.x; vv[1] = a.y; vv[2] = b2.x; vv[3] = b2.y;
        } else {
          const float2 a = bf16x2_to_f2(*reinterpret_cast<const uint32_t*>(src));
          vv[0] = a.x; vv[1] = a.y;
        }
      } else {
        if constexpr (kDL == 4) {
          const float4 a = *reinterpret_cast<const float4*>(src);
          vv[0] = a.x; vv[1] = a.y; vv[2] = a.z; vv[3] = a.w;
        } else {
          const float2 a = *reinterpret_cast<const float2*>(src);
          vv[0] = a.x; vv[1] = a.y;
        }
      }
      const float2* pr = pbuf + r * kMaxGroup;
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float2 pp = pr[h];
#pragma unroll
        for (int j = 0; j < kDL / 2; ++j)
          acc[h][j] = ffma2(pp, make_float2(vv[2 * j], vv[2 * j + 1]), acc[h][j]);
      }
    }
    __syncwarp();
    mask_cur = mask_next;
    stage ^= 1;
  }

  // ---- merge the warps of the CTA and write the split partial ----
  __syncthreads();
  float* mw = reinterpret_cast<float*>(wbase);             // [nw][G]   m
  float* lw = mw + nw * kMaxGroup;                         // [nw][G]   l
  float* aw = lw + nw * kMaxGroup;                         // [nw][G][D]
#pragma unroll
  for (int h = 0; h < G; ++h) {
    float l = l_lane[h];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) l += __shfl_xor_sync(0xffffffffu, l, off);
    if (lane == 0) {
      mw[warp * kMaxGroup + h] = m_run[h];
      lw[warp * kMaxGroup + h] = l;
    }
#pragma unroll
    for (int j = 0; j < kDL / 2; ++j) {
      aw[(warp * kMaxGroup + h) * D + lane * kDL + 2 * j] = acc[h][j].x;
      aw[(warp * kMaxGroup + h) * D + lane * kDL + 2 * j + 1] = acc[h][j].y;
    }
  }
  __syncthreads();
  float* out = p.part + ((int64_t)unit * p.S + split) * G * (D + 2);
  for (int e = tid; e < G * D; e += blockDim.x) {
    const int h = e / D, i = e % D;
    float M = -INFINITY;
    for (int w = 0; w < nw; ++w) M = fmaxf(M, mw[w * kMaxGroup + h]);
    float a = 0.0f, l = 0.0f;
    if (M != -INFINITY) {
      for (int w = 0; w < nw; ++w) {
        const float sc2 = exp2f(mw[w * kMaxGroup + h] - M);
        a += aw[(w * kMaxGroup + h) * D + i] * sc2;
        l += lw[w * kMaxGroup + h] * sc2;
      }
    }
    out[h * (D + 2) + i] = a;
    if (i == 0) {
      out[h * (D + 2) + D] = M;
      out[h * (D + 2) + D + 1] = l;
    }
  }
}

// ---------------------------------------------------------------------------
// bf16 GQA-group path on warp-level tensor-core MMA.
//
// The G <= 8 query heads of a KV head form the M side of an m16n8k16 MMA
// (rows G..15 are zero), so per 32 keys a warp issues 32 MMAs for S = Q K^T
// and 32 for O += P V, with K/V fragments read by ldmatrix from the swizzled
// tiles. The group contraction is tiny (8 x 128 x n); the point is to keep the
// FP32/ALU pipes out of the way so the kernel stays bound by HBM.
// ---------------------------------------------------------------------------
template <int D>
struct MmaCfg {
  static constexpr int kRowBytes = D * 2;
  // 6 warps x 2 stages (one block in flight while one is computed): more
  // warps to issue the per-block work than 4 x 3, with the same shared memory
  static constexpr int kStages = 2;
  static constexpr int kStageBytes = 32 * kRowBytes * 2;             // K and V of 32 rows
  static constexpr int kWarpBytes = kStages * kStageBytes + kStages * 32;  // + row masks
  static constexpr int kWarps = 6;
  static constexpr int kKeptCap = 5120;   // kept-list entries staged in shared memory
  static constexpr int kThreads = 32 * kWarps;
  static constexpr int kKSteps = D / 16;   // QK k-steps
  static constexpr int kNTiles = D / 8;    // PV n-tiles
};

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// D = A(16x16 bf16, rows 8..15 zero) * B(16x8 bf16) + C, fp32 accumulate.
__device__ __forceinline__ void mma_bf16(float* c, uint32_t a0, uint32_t a2, uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(0u), "r"(a2), "r"(0u), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

template <int D, int G>
__global__ void __launch_bounds__(MmaCfg<D>::kThreads, 1) attend_mma_kernel(AttParams p) {
  using C = MmaCfg<D>;
  using T = __nv_bfloat16;
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ unsigned int s_segbase[kMaxCluster + 1];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t4 = lane & 3;   // MMA fragment coordinates
  unsigned char* my = smem + warp * C::kWarpBytes;
  uint8_t* rmask = my + C::kStages * C::kStageBytes;  // [stage][32]

  const int unit = p.unit0 + (int)(blockIdx.x / p.S);
  const int split = blockIdx.x % p.S;
  const uint32_t all = (1u << G) - 1u;

  Span s{};
  const int qi = unit / p.Hkv, kvh = unit % p.Hkv;
  int seq = p.q_pos ? p.q_seq[qi] : qi;
  int64_t t = p.q_pos ? (int64_t)p.q_pos[qi] : (int64_t)p.seq_len[seq] - 1;
  if (seq < 0 || seq >= p.B) {
    seq = 0;
    t = -1;
  } else {
    int64_t n = p.seq_len[seq];
    if (n > p.ncap) n = p.ncap;
    if (t > n - 1) t = n - 1;
  }
  s.kv_unit = (int64_t)seq * p.Hkv + kvh;
  const T* qrow = static_cast<const T*>(p.q) + ((int64_t)qi * p.Hq + (int64_t)kvh * G) * D;
  if (p.kind == kStreamDense) {
    s.t0 = (t + 1) * split / p.S;
    s.t1 = (t + 1) * (split + 1) / p.S;
    s.rows = s.t1 - s.t0;
  } else {
    const int64_t T_top = (t + 1) / p.span_L;
    s.tail_start = p.span_L * T_top;
    const int64_t tail_len = t + 1 - s.tail_start;
    if (tid < 32) seg_prefix(p, unit, T_top, s_segbase);
    __syncthreads();
    const int64_t nk = s_segbase[p.kept_segs];
    s.kept = p.kept + (int64_t)unit * p.kept_segs * p.kept_stride;
    s.segbase = s_segbase;
    s.stride = p.kept_stride;
    s.tok0 = (T_top > 0 && split == 0) ? 1 : 0;
    s.n0 = nk * split / p.S;
    s.n1 = nk * (split + 1) / p.S;
    s.t0 = tail_len * split / p.S;
    s.t1 = tail_len * (split + 1) / p.S;
    s.rows = s.tok0 + (s.n1 - s.n0) * p.b + (s.t1 - s.t0);
    if (s.n1 - s.n0 <= C::kKeptCap) {  // stage this CTA's kept entries in smem once
      // every entry's 4-byte asynchronous copy is issued before the one wait:
      // the streaming below waits for this prologue
      uint32_t* kl = reinterpret_cast<uint32_t*>(smem + C::kWarps * C::kWarpBytes);
      int r = 0;  // segment cursor: this thread's entries only grow
      for (int64_t j = s.n0 + tid; j < s.n1; j += C::kThreads) {
        while ((int64_t)s_segbase[r + 1] <= j) ++r;
        cp_async4(kl + (j - s.n0), s.kept + r * s.stride + (j - s_segbase[r]));
      }
      cp_async_commit();
      cp_async_wait<0>();
      s.kept_local = kl;
      __syncthreads();
    }
  }

  // Q fragments (rows g < G; exact bf16 inputs), kept in registers
  uint32_t qa0[C::kKSteps], qa2[C::kKSteps];
#pragma unroll
  for (int ks = 0; ks < C::kKSteps; ++ks) {
    if (g < G) {
      const uint32_t* qr = reinterpret_cast<const uint32_t*>(qrow + (int64_t)g * D);
      qa0[ks] = qr[(ks * 16 + 2 * t4) / 2];
      qa2[ks] = qr[(ks * 16 + 8 + 2 * t4) / 2];
    } else {
      qa0[ks] = 0u;
      qa2[ks] = 0u;
    }
  }
  // stale tiles must hold finite values: masked rows still meet P = 0 in the MMA
  for (int e = lane; e < C::kWarpBytes / 16; e += 32)
    reinterpret_cast<uint4*>(my)[e] = make_uint4(0u, 0u, 0u, 0u);
  __syncwarp();

  const T* kbase = static_cast<const T*>(p.k) + s.kv_unit * p.ncap * D;
  const T* vbase = static_cast<const T*>(p.v) + s.kv_unit * p.ncap * D;
  const int nw = C::kWarps;
  const int64_t nblk = (s.rows + 31) / 32;

  // Row metadata of the next block to issue is computed one block ahead, so the
  // kept-list load it needs completes while the current block is computed.
  int64_t nxt_blk = warp;
  int64_t pr_row = 0;
  uint32_t pr_m = 0;
  auto fetch_row = [&]() {
    const int64_t v = nxt_blk * 32 + lane;
    pr_m = 0;
    pr_row = 0;
    if (nxt_blk < nblk && v < s.rows) {
      row_of(p, s, v, &pr_row, &pr_m, all);
      if (pr_row < 0 || pr_row >= p.ncap) pr_m = 0u;
    }
  };
  fetch_row();
  auto issue = [&](int stage) {
    rmask[stage * 32 + lane] = (uint8_t)pr_m;
    // every instruction moves whole rows: lanes 16j..16j+15 copy the 16-byte
    // chunks of one row, so each warp request is a few full 128-byte lines
    constexpr int kCh = C::kRowBytes / 16;   // chunks per row (8 or 16)
    constexpr int kRowsPerInstr = 32 / kCh;  // rows per warp instruction
    const int c = lane % kCh;
    unsigned char* st = my + stage * C::kStageBytes;
#pragma unroll
    for (int i = 0; i < 32 / kRowsPerInstr; ++i) {
      const int r = i * kRowsPerInstr + lane / kCh;
      const int64_t rr = __shfl_sync(0xffffffffu, pr_row, r);
      const uint32_t mm = __shfl_sync(0xffffffffu, pr_m, r);
      if (mm) {
        const int64_t off = rr * C::kRowBytes + c * 16;
        const int dst = r * C::kRowBytes + swz(c, r) * 16;
        cp_async16(st + dst, reinterpret_cast<const unsigned char*>(kbase) + off);
        cp_async16(st + 32 * C::kRowBytes + dst, reinterpret_cast<const unsigned char*>(vbase) + off);
      }
    }
    cp_async_commit();
    nxt_blk += nw;
    fetch_row();
  };

  float o[C::kNTiles][4];
#pragma unroll
  for (int nt = 0; nt < C::kNTiles; ++nt) o[nt][0] = o[nt][1] = o[nt][2] = o[nt][3] = 0.0f;
  float m_run = -INFINITY, l_part = 0.0f;

  // prologue: stages 0 .. kStages-2
  int64_t blk = warp;
#pragma unroll
  for (int st = 0; st < C::kStages - 1; ++st) issue(st);
  int stage = 0;
  for (; blk < nblk; blk += nw) {
    issue((stage + C::kStages - 1) % C::kStages);
    cp_async_wait<C::kStages - 1>();
    __syncwarp();
    const unsigned char* kst = my + stage * C::kStageBytes;
    const unsigned char* vst = kst + 32 * C::kRowBytes;
    const uint32_t kaddr = smem_u32(kst), vaddr = smem_u32(vst);
    // ---- S = Q K^T over 32 keys: 4 n-tiles of 8 keys ----
    float sc[4][4];
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
      sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.0f;
      const int row = nt * 8 + (lane & 7);
#pragma unroll
      for (int ks = 0; ks < C::kKSteps; ks += 2) {
        const int chunk = 2 * ks + (lane >> 3);
        uint32_t b0, b1, b2, b3;
        ldsm_x4(kaddr + row * C::kRowBytes + swz(chunk, row) * 16, b0, b1, b2, b3);
        mma_bf16(sc[nt], qa0[ks], qa2[ks], b0, b1);
        mma_bf16(sc[nt], qa0[ks + 1], qa2[ks + 1], b2, b3);
      }
    }
    // ---- masks, online softmax for head g ----
    const uint8_t* mk = rmask + stage * 32;
    float sv[4][2];
    float mb = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int key = nt * 8 + 2 * t4 + j;
        const bool ok = (mk[key] >> g) & 1u;
        sv[nt][j] = ok ? sc[nt][j] * p.qscale : -INFINITY;
        mb = fmaxf(mb, sv[nt][j]);
      }
    }
    mb = fmaxf(mb, __shfl_xor_sync(0xffffffffu, mb, 1));
    mb = fmaxf(mb, __shfl_xor_sync(0xffffffffu, mb, 2));
    const float mn = fmaxf(m_run, mb);
    const float alpha = (mn == -INFINITY) ? 1.0f : exp2f(m_run - mn);
    m_run = mn;
    uint32_t pa[2][2];
    float lsum = 0.0f;
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
      const float p0 = (mn == -INFINITY) ? 0.0f : exp2f(sv[nt][0] - mn);
      const float p1 = (mn == -INFINITY) ? 0.0f : exp2f(sv[nt][1] - mn);
      lsum += p0 + p1;
      pa[nt >> 1][nt & 1] = pack_bf16(p0, p1);
    }
    l_part = l_part * alpha + lsum;
#pragma unroll
    for (int nt = 0; nt < C::kNTiles; ++nt) {
      o[nt][0] *= alpha;
      o[nt][1] *= alpha;
    }
    // ---- O += P V: 2 k-steps of 16 keys x kNTiles n-tiles of 8 dims ----
#pragma unroll
    for (int ks = 0; ks < 2; ++ks) {
      const int row = ks * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
      for (int nt = 0; nt < C::kNTiles; nt += 2) {
        const int chunk = nt + (lane >> 4);
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(vaddr + row * C::kRowBytes + swz(chunk, row) * 16, b0, b1, b2, b3);
        mma_bf16(o[nt], pa[ks][0], pa[ks][1], b0, b1);
        mma_bf16(o[nt + 1], pa[ks][0], pa[ks][1], b2, b3);
      }
    }
    __syncwarp();
    stage = (stage + 1) % C::kStages;
  }
  cp_async_wait<0>();

  // ---- merge the warps and write the split partial ----
  l_part += __shfl_xor_sync(0xffffffffu, l_part, 1);
  l_part += __shfl_xor_sync(0xffffffffu, l_part, 2);
  __syncthreads();
  float* mw = reinterpret_cast<float*>(smem);              // [nw][8]
  float* lw = mw + nw * kMaxGroup;                         // [nw][8]
  float* aw = lw + nw * kMaxGroup;                         // [nw][8][D]
  if (g < G) {
    if (t4 == 0) {
      mw[warp * kMaxGroup + g] = m_run;
      lw[warp * kMaxGroup + g] = l_part;
    }
#pragma unroll
    for (int nt = 0; nt < C::kNTiles; ++nt) {
      aw[(warp * kMaxGroup + g) * D + nt * 8 + 2 * t4] = o[nt][0];
      aw[(warp * kMaxGroup + g) * D + nt * 8 + 2 * t4 + 1] = o[nt][1];
    }
  }
  __syncthreads();
  float* out = p.part + ((int64_t)unit * p.S + split) * G * (D + 2);
  for (int e = tid; e < G * D; e += blockDim.x) {
    const int h = e / D, i = e % D;
    float M = -INFINITY;
    for (int w = 0; w < nw; ++w) M = fmaxf(M, mw[w * kMaxGroup + h]);
    float a = 0.0f, l = 0.0f;
    if (M != -INFINITY) {
      for (int w = 0; w < nw; ++w) {
        const float f = exp2f(mw[w * kMaxGroup + h] - M);
        a += aw[(w * kMaxGroup + h) * D + i] * f;
        l += lw[w * kMaxGroup + h] * f;
      }
    }
    out[h * (D + 2) + i] = a;
    if (i == 0) {
      out[h * (D + 2) + D] = M;
      out[h * (D + 2) + D + 1] = l;
    }
  }
}

// Merge the S split partials of each (unit, head) and write the output row.
template <typename T, int D, int G>
__global__ void combine_kernel(AttParams p, void* out_v) {
  const int unit = p.unit0 + (int)(blockIdx.x / G);
  const int h = blockIdx.x % G;
  const int i = threadIdx.x;
  const float* base = p.part + (int64_t)unit * p.S * G * (D + 2);
  float M = -INFINITY;
  for (int k = 0; k < p.S; ++k) M = fmaxf(M, base[(k * G + h) * (D + 2) + D]);
  float a = 0.0f, l = 0.0f;
  for (int k = 0; k < p.S; ++k) {
    const float* pk = base + (k * G + h) * (D + 2);
    const float m = pk[D];
    if (m == -INFINITY) continue;
    const float sc = exp2f(m - M);
    a += pk[i] * sc;
    l += pk[D + 1] * sc;
  }
  int64_t orow;
  if (p.kind == kStreamList) {
    orow = unit;  // unit = query token * Hq + head
  } else {
    const int qi = unit / p.Hkv, kvh = unit % p.Hkv;
    orow = (int64_t)qi * p.Hq + (int64_t)kvh * G + h;
  }
  T* out = static_cast<T*>(out_v) + orow * D;
  out[i] = Elem<T>::from_f(l > 0.0f ? a / l : 0.0f);
}

template <typename T, int D, int G>
cudaError_t launch_t(const AttParams& p, int64_t units, void* out, cudaStream_t stream) {
  const int64_t grid = units * p.S;
  cudaError_t e;
  if constexpr (sizeof(T) == 2 && G >= 2) {
    if (p.kind != kStreamList) {
      using M = MmaCfg<D>;
      const size_t smem = (size_t)M::kWarps * M::kWarpBytes + sizeof(uint32_t) * M::kKeptCap;
      auto kern = attend_mma_kernel<D, G>;
      e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e != cudaSuccess) return e;
      kern<<<(unsigned)grid, M::kThreads, smem, stream>>>(p);
      e = cudaGetLastError();
      if (e != cudaSuccess) return e;
      combine_kernel<T, D, G><<<(unsigned)(units * G), D, 0, stream>>>(p, out);
      return cudaGetLastError();
    }
  }
  using C = Cfg<T, D>;
  const size_t smem = D * kMaxGroup * sizeof(float) + (size_t)C::kWarps * C::kWarpBytes;
  auto kern = attend_kernel<T, D, G>;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  kern<<<(unsigned)grid, C::kThreads, smem, stream>>>(p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  combine_kernel<T, D, G><<<(unsigned)(units * G), D, 0, stream>>>(p, out);
  return cudaGetLastError();
}

template <typename T, int D>
cudaError_t launch_g(int G, const AttParams& p, int64_t units, void* out, cudaStream_t s) {
  switch (G) {
    case 1: return launch_t<T, D, 1>(p, units, out, s);
    case 2: return launch_t<T, D, 2>(p, units, out, s);
    case 4: return launch_t<T, D, 4>(p, units, out, s);
    case 8: return launch_t<T, D, 8>(p, units, out, s);
    default: return cudaErrorInvalidValue;
  }
}

int64_t units_of(const Geometry& g, int kind, int64_t nq) {
  return kind == kStreamList ? nq * g.Hq : nq * g.Hkv;
}

int splits_of(const Geometry& g, int kind, int64_t nq, int num_sms) {
  const int64_t units = units_of(g, kind, nq);
  // about two CTAs per SM in total, rounded down so the last wave is full
  int64_t S = (2 * (int64_t)num_sms) / units;
  if (S < 1) S = 1;
  if (S > 256) S = 256;
  return (int)S;
}

}  // namespace

size_t attend_ws_bytes(const Geometry& g, int kind, int64_t nq, int num_sms) {
  const int64_t units = units_of(g, kind, nq);
  const int G = kind == kStreamList ? 1 : g.G;
  const int S = splits_of(g, kind, nq, num_sms);
  return sizeof(float) * (size_t)units * S * G * (g.d + 2) + 256;
}

cudaError_t launch_attend(const Geometry& g, const AttendArgs& a, void* ws, size_t ws_bytes,
                          int num_sms, cudaStream_t stream) {
  (void)ws_bytes;
  AttParams p{};
  p.kind = a.kind;
  p.k = a.k;
  p.v = a.v;
  p.q = a.q;
  p.seq_len = a.seq_len;
  p.q_seq = a.q_seq;
  p.q_pos = a.q_pos;
  p.ncap = g.ncap;
  p.Hq = g.Hq;
  p.Hkv = g.Hkv;
  p.B = g.B;
  p.G = a.kind == kStreamList ? 1 : g.G;
  p.b = g.b;
  p.b_shift = (g.b & (g.b - 1)) == 0 ? __builtin_ctz((unsigned)g.b) : -1;
  p.L = g.L;
  p.span_L = g.span[g.L];
  p.qscale = kLog2e * g.inv_sqrt_d;
  p.kept = a.kept;
  p.n_kept = a.n_kept;
  p.kept_stride = a.kept_stride;
  p.kept_segs = a.kept_segs;
  p.idx = a.idx;
  p.idx_cap = a.idx_cap;
  p.n_idx = a.n_idx;
  p.S = splits_of(g, a.kind, a.nq, num_sms);
  p.part = static_cast<float*>(ws);
  const int64_t all_units = units_of(g, a.kind, a.nq);
  const int64_t units = a.n_units > 0 ? a.n_units : all_units;
  p.unit0 = (int)a.unit0;
  if (units <= 0) return cudaSuccess;
  if (a.unit0 < 0 || a.unit0 + units > all_units) return cudaErrorInvalidValue;
  if (g.dtype == ZHA_BF16) {
    if (g.d == 128) return launch_g<__nv_bfloat16, 128>(p.G, p, units, a.out, stream);
    return launch_g<__nv_bfloat16, 64>(p.G, p, units, a.out, stream);
  }
  if (g.d == 128) return launch_g<float, 128>(p.G, p, units, a.out, stream);
  return launch_g<float, 64>(p.G, p, units, a.out, stream);
}

}  // namespace zha
