// Decode selection with every summary row scored up front.
//
// lefilia.fr page "Zyphra presente Zyphra Hierarchical Attention (ZHA) ...",
// paragraph 1: a query scores the top nodes, keeps the fewest nodes whose
// estimated attention mass reaches the fraction p, and descends only into the
// kept branches, level by level, down to individual keys.
//
// The selection of a decode step is computed here in three launches:
//   1. dense_score_kernel -- every summary row that lies under a complete top
//      node is scored against the G query heads of its KV head, all levels at
//      once: a grid-wide stream over the tree prefix in contiguous tiles, with
//      no dependence between levels. The scores are the canonical ones
//      (sequential fmaf chains, z = fl(fl(dot * 1/sqrt(d)) + l ln b)).
//   2. head_cut_kernel -- one CTA per (sequence, KV head, query head) walks the
//      levels top-down: its frontier at a level is the children of the nodes it
//      kept one level up, and the canonical top-p cut of the frontier (exact
//      fixed-point masses, ties to the lower node) is found from the stored
//      scores with CTA-local passes only, as a threshold (key*, node*) on the
//      frontier's (score desc, node asc) order. The descent is exactly the
//      method's; scores of nodes outside the frontier are computed but never
//      read. Levels L..2 list their kept nodes; level 1 stops at its threshold.
//   3. union_kernel -- many CTAs per (sequence, KV head) apply every head's
//      level-1 threshold to the children of that head's kept level-2 nodes and
//      merge the heads' kept level-1 nodes into one ascending list with an
//      8-bit head mask per node, in the segments the decode attention reads.
// Reading every row under the complete top nodes costs the same bytes as
// reading the union of the heads' frontiers whenever that union covers the
// tree (as on diffuse queries), and it removes the per-level dependence of
// the reads on the cuts. The host uses this path when that prefix is small
// enough (decode_dense_ok) and the frontier traversal otherwise.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "zha_device.cuh"
#include "zha_internal.h"

namespace zha {
namespace {

// ---------------------------------------------------------------------------
// parameters
// ---------------------------------------------------------------------------
struct DenseParams {
  const void* tree;
  int64_t level_off[kMaxLevels];
  int64_t level_rows[kMaxLevels];
  int64_t span[kMaxLevels + 1];
  float lnsize[kMaxLevels];
  float inv_sqrt_d;
  const void* q;           // [B][Hq][D]
  const int32_t* seq_len;  // [B]
  int Hq, Hkv, G, b, L, B;
  int64_t ncap;
  // scores: unit u, head h, level l, node j at z[(u * G + h) * zrows + zoff[l-1] + j]
  float* z;
  int64_t zoff[kMaxLevels];
  int64_t zrows;
  int32_t* stats;          // [units][L] rows scored per level (nullable)
  // cut
  uint64_t p_q;
  int keep_all;
  int32_t* klist;          // [units][G][2][klcap] kept nodes, ascending
  int64_t klcap;
  uint32_t* bitmap;        // [units][G][bmw] kept level-2 nodes (L >= 2)
  int64_t bmw;
  uint4* cutpar;           // [units][G] level-1 cut: mode, key*, node*, kept count
  int32_t* level_counts;   // [B][Hq][L] (nullable)
  int32_t* status;
  // union
  uint32_t* kept;          // [units][segs][stride]
  int32_t* n_kept;         // [units][segs]
  int64_t kept_stride;
  int segs;
  int unit0;               // first unit of this launch (grid y: its units)
  // FP4 router variant (nullable): block-scaled 4-bit summary rows scored in
  // place of the tree's rows (d = 128)
  const unsigned char* fp4_codes;
  const int16_t* fp4_exps;
};

// Complete top nodes visible to the decode query of sequence `seq` (at
// position seq_len - 1), 0 for an invalid sequence.
__device__ __forceinline__ int64_t decode_top(const DenseParams& p, int seq) {
  if (seq < 0 || seq >= p.B) return 0;
  int64_t n = p.seq_len[seq];
  if (n > p.ncap) n = p.ncap;
  if (n < 0) n = 0;
  return n / p.span[p.L];
}

// ---------------------------------------------------------------------------
// 1. scoring: tiles of 512 contiguous rows of one level of one unit; each of
//    the 128 threads runs the G chains of 4 rows (rows t, t+128, t+256, t+384
//    of the tile), three CTAs per SM. Rows are staged 64 bytes (4 chunks) at a time, two stages
//    in flight; a warp's load instruction covers 8 rows x 64 contiguous bytes.
// ---------------------------------------------------------------------------
constexpr int kSThreads = 128;
constexpr int kSTile = 4 * kSThreads;          // rows per tile
constexpr int kSStageBytes = kSTile * 64;      // 4 chunks of every row of a tile

template <typename T, int D>
struct ScoreCfg {
  static constexpr int kPer = Elem<T>::kPerChunk;
  static constexpr int kNch = D * (int)sizeof(T) / 16;
  static constexpr int kSteps = kNch / 4;       // stages per row
  static constexpr int kSmem = 2 * kSStageBytes + D * kMaxGroup * 4;
};
static_assert(kSTile == 128 * (kSThreads / 32), "a warp stages 128 rows of the tile");

// Chunk c (0..3) of staged row r sits at slot c ^ ((r >> 1) & 3) of the row's
// 64 bytes: 8 consecutive rows read by 8 consecutive lanes then cover all 32
// banks.
__device__ __forceinline__ int sswz(int c, int r) { return c ^ ((r >> 1) & 3); }

// Rows of level l (1-based) of unit u scored in this call.
__device__ __forceinline__ int64_t level_prefix_rows(const DenseParams& p, int64_t T_top, int l) {
  return T_top * p.span[p.L - l];
}

template <typename T, int D>
__device__ __forceinline__ void stage_rows(const T* lvl, int64_t r0, int n, int step,
                                           unsigned char* dst) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c = lane & 3;
#pragma unroll 4
  for (int m = 0; m < 16; ++m) {
    const int row = warp * 128 + m * 8 + (lane >> 2);
    if (row < n)
      cp_async16(dst + row * 64 + sswz(c, row) * 16,
                 reinterpret_cast<const uint4*>(lvl + (r0 + row) * D) + 4 * step + c);
  }
}

template <typename T, int D, int G>
__global__ void __launch_bounds__(kSThreads, 3) dense_score_kernel(const __grid_constant__ DenseParams p) {
  using C = ScoreCfg<T, D>;
  constexpr int kPer = C::kPer, kSteps = C::kSteps;
  extern __shared__ __align__(16) unsigned char sm[];
  float* qs = reinterpret_cast<float*>(sm + 2 * kSStageBytes);  // [D][8]
  const int unit = p.unit0 + (int)blockIdx.y;
  const int seq = unit / p.Hkv, kvh = unit % p.Hkv;
  const int tid = threadIdx.x;
  const int64_t T_top = decode_top(p, seq);
  // tiles of this unit, levels from the top down
  int64_t n_tiles = 0;
  for (int l = p.L; l >= 1; --l) n_tiles += (level_prefix_rows(p, T_top, l) + kSTile - 1) / kSTile;
  if (p.stats && blockIdx.x == 0 && tid < p.L)
    p.stats[(int64_t)unit * p.L + tid] = (int32_t)level_prefix_rows(p, T_top, p.L - tid);
  if ((int64_t)blockIdx.x >= n_tiles) return;  // uniform over the CTA
  for (int e = tid; e < D * kMaxGroup; e += kSThreads) {
    const int i = e / kMaxGroup, h = e % kMaxGroup;
    qs[e] = h < G ? Elem<T>::to_f(static_cast<const T*>(p.q)[((int64_t)seq * p.Hq + kvh * G + h) * D + i])
                  : 0.0f;
  }
  // (tile, step) sequence of this CTA: tiles blockIdx.x, + gridDim.x, ...
  auto locate = [&](int64_t tile, int* level, int64_t* r0, int* n) {
    int64_t t = tile;
    for (int l = p.L; l >= 1; --l) {
      const int64_t rows = level_prefix_rows(p, T_top, l);
      const int64_t nt = (rows + kSTile - 1) / kSTile;
      if (t < nt) {
        *level = l;
        *r0 = t * kSTile;
        *n = (int)(rows - *r0 < kSTile ? rows - *r0 : kSTile);
        return;
      }
      t -= nt;
    }
    *level = 0;
    *r0 = 0;
    *n = 0;
  };
  auto lvl_ptr = [&](int level) {
    return static_cast<const T*>(p.tree) + p.level_off[level - 1] +
           (int64_t)unit * p.level_rows[level - 1] * D;
  };
  const int64_t my_tiles = (n_tiles - blockIdx.x + gridDim.x - 1) / gridDim.x;
  const int64_t n_items = my_tiles * kSteps;
  int cur_level, nxt_level;
  int64_t cur_r0, nxt_r0;
  int cur_n, nxt_n;
  locate(blockIdx.x, &cur_level, &cur_r0, &cur_n);
  stage_rows<T, D>(lvl_ptr(cur_level), cur_r0, cur_n, 0, sm);
  cp_async_commit();
  float2 acc[4][(G + 1) / 2];
  float acc1[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    acc1[k] = 0.0f;
#pragma unroll
    for (int j = 0; j < (G + 1) / 2; ++j) acc[k][j] = make_float2(0.0f, 0.0f);
  }
  for (int64_t it = 0; it < n_items; ++it) {
    const int step = (int)(it % kSteps);
    const int64_t tile = blockIdx.x + (it / kSteps) * gridDim.x;
    if (it + 1 < n_items) {  // prefetch the next (tile, step) into the other stage
      const int nstep = (int)((it + 1) % kSteps);
      if (nstep == 0) locate(tile + gridDim.x, &nxt_level, &nxt_r0, &nxt_n);
      else {
        nxt_level = cur_level;
        nxt_r0 = cur_r0;
        nxt_n = cur_n;
      }
      stage_rows<T, D>(lvl_ptr(nxt_level), nxt_r0, nxt_n, nstep, sm + ((it + 1) & 1) * kSStageBytes);
    }
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    const unsigned char* st = sm + (it & 1) * kSStageBytes;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      float x[4][kPer];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int row = tid + k * kSThreads;
        Elem<T>::unpack(lds128(st + row * 64 + sswz(c, row) * 16), x[k]);
      }
#pragma unroll
      for (int e = 0; e < kPer; ++e) {
        const float* qv = qs + ((4 * step + c) * kPer + e) * kMaxGroup;
        if constexpr (G == 1) {
#pragma unroll
          for (int k = 0; k < 4; ++k) acc1[k] = __fmaf_rn(qv[0], x[k][e], acc1[k]);
        } else if constexpr (G == 2) {
          const float2 q2 = *reinterpret_cast<const float2*>(qv);
#pragma unroll
          for (int k = 0; k < 4; ++k) acc[k][0] = ffma2(q2, make_float2(x[k][e], x[k][e]), acc[k][0]);
        } else {
          float4 q4[G / 4];
#pragma unroll
          for (int j = 0; j < G / 4; ++j) q4[j] = *reinterpret_cast<const float4*>(qv + 4 * j);
#pragma unroll
          for (int k = 0; k < 4; ++k) {
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
    if (step == kSteps - 1) {  // the rows' chains are complete: store their scores
      const float lns = p.lnsize[cur_level - 1];
      float* zl = p.z + (int64_t)unit * G * p.zrows + p.zoff[cur_level - 1] + cur_r0;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int row = tid + k * kSThreads;
        if (row < cur_n) {
#pragma unroll
          for (int h = 0; h < G; ++h) {
            const float raw = (G == 1) ? acc1[k] : ((h & 1) ? acc[k][h / 2].y : acc[k][h / 2].x);
            zl[(int64_t)h * p.zrows + row] = __fadd_rn(__fmul_rn(raw, p.inv_sqrt_d), lns);
          }
        }
        acc1[k] = 0.0f;
#pragma unroll
        for (int j = 0; j < (G + 1) / 2; ++j) acc[k][j] = make_float2(0.0f, 0.0f);
      }
    }
    __syncthreads();  // this stage is refilled by the next iteration's prefetch
    if (it + 1 < n_items && (it + 1) % kSteps == 0) {
      cur_level = nxt_level;
      cur_r0 = nxt_r0;
      cur_n = nxt_n;
    }
  }
  cp_async_wait<0>();
}

// ---------------------------------------------------------------------------
// 1b. scoring the FP4 router variant's rows (d = 128): 64 bytes of 4-bit codes
//     per row, one stage per tile, and the row's four block exponents (8
//     bytes, loaded while the codes land). Each code becomes its exact fp32
//     value sign * mag[k] * 2^e (k the e2m1 magnitude index), which enters the
//     same canonical chains as a bf16 or fp32 element would.
// ---------------------------------------------------------------------------

// The two e2m1 codes of byte `byte` (bits 0-7) as exact fp32 values (the
// low nibble in .x), by the sm_100 hardware conversion to f16x2.
__device__ __forceinline__ float2 e2m1x2_to_f2(uint32_t byte) {
  uint32_t h2;
  asm("{\n .reg .b8 t;\n cvt.u8.u32 t, %1;\n cvt.rn.f16x2.e2m1x2 %0, t;\n}" : "=r"(h2) : "r"(byte));
  const __half2 h = *reinterpret_cast<const __half2*>(&h2);
  return __half22float2(h);
}

// The fp32 value of code `nib` times 2^e for any e (exact ldexpf scaling):
// the path of blocks whose scale 2^e is not a normal float.
__device__ __forceinline__ float fp4_value_any(uint32_t nib, int e) {
  const uint32_t k = nib & 7u;
  const float m = k <= 4u ? 0.5f * (float)k : (k == 5u ? 3.0f : (k == 6u ? 4.0f : 6.0f));
  const float v = ldexpf(m, e);
  return k == 0u ? 0.0f : ((nib & 8u) ? -v : v);
}

// One canonical chain step for the 4 rows of a thread: acc_h += q_h[i] * x_k.
template <int G>
__device__ __forceinline__ void chain_step(const float* qv, const float* x, float2 (&acc)[4][(G + 1) / 2],
                                           float (&acc1)[4]) {
  if constexpr (G == 1) {
#pragma unroll
    for (int k = 0; k < 4; ++k) acc1[k] = __fmaf_rn(qv[0], x[k], acc1[k]);
  } else if constexpr (G == 2) {
    const float2 q2 = *reinterpret_cast<const float2*>(qv);
#pragma unroll
    for (int k = 0; k < 4; ++k) acc[k][0] = ffma2(q2, make_float2(x[k], x[k]), acc[k][0]);
  } else {
    float4 q4[G / 4];
#pragma unroll
    for (int jj = 0; jj < G / 4; ++jj) q4[jj] = *reinterpret_cast<const float4*>(qv + 4 * jj);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float2 xx = make_float2(x[k], x[k]);
#pragma unroll
      for (int jj = 0; jj < G / 4; ++jj) {
        acc[k][2 * jj] = ffma2(make_float2(q4[jj].x, q4[jj].y), xx, acc[k][2 * jj]);
        acc[k][2 * jj + 1] = ffma2(make_float2(q4[jj].z, q4[jj].w), xx, acc[k][2 * jj + 1]);
      }
    }
  }
}

__device__ __forceinline__ uint32_t word_of(const uint4& v, int w) {
  return w == 0 ? v.x : (w == 1 ? v.y : (w == 2 ? v.z : v.w));
}

__device__ __forceinline__ void stage_fp4_rows(const unsigned char* lvl, int64_t r0, int n,
                                               unsigned char* dst) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c = lane & 3;
#pragma unroll 4
  for (int m = 0; m < 16; ++m) {
    const int row = warp * 128 + m * 8 + (lane >> 2);
    if (row < n)
      cp_async16(dst + row * 64 + sswz(c, row) * 16,
                 reinterpret_cast<const uint4*>(lvl + (r0 + row) * 64) + c);
  }
}

template <typename T, int G>
__global__ void __launch_bounds__(kSThreads, 3)
    dense_score_fp4_kernel(const __grid_constant__ DenseParams p) {
  constexpr int D = 128;
  extern __shared__ __align__(16) unsigned char sm[];
  float* qs = reinterpret_cast<float*>(sm + 2 * kSStageBytes);  // [D][8]
  const int unit = p.unit0 + (int)blockIdx.y;
  const int seq = unit / p.Hkv, kvh = unit % p.Hkv;
  const int tid = threadIdx.x;
  const int64_t T_top = decode_top(p, seq);
  int64_t n_tiles = 0;
  for (int l = p.L; l >= 1; --l) n_tiles += (level_prefix_rows(p, T_top, l) + kSTile - 1) / kSTile;
  if (p.stats && blockIdx.x == 0 && tid < p.L)
    p.stats[(int64_t)unit * p.L + tid] = (int32_t)level_prefix_rows(p, T_top, p.L - tid);
  if ((int64_t)blockIdx.x >= n_tiles) return;  // uniform over the CTA
  for (int e = tid; e < D * kMaxGroup; e += kSThreads) {
    const int i = e / kMaxGroup, h = e % kMaxGroup;
    qs[e] = h < G ? Elem<T>::to_f(static_cast<const T*>(p.q)[((int64_t)seq * p.Hq + kvh * G + h) * D + i])
                  : 0.0f;
  }
  auto locate = [&](int64_t tile, int* level, int64_t* r0, int* n) {
    int64_t t = tile;
    for (int l = p.L; l >= 1; --l) {
      const int64_t rows = level_prefix_rows(p, T_top, l);
      const int64_t nt = (rows + kSTile - 1) / kSTile;
      if (t < nt) {
        *level = l;
        *r0 = t * kSTile;
        *n = (int)(rows - *r0 < kSTile ? rows - *r0 : kSTile);
        return;
      }
      t -= nt;
    }
    *level = 0;
    *r0 = 0;
    *n = 0;
  };
  // element offset of the unit's level `level` in the tree's element order
  auto elem0 = [&](int level) {
    return p.level_off[level - 1] + (int64_t)unit * p.level_rows[level - 1] * D;
  };
  const int64_t my_tiles = (n_tiles - blockIdx.x + gridDim.x - 1) / gridDim.x;
  int cur_level;
  int64_t cur_r0;
  int cur_n;
  locate(blockIdx.x, &cur_level, &cur_r0, &cur_n);
  stage_fp4_rows(p.fp4_codes + elem0(cur_level) / 2, cur_r0, cur_n, sm);
  cp_async_commit();
  for (int64_t it = 0; it < my_tiles; ++it) {
    const int64_t tile = blockIdx.x + it * gridDim.x;
    int nxt_level = 0;
    int64_t nxt_r0 = 0;
    int nxt_n = 0;
    if (it + 1 < my_tiles) {  // prefetch the next tile into the other stage
      locate(tile + gridDim.x, &nxt_level, &nxt_r0, &nxt_n);
      stage_fp4_rows(p.fp4_codes + elem0(nxt_level) / 2, nxt_r0, nxt_n,
                     sm + ((it + 1) & 1) * kSStageBytes);
    }
    cp_async_commit();
    uint2 ex[4];  // the 4 block exponents of each of the thread's rows
    {
      const int16_t* el = p.fp4_exps + elem0(cur_level) / 32;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int row = tid + k * kSThreads;
        ex[k] = row < cur_n ? __ldg(reinterpret_cast<const uint2*>(el + (cur_r0 + row) * 4))
                            : make_uint2(0u, 0u);
      }
    }
    cp_async_wait<1>();
    __syncthreads();
    const unsigned char* st = sm + (it & 1) * kSStageBytes;
    float2 acc[4][(G + 1) / 2];
    float acc1[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      acc1[k] = 0.0f;
#pragma unroll
      for (int j = 0; j < (G + 1) / 2; ++j) acc[k][j] = make_float2(0.0f, 0.0f);
    }
#pragma unroll 1
    for (int c = 0; c < 4; ++c) {  // block c: elements 32c .. 32c + 31
      uint4 cw[4];
      int eb[4];
      float sc[4];
      bool fast = true;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int row = tid + k * kSThreads;
        cw[k] = lds128(st + row * 64 + sswz(c, row) * 16);
        const uint32_t pair = c < 2 ? ex[k].x : ex[k].y;
        eb[k] = (int)(int16_t)((c & 1) ? (pair >> 16) : (pair & 0xffffu));
        fast = fast && eb[k] >= -126 && eb[k] <= 127;
        sc[k] = __int_as_float((eb[k] + 127) << 23);  // 2^e while it is a normal float
      }
      if (fast) {  // value = e2m1 value * 2^e, an exact product
#pragma unroll
        for (int w = 0; w < 4; ++w)
#pragma unroll
          for (int jb = 0; jb < 4; ++jb) {
            float x0[4], x1[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const float2 v = e2m1x2_to_f2((word_of(cw[k], w) >> (8 * jb)) & 0xffu);
              x0[k] = __fmul_rn(v.x, sc[k]);
              x1[k] = __fmul_rn(v.y, sc[k]);
            }
            const int i = 32 * c + 8 * w + 2 * jb;
            chain_step<G>(qs + i * kMaxGroup, x0, acc, acc1);
            chain_step<G>(qs + (i + 1) * kMaxGroup, x1, acc, acc1);
          }
      } else {
#pragma unroll 1
        for (int j = 0; j < 32; ++j) {
          float x[4];
#pragma unroll
          for (int k = 0; k < 4; ++k)
            x[k] = fp4_value_any((word_of(cw[k], j >> 3) >> (4 * (j & 7))) & 15u, eb[k]);
          chain_step<G>(qs + (32 * c + j) * kMaxGroup, x, acc, acc1);
        }
      }
    }
    {  // the rows' chains are complete: store their scores
      const float lns = p.lnsize[cur_level - 1];
      float* zl = p.z + (int64_t)unit * G * p.zrows + p.zoff[cur_level - 1] + cur_r0;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int row = tid + k * kSThreads;
        if (row < cur_n) {
#pragma unroll
          for (int h = 0; h < G; ++h) {
            const float raw = (G == 1) ? acc1[k] : ((h & 1) ? acc[k][h / 2].y : acc[k][h / 2].x);
            zl[(int64_t)h * p.zrows + row] = __fadd_rn(__fmul_rn(raw, p.inv_sqrt_d), lns);
          }
        }
      }
    }
    __syncthreads();  // this stage is refilled by the next iteration's prefetch
    cur_level = nxt_level;
    cur_r0 = nxt_r0;
    cur_n = nxt_n;
  }
  cp_async_wait<0>();
}

// ---------------------------------------------------------------------------
// 2. the cut chain of one query head
//
// Per level, with zmax / zmin the score extremes of the head's frontier:
//   M_i = trunc(exp(z_i - zmax) 2^40), T = sum M_i, need = ceil(T p_q / 2^32),
// and the kept set is the shortest prefix of (z desc, node asc) whose mass
// reaches need. It is found as a threshold (key*, node*) on the order key of
// z: the masses are histogrammed over 256 linear score buckets (exact
// sums), the bucket where the mass crosses need is narrowed by 8-bit key
// digits while it holds more than kCList candidates, and its members are then
// ranked; a group that narrows to one key with more than kCList members (all
// with one mass) is resolved by node order.
//
// Frontiers of at most kZCap candidates live in shared memory (score and node
// of every candidate), filled in one batched round of loads from the kept
// nodes of the level above. Larger frontiers are streamed: the frontier is
// walked in ITEMS of up to 4 consecutive candidates (children 4q..4q+3 of the
// j-th kept parent, or top nodes 4i..4i+3), a thread taking U consecutive
// items per iteration and issuing all their loads before using any.
// ---------------------------------------------------------------------------
constexpr int kCThreads = 512;
constexpr int kCWarps = kCThreads / 32;
constexpr int kCBuckets = 256;
constexpr int kCCopies = 16;  // histogram copies (lane % 16)
constexpr int kCList = 1024;  // groups this small are ranked directly
// largest U: 2 items (8 candidates) per thread and iteration. Larger U
// batches more loads, but the unrolled per-slot code of every pass grows with
// it; measured at the headline, U <= 2 gave the fastest cut (U <= 4 cost
// 20 us per step, U <= 3 10 us, U <= 1 the same as 2).
constexpr int kCU = 2;
constexpr int kZCap = 8192;   // frontier candidates held in shared memory
constexpr int kKCap = 16384;  // kept nodes held in shared memory

struct CutSmem {
  // histogram copies, bucket-major: mass low / high words and counts
  unsigned int hlo[kCBuckets][kCCopies];
  unsigned int hhi[kCBuckets][kCCopies];
  unsigned int hc[kCBuckets][kCCopies];
  unsigned long long bm[kCBuckets];   // reduced bucket masses
  unsigned int bc[kCBuckets];         // reduced bucket counts
  unsigned long long list[kCList];    // group members: (key << 32) | ~node
  unsigned long long srt[kCList];     // the members sorted (descending)
  unsigned long long mr[kCList];      // their masses in that order
  float zc[kZCap];                    // small frontier: scores
  int32_t nc[kZCap];                  // ... and nodes
  int32_t ks[kKCap];                  // kept nodes of the last level (ascending)
  unsigned int n_list;
  float red_f[kCWarps][2];
  unsigned int red_u[kCWarps][2];
  unsigned long long red_m[kCWarps];
  float zmax, zmin;
  unsigned long long above, need, bmass;
  unsigned int cabove, bcnt, beta, kgmin, kgmax, mode, count;
  unsigned int thr_key, thr_node, tie_n, rank_hit;
  int ok;
};
// the head's level-2 kept bitmap follows the struct (bmw words)

enum CutMode : unsigned { kCutAll = 0, kCutThr = 1, kCutTie = 2 };

// Block reduction of a float pair (max of a, min of b).
__device__ __forceinline__ void block_minmax(CutSmem& S, float a, float b, float* mx, float* mn) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, off));
    b = fminf(b, __shfl_xor_sync(0xffffffffu, b, off));
  }
  if (lane == 0) {
    S.red_f[warp][0] = a;
    S.red_f[warp][1] = b;
  }
  __syncthreads();
  float x = -INFINITY, y = INFINITY;
#pragma unroll
  for (int w = 0; w < kCWarps; ++w) {
    x = fmaxf(x, S.red_f[w][0]);
    y = fminf(y, S.red_f[w][1]);
  }
  *mx = x;
  *mn = y;
  __syncthreads();
}

// Exclusive scan of v over the CTA (thread order); *total gets the sum.
__device__ __forceinline__ unsigned block_scan(CutSmem& S, unsigned v, unsigned* total, int slot) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  unsigned x = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const unsigned y = __shfl_up_sync(0xffffffffu, x, off);
    if (lane >= off) x += y;
  }
  if (lane == 31) S.red_u[warp][slot] = x;
  __syncthreads();
  unsigned base = 0, tot = 0;
#pragma unroll
  for (int w = 0; w < kCWarps; ++w) {
    const unsigned s = S.red_u[w][slot];
    if (w < warp) base += s;
    tot += s;
  }
  __syncthreads();
  *total = tot;
  return base + x - v;
}

__device__ __forceinline__ void hist_clear(CutSmem& S) {
  for (int e = threadIdx.x; e < kCBuckets * kCCopies; e += kCThreads) {
    (&S.hlo[0][0])[e] = 0u;
    (&S.hhi[0][0])[e] = 0u;
    (&S.hc[0][0])[e] = 0u;
  }
}

// Adds mass m (< 2^40) and one member to bucket d: the low word with its
// carry into the high word (32-bit shared-memory atomics).
__device__ __forceinline__ void hist_add(CutSmem& S, uint32_t d, unsigned long long m) {
  const int cp = threadIdx.x & (kCCopies - 1);
  const unsigned lo = (unsigned)m;
  const unsigned old = atomicAdd(&S.hlo[d][cp], lo);
  const unsigned hi = (unsigned)(m >> 32) + (old + lo < old ? 1u : 0u);
  if (hi) atomicAdd(&S.hhi[d][cp], hi);
  atomicAdd(&S.hc[d][cp], 1u);
}

// The same for a pass that needs no counts (the first one of a level).
__device__ __forceinline__ void hist_add_mass(CutSmem& S, uint32_t d, unsigned long long m) {
  const int cp = threadIdx.x & (kCCopies - 1);
  const unsigned lo = (unsigned)m;
  const unsigned old = atomicAdd(&S.hlo[d][cp], lo);
  const unsigned hi = (unsigned)(m >> 32) + (old + lo < old ? 1u : 0u);
  if (hi) atomicAdd(&S.hhi[d][cp], hi);
}

// Sums the copies of every bucket into S.bm / S.bc: thread t sums 8 copies of
// bucket t / 2 (starting at a copy that depends on the bucket, so that a
// warp's reads spread over the banks) and the thread pair combines.
__device__ __forceinline__ void hist_reduce(CutSmem& S) {
  const int t = threadIdx.x;
  const int d = t >> 1, half = t & 1;
  unsigned long long m = 0;
  unsigned int c = 0;
#pragma unroll
  for (int i = 0; i < kCCopies / 2; ++i) {
    const int cp = (kCCopies / 2) * half + ((i + d) & (kCCopies / 2 - 1));
    m += ((unsigned long long)S.hhi[d][cp] << 32) + S.hlo[d][cp];
    c += S.hc[d][cp];
  }
  m += __shfl_xor_sync(0xffffffffu, m, 1);
  c += __shfl_xor_sync(0xffffffffu, c, 1);
  if (!half) {
    S.bm[d] = m;
    S.bc[d] = c;
  }
  __syncthreads();
}

// Warp 0: the bucket (of nb, higher first) where the mass taken in descending
// order reaches `need`, given the mass `above` ranked before all buckets.
// Returns false if no bucket crosses (cannot happen with exact sums).
__device__ __forceinline__ bool find_crossing(const CutSmem& S, int nb, unsigned long long above,
                                              unsigned long long need, unsigned* beta,
                                              unsigned long long* b_above, unsigned* c_above) {
  const int lane = threadIdx.x & 31;
  constexpr int kPer = kCBuckets / 32;
  unsigned long long m[kPer], tm = 0;
  unsigned c[kPer], tc = 0;
#pragma unroll
  for (int j = 0; j < kPer; ++j) {
    const int d = lane * kPer + j;
    m[j] = d < nb ? S.bm[d] : 0ull;
    c[j] = d < nb ? S.bc[d] : 0u;
    tm += m[j];
    tc += c[j];
  }
  unsigned long long xs = tm;
  unsigned xc = tc;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {  // inclusive suffix sums over lanes
    const unsigned long long ym = __shfl_down_sync(0xffffffffu, xs, off);
    const unsigned yc = __shfl_down_sync(0xffffffffu, xc, off);
    if (lane + off < 32) {
      xs += ym;
      xc += yc;
    }
  }
  unsigned long long run = above + (xs - tm);
  unsigned runc = xc - tc;
  int f = -1;
  unsigned long long fa = 0;
  unsigned fc = 0;
#pragma unroll
  for (int j = kPer - 1; j >= 0; --j) {
    const int d = lane * kPer + j;
    if (d < nb && run < need && run + m[j] >= need) {
      f = d;
      fa = run;
      fc = runc;
    }
    run += m[j];
    runc += c[j];
  }
  const unsigned fm = __ballot_sync(0xffffffffu, f >= 0);
  if (!fm) return false;
  const int src = __ffs(fm) - 1;
  *beta = (unsigned)__shfl_sync(0xffffffffu, f, src);
  *b_above = __shfl_sync(0xffffffffu, fa, src);
  *c_above = __shfl_sync(0xffffffffu, fc, src);
  return true;
}

// Scores of nodes node0 .. node0+3 (node0 even; rows past the level's end are
// padding and are never used).
__device__ __forceinline__ float4 load_z4(const float* zl, int64_t node0) {
  if ((node0 & 3) == 0) return __ldcg(reinterpret_cast<const float4*>(zl + node0));
  const float2 v = __ldcg(reinterpret_cast<const float2*>(zl + node0));
  return make_float4(v.x, v.y, 0.0f, 0.0f);
}

__device__ __forceinline__ float f4get(const float4& v, int c) {
  return c == 0 ? v.x : c == 1 ? v.y : c == 2 ? v.z : v.w;
}

// One level of the head's descent as seen by the passes.
struct Frontier {
  bool cached;          // candidates in S.zc / S.nc
  bool top;             // streamed top level: node = candidate index
  int b, nq, U;         // children per parent, items per parent, items per thread
  int64_t nF, nItems, T_top;
  const int32_t* kin;   // streamed, below the top: kept parents (shared or global)
  const float* zl;      // scores of the level
};

// The candidates of this thread in one iteration, in frontier order: slot s
// holds score z[s] and node nd[s]; bit s of `valid` marks slots in use. A
// cached frontier gives each thread up to 4 U consecutive candidates, a
// streamed one U consecutive items (4 slots each); every load is issued
// before any is used.
struct Slots {
  float z[4 * kCU];
  uint32_t nd[4 * kCU];  // node ids fit in 24 bits
  uint32_t valid;
};

__device__ __forceinline__ void load_slots(const CutSmem& S, const Frontier& V, int64_t base,
                                           Slots& q) {
  const int tid = threadIdx.x;
  q.valid = 0;
  if (V.cached) {
    const int64_t k0 = base * 4 + (int64_t)tid * 4 * V.U;
#pragma unroll
    for (int s = 0; s < 4 * kCU; ++s) {
      const int64_t k = k0 + s;
      const bool in = s < 4 * V.U && k < V.nF;
      q.z[s] = in ? S.zc[k] : 0.0f;
      q.nd[s] = in ? (uint32_t)S.nc[k] : 0u;
      q.valid |= (in ? 1u : 0u) << s;
    }
    return;
  }
  const int64_t i0 = base + (int64_t)tid * V.U;
  uint32_t n0[kCU];
  int cnt[kCU];
#pragma unroll
  for (int u = 0; u < kCU; ++u) {
    const int64_t i = i0 + u;
    const bool in = u < V.U && i < V.nItems;
    cnt[u] = 0;
    n0[u] = 0;
    if (in) {
      if (V.top) {
        n0[u] = (uint32_t)(4 * i);
        const int64_t r = V.T_top - 4 * i;
        cnt[u] = r < 4 ? (int)r : 4;
      } else {
        const int64_t j = i / V.nq;
        const int qq = (int)(i - j * V.nq);
        n0[u] = (uint32_t)V.kin[j] * (uint32_t)V.b + 4u * (uint32_t)qq;
        const int r = V.b - 4 * qq;
        cnt[u] = r < 4 ? r : 4;
      }
    }
  }
  float4 zz[kCU];
#pragma unroll
  for (int u = 0; u < kCU; ++u) zz[u] = cnt[u] ? load_z4(V.zl, n0[u]) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
  for (int u = 0; u < kCU; ++u)
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      q.z[4 * u + c] = f4get(zz[u], c);
      q.nd[4 * u + c] = n0[u] + c;
      q.valid |= (c < cnt[u] ? 1u : 0u) << (4 * u + c);
    }
}

// The first node and candidate count of items i0 .. i0 + U - 1 of a streamed
// frontier (count 0 past the end).
__device__ __forceinline__ void load_item_nodes(const Frontier& V, int64_t i0, uint32_t* n0, int* cnt) {
#pragma unroll
  for (int u = 0; u < kCU; ++u) {
    const int64_t i = i0 + u;
    cnt[u] = 0;
    n0[u] = 0;
    if (u < V.U && i < V.nItems) {
      if (V.top) {
        n0[u] = (uint32_t)(4 * i);
        const int64_t r = V.T_top - 4 * i;
        cnt[u] = r < 4 ? (int)r : 4;
      } else {
        const int64_t j = i / V.nq;
        const int qq = (int)(i - j * V.nq);
        n0[u] = (uint32_t)V.kin[j] * (uint32_t)V.b + 4u * (uint32_t)qq;
        const int r = V.b - 4 * qq;
        cnt[u] = r < 4 ? r : 4;
      }
    }
  }
}

// Ranks the n entries of S.list (all distinct), leaving them sorted
// descending in S.srt with their masses in S.mr, scans the masses and finds
// the rank where the mass taken after `above` reaches `need`: S.rank_hit,
// 0xffffffff if never.
__device__ void rank_group(CutSmem& S, int n, float zmax, unsigned long long above,
                           unsigned long long need) {
  const int tid = threadIdx.x, lane = tid & 31;
  for (int i = tid; i < n; i += kCThreads) {
    const unsigned long long e = S.list[i];
    unsigned r = 0;
    for (int j = 0; j < n; ++j) r += S.list[j] > e ? 1u : 0u;
    S.srt[r] = e;
    S.mr[r] = mass_fixed(key_float((uint32_t)(e >> 32)), zmax);
  }
  __syncthreads();
  const int r0 = 2 * tid;  // thread t owns ranks 2t, 2t + 1
  const unsigned long long m0 = r0 < n ? S.mr[r0] : 0ull;
  const unsigned long long m1 = r0 + 1 < n ? S.mr[r0 + 1] : 0ull;
  unsigned long long x = m0 + m1;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const unsigned long long y = __shfl_up_sync(0xffffffffu, x, off);
    if (lane >= off) x += y;
  }
  if (lane == 31) S.red_m[tid >> 5] = x;
  if (tid == 0) S.rank_hit = 0xffffffffu;
  __syncthreads();
  unsigned long long run = 0;
  for (int w = 0; w < (tid >> 5); ++w) run += S.red_m[w];
  run += x - (m0 + m1);
  const unsigned long long rem = need - above;  // > 0
  if (r0 < n && run < rem && run + m0 >= rem) S.rank_hit = (unsigned)r0;
  if (r0 + 1 < n && run + m0 < rem && run + m0 + m1 >= rem) S.rank_hit = (unsigned)r0 + 1u;
  __syncthreads();
}

// The candidates of one iteration (as load_slots gives them) with their keep
// bits -- key > key*, or key == key* and node <= node*; every candidate in
// kCutAll -- and their exact-tie bits (key == key*). by_bytes: every candidate
// outside the crossing bucket beta is decided by its bucket byte, and scores
// are loaded only for the items that hold members of beta.
__device__ __forceinline__ void classify(const CutSmem& S, const Frontier& V, int64_t base,
                                         bool by_bytes, const uint32_t* qbw, unsigned mode,
                                         uint32_t thr_key, uint32_t thr_node, uint32_t beta,
                                         Slots& q, uint32_t* keepm, uint32_t* tiem) {
  uint32_t km = 0, tm = 0;
  if (by_bytes) {
    const int64_t i0 = base + (int64_t)threadIdx.x * V.U;
    uint32_t n0[kCU];
    int cnt[kCU];
    uint32_t qw[kCU];
    load_item_nodes(V, i0, n0, cnt);
#pragma unroll
    for (int u = 0; u < kCU; ++u) qw[u] = cnt[u] ? qbw[i0 + u] : 0u;
    const uint32_t bpat = beta * 0x01010101u;
    float4 zz[kCU];
#pragma unroll
    for (int u = 0; u < kCU; ++u)
      zz[u] = (cnt[u] && __vcmpeq4(qw[u], bpat)) ? load_z4(V.zl, n0[u])
                                                 : make_float4(0.f, 0.f, 0.f, 0.f);
    q.valid = 0;
#pragma unroll
    for (int u = 0; u < kCU; ++u)
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int sl = 4 * u + c;
        q.nd[sl] = n0[u] + c;
        if (c >= cnt[u]) continue;
        q.valid |= 1u << sl;
        const uint32_t d = (qw[u] >> (8 * c)) & 0xffu;
        if (d > beta) {
          km |= 1u << sl;
        } else if (d == beta) {
          const uint32_t key = order_key(f4get(zz[u], c));
          const bool gt = key > thr_key, eq = key == thr_key;
          km |= (gt || (eq && mode == kCutThr && q.nd[sl] <= thr_node) ? 1u : 0u) << sl;
          tm |= (eq ? 1u : 0u) << sl;
        }
      }
  } else {
    load_slots(S, V, base, q);
#pragma unroll
    for (int sl = 0; sl < 4 * kCU; ++sl) {
      if (!((q.valid >> sl) & 1u)) continue;
      const uint32_t key = order_key(q.z[sl]);
      const bool gt = key > thr_key, eq = key == thr_key;
      km |= (mode == kCutAll || gt || (eq && mode == kCutThr && q.nd[sl] <= thr_node) ? 1u : 0u)
            << sl;
      tm |= (eq ? 1u : 0u) << sl;
    }
  }
  *keepm = km;
  *tiem = tm;
}

__global__ void __launch_bounds__(kCThreads, 1) head_cut_kernel(const __grid_constant__ DenseParams p) {
  extern __shared__ __align__(16) unsigned char smc[];
  CutSmem& S = *reinterpret_cast<CutSmem*>(smc);
  uint32_t* bm2 = reinterpret_cast<uint32_t*>(smc + ((sizeof(CutSmem) + 15) & ~(size_t)15));
  const int h = blockIdx.x, unit = p.unit0 + (int)blockIdx.y;
  const int G = p.G, b = p.b, L = p.L;
  const int seq = unit / p.Hkv, kvh = unit % p.Hkv;
  const int tid = threadIdx.x;
  const int64_t T_top = decode_top(p, seq);
  // level-2 nodes under complete top nodes, kept ones as bits
  const int64_t words2 = L >= 2 ? (T_top * p.span[L - 2] + 31) / 32 : 0;
  int32_t* lc = p.level_counts && seq >= 0 && seq < p.B
                    ? p.level_counts + ((int64_t)seq * p.Hq + (int64_t)kvh * G + h) * L
                    : nullptr;
  uint32_t* gbm = p.bitmap + ((int64_t)unit * G + h) * p.bmw;
  for (int64_t w = tid; w < words2; w += kCThreads) bm2[w] = 0u;
  if (T_top == 0) {
    if (lc && tid < L) lc[tid] = 0;
    if (tid == 0) p.cutpar[(int64_t)unit * G + h] = make_uint4(kCutAll, 0u, 0u, 0u);
    return;
  }
  // kept nodes in global memory, two buffers: a streamed level reads its
  // parents from one while it writes its kept nodes to the other
  int32_t* kgb = p.klist + ((int64_t)unit * G + h) * 2 * p.klcap;
  int gsel = 0;
  const float* zh = p.z + ((int64_t)unit * G + h) * p.zrows;
  // the top level: cached when small enough
  bool cached = T_top <= kZCap;
  {
    const float* zt = zh + p.zoff[L - 1];
    float mx = -INFINITY, mn = INFINITY;
    for (int64_t k = tid; k < T_top; k += kCThreads) {
      const float zz = __ldcg(zt + k);
      if (cached) {
        S.zc[k] = zz;
        S.nc[k] = (int32_t)k;
      }
      mx = fmaxf(mx, zz);
      mn = fminf(mn, zz);
    }
    float zmax, zmin;
    block_minmax(S, mx, mn, &zmax, &zmin);
    if (tid == 0) {
      S.zmax = zmax;
      S.zmin = zmin;
    }
  }
  int64_t nF = T_top, n_prev = 0;
  __syncthreads();
  for (int level = L; level >= 1; --level) {
    Frontier V;
    V.cached = cached;
    V.top = level == L;
    V.b = b;
    V.nq = (b + 3) / 4;
    V.T_top = T_top;
    V.nF = nF;
    V.nItems = cached ? (nF + 3) / 4 : (V.top ? (T_top + 3) / 4 : n_prev * V.nq);
    {
      const int64_t per = (V.nItems + kCThreads - 1) / kCThreads;
      V.U = per < 1 ? 1 : (per > kCU ? kCU : (int)per);
    }
    const int64_t stride = (int64_t)kCThreads * V.U;  // items per iteration
    V.kin = n_prev <= kKCap ? S.ks : kgb + (int64_t)gsel * p.klcap;
    int32_t* kg_out = kgb + (int64_t)(gsel ^ 1) * p.klcap;
    V.zl = zh + p.zoff[level - 1];
    // a streamed frontier keeps each candidate's first-pass bucket byte in the
    // shared memory the cached frontier uses (slot 4 i + c of item i)
    const bool qb_ok = !cached && 4 * V.nItems <= (int64_t)sizeof(S.zc) + (int64_t)sizeof(S.nc);
    uint32_t* qbw = reinterpret_cast<uint32_t*>(S.zc);
    float zmax = S.zmax, zmin = S.zmin;
    __syncthreads();  // every thread has read the extremes before they are rewritten
    if (!cached && !V.top && !p.keep_all) {  // streamed: extremes of this frontier
      float mx = -INFINITY, mn = INFINITY;
      for (int64_t base = 0; base < V.nItems; base += stride) {
        Slots q;
        load_slots(S, V, base, q);
#pragma unroll
        for (int sl = 0; sl < 4 * kCU; ++sl)
          if ((q.valid >> sl) & 1u) {
            mx = fmaxf(mx, q.z[sl]);
            mn = fminf(mn, q.z[sl]);
          }
      }
      block_minmax(S, mx, mn, &zmax, &zmin);
    }
    if (tid == 0) {
      S.mode = kCutAll;
      S.ok = 1;
      S.n_list = 0u;
      S.kgmin = 0u;
      S.kgmax = 0xffffffffu;
      S.bcnt = 0u;
    }
    __syncthreads();
    const float zlo = fmaxf(zmin, __fsub_rn(zmax, 32.0f));
    const float zscale = zmax > zlo ? __fdiv_rn(256.0f, __fsub_rn(zmax, zlo)) : 0.0f;
    if (!p.keep_all) {
      // -- exact masses per linear score bucket (bucket bytes kept when streamed) --
      hist_clear(S);
      __syncthreads();
      for (int64_t base = 0; base < V.nItems; base += stride) {
        Slots q;
        load_slots(S, V, base, q);
        uint32_t word[kCU];
#pragma unroll
        for (int u = 0; u < kCU; ++u) word[u] = 0u;
#pragma unroll
        for (int sl = 0; sl < 4 * kCU; ++sl)
          if ((q.valid >> sl) & 1u) {
            const uint32_t d = quant_bucket(q.z[sl], zlo, zscale);
            hist_add_mass(S, d, mass_fixed(q.z[sl], zmax));
            word[sl >> 2] |= d << (8 * (sl & 3));
          }
        if (qb_ok) {
          const int64_t i0 = base + (int64_t)tid * V.U;
#pragma unroll
          for (int u = 0; u < kCU; ++u)
            if (u < V.U && i0 + u < V.nItems) qbw[i0 + u] = word[u];
        }
      }
      __syncthreads();
      hist_reduce(S);
      if (tid < 32) {
        const int lane = tid;
        unsigned long long tot = 0;
        for (int d = lane; d < kCBuckets; d += 32) tot += S.bm[d];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) tot += __shfl_xor_sync(0xffffffffu, tot, off);
        const unsigned long long need = ceil_mul_shift32(tot, p.p_q);
        unsigned beta = 0;
        unsigned long long ab = 0;
        unsigned ca = 0;
        const bool ok = find_crossing(S, kCBuckets, 0ull, need, &beta, &ab, &ca);
        if (lane == 0) {
          S.need = need;
          S.ok = ok;
          S.beta = beta;
          S.above = ab;
          S.cabove = 0u;  // counted by the gather below (this pass counts no members)
          S.bmass = ok ? S.bm[beta] : 0ull;
        }
      }
      __syncthreads();
      // -- the crossing bucket's members into the list (counted past its end),
      //    and the count of the candidates in the buckets above it --
      if (S.ok) {
        const unsigned beta = S.beta;
        unsigned n_above = 0;
        if (qb_ok) {  // from the bucket bytes; scores only for the members
          const uint32_t bpat = beta * 0x01010101u;
          for (int64_t base = 0; base < V.nItems; base += stride) {
            const int64_t i0 = base + (int64_t)tid * V.U;
            uint32_t n0[kCU];
            int cnt[kCU];
            uint32_t eqm[kCU];
            bool anym = false;
#pragma unroll
            for (int u = 0; u < kCU; ++u) {
              const bool in = u < V.U && i0 + u < V.nItems;
              const uint32_t w = in ? qbw[i0 + u] : 0u;  // absent candidates hold byte 0
              eqm[u] = in ? __vcmpeq4(w, bpat) : 0u;
              n_above += (unsigned)__popc(__vcmpgtu4(w, bpat)) >> 3;
              anym |= eqm[u] != 0u;
            }
            if (!anym) continue;
            load_item_nodes(V, i0, n0, cnt);
            float4 zz[kCU];
#pragma unroll
            for (int u = 0; u < kCU; ++u)
              zz[u] = (eqm[u] && cnt[u]) ? load_z4(V.zl, n0[u]) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int u = 0; u < kCU; ++u)
#pragma unroll
              for (int c = 0; c < 4; ++c)
                if (c < cnt[u] && ((eqm[u] >> (8 * c)) & 1u)) {
                  const unsigned slot = atomicAdd(&S.n_list, 1u);
                  if (slot < (unsigned)kCList)
                    S.list[slot] = ((unsigned long long)order_key(f4get(zz[u], c)) << 32) |
                                   (0xffffffffu - (n0[u] + c));
                }
          }
        } else {
          for (int64_t base = 0; base < V.nItems; base += stride) {
            Slots q;
            load_slots(S, V, base, q);
#pragma unroll
            for (int sl = 0; sl < 4 * kCU; ++sl) {
              if (!((q.valid >> sl) & 1u)) continue;
              const uint32_t d = quant_bucket(q.z[sl], zlo, zscale);
              n_above += d > beta ? 1u : 0u;
              if (d != beta) continue;
              const unsigned slot = atomicAdd(&S.n_list, 1u);
              if (slot < (unsigned)kCList)
                S.list[slot] = ((unsigned long long)order_key(q.z[sl]) << 32) | (0xffffffffu - q.nd[sl]);
            }
          }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) n_above += __shfl_xor_sync(0xffffffffu, n_above, off);
        if ((tid & 31) == 0 && n_above) atomicAdd(&S.cabove, n_above);
      }
      __syncthreads();
      // -- a group too large to rank: narrow it by key digits, then gather again --
      if (S.ok && S.n_list > (unsigned)kCList) {
        if (tid == 0) {
          S.bcnt = S.n_list;
          if (zscale == 0.0f) {
            S.kgmin = S.kgmax = order_key(zlo);
          } else {
            uint32_t a0, a1;
            quant_interval(zlo, zscale, S.beta, &a0, &a1);
            S.kgmin = a0;
            S.kgmax = a1;
          }
        }
        __syncthreads();
        for (int pass = 0; pass < 4 && S.ok && S.bcnt > (unsigned)kCList && S.kgmin < S.kgmax; ++pass) {
          const unsigned beta = S.beta, kgmin = S.kgmin, kgmax = S.kgmax;
          int sh, w;
          radix_digit(kgmin, kgmax, &sh, &w);
          hist_clear(S);
          __syncthreads();
          for (int64_t base = 0; base < V.nItems; base += stride) {
            Slots q;
            load_slots(S, V, base, q);
#pragma unroll
            for (int sl = 0; sl < 4 * kCU; ++sl) {
              if (!((q.valid >> sl) & 1u) || quant_bucket(q.z[sl], zlo, zscale) != beta) continue;
              const uint32_t key = order_key(q.z[sl]);
              if (key < kgmin || key > kgmax) continue;
              hist_add(S, (key >> sh) & ((1u << w) - 1u), mass_fixed(q.z[sl], zmax));
            }
          }
          __syncthreads();
          hist_reduce(S);
          if (tid < 32) {
            unsigned dig = 0;
            unsigned long long ab = 0;
            unsigned ca = 0;
            const bool ok = find_crossing(S, 1 << w, S.above, S.need, &dig, &ab, &ca);
            if (tid == 0) {
              S.ok = ok;
              if (ok) {
                const uint32_t topb = (uint32_t)(((unsigned long long)kgmin >> (sh + w)) << (sh + w));
                const uint32_t dlo = topb | (dig << sh);
                const uint32_t dhi = dlo | (uint32_t)((1ull << sh) - 1ull);
                S.above = ab;
                S.cabove += ca;
                S.bcnt = S.bc[dig];
                S.bmass = S.bm[dig];
                S.kgmin = dlo > kgmin ? dlo : kgmin;
                S.kgmax = dhi < kgmax ? dhi : kgmax;
              }
            }
          }
          __syncthreads();
        }
        if (S.ok && S.bcnt <= (unsigned)kCList) {
          const unsigned beta = S.beta, kgmin = S.kgmin, kgmax = S.kgmax;
          if (tid == 0) S.n_list = 0u;
          __syncthreads();
          for (int64_t base = 0; base < V.nItems; base += stride) {
            Slots q;
            load_slots(S, V, base, q);
#pragma unroll
            for (int sl = 0; sl < 4 * kCU; ++sl) {
              if (!((q.valid >> sl) & 1u) || quant_bucket(q.z[sl], zlo, zscale) != beta) continue;
              const uint32_t key = order_key(q.z[sl]);
              if (key < kgmin || key > kgmax) continue;
              const unsigned slot = atomicAdd(&S.n_list, 1u);
              if (slot < (unsigned)kCList)
                S.list[slot] = ((unsigned long long)key << 32) | (0xffffffffu - q.nd[sl]);
            }
          }
          __syncthreads();
        }
      }
      // -- resolve the group: rank its members, or take exact ties in node order --
      if (S.ok && S.n_list <= (unsigned)kCList) {
        const int n = (int)S.n_list;
        rank_group(S, n, zmax, S.above, S.need);
        if (tid == 0) {
          const unsigned r = S.rank_hit;
          if (r == 0xffffffffu) {  // cannot happen with exact sums
            S.ok = 0;
          } else {
            S.mode = kCutThr;
            S.thr_key = (uint32_t)(S.srt[r] >> 32);
            S.thr_node = 0xffffffffu - (uint32_t)S.srt[r];
            S.count = S.cabove + r + 1u;
          }
        }
      } else if (S.ok && S.kgmin == S.kgmax) {
        if (tid == 0) {  // bcnt members with one key, hence one mass
          const unsigned long long mt = S.bmass / S.bcnt;
          const unsigned long long rem = S.need - S.above;
          const unsigned long long tn = mt ? (rem + mt - 1) / mt : S.bcnt;
          S.mode = kCutTie;
          S.tie_n = (unsigned)(tn < S.bcnt ? tn : S.bcnt);
          S.thr_key = S.kgmin;
          S.count = S.cabove + S.tie_n;
        }
      } else if (tid == 0) {
        S.ok = 0;
      }
      __syncthreads();
    }
    if (!S.ok) {  // keep everything rather than guess; flagged
      __syncthreads();
      if (tid == 0) {
        raise_status(p.status, ZHA_ERR_INTERNAL);
        S.mode = kCutAll;
      }
      __syncthreads();
    }
    // -- exact ties (one key, too many members to rank): the tie_n-th of them
    //    in frontier (= node) order becomes the node threshold --
    if (S.mode == kCutTie) {
      const unsigned thr_key = S.thr_key, tie_n = S.tie_n, beta = S.beta;
      unsigned tie_run = 0;
      for (int64_t base = 0; base < V.nItems && tie_run < tie_n; base += stride) {
        Slots q;
        uint32_t keepm, tiem;
        classify(S, V, base, qb_ok, qbw, kCutTie, thr_key, 0u, beta, q, &keepm, &tiem);
        unsigned tot;
        unsigned rk = tie_run + block_scan(S, __popc(tiem), &tot, 1);
#pragma unroll
        for (int sl = 0; sl < 4 * kCU; ++sl)
          if ((tiem >> sl) & 1u) {
            if (++rk == tie_n) S.thr_node = q.nd[sl];
          }
        tie_run += tot;
      }
      __syncthreads();
      if (tid == 0) S.mode = kCutThr;
      __syncthreads();
    }
    // the level's kept count: the candidates above the group and the group's
    // members up to the threshold (every candidate when nothing is cut)
    const unsigned kept_n = S.mode == kCutAll ? (unsigned)nF : S.count;
    if (level == 1) {  // the union kernel applies the threshold to the level-1 frontier
      if (tid == 0) {
        p.cutpar[(int64_t)unit * G + h] = make_uint4(S.mode, S.thr_key, S.thr_node, kept_n);
        if (lc) lc[L - 1] = (int32_t)kept_n;
      }
      break;
    }
    // -- emit the kept nodes in frontier (= node) order: key > key*, or key ==
    //    key* and node <= node* (the level-2 ones also as bits) --
    const unsigned mode = S.mode;
    const unsigned thr_key = S.thr_key, thr_node = S.thr_node, beta = S.beta;
    unsigned run = 0;
    for (int64_t base = 0; base < V.nItems; base += stride) {
      Slots q;
      uint32_t keepm, tiem;
      classify(S, V, base, qb_ok && mode != kCutAll, qbw, mode, thr_key, thr_node, beta, q,
               &keepm, &tiem);
      unsigned tot;
      unsigned pos = run + block_scan(S, __popc(keepm), &tot, 0);
      uint32_t cw = 0xffffffffu, acc = 0;  // level 2: a bitmap word OR-ed while it stays
#pragma unroll
      for (int sl = 0; sl < 4 * kCU; ++sl)
        if ((keepm >> sl) & 1u) {
          kg_out[pos] = (int32_t)q.nd[sl];
          // a cached frontier never reads S.ks, so it can take the list at once
          if (cached && pos < (unsigned)kKCap) S.ks[pos] = (int32_t)q.nd[sl];
          ++pos;
          if (level == 2) {
            const uint32_t w = q.nd[sl] >> 5;
            if (w != cw) {
              if (acc) atomicOr(&bm2[cw], acc);
              cw = w;
              acc = 0;
            }
            acc |= 1u << (q.nd[sl] & 31);
          }
        }
      if (acc) atomicOr(&bm2[cw], acc);
      run += tot;
    }
    if (tid == 0) {
      if (lc) lc[L - level] = (int32_t)run;
      if (run != kept_n) raise_status(p.status, ZHA_ERR_INTERNAL);  // the count rule above
    }
    n_prev = run;
    gsel ^= 1;
    __syncthreads();  // kept list complete
    if (!cached && run <= (unsigned)kKCap) {  // a streamed level's list into shared memory
      for (int64_t j = tid; j < run; j += kCThreads) S.ks[j] = __ldcg(kg_out + j);
      __syncthreads();
    }
    // -- the next frontier: children of the kept nodes, cached when small --
    nF = (int64_t)run * b;
    cached = nF <= kZCap;
    if (cached) {
      const float* zn = zh + p.zoff[level - 2];
      float mx = -INFINITY, mn = INFINITY;
      for (int64_t k0 = (int64_t)tid * 4; k0 < nF; k0 += (int64_t)kCThreads * 4) {
        // 4 consecutive candidates per thread (b is even: within one parent
        // when b >= 4, two parents when b == 2)
        float v[4];
        int64_t nd[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int64_t k = k0 + c;
          nd[c] = k < nF ? (int64_t)S.ks[k / b] * b + k % b : 0;
        }
#pragma unroll
        for (int c = 0; c < 4; ++c) v[c] = k0 + c < nF ? __ldcg(zn + nd[c]) : 0.0f;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          if (k0 + c >= nF) break;
          S.zc[k0 + c] = v[c];
          S.nc[k0 + c] = (int32_t)nd[c];
          mx = fmaxf(mx, v[c]);
          mn = fminf(mn, v[c]);
        }
      }
      float zmx, zmn;
      block_minmax(S, mx, mn, &zmx, &zmn);
      if (tid == 0) {
        S.zmax = zmx;
        S.zmin = zmn;
      }
    }
    __syncthreads();
  }
  __syncthreads();  // every level-2 bit is set
  for (int64_t w = tid; w < words2; w += kCThreads) gbm[w] = bm2[w];
}

// ---------------------------------------------------------------------------
// 3. the level-1 cut of every head applied, and the heads' kept level-1 nodes
//    merged, in the decode attention's format
// ---------------------------------------------------------------------------
constexpr int kUThreads = 512;
constexpr int kUNodes = 8;  // consecutive level-1 nodes per thread and iteration

// A thread takes 8 consecutive level-1 nodes n (starting at a multiple of 8,
// within the CTA's share [lo, hi) of the unit): head h keeps n when h kept
// its parent at level 2 (every node is a candidate when the tree has one
// level) and its score passes h's level-1 threshold (key > key*, or key ==
// key* and n <= node*; every candidate in kCutAll). The 8 nodes' parents lie
// in one 32-bit word of each head's level-2 bitmap (b >= 2). Nodes any head
// keeps are placed by a block scan, staged in shared memory and written in
// node order as (head mask << 24) | n.
__global__ void __launch_bounds__(kUThreads) union_kernel(const __grid_constant__ DenseParams p) {
  __shared__ unsigned int s_warp[kUThreads / 32];
  __shared__ uint4 s_par[kMaxGroup];
  __shared__ uint32_t s_out[kUThreads * kUNodes];
  const int r = blockIdx.x, unit = p.unit0 + (int)blockIdx.y;
  const int seq = unit / p.Hkv;
  const int G = p.G;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t n1 = decode_top(p, seq) * p.span[p.L - 1];
  const int64_t lo = n1 * r / p.segs, hi = n1 * (r + 1) / p.segs;
  uint32_t* out = p.kept + ((int64_t)unit * p.segs + r) * p.kept_stride;
  if (tid < G) s_par[tid] = p.cutpar[(int64_t)unit * G + tid];
  __syncthreads();
  const float* z1 = p.z + (int64_t)unit * G * p.zrows + p.zoff[0];
  const uint32_t* bm2 = p.bitmap + (int64_t)unit * G * p.bmw;
  const bool one_level = p.L == 1;
  // b <= 32 is a power of two (parent = n >> bsh); a larger b is a multiple
  // of 32, so the 8 nodes share one parent
  const int bsh = p.b <= 32 ? __ffs(p.b) - 1 : -1;
  unsigned run = 0;
  for (int64_t nb = lo & ~(int64_t)(kUNodes - 1); nb < hi; nb += (int64_t)kUThreads * kUNodes) {
    const int64_t n0 = nb + (int64_t)tid * kUNodes;
    const uint32_t u0 = (uint32_t)n0;  // node ids fit in 24 bits
    const uint32_t par0 = bsh >= 0 ? u0 >> bsh : u0 / (uint32_t)p.b;
    uint32_t m[kUNodes];
#pragma unroll
    for (int j = 0; j < kUNodes; ++j) m[j] = 0u;
    if (n0 < hi) {
      // scores of the 8 nodes (the level's score vector is padded to 64 rows)
      // and the parents' bitmap word, for every head at once
      float4 za[kMaxGroup], zb[kMaxGroup];
      uint32_t pw[kMaxGroup];
#pragma unroll
      for (int h = 0; h < kMaxGroup; ++h) {
        const bool live = h < G && s_par[h].x != kCutAll;
        const float4* zp = reinterpret_cast<const float4*>(z1 + (int64_t)h * p.zrows + n0);
        za[h] = live ? __ldcg(zp) : make_float4(0.f, 0.f, 0.f, 0.f);
        zb[h] = live ? __ldcg(zp + 1) : make_float4(0.f, 0.f, 0.f, 0.f);
        pw[h] = h < G && !one_level ? __ldcg(bm2 + (int64_t)h * p.bmw + (par0 >> 5)) : 0xffffffffu;
      }
#pragma unroll
      for (int h = 0; h < kMaxGroup; ++h) {
        if (h >= G) continue;
        const uint4 c = s_par[h];
        const float zz[kUNodes] = {za[h].x, za[h].y, za[h].z, za[h].w,
                                   zb[h].x, zb[h].y, zb[h].z, zb[h].w};
#pragma unroll
        for (int j = 0; j < kUNodes; ++j) {
          const uint32_t par = bsh >= 0 ? (u0 + j) >> bsh : par0;
          const bool cand = (pw[h] >> (par & 31)) & 1u;
          const uint32_t key = order_key(zz[j]);
          const bool keep = cand && (c.x == kCutAll || key > c.y || (key == c.y && u0 + j <= c.z));
          m[j] |= (keep ? 1u : 0u) << h;
        }
      }
#pragma unroll
      for (int j = 0; j < kUNodes; ++j)
        if (n0 + j < lo || n0 + j >= hi) m[j] = 0u;  // outside the share
    }
    unsigned f = 0;
#pragma unroll
    for (int j = 0; j < kUNodes; ++j) f += m[j] ? 1u : 0u;
    unsigned x = f;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const unsigned y = __shfl_up_sync(0xffffffffu, x, off);
      if (lane >= off) x += y;
    }
    if (lane == 31) s_warp[warp] = x;
    __syncthreads();
    unsigned wbase = 0, tot = 0;
#pragma unroll
    for (int w2 = 0; w2 < kUThreads / 32; ++w2) {
      if (w2 < warp) wbase += s_warp[w2];
      tot += s_warp[w2];
    }
    unsigned pos = wbase + x - f;  // within this iteration's entries
#pragma unroll
    for (int j = 0; j < kUNodes; ++j)
      if (m[j]) s_out[pos++] = (m[j] << 24) | (u0 + (uint32_t)j);
    __syncthreads();
    for (unsigned e = tid; e < tot; e += kUThreads) out[run + e] = s_out[e];
    run += tot;
    __syncthreads();
  }
  if (tid == 0) p.n_kept[(int64_t)unit * p.segs + r] = (int32_t)run;
}

template <typename T, int D, int G>
cudaError_t launch_score(const DenseParams& p, int units, int sms, cudaStream_t s) {
  using C = ScoreCfg<T, D>;
  auto kern = dense_score_kernel<T, D, G>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
  if (e != cudaSuccess) return e;
  int per = 3 * sms / units;  // three CTAs per SM
  if (per < 1) per = 1;
  dense_score_kernel<T, D, G><<<dim3((unsigned)per, (unsigned)units), kSThreads, C::kSmem, s>>>(p);
  return cudaGetLastError();
}

template <typename T, int G>
cudaError_t launch_score_fp4(const DenseParams& p, int units, int sms, cudaStream_t s) {
  auto kern = dense_score_fp4_kernel<T, G>;
  const int smem = 2 * kSStageBytes + 128 * kMaxGroup * 4;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  int per = 3 * sms / units;  // three CTAs per SM
  if (per < 1) per = 1;
  kern<<<dim3((unsigned)per, (unsigned)units), kSThreads, smem, s>>>(p);
  return cudaGetLastError();
}

template <typename T, int D>
cudaError_t launch_score_g(const DenseParams& p, int units, int sms, cudaStream_t s) {
  if constexpr (D == 128) {
    if (p.fp4_codes) {
      switch (p.G) {
        case 1: return launch_score_fp4<T, 1>(p, units, sms, s);
        case 2: return launch_score_fp4<T, 2>(p, units, sms, s);
        case 4: return launch_score_fp4<T, 4>(p, units, sms, s);
        case 8: return launch_score_fp4<T, 8>(p, units, sms, s);
        default: return cudaErrorInvalidValue;
      }
    }
  } else {
    if (p.fp4_codes) return cudaErrorInvalidValue;
  }
  switch (p.G) {
    case 1: return launch_score<T, D, 1>(p, units, sms, s);
    case 2: return launch_score<T, D, 2>(p, units, sms, s);
    case 4: return launch_score<T, D, 4>(p, units, sms, s);
    case 8: return launch_score<T, D, 8>(p, units, sms, s);
    default: return cudaErrorInvalidValue;
  }
}

struct DenseLayout {
  size_t z, klist, bitmap, cutpar, total;
  int64_t zrows, klcap, bmw;
  int64_t zoff[kMaxLevels];
};

DenseLayout dense_layout(const Geometry& g, int64_t units) {
  DenseLayout D{};
  int64_t off = 0;
  for (int l = 1; l <= g.L; ++l) {  // 64-row aligned, so score vectors are 16-byte aligned
    D.zoff[l - 1] = off;
    off += (g.level_rows[l - 1] + 63) / 64 * 64;
  }
  D.zrows = off + 64;  // the last level's vector loads may read 3 rows past its end
  D.klcap = (g.level_rows[0] + 63) / 64 * 64;
  D.bmw = g.L >= 2 ? (g.level_rows[1] + 31) / 32 + 1 : 1;
  auto a256 = [](size_t x) { return (x + 255) & ~(size_t)255; };
  size_t o = 0;
  D.z = o;
  o = a256(o + sizeof(float) * (size_t)units * g.G * D.zrows);
  D.klist = o;
  o = a256(o + sizeof(int32_t) * (size_t)units * g.G * 2 * D.klcap);
  D.bitmap = o;
  o = a256(o + sizeof(uint32_t) * (size_t)units * g.G * D.bmw);
  D.cutpar = o;
  o = a256(o + sizeof(uint4) * (size_t)units * g.G);
  D.total = o;
  return D;
}

size_t cut_smem_bytes(const Geometry& g) {
  return ((sizeof(CutSmem) + 15) & ~(size_t)15) + sizeof(uint32_t) * (size_t)dense_layout(g, 1).bmw;
}

}  // namespace

bool decode_dense_ok(const Geometry& g, int64_t units) {
  // the level-2 bitmap of a head lives in shared memory next to the cut state
  if (cut_smem_bytes(g) > 227 * 1024) return false;
  // every row under the complete top nodes is read: keep that prefix within
  // what the frontier traversal's latency costs anyway (a few hundred us)
  int64_t rows = 0;
  for (int l = 0; l < g.L; ++l) rows += g.level_rows[l];
  return (double)rows * units * g.d * g.elem_bytes <= 1.5e9;
}

size_t decode_dense_ws_bytes(const Geometry& g, int64_t units) {
  return dense_layout(g, units).total;
}

cudaError_t launch_decode_dense(const Geometry& g, const void* tree, const void* q,
                                const int32_t* seq_len, uint64_t p_q, void* ws,
                                int32_t* level_counts, int32_t* stats, uint32_t* kept,
                                int32_t* n_kept, int64_t kept_stride, int segs, int32_t* status,
                                int num_sms, cudaStream_t stream, int64_t unit0, int64_t n_units,
                                const void* fp4_tree) {
  const int64_t all_units = (int64_t)g.B * g.Hkv;
  const int64_t units = n_units > 0 ? n_units : all_units;
  if (unit0 < 0 || unit0 + units > all_units) return cudaErrorInvalidValue;
  const DenseLayout Ly = dense_layout(g, all_units);
  unsigned char* w = static_cast<unsigned char*>(ws);
  DenseParams p{};
  p.tree = tree;
  for (int l = 0; l < g.L; ++l) {
    p.level_off[l] = g.level_off[l];
    p.level_rows[l] = g.level_rows[l];
    p.lnsize[l] = g.lnsize[l];
    p.zoff[l] = Ly.zoff[l];
  }
  for (int l = 0; l <= g.L; ++l) p.span[l] = g.span[l];
  p.inv_sqrt_d = g.inv_sqrt_d;
  p.q = q;
  p.seq_len = seq_len;
  p.Hq = g.Hq;
  p.Hkv = g.Hkv;
  p.G = g.G;
  p.b = g.b;
  p.L = g.L;
  p.B = g.B;
  p.ncap = g.ncap;
  p.z = reinterpret_cast<float*>(w + Ly.z);
  p.zrows = Ly.zrows;
  p.stats = stats;
  p.p_q = p_q;
  p.keep_all = p_q >= (1ull << 32);
  p.klist = reinterpret_cast<int32_t*>(w + Ly.klist);
  p.klcap = Ly.klcap;
  p.bitmap = reinterpret_cast<uint32_t*>(w + Ly.bitmap);
  p.bmw = Ly.bmw;
  p.cutpar = reinterpret_cast<uint4*>(w + Ly.cutpar);
  p.level_counts = level_counts;
  p.status = status;
  p.kept = kept;
  p.n_kept = n_kept;
  p.kept_stride = kept_stride;
  p.segs = segs;
  p.unit0 = (int)unit0;
  if (fp4_tree) {
    p.fp4_codes = static_cast<const unsigned char*>(fp4_tree);
    p.fp4_exps = reinterpret_cast<const int16_t*>(static_cast<const unsigned char*>(fp4_tree) +
                                                  fp4_codes_bytes(g));
  }
  cudaError_t e;
  if (g.dtype == ZHA_BF16)
    e = g.d == 128 ? launch_score_g<__nv_bfloat16, 128>(p, (int)units, num_sms, stream)
                   : launch_score_g<__nv_bfloat16, 64>(p, (int)units, num_sms, stream);
  else
    e = g.d == 128 ? launch_score_g<float, 128>(p, (int)units, num_sms, stream)
                   : launch_score_g<float, 64>(p, (int)units, num_sms, stream);
  if (e != cudaSuccess) return e;
  const size_t csm = cut_smem_bytes(g);
  e = cudaFuncSetAttribute(head_cut_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)csm);
  if (e != cudaSuccess) return e;
  head_cut_kernel<<<dim3((unsigned)g.G, (unsigned)units), kCThreads, csm, stream>>>(p);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  union_kernel<<<dim3((unsigned)segs, (unsigned)units), kUThreads, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace zha
