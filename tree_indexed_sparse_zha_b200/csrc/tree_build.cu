// Summary-key tree build and incremental extension.
//
// lefilia.fr page "Zyphra presente Zyphra Hierarchical Attention (ZHA) ...",
// paragraph 1: keys are cut into contiguous blocks, each summarised by one key
// derived from 16 learned reference queries, and blocks are grouped level by
// level. This library's summary of a node with children x_0..x_{b-1}:
//     s = (1/16) sum_r sum_c softmax_c(R_r . x_c / sqrt(d)) x_c
// computed in the canonical fp32 order:
//     l_rc = dot(R_r, x_c) * inv_sqrt_d      (sequential fmaf chain, i = 0..d-1)
//     mu_r = max_c l_rc ; e_rc = exp(l_rc - mu_r) ; Z_r = sum_c e_rc (c order)
//     w_rc = e_rc / Z_r ; a_c = (sum_r w_rc, r order) * 1/16
//     s_i  = sum_c fmaf(a_c, x_ci, .) in c order from +0, stored RNE in the I/O type
//
// Layout: the level kernels stage child rows in shared memory and give each
// thread a 4 x 4 block of (child, reference query) logit chains, packed two
// per fp32x2 FMA: tiles of whole nodes for b <= 32, one node per CTA
// iteration for b = 64..256; wider blocks take one CTA of b threads per node,
// one child row per thread. The work is FP32-ALU bound: 16 d FMAs per child
// row.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "zha_device.cuh"
#include "zha_internal.h"

namespace zha {
namespace {

struct TreeParams {
  const void* k;
  void* tree;
  const float* r;
  const int32_t* seq_len;
  const int32_t* old_len;   // nullable: build from 0
  int64_t ncap;
  int Hkv, b, L;
  int64_t span[kMaxLevels + 1];
  int64_t level_off[kMaxLevels];
  int64_t level_rows[kMaxLevels];
  float inv_sqrt_d;
};

__device__ __forceinline__ int64_t clamp_len(int64_t n, int64_t ncap) {
  return n < 0 ? 0 : (n > ncap ? ncap : n);
}

// Base pointer of the child rows of level `level` for `unit`.
template <typename T, int D>
__device__ __forceinline__ const T* child_base(const TreeParams& p, int level, int unit) {
  if (level == 1) return static_cast<const T*>(p.k) + (int64_t)unit * p.ncap * D;
  return static_cast<const T*>(p.tree) + p.level_off[level - 2] +
         (int64_t)unit * p.level_rows[level - 2] * D;
}

template <typename T, int D>
__device__ __forceinline__ T* level_base(const TreeParams& p, int level, int unit) {
  return static_cast<T*>(p.tree) + p.level_off[level - 1] +
         (int64_t)unit * p.level_rows[level - 1] * D;
}

// Load R transposed into shared memory: Rt[i * 16 + r] = R[r][i].
template <int D>
__device__ __forceinline__ void load_rt(const float* R, float* Rt) {
  for (int e = threadIdx.x; e < kNRef * D; e += blockDim.x) {
    const int r = e / D, i = e % D;
    Rt[i * kNRef + r] = R[e];
  }
}

// The 16 canonical logit chains of one child row: acc[r] = dot(R_r, x).
template <typename T, int D>
__device__ __forceinline__ void logits16(const T* row, const float* Rt, float* acc) {
  float2 a2[kNRef / 2];
#pragma unroll
  for (int j = 0; j < kNRef / 2; ++j) a2[j] = make_float2(0.0f, 0.0f);
  constexpr int kPer = Elem<T>::kPerChunk;
  const uint4* rowc = reinterpret_cast<const uint4*>(row);
#pragma unroll 2
  for (int ch = 0; ch < D / kPer; ++ch) {
    const uint4 raw = rowc[ch];  // plain load: rows may come from this kernel
    float x[kPer];
    Elem<T>::unpack(raw, x);
#pragma unroll
    for (int e = 0; e < kPer; ++e) {
      const float4* rt = reinterpret_cast<const float4*>(Rt + (ch * kPer + e) * kNRef);
      const float2 xx = make_float2(x[e], x[e]);
#pragma unroll
      for (int j = 0; j < kNRef / 4; ++j) {
        const float4 rv = rt[j];
        a2[2 * j] = ffma2(make_float2(rv.x, rv.y), xx, a2[2 * j]);
        a2[2 * j + 1] = ffma2(make_float2(rv.z, rv.w), xx, a2[2 * j + 1]);
      }
    }
  }
#pragma unroll
  for (int j = 0; j < kNRef / 2; ++j) {
    acc[2 * j] = a2[j].x;
    acc[2 * j + 1] = a2[j].y;
  }
}

// ---------------------------------------------------------------------------
// b <= 32 (b divides 32): the b children of a node sit in b adjacent lanes.
// ---------------------------------------------------------------------------
template <typename T, int D>
__device__ void node_small_b(const TreeParams& p, const float* Rt, float* abuf, int level,
                             int unit, int64_t node, bool active) {
  const int b = p.b;
  const int lane = threadIdx.x & 31;
  const int c = lane % b;            // child index within the node
  const int base = lane - c;         // first lane of the group
  const T* cb = child_base<T, D>(p, level, unit);
  float l[kNRef];
  if (active) {
    logits16<T, D>(cb + (node * b + c) * D, Rt, l);
  } else {
#pragma unroll
    for (int r = 0; r < kNRef; ++r) l[r] = 0.0f;
  }
  float a_acc = 0.0f;
#pragma unroll
  for (int r = 0; r < kNRef; ++r) {
    const float lr = __fmul_rn(l[r], p.inv_sqrt_d);
    float mu = lr;
    for (int off = 1; off < b; off <<= 1) mu = fmaxf(mu, __shfl_xor_sync(0xffffffffu, mu, off));
    const float e = exp_canon(__fsub_rn(lr, mu));
    float Z = 0.0f;
    for (int cc = 0; cc < b; ++cc) Z = __fadd_rn(Z, __shfl_sync(0xffffffffu, e, base + cc));
    a_acc = __fadd_rn(a_acc, __fdiv_rn(e, Z));
  }
  abuf[lane] = __fmul_rn(a_acc, 0.0625f);
  __syncwarp();
  // weighted sum: lane c of the group produces dims [c*D/b, (c+1)*D/b), each
  // element a sequential fmaf chain over the children
  if (active) {
    const int per = D / b;
    const T* node_rows = cb + node * b * D;
    T* out = level_base<T, D>(p, level, unit) + node * D;
    for (int k = c * per; k < (c + 1) * per; ++k) {
      float s = 0.0f;
      for (int cc = 0; cc < b; ++cc) s = __fmaf_rn(abuf[base + cc], Elem<T>::to_f(node_rows[cc * D + k]), s);
      out[k] = Elem<T>::from_f(s);
    }
  }
  __syncwarp();
}

// ---------------------------------------------------------------------------
// Level kernel for b <= 32: a CTA takes tiles of kTileRows consecutive child
// rows (kTileRows / b whole nodes) of one unit. The rows are staged in shared
// memory by cp.async in one stage (49 KB of shared memory per CTA, so four
// CTAs share an SM and overlap one another's loads), then reduced in four
// phases:
//   1. logits: thread (cg, rg) runs the 16 canonical chains of children
//      4cg..4cg+3 against reference queries 4rg..4rg+3 -- every staged x
//      chunk feeds 4 reference queries and every R value 4 children;
//   2. softmax per (node, r) over the node's children, in child order;
//   3. a_c = (sum_r w_rc in r order) / 16 per child;
//   4. the weighted sum per (node, 16-byte output chunk), in child order,
//      stored with one 16-byte write.
// Each value is the same chain of the same rounded operations as in the
// per-node formulation, so the stored summaries are bit-identical.
// ---------------------------------------------------------------------------
constexpr int kTileRows = 128;  // child rows per tile (a multiple of every b <= 32)
constexpr int kTileThreads = 128;

template <typename T, int D>
struct TileCfg {
  static constexpr int kPer = Elem<T>::kPerChunk;        // elements per 16-byte chunk
  static constexpr int kNch = D * (int)sizeof(T) / 16;    // chunks per row
  static constexpr int kStageBytes = kTileRows * D * (int)sizeof(T);
  static constexpr int kRtBytes = kNRef * D * 4;
  static constexpr int kWBytes = kTileRows * kNRef * 4;
  static constexpr int kSmem = kStageBytes + kRtBytes + kWBytes + kTileRows * 4;
  static constexpr int kSmemB4 = kStageBytes + kRtBytes + kTileRows * 4;  // no logit buffer
};

// Chunk ch of staged row r sits at chunk ch ^ ((r >> 2) & 7): the 8 rows one
// warp reads at once in phase 1 (rows 4cg + k, 8 consecutive cg) then fall
// in 8 different bank groups.
__device__ __forceinline__ int tswz(int ch, int r) { return ch ^ ((r >> 2) & 7); }

template <typename T, int D>
__device__ __forceinline__ void stage_tile(const T* src, int rows, unsigned char* dst) {
  using C = TileCfg<T, D>;
  for (int e = threadIdx.x; e < rows * C::kNch; e += kTileThreads) {
    const int r = e / C::kNch, ch = e % C::kNch;
    cp_async16(dst + ((int64_t)r * C::kNch + tswz(ch, r)) * 16,
               reinterpret_cast<const uint4*>(src + (int64_t)r * D) + ch);
  }
}

// B4 (b == 4): a thread's 4 children are exactly one node, so phases 2 to 4
// run in its registers: the softmax over the node's children for its 4
// reference queries, each child's weight sum in r order, handed from the lane
// holding r = 0..3 to the one holding r = 12..15 (the 4 lanes of a node are
// adjacent), then a quarter of the node's output chunks. The same rounded
// operations in the same order as the shared-memory phases, without the
// logit buffer and with one barrier per tile instead of four.
template <typename T, int D, bool B4>
__global__ void __launch_bounds__(kTileThreads) tree_level_tiled(const __grid_constant__ TreeParams p,
                                                                 int level) {
  using C = TileCfg<T, D>;
  constexpr int kPer = C::kPer, kNch = C::kNch;
  extern __shared__ __align__(16) float sm[];
  unsigned char* X = reinterpret_cast<unsigned char*>(sm);  // the tile's staged rows
  float* Rt = reinterpret_cast<float*>(X + C::kStageBytes);  // [D][16]
  float* W = Rt + kNRef * D;                                // [tile rows][16] (not B4)
  float* A = B4 ? W : W + kTileRows * kNRef;                // [tile rows]
  const int tid = threadIdx.x;
  const int unit = blockIdx.y;
  const int seq = unit / p.Hkv;
  const int b = p.b;
  const int64_t span = p.span[level];
  const int64_t n_new = clamp_len(p.seq_len[seq], p.ncap);
  const int64_t n_old = p.old_len ? clamp_len(p.old_len[seq], p.ncap) : 0;
  const int64_t lo = (n_old < n_new ? n_old : n_new) / span;
  const int64_t hi = n_new / span;
  const int64_t rows_total = (hi - lo) * b;  // child rows of the nodes to build
  const int64_t n_tiles = (rows_total + kTileRows - 1) / kTileRows;
  if ((int64_t)blockIdx.x >= n_tiles) return;  // uniform over the CTA
  const T* cb = child_base<T, D>(p, level, unit) + lo * b * D;
  T* ob = level_base<T, D>(p, level, unit) + lo * D;
  load_rt<D>(p.r, Rt);
  const int rg = tid & 3, cg = tid >> 2;  // phase-1 block: 4 children x 4 reference queries
  const float inv_sqrt_d = p.inv_sqrt_d;

  for (int64_t tile = blockIdx.x; tile < n_tiles; tile += gridDim.x) {
    const int64_t r0 = tile * kTileRows;
    const int rows = (int)(rows_total - r0 < kTileRows ? rows_total - r0 : kTileRows);
    stage_tile<T, D>(cb + r0 * D, rows, X);
    cp_async_commit();
    cp_async_wait<0>();  // this thread's copies have landed
    __syncthreads();     // ... and every thread's
    // ---- 1. logits of children 4cg..4cg+3 against queries 4rg..4rg+3 ----
    {
      float2 acc[4][2];
#pragma unroll
      for (int k = 0; k < 4; ++k) acc[k][0] = acc[k][1] = make_float2(0.0f, 0.0f);
#pragma unroll 2
      for (int ch = 0; ch < kNch; ++ch) {
        float x[4][kPer];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int r = 4 * cg + k;
          Elem<T>::unpack(lds128(X + ((int64_t)r * kNch + tswz(ch, r)) * 16), x[k]);
        }
#pragma unroll
        for (int e = 0; e < kPer; ++e) {
          const float4 rv = *reinterpret_cast<const float4*>(Rt + (ch * kPer + e) * kNRef + 4 * rg);
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const float2 xx = make_float2(x[k][e], x[k][e]);
            acc[k][0] = ffma2(make_float2(rv.x, rv.y), xx, acc[k][0]);
            acc[k][1] = ffma2(make_float2(rv.z, rv.w), xx, acc[k][1]);
          }
        }
      }
      if constexpr (B4) {
        float l[4][4];  // [child][reference query 4rg + j]
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          l[k][0] = __fmul_rn(acc[k][0].x, inv_sqrt_d);
          l[k][1] = __fmul_rn(acc[k][0].y, inv_sqrt_d);
          l[k][2] = __fmul_rn(acc[k][1].x, inv_sqrt_d);
          l[k][3] = __fmul_rn(acc[k][1].y, inv_sqrt_d);
        }
        // ---- 2. softmax over the node's children, per reference query ----
        float w[4][4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          float mu = l[0][j];
#pragma unroll
          for (int k = 1; k < 4; ++k) mu = fmaxf(mu, l[k][j]);
          float e[4], Z = 0.0f;
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            e[k] = exp_canon(__fsub_rn(l[k][j], mu));
            Z = __fadd_rn(Z, e[k]);
          }
#pragma unroll
          for (int k = 0; k < 4; ++k) w[k][j] = __fdiv_rn(e[k], Z);
        }
        // ---- 3. child weights a_c: r = 0..15 in order across the node's lanes ----
        float part[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
        for (int step = 0; step < 4; ++step) {
          if (rg == step) {
#pragma unroll
            for (int k = 0; k < 4; ++k)
#pragma unroll
              for (int j = 0; j < 4; ++j) part[k] = __fadd_rn(part[k], w[k][j]);
          }
          if (step < 3) {
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const float v = __shfl_up_sync(0xffffffffu, part[k], 1);
              if (rg == step + 1) part[k] = v;
            }
          }
        }
        // ---- 4. the node's weighted sum: chunks rg, rg + 4, ... of its output
        //    row, each element a chain over the 4 children in order ----
        float a[4];
#pragma unroll
        for (int k = 0; k < 4; ++k)
          a[k] = __shfl_sync(0xffffffffu, __fmul_rn(part[k], 0.0625f), ((tid & 31) & ~3) | 3);
        if (4 * cg < rows) {
#pragma unroll
          for (int m = 0; m < kNch / 4; ++m) {
            const int ch = rg + 4 * m;
            float sum[kPer];
#pragma unroll
            for (int e = 0; e < kPer; ++e) sum[e] = 0.0f;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const int r = 4 * cg + k;
              float x[kPer];
              Elem<T>::unpack(lds128(X + ((int64_t)r * kNch + tswz(ch, r)) * 16), x);
#pragma unroll
              for (int e = 0; e < kPer; ++e) sum[e] = __fmaf_rn(a[k], x[e], sum[e]);
            }
            *reinterpret_cast<uint4*>(ob + (r0 / 4 + cg) * D + ch * kPer) = Elem<T>::pack(sum);
          }
        }
      } else {
#pragma unroll
        for (int k = 0; k < 4; ++k)
          *reinterpret_cast<float4*>(W + (4 * cg + k) * kNRef + 4 * rg) =
              make_float4(__fmul_rn(acc[k][0].x, inv_sqrt_d), __fmul_rn(acc[k][0].y, inv_sqrt_d),
                          __fmul_rn(acc[k][1].x, inv_sqrt_d), __fmul_rn(acc[k][1].y, inv_sqrt_d));
      }
    }
    if constexpr (!B4) {
    __syncthreads();
    const int nodes = rows / b;
    // ---- 2. softmax over each node's children, per reference query ----
    for (int task = tid; task < nodes * kNRef; task += kTileThreads) {
      const int n = task / kNRef, r = task % kNRef;
      float* w = W + (n * b) * kNRef + r;
      float mu = w[0];
      for (int c = 1; c < b; ++c) mu = fmaxf(mu, w[c * kNRef]);
      float Z = 0.0f;
      for (int c = 0; c < b; ++c) {
        const float e = exp_canon(__fsub_rn(w[c * kNRef], mu));
        w[c * kNRef] = e;
        Z = __fadd_rn(Z, e);
      }
      for (int c = 0; c < b; ++c) w[c * kNRef] = __fdiv_rn(w[c * kNRef], Z);
    }
    __syncthreads();
    // ---- 3. child weights a_c ----
    for (int c = tid; c < nodes * b; c += kTileThreads) {
      float a = 0.0f;
#pragma unroll
      for (int r = 0; r < kNRef; ++r) a = __fadd_rn(a, W[c * kNRef + r]);
      A[c] = __fmul_rn(a, 0.0625f);
    }
    __syncthreads();
    // ---- 4. weighted sums, one 16-byte output chunk per task ----
    for (int task = tid; task < nodes * kNch; task += kTileThreads) {
      const int n = task / kNch, ch = task % kNch;
      float s[kPer];
#pragma unroll
      for (int e = 0; e < kPer; ++e) s[e] = 0.0f;
      for (int c = 0; c < b; ++c) {
        const int r = n * b + c;
        float x[kPer];
        Elem<T>::unpack(lds128(X + ((int64_t)r * kNch + tswz(ch, r)) * 16), x);
        const float a = A[r];
#pragma unroll
        for (int e = 0; e < kPer; ++e) s[e] = __fmaf_rn(a, x[e], s[e]);
      }
      *reinterpret_cast<uint4*>(ob + (r0 / b + n) * D + ch * kPer) = Elem<T>::pack(s);
    }
    }
    __syncthreads();  // the stage is refilled by the next tile
  }
}

// One CTA per unit walks every level; for small growth (decode steps).
template <typename T, int D>
__global__ void __launch_bounds__(128) tree_extend_fused(TreeParams p) {
  __shared__ __align__(16) float Rt[kNRef * D];
  __shared__ float abuf[128];
  const int unit = blockIdx.x;
  const int seq = unit / p.Hkv;
  const int64_t n_new = clamp_len(p.seq_len[seq], p.ncap);
  const int64_t n_old0 = p.old_len ? clamp_len(p.old_len[seq], p.ncap) : 0;
  const int64_t n_old = n_old0 < n_new ? n_old0 : n_new;
  // most single-token steps complete no node: leave before staging R
  if (n_old / p.span[1] >= n_new / p.span[1]) return;  // uniform over the CTA
  load_rt<D>(p.r, Rt);
  __syncthreads();
  const int groups = blockDim.x / p.b;
  for (int level = 1; level <= p.L; ++level) {
    const int64_t lo = n_old / p.span[level];
    const int64_t hi = n_new / p.span[level];
    if (lo >= hi) break;  // no new node here, so none above either (uniform)
    for (int64_t n0 = lo; n0 < hi; n0 += groups) {
      const int64_t node = n0 + threadIdx.x / p.b;
      const bool active = node < hi;
      if (!__all_sync(0xffffffffu, !active))
        node_small_b<T, D>(p, Rt, abuf + (threadIdx.x & ~31), level, unit, active ? node : lo,
                           active);
    }
    __syncthreads();  // level l rows are read by level l+1 (same CTA)
  }
}

// ---------------------------------------------------------------------------
// b in {64, ..., 1024}, multiple of 32: one CTA of b threads per node.
// ---------------------------------------------------------------------------
template <typename T, int D>
__global__ void __launch_bounds__(1024) tree_level_large_b(TreeParams p, int level) {
  extern __shared__ __align__(16) float sm[];
  float* Rt = sm;                              // [D][16]
  float* E = Rt + kNRef * D;                   // [16][b]
  float* A = E + kNRef * p.b;                  // [b]
  float* red = A + p.b;                        // [32][16]
  float* muZ = red + 32 * kNRef;               // [16] mu then Z
  load_rt<D>(p.r, Rt);
  __syncthreads();
  const int unit = blockIdx.y;
  const int seq = unit / p.Hkv;
  const int64_t span = p.span[level];
  const int64_t n_new = clamp_len(p.seq_len[seq], p.ncap);
  const int64_t n_old = p.old_len ? clamp_len(p.old_len[seq], p.ncap) : 0;
  const int64_t lo = (n_old < n_new ? n_old : n_new) / span;
  const int64_t hi = n_new / span;
  const int b = p.b;
  const int c = threadIdx.x;
  const int warp = c >> 5, lane = c & 31;
  const T* cb = child_base<T, D>(p, level, unit);
  T* ob = level_base<T, D>(p, level, unit);
  for (int64_t node = lo + blockIdx.x; node < hi; node += gridDim.x) {
    float l[kNRef];
    logits16<T, D>(cb + (node * b + c) * D, Rt, l);
#pragma unroll
    for (int r = 0; r < kNRef; ++r) {
      l[r] = __fmul_rn(l[r], p.inv_sqrt_d);
      float m = l[r];
      for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
      if (lane == 0) red[warp * kNRef + r] = m;
    }
    __syncthreads();
    if (c < kNRef) {
      float m = red[c];
      for (int w = 1; w < b / 32; ++w) m = fmaxf(m, red[w * kNRef + c]);
      muZ[c] = m;
    }
    __syncthreads();
#pragma unroll
    for (int r = 0; r < kNRef; ++r) E[r * b + c] = exp_canon(__fsub_rn(l[r], muZ[r]));
    __syncthreads();
    if (c < kNRef) {
      float Z = 0.0f;
      for (int cc = 0; cc < b; ++cc) Z = __fadd_rn(Z, E[c * b + cc]);
      muZ[c] = Z;
    }
    __syncthreads();
    float a = 0.0f;
#pragma unroll
    for (int r = 0; r < kNRef; ++r) a = __fadd_rn(a, __fdiv_rn(E[r * b + c], muZ[r]));
    A[c] = __fmul_rn(a, 0.0625f);
    __syncthreads();
    if (c < D) {
      const T* xr = cb + node * b * D + c;
      float s = 0.0f;
      for (int cc = 0; cc < b; ++cc) s = __fmaf_rn(A[cc], Elem<T>::to_f(xr[(int64_t)cc * D]), s);
      ob[node * D + c] = Elem<T>::from_f(s);
    }
    __syncthreads();
  }
}

// ---------------------------------------------------------------------------
// Level kernel for 64 <= b <= 256 (b a multiple of 32): a CTA takes one node
// at a time, its b child rows staged in shared memory by cp.async (swizzled
// as in the tiled kernel), then
//   1. thread (cg, rg) runs the 16 canonical logit chains of children
//      4cg..4cg+3 against reference queries 4rg..4rg+3 (b threads busy);
//      its maxima over its 4 children go through warp shuffles and one
//      shared slot per warp to the node maxima mu_r;
//   2. the exponentials stay in the thread's registers; one copy goes to
//      shared memory, where 16 threads form Z_r over the children in order;
//   3. w_rc = e_rc / Z_r in registers, and a_c = (sum_r w_rc in r order) / 16
//      handed along the 4 lanes of a child group (r = 0..3 first);
//   4. thread i runs output element i's chain over the children in order.
// The same rounded operations in the same order as the per-node form
// (tree_level_large_b), so the stored summaries are bit-identical.
// ---------------------------------------------------------------------------
constexpr int kBigThreads = 256;
constexpr int kBigMaxB = 256;  // one 4x4 logit block per thread and node

template <typename T, int D>
size_t big_b_smem(int b) {
  // rows [b][D], Rt [D][16], E [16][b + 4], warp maxima [8][16], a [b], Z [16]
  return (size_t)b * D * sizeof(T) +
         sizeof(float) * ((size_t)kNRef * D + (size_t)kNRef * (b + 4) + 8 * kNRef + b + kNRef);
}

template <typename T, int D>
__global__ void __launch_bounds__(kBigThreads) tree_level_big_b(const __grid_constant__ TreeParams p,
                                                                int level) {
  constexpr int kPer = Elem<T>::kPerChunk;
  constexpr int kNch = D * (int)sizeof(T) / 16;  // chunks per row
  extern __shared__ __align__(16) float sm[];
  const int b = p.b;
  const int es = b + 4;  // row stride of E: 16-byte rows, a quarter-warp's float4 stores spread
  unsigned char* X = reinterpret_cast<unsigned char*>(sm);             // [b][kNch] chunks
  float* Rt = reinterpret_cast<float*>(X + (size_t)b * D * sizeof(T));  // [D][16]
  float* E = Rt + kNRef * D;                                           // [16][es]
  float* red = E + kNRef * es;                                         // [8][16]
  float* A = red + 8 * kNRef;                                          // [b]
  float* Zs = A + b;                                                   // [16]
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int rg = tid & 3, cg = tid >> 2;  // logit block: 4 children x 4 reference queries
  const bool blk = tid < b;               // whole warps (b is a multiple of 32)
  const int nw = b >> 5;                  // warps holding a block
  const int unit = blockIdx.y;
  const int seq = unit / p.Hkv;
  const int64_t span = p.span[level];
  const int64_t n_new = clamp_len(p.seq_len[seq], p.ncap);
  const int64_t n_old = p.old_len ? clamp_len(p.old_len[seq], p.ncap) : 0;
  const int64_t lo = (n_old < n_new ? n_old : n_new) / span;
  const int64_t hi = n_new / span;
  if (lo + blockIdx.x >= hi) return;  // uniform over the CTA
  const T* cb = child_base<T, D>(p, level, unit);
  T* ob = level_base<T, D>(p, level, unit);
  load_rt<D>(p.r, Rt);
  const float inv_sqrt_d = p.inv_sqrt_d;
  for (int64_t node = lo + blockIdx.x; node < hi; node += gridDim.x) {
    const T* rows = cb + node * b * D;
    for (int e = tid; e < b * kNch; e += kBigThreads) {
      const int r = e / kNch, ch = e % kNch;
      cp_async16(X + ((int64_t)r * kNch + tswz(ch, r)) * 16,
                 reinterpret_cast<const uint4*>(rows + (int64_t)r * D) + ch);
    }
    cp_async_commit();
    cp_async_wait<0>();
    __syncthreads();  // the rows (and, the first time, R) are in place
    float l[4][4];    // [child 4cg + k][reference query 4rg + j]
    // ---- 1. logits, then the block's maxima per reference query ----
    if (blk) {
      float2 acc[4][2];
#pragma unroll
      for (int k = 0; k < 4; ++k) acc[k][0] = acc[k][1] = make_float2(0.0f, 0.0f);
#pragma unroll 2
      for (int ch = 0; ch < kNch; ++ch) {
        float x[4][kPer];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int r = 4 * cg + k;
          Elem<T>::unpack(lds128(X + ((int64_t)r * kNch + tswz(ch, r)) * 16), x[k]);
        }
#pragma unroll
        for (int e = 0; e < kPer; ++e) {
          const float4 rv = *reinterpret_cast<const float4*>(Rt + (ch * kPer + e) * kNRef + 4 * rg);
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const float2 xx = make_float2(x[k][e], x[k][e]);
            acc[k][0] = ffma2(make_float2(rv.x, rv.y), xx, acc[k][0]);
            acc[k][1] = ffma2(make_float2(rv.z, rv.w), xx, acc[k][1]);
          }
        }
      }
      float m[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        l[k][0] = __fmul_rn(acc[k][0].x, inv_sqrt_d);
        l[k][1] = __fmul_rn(acc[k][0].y, inv_sqrt_d);
        l[k][2] = __fmul_rn(acc[k][1].x, inv_sqrt_d);
        l[k][3] = __fmul_rn(acc[k][1].y, inv_sqrt_d);
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        m[j] = fmaxf(fmaxf(l[0][j], l[1][j]), fmaxf(l[2][j], l[3][j]));
#pragma unroll
        for (int off = 4; off < 32; off <<= 1)  // lanes of the same rg
          m[j] = fmaxf(m[j], __shfl_xor_sync(0xffffffffu, m[j], off));
      }
      if (lane < 4) *reinterpret_cast<float4*>(red + warp * kNRef + 4 * rg) = make_float4(m[0], m[1], m[2], m[3]);
    }
    __syncthreads();
    // ---- 2. exponentials against the node maxima; E for the Z chains ----
    if (blk) {
      float4 mu = *reinterpret_cast<const float4*>(red + 4 * rg);
      for (int w = 1; w < nw; ++w) {
        const float4 v = *reinterpret_cast<const float4*>(red + w * kNRef + 4 * rg);
        mu = make_float4(fmaxf(mu.x, v.x), fmaxf(mu.y, v.y), fmaxf(mu.z, v.z), fmaxf(mu.w, v.w));
      }
      const float muj[4] = {mu.x, mu.y, mu.z, mu.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
#pragma unroll
        for (int k = 0; k < 4; ++k) l[k][j] = exp_canon(__fsub_rn(l[k][j], muj[j]));
        *reinterpret_cast<float4*>(E + (4 * rg + j) * es + 4 * cg) =
            make_float4(l[0][j], l[1][j], l[2][j], l[3][j]);
      }
    }
    __syncthreads();
    if (tid < kNRef) {  // Z_r: the children in order
      const float* e = E + tid * es;
      float Z = 0.0f;
      for (int c = 0; c < b; c += 8) {
        const float4 v0 = *reinterpret_cast<const float4*>(e + c);
        const float4 v1 = *reinterpret_cast<const float4*>(e + c + 4);
        Z = __fadd_rn(Z, v0.x);
        Z = __fadd_rn(Z, v0.y);
        Z = __fadd_rn(Z, v0.z);
        Z = __fadd_rn(Z, v0.w);
        Z = __fadd_rn(Z, v1.x);
        Z = __fadd_rn(Z, v1.y);
        Z = __fadd_rn(Z, v1.z);
        Z = __fadd_rn(Z, v1.w);
      }
      Zs[tid] = Z;
    }
    __syncthreads();
    // ---- 3. child weights a_c: r = 0..15 in order across the group's lanes ----
    if (blk) {
      const float4 z = *reinterpret_cast<const float4*>(Zs + 4 * rg);
      const float zj[4] = {z.x, z.y, z.z, z.w};
      float part[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
      for (int step = 0; step < 4; ++step) {
        if (rg == step) {
#pragma unroll
          for (int k = 0; k < 4; ++k)
#pragma unroll
            for (int j = 0; j < 4; ++j) part[k] = __fadd_rn(part[k], __fdiv_rn(l[k][j], zj[j]));
        }
        if (step < 3) {
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const float v = __shfl_up_sync(0xffffffffu, part[k], 1);
            if (rg == step + 1) part[k] = v;
          }
        }
      }
      if (rg == 3)
        *reinterpret_cast<float4*>(A + 4 * cg) =
            make_float4(__fmul_rn(part[0], 0.0625f), __fmul_rn(part[1], 0.0625f),
                        __fmul_rn(part[2], 0.0625f), __fmul_rn(part[3], 0.0625f));
    }
    __syncthreads();
    // ---- 4. output element tid: a chain over the children in order ----
    if (tid < D) {
      const int ch = tid / kPer, pos = tid % kPer;
      float s = 0.0f;
      for (int c = 0; c < b; c += 8) {
        const float4 a0 = *reinterpret_cast<const float4*>(A + c);
        const float4 a1 = *reinterpret_cast<const float4*>(A + c + 4);
        const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
        float xv[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int cc = c + u;
          xv[u] = Elem<T>::to_f(*(reinterpret_cast<const T*>(X + ((int64_t)cc * kNch + tswz(ch, cc)) * 16) + pos));
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) s = __fmaf_rn(av[u], xv[u], s);
      }
      ob[node * D + tid] = Elem<T>::from_f(s);
    }
    __syncthreads();  // the rows are restaged for the next node
  }
}

template <typename T, int D>
cudaError_t launch_tree_t(const Geometry& g, const TreeParams& p, int64_t max_new_tokens,
                          cudaStream_t stream) {
  const int units = g.B * g.Hkv;
  const bool small_b = g.b <= 32;
  if (small_b && max_new_tokens >= 0 && max_new_tokens <= 64) {
    tree_extend_fused<T, D><<<units, 128, 0, stream>>>(p);
    return cudaGetLastError();
  }
  for (int level = 1; level <= g.L; ++level) {
    int64_t nodes = g.level_rows[level - 1];
    if (max_new_tokens >= 0) {
      const int64_t cap = max_new_tokens / g.span[level] + 1;
      if (cap < nodes) nodes = cap;
    }
    if (nodes <= 0) break;
    if (small_b) {
      using C = TileCfg<T, D>;
      const bool b4 = g.b == 4;
      auto kern = b4 ? tree_level_tiled<T, D, true> : tree_level_tiled<T, D, false>;
      const int smem = b4 ? C::kSmemB4 : C::kSmem;
      cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
      if (e != cudaSuccess) return e;
      int per_sm = 0;
      e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kTileThreads, smem);
      if (e != cudaSuccess) return e;
      // at most one wave (a partial second wave would run a whole CTA's share
      // of tiles after the first): the resident slots shared evenly by the
      // units, each CTA looping over its unit's tiles
      const int64_t tiles = (nodes * g.b + kTileRows - 1) / kTileRows;
      int64_t per_unit = ((int64_t)device_sm_count() * (per_sm > 0 ? per_sm : 1)) / units;
      if (per_unit < 1) per_unit = 1;
      if (per_unit > tiles) per_unit = tiles;
      dim3 grid((unsigned)per_unit, (unsigned)units);
      kern<<<grid, kTileThreads, smem, stream>>>(p, level);
    } else if (g.b <= kBigMaxB) {
      const size_t smem = big_b_smem<T, D>(g.b);
      auto kern = tree_level_big_b<T, D>;
      cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e != cudaSuccess) return e;
      int per_sm = 0;
      e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kBigThreads, smem);
      if (e != cudaSuccess) return e;
      // one wave of resident CTAs shared by the units, each looping over nodes
      int64_t per_unit = ((int64_t)device_sm_count() * (per_sm > 0 ? per_sm : 1)) / units;
      if (per_unit < 1) per_unit = 1;
      if (per_unit > nodes) per_unit = nodes;
      kern<<<dim3((unsigned)per_unit, (unsigned)units), kBigThreads, smem, stream>>>(p, level);
    } else {
      const size_t smem = sizeof(float) * (kNRef * D + kNRef * g.b + g.b + 32 * kNRef + kNRef);
      cudaError_t e = cudaFuncSetAttribute(tree_level_large_b<T, D>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)smem);
      if (e != cudaSuccess) return e;
      const int64_t blocks = nodes < 65535 ? nodes : 65535;
      dim3 grid((unsigned)blocks, (unsigned)units);
      tree_level_large_b<T, D><<<grid, g.b, smem, stream>>>(p, level);
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace

cudaError_t launch_tree(const Geometry& g, const void* k, void* tree, const float* r,
                        const int32_t* seq_len, const int32_t* old_len, int64_t max_new_tokens,
                        cudaStream_t stream) {
  TreeParams p{};
  p.k = k;
  p.tree = tree;
  p.r = r;
  p.seq_len = seq_len;
  p.old_len = old_len;
  p.ncap = g.ncap;
  p.Hkv = g.Hkv;
  p.b = g.b;
  p.L = g.L;
  for (int l = 0; l <= g.L; ++l) p.span[l] = g.span[l];
  for (int l = 0; l < g.L; ++l) {
    p.level_off[l] = g.level_off[l];
    p.level_rows[l] = g.level_rows[l];
  }
  p.inv_sqrt_d = g.inv_sqrt_d;
  if (g.dtype == ZHA_BF16) {
    if (g.d == 128) return launch_tree_t<__nv_bfloat16, 128>(g, p, max_new_tokens, stream);
    return launch_tree_t<__nv_bfloat16, 64>(g, p, max_new_tokens, stream);
  }
  if (g.d == 128) return launch_tree_t<float, 128>(g, p, max_new_tokens, stream);
  return launch_tree_t<float, 64>(g, p, max_new_tokens, stream);
}

}  // namespace zha
