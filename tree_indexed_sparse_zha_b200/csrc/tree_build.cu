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
// Layout: one thread per child row computes its 16 logits (16 independent
// chains, packed two per fp32x2 FMA); the b threads of a node exchange values
// by warp shuffles (b <= 32) or through shared memory (b = 64..1024, one CTA
// per node). The work is FP32-ALU bound: 16 d FMAs per child row.
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

template <typename T, int D>
__global__ void __launch_bounds__(256) tree_level_small_b(TreeParams p, int level) {
  __shared__ __align__(16) float Rt[kNRef * D];
  __shared__ float abuf[256];
  load_rt<D>(p.r, Rt);
  __syncthreads();
  const int unit = blockIdx.y;
  const int seq = unit / p.Hkv;
  const int64_t span = p.span[level];
  const int64_t n_new = clamp_len(p.seq_len[seq], p.ncap);
  const int64_t n_old = p.old_len ? clamp_len(p.old_len[seq], p.ncap) : 0;
  const int64_t lo = (n_old < n_new ? n_old : n_new) / span;
  const int64_t hi = n_new / span;
  const int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t node = lo + g / p.b;
  const bool active = node < hi;
  // whole warp idle -> leave (shuffles only mix lanes of one node group)
  if (__all_sync(0xffffffffu, !active)) return;
  node_small_b<T, D>(p, Rt, abuf + (threadIdx.x & ~31), level, unit, active ? node : lo, active);
}

// One CTA per unit walks every level; for small growth (decode steps).
template <typename T, int D>
__global__ void __launch_bounds__(128) tree_extend_fused(TreeParams p) {
  __shared__ __align__(16) float Rt[kNRef * D];
  __shared__ float abuf[128];
  load_rt<D>(p.r, Rt);
  __syncthreads();
  const int unit = blockIdx.x;
  const int seq = unit / p.Hkv;
  const int64_t n_new = clamp_len(p.seq_len[seq], p.ncap);
  const int64_t n_old0 = p.old_len ? clamp_len(p.old_len[seq], p.ncap) : 0;
  const int64_t n_old = n_old0 < n_new ? n_old0 : n_new;
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
      const int64_t threads = nodes * g.b;
      const int64_t blocks = (threads + 255) / 256;
      dim3 grid((unsigned)blocks, (unsigned)units);
      tree_level_small_b<T, D><<<grid, 256, 0, stream>>>(p, level);
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
