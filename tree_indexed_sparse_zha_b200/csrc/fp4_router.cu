// Block-scaled 4-bit copy of the summary tree, for the FP4 router variant.
//
// lefilia.fr page "Zyphra presente Zyphra Hierarchical Attention (ZHA) ...",
// paragraph 4: an FP4 variant of the router was tried; the page gives no
// format. This library's format: every block of 32 consecutive elements of a
// stored summary row becomes 4-bit codes -- bit 3 the sign, bits 0-2 the
// index k of the magnitude in {0, 0.5, 1, 1.5, 2, 3, 4, 6} (the e2m1
// encoding) -- and one exponent e per block, value = sign * mag[k] * 2^e, e
// the smallest integer with max|x| <= 6 * 2^e (0 for an all-zero block). Each
// |x| / 2^e goes to the nearest magnitude, an exact tie to the even k. A zero
// is stored with sign 0. The scoring then reads these values exactly (a
// 256-byte bf16 row becomes 64 bytes of codes and 8 bytes of exponents).
//
// Layout (zha_fp4_tree_bytes): the code of tree element i (the tree's element
// order) in byte i / 2, the low nibble for even i; from byte codes_bytes =
// round_up(tree_elems / 2, 256) on, the exponent of block i / 32 as an int16
// at codes_bytes + 2 (i / 32).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "zha_device.cuh"
#include "zha_internal.h"

namespace zha {
namespace {

constexpr int kQThreads = 256;

struct Fp4Params {
  const void* tree;
  unsigned char* codes;
  int16_t* exps;
  const int32_t* seq_len;
  const int32_t* old_len;  // nullable: every complete node
  int64_t ncap;
  int Hkv, L;
  int64_t span[kMaxLevels + 1];
  int64_t level_off[kMaxLevels];
  int64_t level_rows[kMaxLevels];
};

__device__ __forceinline__ int64_t clamp_len(int64_t n, int64_t ncap) {
  return n < 0 ? 0 : (n > ncap ? ncap : n);
}

// The e2m1 index of a = |x| / 2^e (0 <= a <= 6): the number of midpoints
// between consecutive magnitudes below a, an exact tie going to the even k.
__device__ __forceinline__ uint32_t e2m1_index(float a) {
  uint32_t k = (a > 0.25f) + (a > 0.75f) + (a > 1.25f) + (a > 1.75f) + (a > 2.5f) + (a > 3.5f) +
               (a > 5.0f);
  const float mid = k < 4u ? __fmaf_rn(0.5f, (float)k, 0.25f) : (k == 4u ? 2.5f : (k == 5u ? 3.5f : 5.0f));
  if (k < 7u && a == mid && (k & 1u)) ++k;
  return k;
}

// One thread per (row, 32-element block) of the nodes to quantize, all levels
// in one launch (levels are independent here: each reads stored rows only).
template <typename T, int D>
__global__ void __launch_bounds__(kQThreads) fp4_quantize_kernel(const __grid_constant__ Fp4Params p) {
  constexpr int kBlocks = D / 32;
  constexpr int kPer = Elem<T>::kPerChunk;
  const int unit = blockIdx.y;
  const int seq = unit / p.Hkv;
  const int64_t n_new = clamp_len(p.seq_len[seq], p.ncap);
  int64_t n_old = p.old_len ? clamp_len(p.old_len[seq], p.ncap) : 0;
  if (n_old > n_new) n_old = n_new;
  for (int level = 1; level <= p.L; ++level) {
    const int64_t lo = n_old / p.span[level], hi = n_new / p.span[level];
    const int64_t e0 = p.level_off[level - 1] + (int64_t)unit * p.level_rows[level - 1] * D;
    const int64_t n_blk = (hi - lo) * kBlocks;
    for (int64_t i = (int64_t)blockIdx.x * kQThreads + threadIdx.x; i < n_blk;
         i += (int64_t)gridDim.x * kQThreads) {
      const int64_t elem = e0 + (lo + i / kBlocks) * D + (i % kBlocks) * 32;
      const uint4* src = reinterpret_cast<const uint4*>(static_cast<const T*>(p.tree) + elem);
      float x[32];
#pragma unroll
      for (int c = 0; c < 32 / kPer; ++c) Elem<T>::unpack(__ldcg(src + c), x + c * kPer);
      float amax = 0.0f;
#pragma unroll
      for (int j = 0; j < 32; ++j) amax = fmaxf(amax, fabsf(x[j]));
      int e = 0;
      if (amax > 0.0f) {  // amax = m 2^E, m in [0.5, 1); 6 2^e = 0.75 2^(e + 3)
        int E = 0;
        const float m = frexpf(amax, &E);
        e = m <= 0.75f ? E - 3 : E - 2;
      }
      uint32_t w[4] = {0u, 0u, 0u, 0u};
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const uint32_t k = e2m1_index(ldexpf(fabsf(x[j]), -e));  // exact scaling
        const uint32_t nib = k | (k && x[j] < 0.0f ? 8u : 0u);
        w[j >> 3] |= nib << (4 * (j & 7));
      }
      *reinterpret_cast<uint4*>(p.codes + elem / 2) = make_uint4(w[0], w[1], w[2], w[3]);
      p.exps[elem / 32] = (int16_t)e;
    }
  }
}

template <typename T, int D>
cudaError_t launch_q(const Fp4Params& p, int units, int sms, cudaStream_t s) {
  int per = 4 * sms / units;  // a few CTAs per SM in total
  if (per < 1) per = 1;
  fp4_quantize_kernel<T, D><<<dim3((unsigned)per, (unsigned)units), kQThreads, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace

size_t fp4_codes_bytes(const Geometry& g) { return ((size_t)g.tree_elems / 2 + 255) & ~(size_t)255; }

size_t fp4_tree_bytes(const Geometry& g) {
  return fp4_codes_bytes(g) + sizeof(int16_t) * ((size_t)g.tree_elems / 32);
}

cudaError_t launch_fp4_quantize(const Geometry& g, const void* tree, void* fp4,
                                const int32_t* seq_len, const int32_t* old_len, int num_sms,
                                cudaStream_t stream) {
  Fp4Params p{};
  p.tree = tree;
  p.codes = static_cast<unsigned char*>(fp4);
  p.exps = reinterpret_cast<int16_t*>(static_cast<unsigned char*>(fp4) + fp4_codes_bytes(g));
  p.seq_len = seq_len;
  p.old_len = old_len;
  p.ncap = g.ncap;
  p.Hkv = g.Hkv;
  p.L = g.L;
  for (int l = 0; l <= g.L; ++l) p.span[l] = g.span[l];
  for (int l = 0; l < g.L; ++l) {
    p.level_off[l] = g.level_off[l];
    p.level_rows[l] = g.level_rows[l];
  }
  const int units = g.B * g.Hkv;
  if (g.dtype == ZHA_BF16)
    return g.d == 128 ? launch_q<__nv_bfloat16, 128>(p, units, num_sms, stream)
                      : launch_q<__nv_bfloat16, 64>(p, units, num_sms, stream);
  return g.d == 128 ? launch_q<float, 128>(p, units, num_sms, stream)
                    : launch_q<float, 64>(p, units, num_sms, stream);
}

}  // namespace zha
