// Device-side helpers shared by the libzha kernels (sm_100a).
//
// The "canonical" functions render the library's fixed fp32 arithmetic for
// the selection-deciding steps: every operation is an explicitly rounded
// intrinsic so that nvcc cannot contract or reassociate it.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace zha {

constexpr int kNRef = 16;         // reference queries per node summary
constexpr int kMaxLevels = 8;
constexpr int kMaxGroup = 8;      // query heads per KV head
constexpr int kMaxCluster = 16;   // CTAs cooperating on one traversal unit

// ---------------------------------------------------------------------------
// canonical arithmetic
// ---------------------------------------------------------------------------

// exp(x) for x <= 0. Cody-Waite range reduction x = n ln2 + r with
// n = rint(x * fp32(log2 e)), ln 2 split into a head with 12 trailing zero bits
// and a tail; degree-7 Taylor polynomial 1/k! in Horner form; scaling by the
// exact power 2^n. Returns 0 below -87 (W. J. Cody and W. Waite, "Software
// Manual for the Elementary Functions", 1980).
__device__ __forceinline__ float exp_canon(float x) {
  // branch-free, so that independent calls interleave; below -87 the result is
  // selected away (the scaling below would not be a valid power of two there)
  const bool zero = x < -87.0f;
  x = zero ? 0.0f : x;
  const float n = rintf(__fmul_rn(x, 0x1.715476p+0f));
  float r = __fmaf_rn(-n, 0x1.62e4p-1f, x);
  r = __fmaf_rn(-n, 0x1.7f7d1cp-20f, r);
  float p = 0x1.a01a02p-13f;
  p = __fmaf_rn(p, r, 0x1.6c16c2p-10f);
  p = __fmaf_rn(p, r, 0x1.111112p-7f);
  p = __fmaf_rn(p, r, 0x1.555556p-5f);
  p = __fmaf_rn(p, r, 0x1.555556p-3f);
  p = __fmaf_rn(p, r, 0.5f);
  p = __fmaf_rn(p, r, 1.0f);
  p = __fmaf_rn(p, r, 1.0f);
  const int ni = __float2int_rn(n);  // in [-126, 0]
  return zero ? 0.0f : __fmul_rn(p, __int_as_float((ni + 127) << 23));
}

// Fixed-point node mass trunc(exp(z - zmax) * 2^40).
__device__ __forceinline__ uint64_t mass_fixed(float z, float zmax) {
  return __float2ull_rz(__fmul_rn(exp_canon(__fsub_rn(z, zmax)), 0x1p40f));
}

// Order-preserving map of a float onto uint32 (larger float -> larger key).
__device__ __forceinline__ uint32_t order_key(float z) {
  const uint32_t u = __float_as_uint(z);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// ---------------------------------------------------------------------------
// top-p cut helpers (exact integer arithmetic and the score -> bucket maps)
// ---------------------------------------------------------------------------

constexpr int kCutDigit = 8;  // key bits resolved per radix pass (256 buckets)

// ceil(T * pq / 2^32) without overflow.
__device__ __forceinline__ unsigned long long ceil_mul_shift32(unsigned long long T,
                                                               unsigned long long pq) {
  const unsigned long long lo = T * pq;
  const unsigned long long hi = __umul64hi(T, pq);
  unsigned long long r = (hi << 32) | (lo >> 32);
  if (lo & 0xffffffffull) r += 1;
  return r;
}

// First-pass bucket of score z: a linear map of [zlo, zlo + 256 / zscale)
// onto 0..255, clamped. Non-decreasing in z, and evaluated with the same
// operations on every CTA.
__device__ __forceinline__ uint32_t quant_bucket(float z, float zlo, float zscale) {
  const float f = __fmul_rn(__fsub_rn(z, zlo), zscale);
  return (uint32_t)fminf(fmaxf(f, 0.0f), 255.0f);  // NaN (inf * 0) maps to 0
}

// Inverse of order_key.
__device__ __forceinline__ float key_float(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

// Smallest key in [lo, hi] whose first-pass bucket is >= beta; the bucket of
// key_float(hi) must be >= beta. Binary search over the key order.
__device__ __forceinline__ uint32_t quant_first_key(float zlo, float zscale, uint32_t beta,
                                                    uint32_t lo, uint32_t hi) {
  while (lo < hi) {
    const uint32_t mid = lo + (hi - lo) / 2;
    if (quant_bucket(key_float(mid), zlo, zscale) >= beta) hi = mid;
    else lo = mid + 1;
  }
  return lo;
}

// First key of bucket beta (beta >= 1): the search starts in a window of 512
// keys around the estimate zlo + beta / zscale and widens to the whole key
// range of the finite scores when the window does not bracket the boundary.
__device__ __forceinline__ uint32_t quant_boundary(float zlo, float zscale, uint32_t beta) {
  const uint32_t kneg = order_key(-INFINITY), kpos = order_key(INFINITY);
  const uint32_t ke = order_key(__fadd_rn(zlo, __fdiv_rn((float)beta, zscale)));
  uint32_t lo = ke > kneg + 256u ? ke - 256u : kneg;
  uint32_t hi = ke < kpos - 256u ? ke + 256u : kpos;
  if (lo < kneg || hi > kpos || lo > hi || quant_bucket(key_float(lo), zlo, zscale) >= beta ||
      quant_bucket(key_float(hi), zlo, zscale) < beta) {
    lo = kneg;
    hi = kpos;
  }
  return quant_first_key(zlo, zscale, beta, lo, hi);
}

// Key interval [*klo, *khi] of the finite scores whose first-pass bucket is
// beta (an interval, as the bucket map is non-decreasing in the score).
__device__ __forceinline__ void quant_interval(float zlo, float zscale, uint32_t beta,
                                               uint32_t* klo, uint32_t* khi) {
  *klo = beta == 0u ? order_key(-INFINITY) : quant_boundary(zlo, zscale, beta);
  *khi = beta >= 255u || zscale == 0.0f
             ? order_key(INFINITY)
             : quant_boundary(zlo, zscale, beta + 1u) - 1u;
}

// Digit width and position of a kModeRadix pass over the group [kgmin, kgmax]
// (kgmin < kgmax): the bits below the range's common prefix, 8 at a time.
__device__ __forceinline__ void radix_digit(unsigned kgmin, unsigned kgmax, int* sh, int* w) {
  const int shift = 32 - __clz(kgmin ^ kgmax);
  *w = shift < kCutDigit ? shift : kCutDigit;
  *sh = shift - *w;
}

// ---------------------------------------------------------------------------
// packed fp32x2 FMA (sm_100): two independent round-to-nearest FMAs, each
// bit-identical to __fmaf_rn on its lane.
// ---------------------------------------------------------------------------
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;"
      : "=l"(d)
      : "l"(*reinterpret_cast<uint64_t*>(&a)), "l"(*reinterpret_cast<uint64_t*>(&b)),
        "l"(*reinterpret_cast<uint64_t*>(&c)));
  return *reinterpret_cast<float2*>(&d);
}

__device__ __forceinline__ float2 fmul2(float2 a, float2 b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;"
      : "=l"(d)
      : "l"(*reinterpret_cast<uint64_t*>(&a)), "l"(*reinterpret_cast<uint64_t*>(&b)));
  return *reinterpret_cast<float2*>(&d);
}

// ---------------------------------------------------------------------------
// element types
// ---------------------------------------------------------------------------

// Two bf16 packed in a uint32 -> (low, high) as exact fp32.
__device__ __forceinline__ float2 bf16x2_to_f2(uint32_t w) {
  return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}

template <typename T>
struct Elem;

template <>
struct Elem<float> {
  static constexpr int kPerChunk = 4;  // elements per 16-byte chunk
  // unpack a 16-byte chunk into kPerChunk floats
  __device__ __forceinline__ static void unpack(const uint4& c, float* out) {
    out[0] = __uint_as_float(c.x);
    out[1] = __uint_as_float(c.y);
    out[2] = __uint_as_float(c.z);
    out[3] = __uint_as_float(c.w);
  }
  // pack kPerChunk floats into a 16-byte chunk
  __device__ __forceinline__ static uint4 pack(const float* v) {
    return make_uint4(__float_as_uint(v[0]), __float_as_uint(v[1]), __float_as_uint(v[2]),
                      __float_as_uint(v[3]));
  }
  __device__ __forceinline__ static float load(const float* p) { return *p; }
  __device__ __forceinline__ static float to_f(float v) { return v; }
  __device__ __forceinline__ static float from_f(float v) { return v; }
};

template <>
struct Elem<__nv_bfloat16> {
  static constexpr int kPerChunk = 8;
  __device__ __forceinline__ static void unpack(const uint4& c, float* out) {
    const float2 a = bf16x2_to_f2(c.x), b = bf16x2_to_f2(c.y), d = bf16x2_to_f2(c.z),
                 e = bf16x2_to_f2(c.w);
    out[0] = a.x; out[1] = a.y; out[2] = b.x; out[3] = b.y;
    out[4] = d.x; out[5] = d.y; out[6] = e.x; out[7] = e.y;
  }
  // round kPerChunk floats to nearest-even bf16 and pack them (element 0 in
  // the low half of the first word)
  __device__ __forceinline__ static uint4 pack(const float* v) {
    uint32_t w[4];
#pragma unroll
    for (int j = 0; j < 4; ++j)
      w[j] = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(v[2 * j])) |
             ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(v[2 * j + 1])) << 16);
    return make_uint4(w[0], w[1], w[2], w[3]);
  }
  __device__ __forceinline__ static float load(const __nv_bfloat16* p) {
    return __bfloat162float(*p);
  }
  __device__ __forceinline__ static float to_f(__nv_bfloat16 v) { return __bfloat162float(v); }
  __device__ __forceinline__ static __nv_bfloat16 from_f(float v) {
    return __float2bfloat16_rn(v);
  }
};

// ---------------------------------------------------------------------------
// async copies
// ---------------------------------------------------------------------------

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gmem_src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(smem_u32(smem_dst)),
               "l"(gmem_src)
               : "memory");
}

// 4-byte asynchronous copy (cached in L1 as well; sizes below 16 bytes take .ca)
__device__ __forceinline__ void cp_async4(void* smem_dst, const void* gmem_src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"(smem_u32(smem_dst)),
               "l"(gmem_src)
               : "memory");
}

__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;\n" ::: "memory");
}

template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

__device__ __forceinline__ uint4 lds128(const void* p) {
  return *reinterpret_cast<const uint4*>(p);
}

// 16-byte chunk index c of a staged row r lives at chunk (c ^ (r & 7)), which
// makes "one row per lane" reads of a fixed logical chunk conflict-free.
__device__ __forceinline__ int swz(int c, int r) { return c ^ (r & 7); }

// ---------------------------------------------------------------------------
// status reporting (never traps)
// ---------------------------------------------------------------------------
__device__ __forceinline__ void raise_status(int32_t* status, int32_t bit) {
  if (status) atomicOr(status, bit);
}

}  // namespace zha
