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
