// Prefill top-level node scoring on the 5th-generation tensor cores, with a
// certificate that the tensor-core scores select exactly what the canonical
// fp32 scores select.
//
// lefilia.fr page "Zyphra presente Zyphra Hierarchical Attention (ZHA) ...",
// paragraph 1: a query scores the top nodes first. In a prefill chunk every
// (token, query head) of a KV head scores the same top-level summaries, so the
// top level is one GEMM per KV head: Z = Q S_top^T with M = tokens x query
// heads of the group, N = top nodes, K = head_dim.
//
// 1. top_norms_kernel: |s_i| of every top summary (fp64 sum of squares).
// 2. top_score_tc_kernel: one CTA per 128-row M tile x 256-column N tile of one
//    KV head. bf16 A (query rows) and B (summaries) tiles are staged in shared
//    memory, K-major with the 128-byte swizzle; one thread issues tcgen05.mma
//    (kind::f16, fp32 accumulation in TMEM, M = 128, N <= 256, K = 16 per
//    instruction) and commits to an mbarrier; four warps read the accumulator
//    back with tcgen05.ld and write z~ = fl(fl(acc * inv_sqrt_d) + ln|node|).
//    The completion wait is bounded (1 s): on a timeout the kernel reports
//    ZHA_ERR_TIMEOUT, waits once more (bounded) for its MMAs, frees TMEM and
//    marks the chunk's scores invalid, so no unit is certified.
// 3. top_certify_kernel: one warp per (token, query head), one CTA per
//    (token, KV head). The tensor core sums the exact bf16 products in its own
//    order, the canonical path in a sequential fmaf chain; both are within
//    d 2^-24 (canonical) and 2 d 2^-24 (tensor core, truncating adds) of the
//    exact dot, relative to sum |q_k s_k| <= |q| |s| (Cauchy-Schwarz). With a
//    safety factor 4 on the accumulation and on the two rounded epilogue
//    operations:
//        |z~_i - z_i| <= delta_i = 12 d 2^-24 inv_sqrt_d |q| |s_i|
//                                  + 2^-21 (2 |z~_i| + ln|node| + 1).
//    The warp picks a candidate set K (top nodes by z~ whose fp64 softmax mass
//    first reaches p) and proves that the canonical cut selects exactly K for
//    every score vector in the box z~ +- delta:
//      (i)   separation: min over K of (z~ - delta) > max outside K of (z~ + delta),
//            so K is the canonical top-|K| set and no tie crosses its border;
//      (ii)  cover: the fixed-point mass of K reaches need = ceil(T p_q / 2^32);
//      (iii) minimality: K without its lowest member stays below need.
//    (ii) and (iii) are checked in fp64 against lower and upper bounds of every
//    fixed-point mass M_i = trunc(exp_c(fl(z_i - zmax)) 2^40): the exp_c
//    relative error (2^-20), the rounding of the subtraction, the truncation
//    and the unknown zmax are all bounded, and an fp64 summation slack is
//    added. A (token, KV head) unit is certified when all of its heads are;
//    the traversal then takes K as the top level's selection and starts one
//    level lower. Uncertified units are scored canonically.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdlib>

#include "zha_device.cuh"
#include "zha_internal.h"

namespace zha {
namespace {

constexpr int kTileM = 128;
constexpr int kTileN = 256;
constexpr int kTcThreads = 128;
constexpr uint32_t kTmemCols = 256;
constexpr int kTcD = 128;                  // head_dim of the tensor-core path
constexpr long long kMbarSpin = 1ll << 24; // iteration cap of the MMA completion wait
constexpr unsigned long long kWaitNs = 1000000000ull;  // and its time limit (1 s)
constexpr int kCertPer = 32;               // top nodes per lane in the certifier
constexpr int kTopCapMax = 32 * kCertPer;  // top nodes per unit on this path

__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// Shared-memory matrix descriptor of a K-major tile with the 128-byte
// swizzle: rows of 128 bytes (64 bf16), 8-row groups 1024 bytes apart. A K
// step of 16 elements inside the 128-byte row advances the start by 32 bytes.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3fffu);  // start address, 16-byte units
  d |= (uint64_t)1u << 16;                  // leading byte offset (unused with this swizzle)
  d |= (uint64_t)(1024u >> 4) << 32;        // stride byte offset: next 8-row group
  d |= (uint64_t)1u << 46;                  // descriptor version of sm_100
  d |= (uint64_t)2u << 61;                  // 128-byte swizzle
  return d;
}

// Instruction descriptor of kind::f16: bf16 A and B, fp32 accumulator, both
// operands K-major, shape M x N.
__host__ __device__ constexpr uint32_t mma_idesc(int M, int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) |
         ((uint32_t)(M >> 4) << 24);
}

// Byte offset of 16-byte chunk c (0..15) of row r in a K-major SW128 tile of
// `rows` rows stored as two 64-element K halves of rows x 128 bytes each.
__device__ __forceinline__ uint32_t sw128_offset(int r, int c, int rows) {
  const int half = c >> 3, cc = c & 7;
  return (uint32_t)(half * rows * 128 + (r >> 3) * 1024 + (r & 7) * 128 + ((cc ^ (r & 7)) << 4));
}

// |s_i| of every top-level summary of the sequence, per KV head: snorm[kvh][i].
// It also sets *tc_valid = 1 ahead of the scoring kernel, which clears it if a
// completion wait gives up.
__global__ void top_norms_kernel(const __nv_bfloat16* top, int64_t top_stride, int64_t n_top,
                                 int64_t cap, int Hkv, float* snorm, int32_t* tc_valid) {
  if (blockIdx.x == 0 && threadIdx.x == 0) *tc_valid = 1;
  const int64_t w = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (w >= (int64_t)Hkv * cap) return;
  const int kvh = (int)(w / cap);
  const int64_t i = w % cap;
  double ss = 0.0;
  if (i < n_top) {
    const __nv_bfloat16* row = top + kvh * top_stride + i * kTcD;
    for (int k = lane; k < kTcD; k += 32) {
      const double v = (double)__bfloat162float(row[k]);
      ss += v * v;
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
  // rounded up: the bound only ever needs an upper estimate of the norm
  if (lane == 0) snorm[w] = (float)(sqrt(ss) * (1.0 + 0x1p-20));
}

// z~ of one KV head's M tile against one N tile of top summaries. Rows of a
// KV head: row r is token r / G, query head kvh * G + r % G. zt is
// [Hkv][rows][zt_stride] with zt_stride a multiple of 4.
__global__ void __launch_bounds__(kTcThreads, 1)
    top_score_tc_kernel(const __nv_bfloat16* q, int64_t rows, int Hq, int G,
                        const __nv_bfloat16* top, int64_t top_stride, int64_t n_top,
                        float inv_sqrt_d, float lnsize, float* zt, int64_t zt_stride,
                        int32_t* status, int32_t* tc_valid, uint32_t wait_parity) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  // tiles on 1024-byte boundaries: the swizzle pattern repeats every 1024 bytes
  unsigned char* base = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  unsigned char* sa = base;                         // A: 128 rows x 256 bytes
  unsigned char* sb = base + kTileM * kTcD * 2;     // B: 256 rows x 256 bytes
  uint64_t* mbar = reinterpret_cast<uint64_t*>(sb + kTileN * kTcD * 2);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mbar + 1);
  int* done_flag = reinterpret_cast<int*>(tmem_slot + 1);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int kvh = blockIdx.z;
  const int64_t m0 = (int64_t)blockIdx.x * kTileM, n0 = (int64_t)blockIdx.y * kTileN;
  const int n_here = (int)(n_top - n0 < kTileN ? n_top - n0 : kTileN);
  const int n_mma = (n_here + 15) / 16 * 16;  // N of the MMA: a multiple of 16

  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(
                     smem_addr(tmem_slot)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
    asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
  }
  if (tid == 0) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;\n" ::"r"(smem_addr(mbar)) : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  }
  // stage A and B; rows past the valid ones are zero
  constexpr int kChunks = kTcD * 2 / 16;  // 16-byte chunks per row
  for (int e = tid; e < kTileM * kChunks; e += kTcThreads) {
    const int r = e / kChunks, c = e % kChunks;
    const int64_t row = m0 + r;
    unsigned char* dst = sa + sw128_offset(r, c, kTileM);
    if (row < rows) {
      const int64_t tok = row / G, h = (int64_t)kvh * G + row % G;
      cp_async16(dst, reinterpret_cast<const unsigned char*>(q + (tok * Hq + h) * kTcD) + c * 16);
    } else {
      *reinterpret_cast<uint4*>(dst) = make_uint4(0u, 0u, 0u, 0u);
    }
  }
  const __nv_bfloat16* topk = top + kvh * top_stride;
  for (int e = tid; e < kTileN * kChunks; e += kTcThreads) {
    const int r = e / kChunks, c = e % kChunks;
    unsigned char* dst = sb + sw128_offset(r, c, kTileN);
    if (r < n_here) {
      cp_async16(dst, reinterpret_cast<const unsigned char*>(topk + (n0 + r) * kTcD) + c * 16);
    } else {
      *reinterpret_cast<uint4*>(dst) = make_uint4(0u, 0u, 0u, 0u);
    }
  }
  cp_async_commit();
  cp_async_wait<0>();
  // the generic-proxy writes become visible to the tensor core (async proxy)
  asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
  const uint32_t tmem = *tmem_slot;

  if (tid == 0) {
    const uint32_t idesc = mma_idesc(kTileM, n_mma);
#pragma unroll
    for (int k = 0; k < kTcD / 16; ++k) {
      const uint32_t koff = (uint32_t)(k & 3) * 32u;  // K step inside the 128-byte row
      const uint64_t da = sw128_desc(smem_addr(sa + (k >> 2) * kTileM * 128) + koff);
      const uint64_t db = sw128_desc(smem_addr(sb + (k >> 2) * kTileN * 128) + koff);
      const uint32_t accumulate = k > 0 ? 1u : 0u;
      asm volatile(
          "{\n\t.reg .pred p;\n\t"
          "setp.ne.b32 p, %4, 0;\n\t"
          "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t"
          "}\n" ::"r"(tmem),
          "l"(da), "l"(db), "r"(idesc), "r"(accumulate)
          : "memory");
    }
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(
            smem_addr(mbar))
        : "memory");
    // bounded wait (time and iterations) for the completion phase of the
    // barrier. wait_parity is 0; a test sets 1, a phase that never completes,
    // to run the timeout path without any fault
    auto wait_mma = [&](uint32_t parity) -> int {
      const unsigned long long t0 = global_ns();
      int ok = 0;
      for (long long it = 0; it < kMbarSpin && !ok; ++it) {
        uint32_t r;
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.b32 %0, 1, 0, p;\n\t"
            "}\n"
            : "=r"(r)
            : "r"(smem_addr(mbar)), "r"(parity)
            : "memory");
        ok = (int)r;
        if (!ok && global_ns() - t0 > kWaitNs) break;
      }
      return ok;
    };
    const int ok = wait_mma(wait_parity);
    if (!ok) {
      raise_status(status, ZHA_ERR_TIMEOUT);
      *tc_valid = 0;  // the certifier then certifies nothing: canonical top level
      // a second bounded wait for the MMAs in flight before TMEM is freed
      (void)wait_mma(0u);
    }
    *done_flag = ok;
  }
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
  if (*done_flag) {
    // warp w owns TMEM lanes (rows) 32w .. 32w+31; 32 columns per load
    const int64_t row = m0 + warp * 32 + lane;
    float* out = zt + ((int64_t)kvh * rows + row) * zt_stride + n0;
    for (int cb = 0; cb < n_mma; cb += 32) {
      uint32_t v[32];
      const uint32_t taddr = tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)cb;
      asm volatile(
          "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
          "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
          "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n"
          : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
            "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]),
            "=r"(v[13]), "=r"(v[14]), "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]),
            "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]),
            "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]),
            "=r"(v[31])
          : "r"(taddr)
          : "memory");
      asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory");
      if (row < rows) {
        float z[32];
#pragma unroll
        for (int j = 0; j < 32; ++j)
          z[j] = __fadd_rn(__fmul_rn(__uint_as_float(v[j]), inv_sqrt_d), lnsize);
        if (cb + 32 <= n_here) {
#pragma unroll
          for (int j = 0; j < 8; ++j)
            reinterpret_cast<float4*>(out + cb)[j] =
                make_float4(z[4 * j], z[4 * j + 1], z[4 * j + 2], z[4 * j + 3]);
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (cb + j < n_here) out[cb + j] = z[j];
        }
      }
    }
  }
  asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
  __syncthreads();
  if (warp == 0)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem),
                 "r"(kTmemCols)
                 : "memory");
}

struct CertParams {
  const float* zt;          // [Hkv][rows][zt_stride] tensor-core scores
  int64_t zt_stride, rows;  // rows = tokens * G
  const float* snorm;       // [Hkv][cap] |s_i|, rounded up
  const __nv_bfloat16* q;   // [tokens][Hq][128]
  const int32_t* seq_len;
  int seq;
  int64_t pos0;             // position of the chunk's first token
  int64_t ncap, span_top, cap;
  int Hq, Hkv, G;
  float inv_sqrt_d, lns;
  uint64_t p_q;
  int32_t* ok;              // [tokens * Hkv]
  uint8_t* mask;            // [tokens * Hkv][cap]
  int32_t* cnt;             // [tokens * Hkv][G]
  float* z_out;             // nullable: [tokens][Hq][cap]
  int32_t* cert_out;        // nullable: [tokens][Hq]
  const int32_t* tc_valid;  // 0: a scoring wait gave up, the scores are not to be used
};

__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  return v;
}
__device__ __forceinline__ double warp_min_d(double v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v = fmin(v, __shfl_xor_sync(0xffffffffu, v, off));
  return v;
}
__device__ __forceinline__ double warp_max_d(double v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v = fmax(v, __shfl_xor_sync(0xffffffffu, v, off));
  return v;
}
__device__ __forceinline__ float warp_sum_f(float v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  return v;
}

// One CTA of G warps per (token, KV head) unit; warp h certifies query head h.
// PER top nodes per lane: the unit's top level holds at most 32 PER nodes.
template <int PER>
__global__ void __launch_bounds__(32 * kMaxGroup) top_certify_kernel(CertParams p) {
  __shared__ uint32_t kbits[kTopCapMax / 4];  // byte i: heads keeping top node i
  __shared__ int all_ok;
  const int64_t u = blockIdx.x;
  const int64_t i = u / p.Hkv;
  const int kvh = (int)(u % p.Hkv);
  const int h = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // complete top nodes visible to this token (the traversal's clamping)
  int64_t nseq = p.seq_len[p.seq];
  if (nseq > p.ncap) nseq = p.ncap;
  int64_t t = p.pos0 + i;
  if (t > nseq - 1) t = nseq - 1;
  int64_t nt = (t + 1) / p.span_top;
  if (nt > p.cap) nt = p.cap;
  const int n = (int)nt;
  for (int e = threadIdx.x; e < kTopCapMax / 4; e += blockDim.x) kbits[e] = 0u;
  if (threadIdx.x == 0) all_ok = n > 0 ? 1 : 0;
  __syncthreads();

  const int qh = kvh * p.G + h;
  // |q| (exact products, fp64 sum), rounded up
  const __nv_bfloat16* qrow = p.q + (i * p.Hq + qh) * kTcD;
  double qq = 0.0;
  for (int k = lane; k < kTcD; k += 32) {
    const double v = (double)__bfloat162float(qrow[k]);
    qq += v * v;
  }
  const double qn = sqrt(warp_sum_d(qq)) * (1.0 + 0x1p-20);
  const double cdot = 12.0 * kTcD * 0x1p-24 * (double)p.inv_sqrt_d * qn;
  const float* zrow = p.zt + ((int64_t)kvh * p.rows + i * p.G + h) * p.zt_stride;
  const float* sn = p.snorm + (int64_t)kvh * p.cap;

  // scores and their error bounds, 32 nodes per lane at most
  float zv[PER], dl[PER];
  bool finite = true;
  float zm = -INFINITY;
#pragma unroll
  for (int j = 0; j < PER; ++j) {
    const int idx = lane + 32 * j;
    zv[j] = -INFINITY;
    dl[j] = 0.0f;
    if (idx < n) {
      const float z = zrow[idx];
      finite = finite && isfinite(z);
      zv[j] = z;
      const double d =
          cdot * (double)sn[idx] + 0x1p-21 * (2.0 * fabs((double)z) + (double)p.lns + 1.0);
      dl[j] = (float)(d * (1.0 + 0x1p-20));
      zm = fmaxf(zm, z);
    }
  }
  finite = __all_sync(0xffffffffu, finite);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) zm = fmaxf(zm, __shfl_xor_sync(0xffffffffu, zm, off));

  const bool keep_all = p.p_q >= (1ull << 32);
  const double pr = (double)p.p_q * 0x1p-32;
  // scores of a chunk whose scoring wait gave up are not used: no certificate
  const bool tc_ok = n > 0 && *p.tc_valid != 0;
  bool cert = keep_all && tc_ok;
  uint32_t tau = 0u;  // candidate set: nodes whose order key is >= tau
  if (!keep_all && finite && tc_ok) {
    // the smallest descending prefix whose softmax mass reaches p (approximate:
    // only the certificate below has to be exact)
    float w[PER];
    float tot = 0.0f;
#pragma unroll
    for (int j = 0; j < PER; ++j) {
      w[j] = lane + 32 * j < n ? expf(zv[j] - zm) : 0.0f;
      tot += w[j];
    }
    const float target = (float)pr * warp_sum_f(tot);
    for (int bit = 31; bit >= 0; --bit) {
      const uint32_t cand = tau | (1u << bit);
      float s = 0.0f;
#pragma unroll
      for (int j = 0; j < PER; ++j) s += order_key(zv[j]) >= cand ? w[j] : 0.0f;
      if (warp_sum_f(s) >= target) tau = cand;  // identical on every lane
    }
    // the certificate, in fp64
    double zr = -INFINITY;
#pragma unroll
    for (int j = 0; j < PER; ++j)
      if (lane + 32 * j < n) zr = fmax(zr, (double)zv[j] + (double)dl[j]);
    zr = warp_max_d(zr);
    const double eta = 0x1p-20;  // relative error bound of exp_c
    int kk = 0;
    double min_a_k = INFINITY, max_b_r = -INFINITY;
    double s_ka = 0.0, s_kb = 0.0, m_ka = INFINITY, s_rb = 0.0, s_ra = 0.0;
#pragma unroll
    for (int j = 0; j < PER; ++j) {
      if (lane + 32 * j >= n) continue;
      const double a = (double)zv[j] - (double)dl[j], b = (double)zv[j] + (double)dl[j];
      // |fl(z - zmax) - (z - zmax)| <= 2^-24 (zr - a): mass factor bounds
      const double x = 0x1p-24 * (zr - a);
      const double lo = (1.0 - eta) * (1.0 - x), hi = (1.0 + eta) * (1.0 + x + x * x);
      const double ea = exp(a - zr) * lo, eb = exp(b - zr) * hi;
      if (order_key(zv[j]) >= tau) {
        ++kk;
        min_a_k = fmin(min_a_k, a);
        s_ka += ea;
        s_kb += eb;
        m_ka = fmin(m_ka, ea);
      } else {
        max_b_r = fmax(max_b_r, b);
        s_rb += eb;
        s_ra += ea;
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) kk += __shfl_xor_sync(0xffffffffu, kk, off);
    min_a_k = warp_min_d(min_a_k);
    max_b_r = warp_max_d(max_b_r);
    m_ka = warp_min_d(m_ka);
    s_ka = warp_sum_d(s_ka);
    s_kb = warp_sum_d(s_kb);
    s_rb = warp_sum_d(s_rb);
    s_ra = warp_sum_d(s_ra);
    const int rr = n - kk;
    const bool sep = rr == 0 || min_a_k > max_b_r;
    // cover: (1 - p) S_K - p S_R >= 1 for every mass vector in the box
    const double ha = (1.0 - pr) * s_ka - pr * s_rb;
    const double slack_a = 0x1p-36 * ((1.0 - pr) * s_ka + pr * s_rb);
    const bool cover = rr == 0 || ha - slack_a >= (1.0 + (1.0 - pr) * kk) * 0x1p-40;
    // minimality: (1 - p) S_K - M_last - p S_R < 0 for every mass vector
    const double hb = (1.0 - pr) * s_kb - m_ka - pr * s_ra;
    const double slack_b = 0x1p-36 * ((1.0 - pr) * s_kb + m_ka + pr * s_ra);
    const bool minimal = hb + slack_b <= -(1.0 + pr * rr) * 0x1p-40;
    cert = sep && cover && minimal;
  }
  int kept = 0;
#pragma unroll
  for (int j = 0; j < PER; ++j) {
    const int idx = lane + 32 * j;
    if (idx < n && (keep_all || order_key(zv[j]) >= tau)) {
      atomicOr(&kbits[idx >> 2], 1u << (8 * (idx & 3) + h));
      ++kept;
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) kept += __shfl_xor_sync(0xffffffffu, kept, off);
  if (lane == 0) {
    p.cnt[u * p.G + h] = kept;
    if (!cert) all_ok = 0;
    if (p.cert_out) p.cert_out[i * p.Hq + qh] = cert ? 1 : 0;
  }
  if (p.z_out) {
    float* zo = p.z_out + (i * p.Hq + qh) * p.cap;
#pragma unroll
    for (int j = 0; j < PER; ++j)
      if (lane + 32 * j < n) zo[lane + 32 * j] = zv[j];
  }
  __syncthreads();
  const bool ok = all_ok != 0;
  if (ok)
    for (int idx = threadIdx.x; idx < n; idx += blockDim.x)
      p.mask[u * p.cap + idx] = (uint8_t)((kbits[idx >> 2] >> (8 * (idx & 3))) & 0xffu);
  if (threadIdx.x == 0) p.ok[u] = ok ? 1 : 0;
}

}  // namespace

int64_t top_cap(const Geometry& g) { return g.level_rows[g.L - 1]; }

bool top_tc_supported(const Geometry& g) {
  return g.dtype == ZHA_BF16 && g.d == kTcD && g.L >= 2 && g.G >= 1 && g.G <= kMaxGroup &&
         top_cap(g) >= 1 && top_cap(g) <= kTopCapMax;
}

namespace {

struct TopLayout {
  size_t snorm, zt, ok, cnt, mask, valid, total;
  int64_t zs;  // row stride of the score buffer (floats)
};

size_t align256_(size_t x) { return (x + 255) & ~(size_t)255; }

TopLayout top_layout(const Geometry& g, int64_t n_tok) {
  TopLayout T{};
  const int64_t cap = top_cap(g);
  T.zs = (cap + 31) / 32 * 32;
  size_t off = 0;
  T.snorm = off;
  off = align256_(off + sizeof(float) * (size_t)g.Hkv * cap);
  T.zt = off;
  off = align256_(off + sizeof(float) * (size_t)g.Hkv * n_tok * g.G * T.zs);
  T.ok = off;
  off = align256_(off + sizeof(int32_t) * (size_t)n_tok * g.Hkv);
  T.cnt = off;
  off = align256_(off + sizeof(int32_t) * (size_t)n_tok * g.Hkv * g.G);
  T.mask = off;
  off = align256_(off + (size_t)n_tok * g.Hkv * cap);
  T.valid = off;
  off = align256_(off + sizeof(int32_t));
  T.total = off;
  return T;
}

size_t top_score_tc_smem() {
  // A and B tiles, barrier, TMEM address and flag, and the 1024-byte alignment slack
  return (size_t)kTileM * kTcD * 2 + (size_t)kTileN * kTcD * 2 + 16 + 1024;
}

}  // namespace

size_t top_tc_ws_bytes(const Geometry& g, int64_t n_tok) {
  return top_tc_supported(g) ? top_layout(g, n_tok).total : 0;
}

cudaError_t launch_top_select(const Geometry& g, const void* tree, const int32_t* seq_len,
                              int seq, const void* q, int64_t pos0, int64_t n_tok, uint64_t p_q,
                              void* ws, size_t ws_bytes, TopSeeds* seeds, float* z_out,
                              int32_t* cert_out, int32_t* status, cudaStream_t stream) {
  if (!top_tc_supported(g) || n_tok < 1 || !seeds) return cudaErrorInvalidValue;
  const TopLayout T = top_layout(g, n_tok);
  if (ws_bytes < T.total) return cudaErrorInvalidValue;
  const int64_t cap = top_cap(g);
  // the GEMM's N: top nodes the chunk's last token can see (the certifier
  // applies each token's own count)
  int64_t n_top = (pos0 + n_tok) / g.span[g.L];
  if (n_top > cap) n_top = cap;
  unsigned char* w = static_cast<unsigned char*>(ws);
  float* snorm = reinterpret_cast<float*>(w + T.snorm);
  float* zt = reinterpret_cast<float*>(w + T.zt);
  int32_t* ok = reinterpret_cast<int32_t*>(w + T.ok);
  int32_t* cnt = reinterpret_cast<int32_t*>(w + T.cnt);
  uint8_t* mask = reinterpret_cast<uint8_t*>(w + T.mask);
  int32_t* tc_valid = reinterpret_cast<int32_t*>(w + T.valid);
  // test hook: ZHA_TEST_TC_WAIT_PARITY=1 makes the scoring kernel wait for a
  // barrier phase that never completes, so its bounded wait runs out (the
  // MMAs themselves complete); the call then reports ZHA_ERR_TIMEOUT and the
  // top level falls back to canonical scoring
  const char* hook = getenv("ZHA_TEST_TC_WAIT_PARITY");
  const uint32_t wait_parity = (hook && hook[0] == '1') ? 1u : 0u;
  seeds->ok = ok;
  seeds->mask = mask;
  seeds->cnt = cnt;
  seeds->stride = cap;
  const int64_t rows = n_tok * g.G;
  const int64_t top_stride = cap * kTcD;  // elements between KV heads' top levels
  const __nv_bfloat16* top = static_cast<const __nv_bfloat16*>(tree) + g.level_off[g.L - 1] +
                             (int64_t)seq * g.Hkv * top_stride;
  if (n_top > 0) {
    const int64_t warps = (int64_t)g.Hkv * cap;
    top_norms_kernel<<<(unsigned)((warps * 32 + 255) / 256), 256, 0, stream>>>(
        top, top_stride, n_top, cap, g.Hkv, snorm, tc_valid);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const size_t smem = top_score_tc_smem();
    e = cudaFuncSetAttribute(top_score_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)((rows + kTileM - 1) / kTileM), (unsigned)((n_top + kTileN - 1) / kTileN),
              (unsigned)g.Hkv);
    top_score_tc_kernel<<<grid, kTcThreads, smem, stream>>>(
        static_cast<const __nv_bfloat16*>(q), rows, g.Hq, g.G, top, top_stride, n_top,
        g.inv_sqrt_d, g.lnsize[g.L - 1], zt, T.zs, status, tc_valid, wait_parity);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  CertParams c{};
  c.zt = zt;
  c.zt_stride = T.zs;
  c.rows = rows;
  c.snorm = snorm;
  c.q = static_cast<const __nv_bfloat16*>(q);
  c.seq_len = seq_len;
  c.seq = seq;
  c.pos0 = pos0;
  c.ncap = g.ncap;
  c.span_top = g.span[g.L];
  c.cap = cap;
  c.Hq = g.Hq;
  c.Hkv = g.Hkv;
  c.G = g.G;
  c.inv_sqrt_d = g.inv_sqrt_d;
  c.lns = g.lnsize[g.L - 1];
  c.p_q = p_q;
  c.ok = ok;
  c.mask = mask;
  c.cnt = cnt;
  c.z_out = z_out;
  c.cert_out = cert_out;
  c.tc_valid = tc_valid;
  const unsigned grid = (unsigned)(n_tok * g.Hkv), block = 32u * (unsigned)g.G;
  if (cap <= 32 * 4) top_certify_kernel<4><<<grid, block, 0, stream>>>(c);
  else if (cap <= 32 * 8) top_certify_kernel<8><<<grid, block, 0, stream>>>(c);
  else if (cap <= 32 * 16) top_certify_kernel<16><<<grid, block, 0, stream>>>(c);
  else top_certify_kernel<kCertPer><<<grid, block, 0, stream>>>(c);
  return cudaGetLastError();
}

}  // namespace zha
