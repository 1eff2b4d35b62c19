// Prefill attention over a tile of query tokens at once.
//
// lefilia.fr page "Zyphra presente Zyphra Hierarchical Attention (ZHA) ...",
// paragraph 1: each query attends the raw K/V entries under the nodes it kept,
// plus (by the causal reading) token 0 and the tail of tokens not yet in a
// complete top node:
//     o = sum_{j in S} softmax_j(q . k_j / sqrt(d)) v_j .
//
// In a prefill chunk consecutive tokens of one sequence keep nearly the same
// nodes, so instead of streaming each (token, KV head)'s kept rows separately
// (once per token), one CTA takes 16 tokens x 8 query heads = 128 query rows of
// one KV head and a range of keys: every 64-key K/V block is loaded once and
// serves all 128 rows through m16n8k16 bf16 tensor-core MMAs (fp32
// accumulation), and a per-(token, node) keep map masks the scores:
//   key j is attended by (token i, head h) iff j <= t_i and (j == 0, or j is in
//   i's tail [b^L T_top(t_i), t_i], or bit h of keep[i][j / b] is set).
// The selection comes from the traversal (its kept level-1 lists, scattered
// into the map); the arithmetic is that of the gather kernel: scores scaled by
// log2(e)/sqrt(d), exp2, P rounded to bf16 for P V, fp32 accumulators, split-K
// partials (m, l, acc) merged by a combine step.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "zha_device.cuh"
#include "zha_internal.h"

namespace zha {
namespace {

constexpr float kLog2eT = 1.4426950408889634f;
constexpr int kTD = 128;            // head_dim
constexpr int kTRows = 128;         // query rows per CTA
constexpr int kTWarps = 8;          // 16 rows each
constexpr int kTThreads = 32 * kTWarps;
constexpr int kTKB = 64;            // keys per block
constexpr int kTStages = 3;
constexpr int kTRowBytes = kTD * 2;
constexpr int kTKVBytes = kTKB * kTRowBytes;           // one K (or V) block: 16 KB
constexpr int kTMaskBytes = (kTRows / 2) * (kTKB / 2);  // tokens x nodes per block, b >= 2
constexpr int kTStageBytes = 2 * kTKVBytes + kTMaskBytes;

struct TileParams {
  const __nv_bfloat16* k;   // [B][Hkv][ncap][D]
  const __nv_bfloat16* v;
  const __nv_bfloat16* q;   // [n][Hq][D] (the tile)
  const int32_t* seq_len;
  int seq;
  int64_t pos0;             // position of the tile's first token
  int n;                    // tokens in the tile
  int64_t ncap;
  int Hq, Hkv, b, b_shift;
  int64_t span_L;
  float qscale;
  const uint8_t* keep;      // [Hkv][n][map_stride]
  int64_t map_stride;
  int S;                    // key splits
  float* part;              // [n * Hkv][S][G][D + 2]
};

__device__ __forceinline__ void ldsm4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                      uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void ldsm4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// C += A (16x16 bf16) * B (16x8 bf16), fp32 accumulate.
__device__ __forceinline__ void mma16816(float* c, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

__device__ __forceinline__ void cp_async4(void* dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"(smem_u32(dst)), "l"(src));
}

// Scatters the kept level-1 lists of the tile's units (unit = token * Hkv +
// KV head; `segs` ordered segments of `stride` entries each) into the keep
// map: keep[kvh][token][node] = head mask. The map was zeroed before.
__global__ void keep_scatter_kernel(const uint32_t* kept, const int32_t* n_kept, int64_t stride,
                                    int segs, int units, int Hkv, int n, uint8_t* keep,
                                    int64_t map_stride) {
  const int u = blockIdx.y;
  if (u >= units) return;
  const int i = u / Hkv, kvh = u % Hkv;
  uint8_t* row = keep + ((int64_t)kvh * n + i) * map_stride;
  for (int r = 0; r < segs; ++r) {
    const int64_t cnt = n_kept[(int64_t)u * segs + r];
    const uint32_t* src = kept + ((int64_t)u * segs + r) * stride;
    for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < cnt;
         e += (int64_t)gridDim.x * blockDim.x) {
      const uint32_t w = src[e];
      const int64_t node = w & 0x00ffffffu;
      if (node < map_stride) row[node] = (uint8_t)(w >> 24);
    }
  }
}

// One CTA: kTRows / G tokens x G heads of KV head blockIdx.z, key blocks of
// split blockIdx.y. Warp w owns rows 16w .. 16w + 15 (row r = token r / G,
// head r % G); each thread holds rows g and g + 8 of its warp's MMA tiles.
template <int G>
__global__ void __launch_bounds__(kTThreads, 1) attend_tile_kernel(TileParams p) {
  constexpr int kTok = kTRows / G;
  extern __shared__ __align__(128) unsigned char smem[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t4 = lane & 3;
  const int kvh = blockIdx.z, split = blockIdx.y;
  const int tok0 = blockIdx.x * kTok;
  int64_t nseq = p.seq_len[p.seq];
  if (nseq > p.ncap) nseq = p.ncap;
  const int ntok = p.n - tok0 < kTok ? p.n - tok0 : kTok;
  // positions of the CTA's tokens (clamped like the traversal's)
  int64_t kmax = p.pos0 + tok0 + ntok - 1;
  if (kmax > nseq - 1) kmax = nseq - 1;
  const int64_t nblk = kmax >= 0 ? (kmax + kTKB) / kTKB : 0;
  const int64_t blk0 = nblk * split / p.S, blk1 = nblk * (split + 1) / p.S;

  const int r0 = warp * 16 + g, r1 = r0 + 8;
  const int tl[2] = {r0 / G, r1 / G};
  const int hh[2] = {r0 % G, r1 % G};
  bool valid[2];
  int64_t tpos[2], tstart[2];
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    valid[k] = tok0 + tl[k] < p.n;
    int64_t t = p.pos0 + tok0 + tl[k];
    if (t > nseq - 1) t = nseq - 1;
    tpos[k] = valid[k] ? t : -1;
    tstart[k] = p.span_L * ((tpos[k] + 1) / p.span_L);
  }
  // the lowest tail start among the CTA's tokens (keys below it are decided by
  // the keep map alone, except key 0)
  int64_t tail_min;
  {
    int64_t t = p.pos0 + tok0;
    if (t > nseq - 1) t = nseq - 1;
    tail_min = ntok > 0 && t >= 0 ? p.span_L * ((t + 1) / p.span_L) : 0;
  }
  // Q fragments of rows g (a0, a2) and g + 8 (a1, a3), exact bf16 inputs
  uint32_t qa[kTD / 16][4];
  {
    const __nv_bfloat16* qr[2];
#pragma unroll
    for (int k = 0; k < 2; ++k)
      qr[k] = p.q + ((int64_t)(tok0 + tl[k]) * p.Hq + (int64_t)kvh * G + hh[k]) * kTD;
#pragma unroll
    for (int ks = 0; ks < kTD / 16; ++ks) {
      qa[ks][0] = valid[0] ? *reinterpret_cast<const uint32_t*>(qr[0] + ks * 16 + 2 * t4) : 0u;
      qa[ks][1] = valid[1] ? *reinterpret_cast<const uint32_t*>(qr[1] + ks * 16 + 2 * t4) : 0u;
      qa[ks][2] = valid[0] ? *reinterpret_cast<const uint32_t*>(qr[0] + ks * 16 + 8 + 2 * t4) : 0u;
      qa[ks][3] = valid[1] ? *reinterpret_cast<const uint32_t*>(qr[1] + ks * 16 + 8 + 2 * t4) : 0u;
    }
  }
  const int64_t kv_unit = (int64_t)p.seq * p.Hkv + kvh;
  const unsigned char* kbase = reinterpret_cast<const unsigned char*>(p.k + kv_unit * p.ncap * kTD);
  const unsigned char* vbase = reinterpret_cast<const unsigned char*>(p.v + kv_unit * p.ncap * kTD);
  const uint8_t* keep = p.keep + ((int64_t)kvh * p.n + tok0) * p.map_stride;
  const int npb = kTKB >> p.b_shift;  // nodes per key block: 32, 16, 8 or 4
  const int words = npb >> 2;

  // CTA-wide stage fill: K and V rows (zero past kmax) and the keep bytes
  auto issue = [&](int64_t kb, int st) {
    unsigned char* base = smem + st * kTStageBytes;
    if (kb < blk1) {
      const int64_t k0 = kb * kTKB;
      for (int e = tid; e < kTKB * (kTRowBytes / 16); e += kTThreads) {
        const int r = e >> 4, c = e & 15;
        const int64_t key = k0 + r;
        const int dst = r * kTRowBytes + (swz(c, r) << 4);
        if (key <= kmax) {
          cp_async16(base + dst, kbase + key * kTRowBytes + c * 16);
          cp_async16(base + kTKVBytes + dst, vbase + key * kTRowBytes + c * 16);
        } else {
          *reinterpret_cast<uint4*>(base + dst) = make_uint4(0u, 0u, 0u, 0u);
          *reinterpret_cast<uint4*>(base + kTKVBytes + dst) = make_uint4(0u, 0u, 0u, 0u);
        }
      }
      const int64_t node0 = k0 >> p.b_shift;
      for (int e = tid; e < kTok * words; e += kTThreads) {
        const int t = e / words, w = e % words;
        unsigned char* dst = base + 2 * kTKVBytes + t * (kTKB / 2) + w * 4;
        if (t < ntok) cp_async4(dst, keep + (int64_t)t * p.map_stride + node0 + w * 4);
        else *reinterpret_cast<uint32_t*>(dst) = 0u;
      }
    }
    cp_async_commit();
  };

  float o[kTD / 8][4];
#pragma unroll
  for (int nt = 0; nt < kTD / 8; ++nt) o[nt][0] = o[nt][1] = o[nt][2] = o[nt][3] = 0.0f;
  float m_run[2] = {-INFINITY, -INFINITY}, l_part[2] = {0.0f, 0.0f};

  int64_t kb_next = blk0;
#pragma unroll
  for (int st = 0; st < kTStages - 1; ++st) issue(kb_next++, st);
  int st = 0;
  for (int64_t kb = blk0; kb < blk1; ++kb) {
    issue(kb_next++, (st + kTStages - 1) % kTStages);
    cp_async_wait<kTStages - 1>();
    __syncthreads();
    const unsigned char* base = smem + st * kTStageBytes;
    const uint32_t kaddr = smem_u32(base), vaddr = smem_u32(base + kTKVBytes);
    const uint8_t* mk = base + 2 * kTKVBytes;
    // ---- S = Q K^T: 16 rows x 64 keys per warp (8 n-tiles) ----
    float sc[kTKB / 8][4];
#pragma unroll
    for (int nt = 0; nt < kTKB / 8; ++nt) {
      sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.0f;
      const int row = nt * 8 + (lane & 7);
#pragma unroll
      for (int ks = 0; ks < kTD / 16; ks += 2) {
        const int chunk = 2 * ks + (lane >> 3);
        uint32_t b0, b1, b2, b3;
        ldsm4(kaddr + row * kTRowBytes + swz(chunk, row) * 16, b0, b1, b2, b3);
        mma16816(sc[nt], qa[ks], b0, b1);
        mma16816(sc[nt], qa[ks + 1], b2, b3);
      }
    }
    // ---- selection mask, scale, online softmax (rows g and g + 8) ----
    // A thread's keys 2 t4 and 2 t4 + 1 of n-tile nt share one node (b >= 2):
    // one keep byte per (row, n-tile). Blocks past key 0 and below every
    // token's tail need nothing else; the others also test positions,
    // relative to the block start.
    const int64_t k0 = kb * kTKB;
    const bool plain = k0 > 0 && k0 + kTKB <= tail_min;
    float mb[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const uint8_t* mrow = mk + tl[k] * (kTKB / 2);
      const int lim = (int)(tpos[k] - k0 < kTKB ? tpos[k] - k0 : kTKB);      // last key <= t
      const int tst = (int)(tstart[k] - k0 < kTKB ? tstart[k] - k0 : kTKB);  // first tail key
#pragma unroll
      for (int nt = 0; nt < kTKB / 8; ++nt) {
        const bool keep = (mrow[(nt * 8 + 2 * t4) >> p.b_shift] >> hh[k]) & 1u;
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const int kk = nt * 8 + 2 * t4 + j;
          const bool ok = plain ? keep
                                : kk <= lim && (keep || kk >= tst || (k0 == 0 && kk == 0));
          const float s = ok ? sc[nt][2 * k + j] * p.qscale : -INFINITY;
          sc[nt][2 * k + j] = s;
          mb[k] = fmaxf(mb[k], s);
        }
      }
    }
    float alpha[2], mn[2];
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      mb[k] = fmaxf(mb[k], __shfl_xor_sync(0xffffffffu, mb[k], 1));
      mb[k] = fmaxf(mb[k], __shfl_xor_sync(0xffffffffu, mb[k], 2));
      mn[k] = fmaxf(m_run[k], mb[k]);
      alpha[k] = (mn[k] == -INFINITY) ? 1.0f : exp2f(m_run[k] - mn[k]);
      m_run[k] = mn[k];
    }
    float lsum[2] = {0.0f, 0.0f};
#pragma unroll
    for (int nt = 0; nt < kTKB / 8; ++nt) {
#pragma unroll
      for (int k = 0; k < 2; ++k) {
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const float pv = (mn[k] == -INFINITY) ? 0.0f : exp2f(sc[nt][2 * k + j] - mn[k]);
          sc[nt][2 * k + j] = pv;
          lsum[k] += pv;
        }
      }
    }
#pragma unroll
    for (int k = 0; k < 2; ++k) l_part[k] = l_part[k] * alpha[k] + lsum[k];
    // the accumulators need rescaling only after a row's maximum moved (rare
    // once a few blocks are in); multiplying by exactly 1 changes nothing
    if (!__all_sync(0xffffffffu, alpha[0] == 1.0f && alpha[1] == 1.0f)) {
#pragma unroll
      for (int nt = 0; nt < kTD / 8; ++nt) {
        o[nt][0] *= alpha[0];
        o[nt][1] *= alpha[0];
        o[nt][2] *= alpha[1];
        o[nt][3] *= alpha[1];
      }
    }
    // ---- O += P V: 4 k-steps of 16 keys x 16 n-tiles of 8 dims ----
#pragma unroll
    for (int ks = 0; ks < kTKB / 16; ++ks) {
      uint32_t pa[4];
      pa[0] = pack2(sc[2 * ks][0], sc[2 * ks][1]);
      pa[1] = pack2(sc[2 * ks][2], sc[2 * ks][3]);
      pa[2] = pack2(sc[2 * ks + 1][0], sc[2 * ks + 1][1]);
      pa[3] = pack2(sc[2 * ks + 1][2], sc[2 * ks + 1][3]);
      const int row = ks * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
      for (int nt = 0; nt < kTD / 8; nt += 2) {
        const int chunk = nt + (lane >> 4);
        uint32_t b0, b1, b2, b3;
        ldsm4_t(vaddr + row * kTRowBytes + swz(chunk, row) * 16, b0, b1, b2, b3);
        mma16816(o[nt], pa, b0, b1);
        mma16816(o[nt + 1], pa, b2, b3);
      }
    }
    __syncthreads();  // the stage may be refilled
    st = (st + 1) % kTStages;
  }
  cp_async_wait<0>();

  // ---- split partial of every (token, head) row: (acc[D], m, l) ----
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    float l = l_part[k];
    l += __shfl_xor_sync(0xffffffffu, l, 1);
    l += __shfl_xor_sync(0xffffffffu, l, 2);
    if (!valid[k]) continue;
    const int64_t unit = (int64_t)(tok0 + tl[k]) * p.Hkv + kvh;
    float* out = p.part + ((unit * p.S + split) * G + hh[k]) * (kTD + 2);
#pragma unroll
    for (int nt = 0; nt < kTD / 8; ++nt) {
      out[nt * 8 + 2 * t4] = o[nt][2 * k];
      out[nt * 8 + 2 * t4 + 1] = o[nt][2 * k + 1];
    }
    if (t4 == 0) {
      out[kTD] = m_run[k];
      out[kTD + 1] = l;
    }
  }
}

// Merges the S split partials of each (token, head) row into the output.
template <int G>
__global__ void tile_combine_kernel(const float* part, int S, int Hq, int Hkv,
                                    __nv_bfloat16* out) {
  const int64_t unit = blockIdx.x / G;
  const int h = blockIdx.x % G;
  const int i = threadIdx.x;
  const float* base = part + unit * S * G * (kTD + 2);
  float M = -INFINITY;
  for (int k = 0; k < S; ++k) M = fmaxf(M, base[(k * G + h) * (kTD + 2) + kTD]);
  float a = 0.0f, l = 0.0f;
  for (int k = 0; k < S; ++k) {
    const float* pk = base + (k * G + h) * (kTD + 2);
    const float m = pk[kTD];
    if (m == -INFINITY) continue;
    const float sc = exp2f(m - M);
    a += pk[i] * sc;
    l += pk[kTD + 1] * sc;
  }
  const int64_t orow = (unit / Hkv) * Hq + (unit % Hkv) * G + h;
  out[orow * kTD + i] = __float2bfloat16_rn(l > 0.0f ? a / l : 0.0f);
}

int tile_tokens(const Geometry& g) { return kTRows / g.G; }

int tile_splits(const Geometry& g, int64_t n, int num_sms) {
  const int64_t ctas = (n + tile_tokens(g) - 1) / tile_tokens(g) * g.Hkv;
  int64_t S = (int64_t)num_sms / (ctas > 0 ? ctas : 1);
  if (S < 1) S = 1;
  if (S > 64) S = 64;
  return (int)S;
}

size_t align256t(size_t x) { return (x + 255) & ~(size_t)255; }

}  // namespace

bool tile_attend_supported(const Geometry& g) {
  return g.dtype == ZHA_BF16 && g.d == kTD && (g.G == 2 || g.G == 4 || g.G == 8) &&
         (g.b == 2 || g.b == 4 || g.b == 8 || g.b == 16);
}

int64_t tile_map_stride(const Geometry& g) {
  // covers the nodes of every key block up to the cache capacity
  const int64_t nodes = (g.ncap + kTKB + g.b - 1) / g.b;
  return (nodes + 63) / 64 * 64;
}

// Scratch for any tile of at most n tokens: the keep map grows with the
// tile, the split partials do not (a smaller tile takes more key splits).
size_t tile_attend_ws_bytes(const Geometry& g, int64_t n, int num_sms) {
  if (!tile_attend_supported(g) || n < 1) return 0;
  int64_t rows_splits = 0;  // max over tile sizes m <= n of m * splits(m)
  for (int64_t m = 1; m <= n; ++m) {
    const int64_t v = m * tile_splits(g, m, num_sms);
    if (v > rows_splits) rows_splits = v;
  }
  return align256t((size_t)g.Hkv * n * tile_map_stride(g)) +
         align256t(sizeof(float) * (size_t)rows_splits * g.Hkv * g.G * (kTD + 2));
}

cudaError_t launch_attend_tile(const Geometry& g, const void* k, const void* v,
                               const int32_t* seq_len, int seq, int64_t pos0, int64_t n,
                               const void* q, void* out, const uint32_t* kept,
                               const int32_t* n_kept, int64_t kept_stride, int kept_segs,
                               void* ws, size_t ws_bytes, int num_sms, cudaStream_t stream) {
  if (!tile_attend_supported(g) || n < 1) return cudaErrorInvalidValue;
  if (ws_bytes < tile_attend_ws_bytes(g, n, num_sms)) return cudaErrorInvalidValue;
  const int64_t stride = tile_map_stride(g);
  const size_t map_bytes = (size_t)g.Hkv * n * stride;
  uint8_t* map = static_cast<uint8_t*>(ws);
  float* part = reinterpret_cast<float*>(static_cast<unsigned char*>(ws) + align256t(map_bytes));
  cudaError_t e = cudaMemsetAsync(map, 0, map_bytes, stream);
  if (e != cudaSuccess) return e;
  const int units = (int)(n * g.Hkv);
  keep_scatter_kernel<<<dim3(32, (unsigned)units), 256, 0, stream>>>(
      kept, n_kept, kept_stride, kept_segs, units, g.Hkv, (int)n, map, stride);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  TileParams p{};
  p.k = static_cast<const __nv_bfloat16*>(k);
  p.v = static_cast<const __nv_bfloat16*>(v);
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.seq_len = seq_len;
  p.seq = seq;
  p.pos0 = pos0;
  p.n = (int)n;
  p.ncap = g.ncap;
  p.Hq = g.Hq;
  p.Hkv = g.Hkv;
  p.b = g.b;
  p.b_shift = __builtin_ctz((unsigned)g.b);
  p.span_L = g.span[g.L];
  p.qscale = kLog2eT * g.inv_sqrt_d;
  p.keep = map;
  p.map_stride = stride;
  p.S = tile_splits(g, n, num_sms);
  p.part = part;
  const size_t smem = (size_t)kTStages * kTStageBytes;
  const dim3 grid((unsigned)((n + tile_tokens(g) - 1) / tile_tokens(g)), (unsigned)p.S,
                  (unsigned)g.Hkv);
  auto run = [&](auto kern, auto comb, int G) -> cudaError_t {
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)smem);
    if (err != cudaSuccess) return err;
    kern<<<grid, kTThreads, smem, stream>>>(p);
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
    comb<<<(unsigned)(units * G), kTD, 0, stream>>>(part, p.S, g.Hq, g.Hkv,
                                                    static_cast<__nv_bfloat16*>(out));
    return cudaGetLastError();
  };
  if (g.G == 8) return run(attend_tile_kernel<8>, tile_combine_kernel<8>, 8);
  if (g.G == 4) return run(attend_tile_kernel<4>, tile_combine_kernel<4>, 4);
  return run(attend_tile_kernel<2>, tile_combine_kernel<2>, 2);
}

}  // namespace zha
