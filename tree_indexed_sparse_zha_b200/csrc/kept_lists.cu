// zha_decode_kept_lists: the token list each query head of a decode step
// attends, expanded from the traversal's decode-mode output.
//
// lefilia.fr page "Zyphra presente Zyphra Hierarchical Attention (ZHA) ...",
// paragraph 1: a query attends the raw keys under the level-1 nodes it kept,
// plus the first token. The decode traversal leaves, per (sequence, KV head),
// the union of the kept level-1 nodes of its G query heads as C ordered
// segments of (head mask << 24) | node entries; the decode attention reads,
// for head h, token 0, then the b tokens of every entry whose mask has bit h
// (token 0 of node 0 once only), then the causal tail [b^L T_top, t]. This
// kernel writes exactly that row sequence per head, which is the ascending
// set S = tokens of kept level-1 nodes U {0} U tail, so that it can be
// compared element by element with an independent selection.
#include <cuda_runtime.h>

#include "zha_device.cuh"
#include "zha_internal.h"

namespace zha {
namespace {

constexpr int kThreads = 256;

struct KeptArgs {
  const uint32_t* kept;   // [units][segs][stride]
  const int32_t* n_kept;  // [units][segs]
  int64_t stride;
  int segs;
  const int32_t* seq_len;
  int64_t ncap, span_L;
  int Hq, Hkv, G, b;
  int32_t* idx;           // [B][Hq][idx_cap]
  int64_t idx_cap;
  int32_t* n_idx;         // [B][Hq]
  int32_t* status;
};

// One CTA per (sequence, query head): a block-wide scan over the unit's kept
// entries in segment order gives every node the head keeps its place.
__global__ void __launch_bounds__(kThreads) kept_lists_kernel(KeptArgs a) {
  __shared__ unsigned int s_warp[kThreads / 32];
  __shared__ unsigned int s_run;
  __shared__ int s_shift;
  const int qh = blockIdx.x;  // seq * Hq + h
  const int seq = qh / a.Hq, h = qh % a.Hq;
  const int kvh = h / a.G, bit = h % a.G;
  const int unit = seq * a.Hkv + kvh;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int64_t n = a.seq_len[seq];
  if (n > a.ncap) n = a.ncap;
  if (n < 0) n = 0;
  const int64_t t = n - 1;
  const int64_t T_top = (t + 1) / a.span_L;
  const int64_t tail_start = a.span_L * T_top;
  int32_t* out = a.idx + (int64_t)qh * a.idx_cap;
  // token 0 leads the list whenever a top node is complete (the attention
  // reads it as a separate row and skips it inside node 0)
  const int64_t lead = T_top > 0 ? 1 : 0;
  if (tid == 0) {
    s_run = 0u;
    s_shift = 0;
    if (T_top > 0) {
      if (a.idx_cap > 0) out[0] = 0;
      // node 0, when the head keeps it, is the first entry of the first
      // non-empty segment: its token 0 is already in the list
      for (int r = 0; r < a.segs; ++r) {
        if (a.n_kept[(int64_t)unit * a.segs + r] > 0) {
          const uint32_t e = a.kept[((int64_t)unit * a.segs + r) * a.stride];
          s_shift = ((e & 0x00ffffffu) == 0u && ((e >> (24 + bit)) & 1u)) ? 1 : 0;
          break;
        }
      }
    }
  }
  __syncthreads();
  const int64_t shift = s_shift;
  if (T_top > 0) {
    for (int r = 0; r < a.segs; ++r) {
      const int64_t cnt = a.n_kept[(int64_t)unit * a.segs + r];
      const uint32_t* seg = a.kept + ((int64_t)unit * a.segs + r) * a.stride;
      for (int64_t base = 0; base < cnt; base += kThreads) {
        const int64_t i = base + tid;
        const uint32_t e = i < cnt ? seg[i] : 0u;
        const unsigned f = (i < cnt && ((e >> (24 + bit)) & 1u)) ? 1u : 0u;
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
        for (int w = 0; w < kThreads / 32; ++w) {
          if (w < warp) wbase += s_warp[w];
          tot += s_warp[w];
        }
        const unsigned run = s_run;
        if (f) {
          const int64_t node = e & 0x00ffffffu;
          const int64_t k = (int64_t)run + wbase + x - 1;  // the head's k-th kept node
          for (int c = 0; c < a.b; ++c) {
            const int64_t tok = node * a.b + c;
            if (tok == 0) continue;
            const int64_t at = lead + k * a.b + c - shift;
            if (at < a.idx_cap) out[at] = (int32_t)tok;
          }
        }
        __syncthreads();
        if (tid == 0) s_run = run + tot;
        __syncthreads();
      }
    }
  }
  const int64_t head = lead + (int64_t)s_run * a.b - shift;  // entries before the tail
  const int64_t tail_len = t + 1 - tail_start;
  for (int64_t j = tid; j < tail_len; j += kThreads)
    if (head + j < a.idx_cap) out[head + j] = (int32_t)(tail_start + j);
  if (tid == 0) {
    const int64_t total = head + (tail_len > 0 ? tail_len : 0);
    a.n_idx[qh] = (int32_t)total;
    if (total > a.idx_cap) raise_status(a.status, ZHA_ERR_CAPACITY);
  }
}

}  // namespace

cudaError_t launch_kept_lists(const Geometry& g, const uint32_t* kept, const int32_t* n_kept,
                              int64_t stride, int segs, const int32_t* seq_len, int32_t* idx,
                              int64_t idx_cap, int32_t* n_idx, int32_t* status,
                              cudaStream_t stream) {
  KeptArgs a{};
  a.kept = kept;
  a.n_kept = n_kept;
  a.stride = stride;
  a.segs = segs;
  a.seq_len = seq_len;
  a.ncap = g.ncap;
  a.span_L = g.span[g.L];
  a.Hq = g.Hq;
  a.Hkv = g.Hkv;
  a.G = g.G;
  a.b = g.b;
  a.idx = idx;
  a.idx_cap = idx_cap;
  a.n_idx = n_idx;
  a.status = status;
  kept_lists_kernel<<<(unsigned)(g.B * g.Hq), kThreads, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace zha
