/*
 * zha_oracle.c -- plain, slow, single-threaded CPU oracle for the ZHA hot path.
 *
 * TEST INFRASTRUCTURE. Only tests/, __graft_entry__.smoke() and bench.py's
 * cpu_baseline / reference leg may load this library. The CUDA path shares
 * no source, header, table or constant generator with it.
 *
 * What it follows (pages cited by title and paragraph):
 *   [lefilia] "Zyphra presente Zyphra Hierarchical Attention (ZHA), une voie
 *             vers une attention vraiment sous-quadratique" (lefilia.fr), par. 1:
 *             the KV cache stays complete and the tree only decides which keys
 *             a query reads; keys are cut into contiguous blocks, each block is
 *             summarised by one key derived from 16 learned reference queries,
 *             and each higher level summarises groups of b nodes of the level
 *             below; a query scores the top
 *             nodes, keeps the fewest nodes whose estimated attention mass
 *             reaches the fraction p, descends only into the kept branches
 *             until it reaches individual keys, and always keeps token 0.
 *   [lefilia] par. 2: p = 0.95; deep tree (blocks of 4, 6 levels) and wide tree
 *             (blocks of 256, 1 level).
 * The pages leave the formulas open. This library fixes them as:
 *   summary   s = (1/16) sum_r sum_c softmax_c(R_r . x_c / sqrt(d)) x_c,
 *             c over the node's children (raw keys at level 1, stored level l-1
 *             summaries above), R a 16 x d matrix shared by all KV heads;
 *   node mass exp(q . s / sqrt(d) + ln|node|), |node| = b^l tokens;
 *   causal tail: tokens not yet inside a complete top-level node are always
 *             attended; a top node is visible to a query at position t when it
 *             ends at or before t;
 *   GQA:      selection runs per query head on its KV head's tree.
 *
 * Every floating-point step that decides an integer result (summary values,
 * node scores, the top-p cut) uses the library's CANONICAL fp32 arithmetic, so
 * that index sets can be compared bit for bit. The canonical arithmetic is a
 * definition, restated here from its prose specification:
 *   - round to nearest even everywhere, no contraction of a*b+c unless written
 *     as fmaf, subnormals kept;
 *   - dot(a, x) = sequential fmaf chain over i = 0..d-1 starting from +0;
 *   - inv_sqrt_d = fp32(1/sqrt(d)), lnsize_l = fp32(l * ln b), both rounded from
 *     double;
 *   - exp_c(x), x <= 0: Cody-Waite reduction x = n ln2 + r with
 *     n = rint(x * fp32(log2 e)) and ln2 split into a 12-bit head and a tail,
 *     a degree-7 Taylor polynomial in Horner form with fmaf, then scaling by
 *     the exact power 2^n; 0 for x < -87 (W. J. Cody and W. Waite, "Software
 *     Manual for the Elementary Functions", 1980, exponential chapter);
 *   - masses are fixed point: M = trunc(exp_c(z - zmax) * 2^40) as uint64,
 *     summed exactly; need = ceil(T * p_q / 2^32) with p_q = floor(p*2^32+0.5);
 *     p_q >= 2^32 keeps every candidate.
 * Attention itself is computed in fp64 (it is compared within a tolerance).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ZO_NREF 16

/* ------------------------------------------------------------------------ */
/* canonical scalar helpers                                                  */
/* ------------------------------------------------------------------------ */

static float zo_f32_from_bits(uint32_t u) {
  float f;
  memcpy(&f, &u, 4);
  return f;
}

static uint32_t zo_bits_from_f32(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  return u;
}

/* exp(x) for x <= 0 in the canonical form described in the file header. */
float zo_exp_c(float x) {
  if (x < -87.0f) return 0.0f;
  const float log2e = 0x1.715476p+0f;  /* fp32(1/ln 2) */
  const float ln2_hi = 0x1.62e4p-1f;   /* ln 2 with the low 12 mantissa bits cleared */
  const float ln2_lo = 0x1.7f7d1cp-20f; /* fp32(ln 2 - ln2_hi) */
  float n = rintf(x * log2e);
  float r = fmaf(-n, ln2_hi, x);
  r = fmaf(-n, ln2_lo, r);
  /* Taylor coefficients fp32(1/k!), k = 7 .. 0 */
  float p = 0x1.a01a02p-13f;          /* 1/5040 */
  p = fmaf(p, r, 0x1.6c16c2p-10f);    /* 1/720 */
  p = fmaf(p, r, 0x1.111112p-7f);     /* 1/120 */
  p = fmaf(p, r, 0x1.555556p-5f);     /* 1/24 */
  p = fmaf(p, r, 0x1.555556p-3f);     /* 1/6 */
  p = fmaf(p, r, 0.5f);
  p = fmaf(p, r, 1.0f);
  p = fmaf(p, r, 1.0f);
  int ni = (int)n; /* in [-126, 0] because -87 <= x <= 0 */
  float scale = zo_f32_from_bits((uint32_t)(ni + 127) << 23);
  return p * scale;
}

/* dot(a, x): sequential fmaf chain from +0 over i = 0..d-1. */
float zo_dot(const float* a, const float* x, int d) {
  float acc = 0.0f;
  for (int i = 0; i < d; ++i) acc = fmaf(a[i], x[i], acc);
  return acc;
}

/* Round a finite fp32 value to the nearest bf16 (ties to even); the result is
 * returned widened back to fp32, which is exact. */
float zo_round_bf16(float x) {
  uint32_t u = zo_bits_from_f32(x);
  uint32_t lsb = (u >> 16) & 1u;
  u += 0x7FFFu + lsb;
  u &= 0xFFFF0000u;
  return zo_f32_from_bits(u);
}

float zo_inv_sqrt_d(int d) { return (float)(1.0 / sqrt((double)d)); }

float zo_lnsize(int level, int b) { return (float)((double)level * log((double)b)); }

/* ------------------------------------------------------------------------ */
/* summary keys  [lefilia page, par. 1: one key per node, derived from 16  */
/* learned reference queries; the tree is built one level at a time]        */
/* ------------------------------------------------------------------------ */

/*
 * One node from its b children rows (children[c*d + i]). out[i] receives the
 * canonical fp32 value; if store_bf16 it is rounded to bf16 (the storage type).
 * Canonical steps:
 *   l_rc = dot(R_r, x_c) * inv_sqrt_d
 *   mu_r = max_c l_rc;  e_rc = exp_c(l_rc - mu_r);  Z_r = sum_c e_rc (c order)
 *   w_rc = e_rc / Z_r
 *   a_c  = (sum_r w_rc, r order) * 0.0625
 *   s_i  = sum_c fmaf(a_c, x_ci, .) in c order from +0
 */
void zo_build_node(const float* children, int b, int d, const float* R, int store_bf16,
                   float* out) {
  const float inv_sqrt_d = zo_inv_sqrt_d(d);
  float* logit = (float*)malloc(sizeof(float) * (size_t)ZO_NREF * (size_t)b);
  float* a = (float*)malloc(sizeof(float) * (size_t)b);
  for (int r = 0; r < ZO_NREF; ++r)
    for (int c = 0; c < b; ++c)
      logit[r * b + c] = zo_dot(R + (size_t)r * d, children + (size_t)c * d, d) * inv_sqrt_d;
  for (int c = 0; c < b; ++c) a[c] = 0.0f;
  for (int r = 0; r < ZO_NREF; ++r) {
    float mu = logit[r * b];
    for (int c = 1; c < b; ++c)
      if (logit[r * b + c] > mu) mu = logit[r * b + c];
    float Z = 0.0f;
    for (int c = 0; c < b; ++c) {
      logit[r * b + c] = zo_exp_c(logit[r * b + c] - mu); /* now e_rc */
      Z = Z + logit[r * b + c];
    }
    for (int c = 0; c < b; ++c) logit[r * b + c] = logit[r * b + c] / Z; /* now w_rc */
  }
  for (int c = 0; c < b; ++c) {
    float acc = 0.0f;
    for (int r = 0; r < ZO_NREF; ++r) acc = acc + logit[r * b + c];
    a[c] = acc * 0.0625f;
  }
  for (int i = 0; i < d; ++i) {
    float acc = 0.0f;
    for (int c = 0; c < b; ++c) acc = fmaf(a[c], children[(size_t)c * d + i], acc);
    out[i] = store_bf16 ? zo_round_bf16(acc) : acc;
  }
  free(logit);
  free(a);
}

/*
 * Build every complete node of levels 1..L for one (sequence, KV head) whose
 * first n keys are K[0..n) (row-major n x d, values already widened to fp32).
 * tree + level_row_off[l-1]*d holds level l, row j = node (l, j); a level-l node
 * j covers tokens [j b^l, (j+1) b^l) and is complete when (j+1) b^l <= n.
 * Returns the number of nodes written.
 */
int64_t zo_build_tree(const float* K, int64_t n, int d, const float* R, int b, int L,
                      int store_bf16, float* tree, const int64_t* level_row_off) {
  int64_t written = 0;
  int64_t span = 1;
  for (int l = 1; l <= L; ++l) {
    span *= b;
    const int64_t nodes = n / span;
    const float* child_base = (l == 1) ? K : tree + level_row_off[l - 2] * (int64_t)d;
    float* out_base = tree + level_row_off[l - 1] * (int64_t)d;
    for (int64_t j = 0; j < nodes; ++j) {
      zo_build_node(child_base + j * (int64_t)b * d, b, d, R, store_bf16, out_base + j * d);
      ++written;
    }
  }
  return written;
}

/* ------------------------------------------------------------------------ */
/* top-p cut at one level  [lefilia page, par. 1: the fewest nodes whose    */
/* estimated attention mass reaches the fraction p]                          */
/* ------------------------------------------------------------------------ */

typedef struct {
  float z;
  int64_t node;
  uint64_t mass;
} zo_cand;

static int zo_cmp_cand(const void* pa, const void* pb) {
  const zo_cand* a = (const zo_cand*)pa;
  const zo_cand* b = (const zo_cand*)pb;
  if (a->z > b->z) return -1; /* larger score first */
  if (a->z < b->z) return 1;
  if (a->node < b->node) return -1; /* equal scores: lower node index first */
  if (a->node > b->node) return 1;
  return 0;
}

static int zo_cmp_i64(const void* pa, const void* pb) {
  int64_t a = *(const int64_t*)pa, b = *(const int64_t*)pb;
  return (a > b) - (a < b);
}

uint64_t zo_p_fixed(double p) { return (uint64_t)floor(p * 4294967296.0 + 0.5); }

/*
 * Canonical cut over n candidates (scores z[i] of nodes node[i]). Writes the
 * kept node ids in ascending order to kept[] and returns k = their count.
 *   zmax = max z;  M_i = trunc(exp_c(z_i - zmax) * 2^40);  T = sum M_i;
 *   need = ceil(T * p_q / 2^32);  order by (z desc, node asc);
 *   k = smallest prefix length whose mass reaches need (all if p_q >= 2^32).
 * near_tie (nullable) is set to 1 if the cutoff score z_(k) lies within 1e-6
 * relative of a sorted neighbour (|dz| <= 1e-6 max(|z_(k)|, 1)), or if the
 * target need lies within 1e-6 T of the prefix mass on either side of the
 * cut (need - C_(k-1) or C_k - need, where C_j is the mass of the first j).
 * T_out / need_out (nullable) receive T and need.
 */
int64_t zo_cut(const float* z, const int64_t* node, int64_t n, uint64_t p_q, int64_t* kept,
               uint64_t* T_out, uint64_t* need_out, int* near_tie) {
  if (n <= 0) return 0;
  zo_cand* c = (zo_cand*)malloc(sizeof(zo_cand) * (size_t)n);
  float zmax = z[0];
  for (int64_t i = 1; i < n; ++i)
    if (z[i] > zmax) zmax = z[i];
  uint64_t T = 0;
  for (int64_t i = 0; i < n; ++i) {
    c[i].z = z[i];
    c[i].node = node[i];
    c[i].mass = (uint64_t)(zo_exp_c(z[i] - zmax) * 0x1p40f);
    T += c[i].mass;
  }
  const unsigned __int128 prod = (unsigned __int128)T * (unsigned __int128)p_q;
  const uint64_t need = (uint64_t)((prod + (((unsigned __int128)1 << 32) - 1)) >> 32);
  qsort(c, (size_t)n, sizeof(zo_cand), zo_cmp_cand);
  int64_t k;
  const int all = p_q >= ((uint64_t)1 << 32);
  uint64_t cum = 0; /* C_k, the mass of the kept prefix */
  if (all) {
    k = n;
  } else {
    k = n;
    for (int64_t i = 0; i < n; ++i) {
      cum += c[i].mass;
      if (cum >= need) {
        k = i + 1;
        break;
      }
    }
  }
  if (near_tie) {
    *near_tie = 0;
    const float zk = c[k - 1].z;
    const float band = 1e-6f * (fabsf(zk) > 1.0f ? fabsf(zk) : 1.0f);
    if (k < n && fabsf(zk - c[k].z) <= band) *near_tie = 1;
    if (k >= 2 && fabsf(c[k - 2].z - zk) <= band) *near_tie = 1;
    /* the cut's mass margin: C_(k-1) < need <= C_k, either side within 1e-6 T */
    if (!all) {
      const double mband = 1e-6 * (double)T;
      const uint64_t prev = cum - c[k - 1].mass; /* C_(k-1) */
      if ((double)(need - prev) <= mband || (double)(cum - need) <= mband) *near_tie = 1;
    }
  }
  for (int64_t i = 0; i < k; ++i) kept[i] = c[i].node;
  qsort(kept, (size_t)k, sizeof(int64_t), zo_cmp_i64);
  if (T_out) *T_out = T;
  if (need_out) *need_out = need;
  free(c);
  return k;
}

/* ------------------------------------------------------------------------ */
/* per-query traversal  [lefilia page, par. 1: start from the top nodes,   */
/* descend only into kept branches, down to the individual keys; token 0 is */
/* always part of the selection]                                            */
/* ------------------------------------------------------------------------ */

/* z = (dot(q, s) * inv_sqrt_d) + lnsize_l, two separately rounded fp32 ops. */
float zo_score(const float* q, const float* s, int d, int level, int b) {
  return zo_dot(q, s, d) * zo_inv_sqrt_d(d) + zo_lnsize(level, b);
}

/*
 * Selection for one query head at position t over one (sequence, KV head)
 * tree. Candidates at level L are the complete top nodes ending at or before
 * t: (L, 0 .. T_top-1) with T_top = floor((t+1) / b^L). At each level l = L..1
 * the canonical cut keeps k_l nodes (level_counts[L-l] = k_l) and the
 * candidates of level l-1 are the children of the kept nodes. The selected
 * token set is
 *   S = ascending( tokens of kept level-1 nodes  U  {0}  U  [b^L T_top, t] ).
 * Up to cap indices are written to idx; the return value is |S| (compare with
 * cap for truncation). level_ncand (nullable, [L]) receives the candidate
 * counts; near_tie (nullable) is OR-ed over levels.
 */
int64_t zo_select(const float* q, int d, const float* tree, const int64_t* level_row_off, int b,
                  int L, int64_t t, uint64_t p_q, int32_t* idx, int64_t cap,
                  int32_t* level_counts, int64_t* level_ncand, int* near_tie) {
  int64_t bL = 1;
  for (int l = 0; l < L; ++l) bL *= b;
  const int64_t T_top = (t + 1) / bL;
  const int64_t tail_start = bL * T_top;
  for (int l = 0; l < L; ++l) {
    level_counts[l] = 0;
    if (level_ncand) level_ncand[l] = 0;
  }
  if (near_tie) *near_tie = 0;

  int64_t n_sel = 0;
#define ZO_EMIT(tok)                                  \
  do {                                                \
    if (n_sel < cap) idx[n_sel] = (int32_t)(tok);     \
    ++n_sel;                                          \
  } while (0)

  if (T_top == 0) {
    for (int64_t j = 0; j <= t; ++j) ZO_EMIT(j);
    return n_sel;
  }

  /* level-1 node count bounds every candidate list */
  const int64_t max_nodes = (t + 1) / b + 1;
  int64_t* cand = (int64_t*)malloc(sizeof(int64_t) * (size_t)max_nodes);
  int64_t* kept = (int64_t*)malloc(sizeof(int64_t) * (size_t)max_nodes);
  float* z = (float*)malloc(sizeof(float) * (size_t)max_nodes);
  int64_t n_cand = T_top;
  for (int64_t j = 0; j < n_cand; ++j) cand[j] = j;
  int64_t k = 0;
  for (int l = L; l >= 1; --l) {
    const float* level_base = tree + level_row_off[l - 1] * (int64_t)d;
    for (int64_t i = 0; i < n_cand; ++i) z[i] = zo_score(q, level_base + cand[i] * d, d, l, b);
    int tie = 0;
    k = zo_cut(z, cand, n_cand, p_q, kept, NULL, NULL, &tie);
    if (near_tie && tie) *near_tie = 1;
    level_counts[L - l] = (int32_t)k;
    if (level_ncand) level_ncand[L - l] = n_cand;
    if (l > 1) {
      n_cand = 0;
      for (int64_t i = 0; i < k; ++i)
        for (int c = 0; c < b; ++c) cand[n_cand++] = kept[i] * b + c;
    }
  }
  /* kept[] now holds the kept level-1 nodes in ascending order */
  if (k == 0 || kept[0] != 0) ZO_EMIT(0);
  for (int64_t i = 0; i < k; ++i)
    for (int c = 0; c < b; ++c) ZO_EMIT(kept[i] * b + c);
  for (int64_t j = tail_start; j <= t; ++j) ZO_EMIT(j);
#undef ZO_EMIT
  free(cand);
  free(kept);
  free(z);
  return n_sel;
}

/* ------------------------------------------------------------------------ */
/* exact attention over the selected keys, fp64  [lefilia par. 1: the full   */
/* KV cache is kept and attention reads the selected raw entries]            */
/* ------------------------------------------------------------------------ */

/* out[i] = sum_{j in S} softmax_j(q . k_j / sqrt(d)) v_ji, in double. K and V are
 * the (sequence, KV head) rows, row-major, fp32 values. */
void zo_attend_f64(const float* q, int d, const float* K, const float* V, const int32_t* idx,
                   int64_t n, double* out) {
  const double scale = 1.0 / sqrt((double)d);
  double* s = (double*)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
  double m = -INFINITY;
  for (int64_t j = 0; j < n; ++j) {
    const float* k = K + (int64_t)idx[j] * d;
    double acc = 0.0;
    for (int i = 0; i < d; ++i) acc += (double)q[i] * (double)k[i];
    s[j] = acc * scale;
    if (s[j] > m) m = s[j];
  }
  double denom = 0.0;
  for (int i = 0; i < d; ++i) out[i] = 0.0;
  for (int64_t j = 0; j < n; ++j) {
    const double w = exp(s[j] - m);
    denom += w;
    const float* v = V + (int64_t)idx[j] * d;
    for (int i = 0; i < d; ++i) out[i] += w * (double)v[i];
  }
  for (int i = 0; i < d; ++i) out[i] /= denom;
  free(s);
}

/* ------------------------------------------------------------------------ */
/* fp64 "faithful" mode: the same formulas in double with libm exp and a     */
/* plain sort; used only to show that the canonical fp32 spec renders the    */
/* mathematics faithfully (selections agree wherever the decision is not     */
/* within a rounding-sized margin).                                          */
/* ------------------------------------------------------------------------ */

void zo_build_node_f64(const float* children, int b, int d, const float* R, double* out) {
  const double inv = 1.0 / sqrt((double)d);
  double* a = (double*)calloc((size_t)b, sizeof(double));
  double* lg = (double*)malloc(sizeof(double) * (size_t)b);
  for (int r = 0; r < ZO_NREF; ++r) {
    double mu = -INFINITY;
    for (int c = 0; c < b; ++c) {
      double acc = 0.0;
      for (int i = 0; i < d; ++i) acc += (double)R[r * d + i] * (double)children[c * d + i];
      lg[c] = acc * inv;
      if (lg[c] > mu) mu = lg[c];
    }
    double Z = 0.0;
    for (int c = 0; c < b; ++c) Z += exp(lg[c] - mu);
    for (int c = 0; c < b; ++c) a[c] += exp(lg[c] - mu) / Z / (double)ZO_NREF;
  }
  for (int i = 0; i < d; ++i) {
    double acc = 0.0;
    for (int c = 0; c < b; ++c) acc += a[c] * (double)children[c * d + i];
    out[i] = acc;
  }
  free(a);
  free(lg);
}

typedef struct {
  double z;
  int64_t node;
  double mass;
} zo_cand64;

static int zo_cmp_cand64(const void* pa, const void* pb) {
  const zo_cand64* a = (const zo_cand64*)pa;
  const zo_cand64* b = (const zo_cand64*)pb;
  if (a->z > b->z) return -1;
  if (a->z < b->z) return 1;
  return (a->node > b->node) - (a->node < b->node);
}

/*
 * Same traversal as zo_select but in double: z = q.s/sqrt(d) + l ln b, masses
 * exp(z - zmax), cut at the first prefix with cumulative mass >= p T. margin
 * receives the smallest decision margin met on the way, relative: the score gap
 * at the cut |z_(k) - z_(k+/-1)| / max(|z_(k)|, 1) and the mass gap
 * |C - pT| / T for C in {C_(k-1), C_k}.
 */
int64_t zo_select_f64(const float* q, int d, const float* tree, const int64_t* level_row_off,
                      int b, int L, int64_t t, double p, int32_t* idx, int64_t cap,
                      int32_t* level_counts, double* margin) {
  int64_t bL = 1;
  for (int l = 0; l < L; ++l) bL *= b;
  const int64_t T_top = (t + 1) / bL;
  const int64_t tail_start = bL * T_top;
  double mmin = INFINITY;
  for (int l = 0; l < L; ++l) level_counts[l] = 0;
  int64_t n_sel = 0;
  if (T_top == 0) {
    for (int64_t j = 0; j <= t; ++j) {
      if (n_sel < cap) idx[n_sel] = (int32_t)j;
      ++n_sel;
    }
    if (margin) *margin = mmin;
    return n_sel;
  }
  const int64_t max_nodes = (t + 1) / b + 1;
  int64_t* cand = (int64_t*)malloc(sizeof(int64_t) * (size_t)max_nodes);
  int64_t* kept = (int64_t*)malloc(sizeof(int64_t) * (size_t)max_nodes);
  zo_cand64* c = (zo_cand64*)malloc(sizeof(zo_cand64) * (size_t)max_nodes);
  int64_t n_cand = T_top, k = 0;
  for (int64_t j = 0; j < n_cand; ++j) cand[j] = j;
  for (int l = L; l >= 1; --l) {
    const float* base = tree + level_row_off[l - 1] * (int64_t)d;
    double zmax = -INFINITY;
    for (int64_t i = 0; i < n_cand; ++i) {
      double acc = 0.0;
      for (int e = 0; e < d; ++e) acc += (double)q[e] * (double)base[cand[i] * d + e];
      c[i].z = acc / sqrt((double)d) + (double)l * log((double)b);
      c[i].node = cand[i];
      if (c[i].z > zmax) zmax = c[i].z;
    }
    double T = 0.0;
    for (int64_t i = 0; i < n_cand; ++i) {
      c[i].mass = exp(c[i].z - zmax);
      T += c[i].mass;
    }
    qsort(c, (size_t)n_cand, sizeof(zo_cand64), zo_cmp_cand64);
    if (p >= 1.0) {
      k = n_cand;
    } else {
      double cum = 0.0;
      k = n_cand;
      for (int64_t i = 0; i < n_cand; ++i) {
        const double prev = cum;
        cum += c[i].mass;
        if (cum >= p * T) {
          k = i + 1;
          const double g1 = fabs(cum - p * T) / T, g0 = fabs(prev - p * T) / T;
          if (g1 < mmin) mmin = g1;
          if (g0 < mmin) mmin = g0;
          break;
        }
      }
      const double zk = c[k - 1].z;
      const double sc = fabs(zk) > 1.0 ? fabs(zk) : 1.0;
      if (k < n_cand && fabs(zk - c[k].z) / sc < mmin) mmin = fabs(zk - c[k].z) / sc;
      if (k >= 2 && fabs(c[k - 2].z - zk) / sc < mmin) mmin = fabs(c[k - 2].z - zk) / sc;
    }
    for (int64_t i = 0; i < k; ++i) kept[i] = c[i].node;
    qsort(kept, (size_t)k, sizeof(int64_t), zo_cmp_i64);
    level_counts[L - l] = (int32_t)k;
    if (l > 1) {
      n_cand = 0;
      for (int64_t i = 0; i < k; ++i)
        for (int cc = 0; cc < b; ++cc) cand[n_cand++] = kept[i] * b + cc;
    }
  }
  if (k == 0 || kept[0] != 0) {
    if (n_sel < cap) idx[n_sel] = 0;
    ++n_sel;
  }
  for (int64_t i = 0; i < k; ++i)
    for (int cc = 0; cc < b; ++cc) {
      if (n_sel < cap) idx[n_sel] = (int32_t)(kept[i] * b + cc);
      ++n_sel;
    }
  for (int64_t j = tail_start; j <= t; ++j) {
    if (n_sel < cap) idx[n_sel] = (int32_t)j;
    ++n_sel;
  }
  if (margin) *margin = mmin;
  free(cand);
  free(kept);
  free(c);
  return n_sel;
}

/* ------------------------------------------------------------------------ */
/* block-scaled 4-bit summary rows (the FP4 router variant)                  */
/* ------------------------------------------------------------------------ */

/* [lefilia] par. 4 reports that a 4-bit (FP4) variant of the router was
 * tried; the pages give no format. This library's reading: every block of 32
 * consecutive elements of a summary row is stored as e2m1 magnitudes
 * {0, 0.5, 1, 1.5, 2, 3, 4, 6} (codes 0..7 in that order) with a sign, times
 * one power of two 2^e per block, e the smallest integer with
 * max|x| <= 6 * 2^e (e = 0 for an all-zero block). Each |x| / 2^e goes to the
 * nearest magnitude, an exact tie to the even code. The rounded values are
 * written to out (zero as +0) and e to exps[row * d/32 + block]. The router
 * then scores these values with the canonical arithmetic. */
void zo_fp4_round_rows(const float* in, int64_t n_rows, int d, float* out, int32_t* exps) {
  static const float mag[8] = {0.0f, 0.5f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 6.0f};
  static const float mid[7] = {0.25f, 0.75f, 1.25f, 1.75f, 2.5f, 3.5f, 5.0f};
  const int nb = d / 32;
  for (int64_t r = 0; r < n_rows; ++r)
    for (int blk = 0; blk < nb; ++blk) {
      const float* x = in + r * d + blk * 32;
      float* y = out + r * d + blk * 32;
      float amax = 0.0f;
      for (int i = 0; i < 32; ++i)
        if (fabsf(x[i]) > amax) amax = fabsf(x[i]);
      int e = 0;
      if (amax > 0.0f) {
        /* amax = m 2^E with m in [0.5, 1); 6 2^e = 0.75 2^(e+3) */
        int E = 0;
        const float m = frexpf(amax, &E);
        e = m <= 0.75f ? E - 3 : E - 2;
      }
      exps[r * nb + blk] = e;
      for (int i = 0; i < 32; ++i) {
        const float a = ldexpf(fabsf(x[i]), -e); /* exact: a power-of-two scaling */
        int k = 0;
        while (k < 7 && a > mid[k]) ++k;
        if (k < 7 && a == mid[k] && (k & 1)) ++k;
        const float v = ldexpf(mag[k], e);
        y[i] = k == 0 ? 0.0f : (x[i] < 0.0f ? -v : v);
      }
    }
}

