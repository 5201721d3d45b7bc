/*
 * rswa_oracle.c -- plain, slow, fp64 CPU statement of what the R-SWA / SR-SWA
 * decode-attention hot path computes.
 *
 * TEST INFRASTRUCTURE. Only the test suite, the package smoke check and the
 * benchmark's CPU-baseline leg may load this library. The product (the CUDA
 * library and its Python binding) never calls it, shares no code with it and
 * has no CPU fallback through it.
 *
 * Every value is widened to double on load and every sum is taken in double,
 * in the plain order of the definition. There is no tiling, no online softmax,
 * no split; OpenMP only distributes independent (sequence, head) problems.
 *
 * Page names used in the citations below:
 *   [R-SWA summary]   "百度Unlimited OCR" paper summary, lshu.cn/news/33052
 *   [R-SWA tutorial]  "百度 Unlimited OCR 深度实战 ... R-SWA注意力革命", chenxutan.com/d/4055.html
 *   [SR-SWA explainer] Unlimited-OCR-2 SR-SWA explainer, nxmr.cn/news/162408
 *   [tech analysis]   "Unlimited-OCR：突破32768上下文限制的视觉语言模型技术解析", pnsm.cn
 *
 * Layouts (row-major, all little-endian):
 *   bf16 tensors are passed as their raw 16-bit patterns (uint16_t).
 *   q, k_new, v_new        [B][H][D]
 *   prefix K/V  pk, pv     [B][H][cap][D]   rows [0, prefix_len[b]) valid
 *   ring K/V               [B][H][n][D]
 *   wp, fill               [B]  next slot to write, number of valid slots
 *   prefill q/k_out/v_out  [B][H][T][D]
 *   k_idx                  [B][cap][DI]     per-token router index keys
 *   q_idx                  [B][DI]          fp32 router query per sequence
 *
 * Parity status of each function is stated at the function.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------ */
/* helpers                                                             */
/* ------------------------------------------------------------------ */

/* bf16 is the upper half of an IEEE binary32; widening is exact. */
static double bf16_to_double(uint16_t bits) {
  uint32_t u = ((uint32_t)bits) << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

static int64_t pos_mod(int64_t a, int64_t n) {
  int64_t r = a % n;
  return r < 0 ? r + n : r;
}

void oracle_set_threads(int n) {
#ifdef _OPENMP
  if (n > 0) omp_set_num_threads(n);
#else
  (void)n;
#endif
}

int oracle_get_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/*
 * One attention read: softmax over an explicit key list.
 *   s_j = scale * <q, k_j> + bias_j
 *   o   = sum_j softmax(s)_j v_j ,  lse = log sum_j exp(s_j)
 * The largest s_j is subtracted before exponentiating (exp(s - M) / sum
 * exp(s - M) is the same quotient); lse adds M back. An empty key list gives
 * o = 0 and lse = -inf.
 * This is the attention formula of [R-SWA tutorial] §2.2.1 (softmax(Q K^T /
 * sqrt(d)) V) over the key set R-SWA makes visible, with an additive bias
 * slot for SR-SWA's log-probability term.
 */
typedef struct {
  const uint16_t** krow;  /* bf16 rows, or NULL when the key is stored as e4m3 codes */
  const uint16_t** vrow;
  const uint8_t** k8;     /* e4m3 rows and their block scales (FP8 prefix) */
  const uint8_t** v8;
  double* kscale;
  double* vscale;
  double* bias;
  double* s;
  int64_t count;
} keylist;

static void* alloc_keys(size_t elem, int64_t max_keys) { return malloc(elem * (size_t)(max_keys > 0 ? max_keys : 1)); }

static void keylist_init(keylist* L, int64_t max_keys) {
  L->krow = (const uint16_t**)alloc_keys(sizeof(*L->krow), max_keys);
  L->vrow = (const uint16_t**)alloc_keys(sizeof(*L->vrow), max_keys);
  L->k8 = (const uint8_t**)alloc_keys(sizeof(*L->k8), max_keys);
  L->v8 = (const uint8_t**)alloc_keys(sizeof(*L->v8), max_keys);
  L->kscale = (double*)alloc_keys(sizeof(double), max_keys);
  L->vscale = (double*)alloc_keys(sizeof(double), max_keys);
  L->bias = (double*)alloc_keys(sizeof(double), max_keys);
  L->s = (double*)alloc_keys(sizeof(double), max_keys);
  L->count = 0;
}

static void keylist_free(keylist* L) {
  free((void*)L->krow);
  free((void*)L->vrow);
  free((void*)L->k8);
  free((void*)L->v8);
  free(L->kscale);
  free(L->vscale);
  free(L->bias);
  free(L->s);
}

static void keylist_push(keylist* L, const uint16_t* k, const uint16_t* v, double bias) {
  L->krow[L->count] = k;
  L->vrow[L->count] = v;
  L->k8[L->count] = NULL;
  L->v8[L->count] = NULL;
  L->bias[L->count] = bias;
  L->count++;
}

double oracle_e4m3_to_double(uint8_t c);

static void keylist_push8(keylist* L, const uint8_t* k, const uint8_t* v, double kscale, double vscale,
                          double bias) {
  L->krow[L->count] = NULL;
  L->vrow[L->count] = NULL;
  L->k8[L->count] = k;
  L->v8[L->count] = v;
  L->kscale[L->count] = kscale;
  L->vscale[L->count] = vscale;
  L->bias[L->count] = bias;
  L->count++;
}

/* element d of key / value j, widened to double (an e4m3 code times its block scale) */
static double key_at(const keylist* L, int64_t j, int d) {
  return L->krow[j] ? bf16_to_double(L->krow[j][d]) : oracle_e4m3_to_double(L->k8[j][d]) * L->kscale[j];
}

static double val_at(const keylist* L, int64_t j, int d) {
  return L->vrow[j] ? bf16_to_double(L->vrow[j][d]) : oracle_e4m3_to_double(L->v8[j][d]) * L->vscale[j];
}

static void attend(const keylist* L, const uint16_t* q, int D, double scale, double* out, double* lse) {
  double qd[1024];
  for (int d = 0; d < D; ++d) qd[d] = bf16_to_double(q[d]);
  for (int d = 0; d < D; ++d) out[d] = 0.0;
  if (L->count == 0) {
    *lse = -INFINITY;
    return;
  }
  double M = -INFINITY;
  for (int64_t j = 0; j < L->count; ++j) {
    double dot = 0.0;
    for (int d = 0; d < D; ++d) dot += qd[d] * key_at(L, j, d);
    L->s[j] = scale * dot + L->bias[j];
    if (L->s[j] > M) M = L->s[j];
  }
  if (M == -INFINITY) { /* every key carries a -inf bias */
    *lse = -INFINITY;
    return;
  }
  double denom = 0.0;
  for (int64_t j = 0; j < L->count; ++j) {
    double w = exp(L->s[j] - M);
    denom += w;
    for (int d = 0; d < D; ++d) out[d] += w * val_at(L, j, d);
  }
  for (int d = 0; d < D; ++d) out[d] /= denom;
  *lse = M + log(denom);
}

/* ------------------------------------------------------------------ */
/* a1: ring append                                                     */
/* ------------------------------------------------------------------ */

/*
 * The sliding part of the cache is a ring of n slots per (sequence, head).
 * A new token's K/V overwrite the slot at the write pointer, then the pointer
 * advances cyclically and the valid count saturates at n
 * ([SR-SWA explainer] "环形缓冲": the newest token overwrites the oldest slot
 * in place and the write pointer wraps; [R-SWA tutorial] §3.3.2: a window of
 * at most n entries to which each new K/V is appended, the oldest dropped).
 * slot_out[b] receives the slot written (nullable).
 * Pinned by: the closed form slot_s = (wp0 + s) mod n, fill = min(n, T)
 * ([R-SWA summary] §二.2, C(T) = L_m + min(n, T)) and by a deque(maxlen=n)
 * model of the ring's contents.
 */
void oracle_append(int B, int H, int n, int D, uint16_t* ring_k, uint16_t* ring_v, const uint16_t* k_new,
                   const uint16_t* v_new, int32_t* wp, int32_t* fill, int32_t* slot_out) {
  for (int b = 0; b < B; ++b) {
    int32_t slot = wp[b];
    for (int h = 0; h < H; ++h) {
      int64_t dst = (((int64_t)b * H + h) * n + slot) * D;
      int64_t src = ((int64_t)b * H + h) * D;
      memcpy(ring_k + dst, k_new + src, sizeof(uint16_t) * (size_t)D);
      memcpy(ring_v + dst, v_new + src, sizeof(uint16_t) * (size_t)D);
    }
    wp[b] = (slot + 1 == n) ? 0 : slot + 1;
    if (fill[b] < n) fill[b] = fill[b] + 1;
    if (slot_out) slot_out[b] = slot;
  }
}

/* The ring's valid slots: the fill[b] most recently written ones, i.e. the
 * slots (wp - fill + i) mod n for i in [0, fill). Their order does not
 * matter to a softmax. */
static void push_ring(keylist* L, const uint16_t* ring_k, const uint16_t* ring_v, int64_t bh, int n, int D,
                      int32_t wp, int32_t fill) {
  for (int32_t i = 0; i < fill; ++i) {
    int64_t slot = pos_mod((int64_t)wp - fill + i, n);
    int64_t off = (bh * n + slot) * D;
    keylist_push(L, ring_k + off, ring_v + off, 0.0);
  }
}

/* ------------------------------------------------------------------ */
/* a2+a3: R-SWA decode (one query per sequence and head)               */
/* ------------------------------------------------------------------ */

/*
 * Each query attends to every prefix token (all page visual tokens plus the
 * prompt, never evicted) and to the valid ring slots, which after this step's
 * append include the query's own token
 * ([R-SWA summary] §二.1; [R-SWA tutorial] §2.2.1 and §3.3.2, where the new
 * K/V is appended to the window before the attention read).
 * out [B][H][D], lse [B][H] (natural log).
 * Pinned by: n >= T reduces to full causal attention; brute force against an
 * explicit R-SWA mask on a flat timeline ([R-SWA tutorial] §3.3.1); m = 0 with
 * one valid slot gives o = v_self; constant V gives o = V.
 */
void oracle_rswa_decode(int B, int H, int D, int n, int64_t cap, const uint16_t* q, const uint16_t* pk,
                        const uint16_t* pv, const int32_t* prefix_len, const uint16_t* ring_k,
                        const uint16_t* ring_v, const int32_t* wp, const int32_t* fill, double scale, double* out,
                        double* lse) {
  int64_t BH = (int64_t)B * H;
#pragma omp parallel
  {
    keylist L;
    keylist_init(&L, cap + n);
#pragma omp for schedule(dynamic, 1)
    for (int64_t bh = 0; bh < BH; ++bh) {
      int64_t b = bh / H;
      L.count = 0;
      for (int64_t j = 0; j < prefix_len[b]; ++j) {
        int64_t off = (bh * cap + j) * D;
        keylist_push(&L, pk + off, pv + off, 0.0);
      }
      push_ring(&L, ring_k, ring_v, bh, n, D, wp[b], fill[b]);
      attend(&L, q + bh * D, D, scale, out + bh * D, lse + bh);
    }
    keylist_free(&L);
  }
}

/* ------------------------------------------------------------------ */
/* a4: R-SWA prefill rows                                              */
/* ------------------------------------------------------------------ */

/*
 * Output-side query i (0 <= i < T) of a chunk sees every prefix token and the
 * output tokens j with i - n < j <= i: the most recent n outputs including
 * itself ([R-SWA tutorial] §3.3.1 mask: reference positions always visible,
 * only the most recent n output positions visible). Positions j < 0 belong
 * to a previous chunk and are read from the ring (position -r is the r-th
 * most recently written slot, (wp - r) mod n, present when r <= fill).
 * Only the listed rows are computed: out [B][H][nrows][D], lse [B][H][nrows].
 * Pinned by: n >= T with an empty ring reduces to causal attention over
 * [prefix; outputs] with the prefix fully visible; row i equals a decode step
 * after appending outputs 0..i; a two-chunk run equals a one-chunk run.
 */
void oracle_rswa_prefill(int B, int H, int D, int n, int64_t cap, int T, const uint16_t* q, const uint16_t* k_out,
                         const uint16_t* v_out, const uint16_t* pk, const uint16_t* pv, const int32_t* prefix_len,
                         const uint16_t* ring_k, const uint16_t* ring_v, const int32_t* wp, const int32_t* fill,
                         double scale, const int32_t* rows, int nrows, double* out, double* lse) {
  int64_t work = (int64_t)B * H * nrows;
#pragma omp parallel
  {
    keylist L;
    keylist_init(&L, cap + n + 1);
#pragma omp for schedule(dynamic, 8)
    for (int64_t w = 0; w < work; ++w) {
      int64_t bh = w / nrows;
      int64_t r = w % nrows;
      int64_t b = bh / H;
      int64_t i = rows[r];
      L.count = 0;
      for (int64_t j = 0; j < prefix_len[b]; ++j) {
        int64_t off = (bh * cap + j) * D;
        keylist_push(&L, pk + off, pv + off, 0.0);
      }
      for (int64_t j = i - n + 1; j <= i; ++j) {
        if (j >= 0) {
          int64_t off = (bh * T + j) * D;
          keylist_push(&L, k_out + off, v_out + off, 0.0);
        } else if (ring_k != NULL) {
          int64_t back = -j; /* 1 = most recent previous token */
          if (back <= fill[b]) {
            int64_t slot = pos_mod((int64_t)wp[b] - back, n);
            int64_t off = (bh * n + slot) * D;
            keylist_push(&L, ring_k + off, ring_v + off, 0.0);
          }
        }
      }
      attend(&L, q + (bh * T + i) * D, D, scale, out + (bh * nrows + r) * D, lse + bh * nrows + r);
    }
    keylist_free(&L);
  }
}

/* ------------------------------------------------------------------ */
/* a5: block index keys                                                */
/* ------------------------------------------------------------------ */

/*
 * The history is cut into blocks of `blk` tokens ([SR-SWA explainer] 稀疏路由
 * step 1, sparse_block_size 32). A block's index key is the mean of its
 * tokens' index keys; a partial last block averages only its valid tokens.
 * Blocks past the prefix are zero.
 * kbar [B][ceil(cap/blk)][DI].
 * Pinned by: constant keys within a block, antithetic pairs, and a partial
 * last block whose invalid tail holds garbage.
 */
void oracle_index_pool(int B, int64_t cap, int DI, int blk, const uint16_t* k_idx, const int32_t* prefix_len,
                       double* kbar) {
  int64_t nb_cap = (cap + blk - 1) / blk;
#pragma omp parallel for schedule(static)
  for (int b = 0; b < B; ++b) {
    int64_t m = prefix_len[b];
    for (int64_t c = 0; c < nb_cap; ++c) {
      double* dst = kbar + ((int64_t)b * nb_cap + c) * DI;
      for (int d = 0; d < DI; ++d) dst[d] = 0.0;
      int64_t t0 = c * blk;
      int64_t t1 = t0 + blk < m ? t0 + blk : m;
      if (t1 <= t0) continue;
      for (int64_t t = t0; t < t1; ++t)
        for (int d = 0; d < DI; ++d) dst[d] += bf16_to_double(k_idx[((int64_t)b * cap + t) * DI + d]);
      for (int d = 0; d < DI; ++d) dst[d] /= (double)(t1 - t0);
    }
  }
}

/* ------------------------------------------------------------------ */
/* a7: exact 1.5-entmax                                                */
/* ------------------------------------------------------------------ */

typedef struct {
  double x;
  int64_t i;
} xi_pair;

static int cmp_desc(const void* a, const void* b) {
  double xa = ((const xi_pair*)a)->x, xb = ((const xi_pair*)b)->x;
  return (xa < xb) - (xa > xb);
}

/*
 * 1.5-entmax of x (x is already (alpha - 1) z = z / 2):
 *   p_i = max(x_i - tau, 0)^2 with tau fixed by sum_i p_i = 1.
 * [SR-SWA explainer] 稀疏路由 step 3 names the 1.5-entmax; the form is the
 * published alpha-entmax (Peters, Niculae & Martins, 2019, "Sparse
 * Sequence-to-Sequence Models"), solved exactly by their sort-based method:
 * sort x descending; for k = 1..K let M_k be the mean and S_k the sum of
 * squares of the k largest, delta_k = (1 - (S_k - k M_k^2)) / k and
 * tau_k = M_k - sqrt(delta_k); the support size is the largest k with
 * delta_k >= 0 and tau_k < x_(k), and tau = tau_k there.
 * Writes p[K] and returns tau. K = 0 returns NaN.
 * Pinned by: bisection on sum max(x - tau, 0)^2 = 1, the two-element closed
 * form, uniform inputs, shift invariance, non-negativity and unit sum.
 */
double oracle_entmax15(int64_t K, const double* x, double* p) {
  if (K <= 0) return NAN;
  xi_pair* s = (xi_pair*)malloc(sizeof(xi_pair) * (size_t)K);
  for (int64_t i = 0; i < K; ++i) {
    s[i].x = x[i];
    s[i].i = i;
  }
  qsort(s, (size_t)K, sizeof(xi_pair), cmp_desc);
  double sum = 0.0, sumsq = 0.0, tau = NAN;
  for (int64_t k = 1; k <= K; ++k) {
    double xk = s[k - 1].x;
    sum += xk;
    sumsq += xk * xk;
    double M = sum / (double)k;
    double delta = (1.0 - (sumsq - (double)k * M * M)) / (double)k;
    if (delta < 0.0) continue;
    double tk = M - sqrt(delta);
    if (tk < xk) tau = tk;
  }
  for (int64_t i = 0; i < K; ++i) {
    double r = x[i] - tau;
    p[i] = r > 0.0 ? r * r : 0.0;
  }
  free(s);
  return tau;
}

/* ------------------------------------------------------------------ */
/* a6-a8: router: block scores, entmax, top-k, log bias                */
/* ------------------------------------------------------------------ */

typedef struct {
  float z;
  int64_t c;
} zc_pair;

/* Descending by the fp32 score; equal scores rank the smaller block first. */
static int cmp_rank(const void* a, const void* b) {
  const zc_pair* A = (const zc_pair*)a;
  const zc_pair* Bp = (const zc_pair*)b;
  if (A->z > Bp->z) return -1;
  if (A->z < Bp->z) return 1;
  return (A->c > Bp->c) - (A->c < Bp->c);
}

/*
 * For each sequence b with NB = ceil(prefix_len[b] / blk) candidate blocks:
 *   z_c   = idx_scale * <q_idx[b], kbar[b][c]>            (step 2: low-dim index score)
 *   p     = 1.5-entmax(z / 2) over all NB candidates       (step 3)
 *   sel   = the topk blocks by z, descending, ties to the smaller index (step 4)
 *   logp  = ln p_c for each selected block (-inf where p_c = 0)   (偏置融合)
 * ([SR-SWA explainer] 稀疏路由 steps 2-4 and the log-bias fusion; top-16 from
 * sparse_topk_blocks.) Candidates are prefix blocks only: tokens in the ring
 * window are not routed. If NB < topk the tail of blk_idx is -1 with logp
 * -inf. The top-k order is decided on the score rounded to fp32, the
 * precision the device router ranks in.
 * Outputs: blk_idx [B][topk], blk_logp [B][topk], probs [B][NBcap] (nullable;
 * zero past NB), tau [B] (nullable, tau of the x = z/2 problem),
 * z_out [B][NBcap] (nullable).
 */
/* One router query against one sequence's NB block keys (the body of oracle_route). */
static void route_one(int64_t NB, int64_t nb_cap, int DI, const float* qv, const double* kb, double idx_scale,
                      int topk, int32_t* blk_idx, double* blk_logp, double* probs, double* tau, double* z_out) {
  double* z = (double*)malloc(sizeof(double) * (size_t)(NB > 0 ? NB : 1));
  double* x = (double*)malloc(sizeof(double) * (size_t)(NB > 0 ? NB : 1));
  double* p = (double*)malloc(sizeof(double) * (size_t)(NB > 0 ? NB : 1));
  zc_pair* r = (zc_pair*)malloc(sizeof(zc_pair) * (size_t)(NB > 0 ? NB : 1));
  for (int64_t c = 0; c < NB; ++c) {
    double dot = 0.0;
    for (int d = 0; d < DI; ++d) dot += (double)qv[d] * kb[c * DI + d];
    z[c] = idx_scale * dot;
    x[c] = z[c] / 2.0;
  }
  double t = oracle_entmax15(NB, x, p);
  for (int64_t c = 0; c < NB; ++c) {
    r[c].z = (float)z[c];
    r[c].c = c;
  }
  qsort(r, (size_t)NB, sizeof(zc_pair), cmp_rank);
  for (int k = 0; k < topk; ++k) {
    if (k < NB) {
      int64_t c = r[k].c;
      blk_idx[k] = (int32_t)c;
      blk_logp[k] = p[c] > 0.0 ? log(p[c]) : -INFINITY;
    } else {
      blk_idx[k] = -1;
      blk_logp[k] = -INFINITY;
    }
  }
  if (probs)
    for (int64_t c = 0; c < nb_cap; ++c) probs[c] = c < NB ? p[c] : 0.0;
  if (z_out)
    for (int64_t c = 0; c < nb_cap; ++c) z_out[c] = c < NB ? z[c] : 0.0;
  if (tau) *tau = t;
  free(z);
  free(x);
  free(p);
  free(r);
}

void oracle_route(int B, int64_t nb_cap, int DI, int blk, const float* q_idx, const double* kbar,
                  const int32_t* prefix_len, double idx_scale, int topk, int32_t* blk_idx, double* blk_logp,
                  double* probs, double* tau, double* z_out) {
#pragma omp parallel for schedule(dynamic, 1)
  for (int b = 0; b < B; ++b) {
    int64_t NB = ((int64_t)prefix_len[b] + blk - 1) / blk;
    route_one(NB, nb_cap, DI, q_idx + (int64_t)b * DI, kbar + (int64_t)b * nb_cap * DI, idx_scale, topk,
              blk_idx + (int64_t)b * topk, blk_logp + (int64_t)b * topk, probs ? probs + (int64_t)b * nb_cap : NULL,
              tau ? tau + b : NULL, z_out ? z_out + (int64_t)b * nb_cap : NULL);
  }
}

/* ------------------------------------------------------------------ */
/* a9: SR-SWA gathered-block decode                                    */
/* ------------------------------------------------------------------ */

/*
 * Each query reads only its routed blocks plus the ring window
 * ([SR-SWA explainer] "三者合起来": a fixed local window plus a fixed number
 * of remote reference blocks). A token of selected block c scores
 * scale * <q, k> + logp_c; ring tokens carry no bias; prefix tokens of
 * unselected blocks are not read. Entries with blk_idx < 0 or logp = -inf are
 * skipped. The route is shared by all heads of a sequence.
 * out [B][H][D], lse [B][H].
 * Pinned by: selecting every block with zero bias equals R-SWA decode; a
 * uniform bias over all selected blocks with an empty ring is a no-op;
 * brute force against a dense biased softmax on tiny inputs.
 */
void oracle_srswa_decode(int B, int H, int D, int n, int64_t cap, int blk, const uint16_t* q, const uint16_t* pk,
                         const uint16_t* pv, const int32_t* prefix_len, const int32_t* blk_idx,
                         const double* blk_logp, int topk, const uint16_t* ring_k, const uint16_t* ring_v,
                         const int32_t* wp, const int32_t* fill, double scale, double* out, double* lse) {
  int64_t BH = (int64_t)B * H;
#pragma omp parallel
  {
    keylist L;
    keylist_init(&L, (int64_t)topk * blk + n);
#pragma omp for schedule(dynamic, 1)
    for (int64_t bh = 0; bh < BH; ++bh) {
      int64_t b = bh / H;
      int64_t m = prefix_len[b];
      L.count = 0;
      for (int k = 0; k < topk; ++k) {
        int64_t c = blk_idx[b * topk + k];
        double bias = blk_logp[b * topk + k];
        if (c < 0 || bias == -INFINITY) continue;
        int64_t t1 = (c + 1) * blk < m ? (c + 1) * blk : m;
        for (int64_t t = c * blk; t < t1; ++t) {
          int64_t off = (bh * cap + t) * D;
          keylist_push(&L, pk + off, pv + off, bias);
        }
      }
      push_ring(&L, ring_k, ring_v, bh, n, D, wp[b], fill[b]);
      attend(&L, q + bh * D, D, scale, out + bh * D, lse + bh);
    }
    keylist_free(&L);
  }
}

/* ------------------------------------------------------------------ */
/* FP8 (e4m3) prefix cache                                             */
/* ------------------------------------------------------------------ */

/*
 * The pages list quantised KV-cache compression among the memory measures
 * ([tech analysis] 内存使用效率, "KV缓存压缩") without fixing a format.
 * Reading adopted: the prefix K and V are stored as OCP FP8 E4M3
 * codes (1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits; exponent 0
 * holds the subnormals m/8 * 2^-6; S.1111.111 is NaN; no infinities; largest
 * finite value 448), one fp32 scale per (sequence, head, 32-token block) for K
 * and one for V. A stored element is code value * scale. The ring stays bf16.
 */

/* Value of an E4M3 code, from the format's definition. Pinned by: the format's
 * landmarks (0x38 = 1, 0x7e = 448, 0x08 = 2^-6, 0x01 = 2^-9, 0x7f NaN) and by
 * exact round trips through the encoder. */
double oracle_e4m3_to_double(uint8_t c) {
  int sign = c >> 7, e = (c >> 3) & 15, m = c & 7;
  double v;
  if (e == 15 && m == 7) return NAN;
  if (e == 0)
    v = ldexp((double)m / 8.0, -6);
  else
    v = ldexp(1.0 + (double)m / 8.0, e - 7);
  return sign ? -v : v;
}

/* Round half to even of a non-negative double holding an exact value. */
static double round_half_even(double x) {
  double f = floor(x), r = x - f;
  if (r > 0.5) return f + 1.0;
  if (r < 0.5) return f;
  return fmod(f, 2.0) == 0.0 ? f : f + 1.0;
}

/* Nearest E4M3 code to x, ties to the even mantissa, magnitudes past 448
 * clamped to 448 (saturating), NaN to 0x7f. The grid spacing in the binade
 * [2^e, 2^(e+1)) is 2^(e-3) (2^-9 below 2^-6), so x / spacing is rounded to an
 * integer; a result of 16 spacings is the next binade's first value.
 * Pinned by: an exhaustive nearest-value search over the 127 non-negative
 * finite codes (tests), round trips of every finite code, and the
 * saturation and tie cases. */
uint8_t oracle_e4m3_encode(float x) {
  if (isnan(x)) return 0x7f;
  int sign = signbit(x) ? 1 : 0;
  double a = fabs((double)x);
  uint8_t code;
  if (a >= 448.0) {
    code = 0x7e;
  } else if (a < ldexp(1.0, -6)) {
    double r = round_half_even(a / ldexp(1.0, -9)); /* 0..8 spacings of 2^-9 */
    code = (uint8_t)r;                               /* 8 -> 0x08 = 2^-6, the first normal */
  } else {
    int e;
    frexp(a, &e);
    e -= 1; /* a in [2^e, 2^(e+1)) */
    double r = round_half_even(a / ldexp(1.0, e - 3)); /* 8..16 spacings */
    if (r >= 16.0) {
      e += 1;
      r = 8.0;
    }
    if (e > 8) { /* rounding past 448 (only from [448, 464) which is caught above) */
      code = 0x7e;
    } else {
      code = (uint8_t)(((e + 7) << 3) | ((int)r - 8));
      if (code == 0x7f) code = 0x7e;
    }
  }
  return (uint8_t)(code | (sign << 7));
}

/*
 * Quantises the prefix K and V: for each (sequence, head, block c) holding
 * valid rows [32c, min(m, 32c + 32)), amax = the largest |x| over those rows
 * and all D dims, scale = amax / 448 (in fp32; 1 when amax = 0), code =
 * e4m3(x / scale) with the quotient in fp32. Rows of the block past m get
 * code 0; blocks past m are not touched. codes [B][H][cap][D], scales
 * [B][H][ceil(cap / 32)]. The fp32 steps are the stated reading (a quantised
 * code is an integer decided by floating point; both sides take it in fp32).
 */
void oracle_quantize_prefix(int B, int H, int D, int64_t cap, int blk, const uint16_t* x, const int32_t* prefix_len,
                            uint8_t* codes, float* scales) {
  int64_t nb_cap = (cap + blk - 1) / blk;
  for (int b = 0; b < B; ++b) {
    int64_t m = prefix_len[b];
    for (int h = 0; h < H; ++h) {
      int64_t bh = (int64_t)b * H + h;
      for (int64_t c = 0; c * blk < m; ++c) {
        int64_t t0 = c * blk, t1 = t0 + blk < m ? t0 + blk : m;
        float amax = 0.0f;
        for (int64_t t = t0; t < t1; ++t)
          for (int d = 0; d < D; ++d) {
            float v = fabsf((float)bf16_to_double(x[(bh * cap + t) * D + d]));
            if (v > amax) amax = v;
          }
        float sc = amax > 0.0f ? amax / 448.0f : 1.0f;
        scales[bh * nb_cap + c] = sc;
        for (int64_t t = t0; t < t0 + blk && t < cap; ++t)
          for (int d = 0; d < D; ++d) {
            int64_t off = (bh * cap + t) * D + d;
            codes[off] = t < t1 ? oracle_e4m3_encode((float)bf16_to_double(x[off]) / sc) : 0;
          }
      }
    }
  }
}

/*
 * R-SWA decode over an FP8 prefix: oracle_rswa_decode with every prefix
 * element read as code value * block scale (exact in double).
 * Pinned by: data on the E4M3 grid with unit scales reproduces the bf16 decode
 * of the same values, plus the bf16 decode's own pins.
 */
void oracle_rswa_decode_fp8(int B, int H, int D, int n, int64_t cap, int blk, const uint16_t* q, const uint8_t* pk8,
                            const uint8_t* pv8, const float* kscale, const float* vscale, const int32_t* prefix_len,
                            const uint16_t* ring_k, const uint16_t* ring_v, const int32_t* wp, const int32_t* fill,
                            double scale, double* out, double* lse) {
  int64_t BH = (int64_t)B * H, nb_cap = (cap + blk - 1) / blk;
#pragma omp parallel
  {
    keylist L;
    keylist_init(&L, cap + n);
#pragma omp for schedule(dynamic, 1)
    for (int64_t bh = 0; bh < BH; ++bh) {
      int64_t b = bh / H;
      L.count = 0;
      for (int64_t j = 0; j < prefix_len[b]; ++j) {
        int64_t off = (bh * cap + j) * D, sc = bh * nb_cap + j / blk;
        keylist_push8(&L, pk8 + off, pv8 + off, kscale[sc], vscale[sc], 0.0);
      }
      push_ring(&L, ring_k, ring_v, bh, n, D, wp[b], fill[b]);
      attend(&L, q + bh * D, D, scale, out + bh * D, lse + bh);
    }
    keylist_free(&L);
  }
}

/* SR-SWA gathered decode over an FP8 prefix: oracle_srswa_decode with the
 * routed blocks' elements read as code value * block scale. */
void oracle_srswa_decode_fp8(int B, int H, int D, int n, int64_t cap, int blk, const uint16_t* q, const uint8_t* pk8,
                             const uint8_t* pv8, const float* kscale, const float* vscale, const int32_t* prefix_len,
                             const int32_t* blk_idx, const double* blk_logp, int topk, const uint16_t* ring_k,
                             const uint16_t* ring_v, const int32_t* wp, const int32_t* fill, double scale, double* out,
                             double* lse) {
  int64_t BH = (int64_t)B * H, nb_cap = (cap + blk - 1) / blk;
#pragma omp parallel
  {
    keylist L;
    keylist_init(&L, (int64_t)topk * blk + n);
#pragma omp for schedule(dynamic, 1)
    for (int64_t bh = 0; bh < BH; ++bh) {
      int64_t b = bh / H;
      int64_t m = prefix_len[b];
      L.count = 0;
      for (int k = 0; k < topk; ++k) {
        int64_t c = blk_idx[b * topk + k];
        double bias = blk_logp[b * topk + k];
        if (c < 0 || bias == -INFINITY) continue;
        int64_t t1 = (c + 1) * blk < m ? (c + 1) * blk : m;
        for (int64_t t = c * blk; t < t1; ++t) {
          int64_t off = (bh * cap + t) * D, sc = bh * nb_cap + c;
          keylist_push8(&L, pk8 + off, pv8 + off, kscale[sc], vscale[sc], bias);
        }
      }
      push_ring(&L, ring_k, ring_v, bh, n, D, wp[b], fill[b]);
      attend(&L, q + bh * D, D, scale, out + bh * D, lse + bh);
    }
    keylist_free(&L);
  }
}

/* Element-wise oracle_e4m3_encode over an array (for the tests). */
void oracle_e4m3_encode_array(int64_t count, const float* x, uint8_t* out) {
  for (int64_t i = 0; i < count; ++i) out[i] = oracle_e4m3_encode(x[i]);
}

/* ------------------------------------------------------------------ */
/* SR-SWA chunked prefill                                              */
/* ------------------------------------------------------------------ */

/*
 * Per-token routing of a prefill chunk: output-side query i of sequence b has
 * its own router query q_idx[b][i] and is routed exactly as a decode query
 * (oracle_route) against the sequence's block keys. The pages name this
 * per-token router for prefill through its [tokens, context/32] score tensor
 * (serving notes, --max-prefill-tokens); its rule is the decode router's.
 * q_idx [B][T][DI]; outputs blk_idx, blk_logp [B][T][topk].
 * Pinned by: every token equals oracle_route called on that token alone.
 */
void oracle_route_tokens(int B, int T, int64_t nb_cap, int DI, int blk, const float* q_idx, const double* kbar,
                         const int32_t* prefix_len, double idx_scale, int topk, int32_t* blk_idx, double* blk_logp) {
  int64_t BT = (int64_t)B * T;
#pragma omp parallel for schedule(dynamic, 16)
  for (int64_t bt = 0; bt < BT; ++bt) {
    int64_t b = bt / T;
    int64_t NB = ((int64_t)prefix_len[b] + blk - 1) / blk;
    route_one(NB, nb_cap, DI, q_idx + bt * DI, kbar + b * nb_cap * DI, idx_scale, topk, blk_idx + bt * topk,
              blk_logp + bt * topk, NULL, NULL, NULL);
  }
}

/*
 * SR-SWA chunked prefill rows: output-side query i of (b, h) attends to its
 * routed prefix blocks (their valid tokens, bias ln p, as in
 * oracle_srswa_decode) and to the outputs j with i - n < j <= i (bias 0),
 * positions j < 0 coming from the previous chunk's ring as in
 * oracle_rswa_prefill. Routes blk_idx / blk_logp [B][T][topk] are inputs.
 * out [B][H][nrows][D], lse [B][H][nrows].
 * Pinned by: row i equals oracle_srswa_decode after appending outputs 0..i
 * with row i's route; every block routed with zero bias equals
 * oracle_rswa_prefill.
 */
void oracle_srswa_prefill(int B, int H, int D, int n, int64_t cap, int T, int blk, const uint16_t* q,
                          const uint16_t* k_out, const uint16_t* v_out, const uint16_t* pk, const uint16_t* pv,
                          const int32_t* prefix_len, const int32_t* blk_idx, const double* blk_logp, int topk,
                          const uint16_t* ring_k, const uint16_t* ring_v, const int32_t* wp, const int32_t* fill,
                          double scale, const int32_t* rows, int nrows, double* out, double* lse) {
  int64_t work = (int64_t)B * H * nrows;
#pragma omp parallel
  {
    keylist L;
    keylist_init(&L, (int64_t)topk * blk + n + 1);
#pragma omp for schedule(dynamic, 8)
    for (int64_t w = 0; w < work; ++w) {
      int64_t bh = w / nrows;
      int64_t r = w % nrows;
      int64_t b = bh / H;
      int64_t i = rows[r];
      int64_t m = prefix_len[b];
      L.count = 0;
      for (int k = 0; k < topk; ++k) {
        int64_t c = blk_idx[(b * T + i) * topk + k];
        double bias = blk_logp[(b * T + i) * topk + k];
        if (c < 0 || bias == -INFINITY) continue;
        int64_t t1 = (c + 1) * blk < m ? (c + 1) * blk : m;
        for (int64_t t = c * blk; t < t1; ++t) {
          int64_t off = (bh * cap + t) * D;
          keylist_push(&L, pk + off, pv + off, bias);
        }
      }
      for (int64_t j = i - n + 1; j <= i; ++j) {
        if (j >= 0) {
          int64_t off = (bh * T + j) * D;
          keylist_push(&L, k_out + off, v_out + off, 0.0);
        } else if (ring_k != NULL) {
          int64_t back = -j;
          if (back <= fill[b]) {
            int64_t slot = pos_mod((int64_t)wp[b] - back, n);
            int64_t off = (bh * n + slot) * D;
            keylist_push(&L, ring_k + off, ring_v + off, 0.0);
          }
        }
      }
      attend(&L, q + (bh * T + i) * D, D, scale, out + (bh * nrows + r) * D, lse + bh * nrows + r);
    }
    keylist_free(&L);
  }
}

/* ------------------------------------------------------------------ */
/* page2d rotary position encoding                                     */
/* ------------------------------------------------------------------ */

/*
 * Nearest bf16 to x, ties to the even pattern, as its bit pattern. The bf16
 * grid in the binade [2^e, 2^(e+1)) has spacing 2^(e-7) (2^-133 below 2^-126);
 * magnitudes that round past the largest finite value give infinity.
 * Pinned by: torch's float32 -> bfloat16 conversion (round to nearest even) on
 * float32-representable inputs, exact round trips of bf16 values, and the
 * tie cases 1 + 2^-8 -> 1 and 1 + 3 * 2^-8 -> 1 + 2^-6.
 */
uint16_t oracle_bf16_round(double x) {
  if (isnan(x)) return 0x7fc0;
  uint16_t sign = signbit(x) ? 0x8000 : 0;
  double a = fabs(x), spacing;
  if (a < ldexp(1.0, -126)) {
    spacing = ldexp(1.0, -133);
  } else {
    int e;
    frexp(a, &e);
    spacing = ldexp(1.0, e - 1 - 7); /* a in [2^(e-1), 2^e) */
  }
  double r = round_half_even(a / spacing) * spacing;
  if (r >= ldexp(1.0, 128)) return (uint16_t)(sign | 0x7f80);
  float f = (float)r; /* exact: r is on the bf16 grid */
  uint32_t u;
  memcpy(&u, &f, sizeof u);
  return (uint16_t)(sign | (u >> 16));
}

void oracle_bf16_round_array(int64_t count, const double* x, uint16_t* out) {
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < count; ++i) out[i] = oracle_bf16_round(x[i]);
}

/*
 * page2d rotary position encoding of rows x [rows][H][D] (bf16), each row with
 * a token-axis position tok_pos[r] (the in-page offset) and a page-axis position
 * page[r] (the page number)
 *   [SR-SWA explainer, 2D 位置编码: two rotary axes, sparse_rope_mode page2d,
 *    the token axis orders tokens inside a page, the page axis (page_mod: 2)
 *    tells pages apart].
 * Readings where the page is silent (constants and layout are not given):
 *   - the head dimension is rotated in the half-split pairing of the LLaMA
 *     family the model's attention derives from: pair i couples dims i and
 *     i + D/2, for i < D/2, rotated by angle a:
 *       out_i = x_i cos a - x_{i+D/2} sin a,  out_{i+D/2} = x_{i+D/2} cos a + x_i sin a;
 *   - pair i has frequency theta_i = base^(-2i/D) (base 10000 in the model
 *     family; a parameter here);
 *   - page_mod interleaves the axes: pair i follows the page axis when
 *     i mod page_mod = page_mod - 1, the token axis otherwise (page_mod 2: odd
 *     pairs on the page axis, even pairs on the token axis); page_mod 0 puts
 *     every pair on the token axis (plain 1-D rotary encoding);
 *   - a = position of the pair's axis * theta_i.
 * out [rows][H][D] in fp64 (the exact rotation of the bf16 inputs).
 * Pinned by: the LLaMA rotary routine of the transformers library (page_mod 0;
 * page_mod 2 with page = tok_pos), axis separation (page 0 leaves the page-axis
 * pairs unchanged and the token-axis pairs equal the library's encoding, and
 * the converse), relative-position invariance of q.k, per-pair norms.
 */
void oracle_rope_page2d(int64_t rows, int H, int D, const uint16_t* x, const int32_t* tok_pos, const int32_t* page,
                        double base, int page_mod, double* out) {
  const int half = D / 2;
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; ++r) {
    for (int i = 0; i < half; ++i) {
      int on_page = page_mod > 0 && i % page_mod == page_mod - 1;
      double pos = on_page ? (double)page[r] : (double)tok_pos[r];
      double theta = pow(base, -2.0 * i / D);
      double c = cos(pos * theta), s = sin(pos * theta);
      for (int h = 0; h < H; ++h) {
        int64_t off = (r * H + h) * (int64_t)D;
        double lo = bf16_to_double(x[off + i]), hi = bf16_to_double(x[off + i + half]);
        out[off + i] = lo * c - hi * s;
        out[off + i + half] = hi * c + lo * s;
      }
    }
  }
}

/* ------------------------------------------------------------------ */
/* FP8 ring                                                            */
/* ------------------------------------------------------------------ */

/*
 * One row quantised on its own: scale = the largest |x| over its D dims / 448
 * in fp32 (1 when that is 0), code = E4M3(x / scale) with the quotient in fp32
 * (the prefix quantiser's rule with a single row as the block).
 */
static void quantize_row(int D, const uint16_t* x, uint8_t* codes, float* scale) {
  float amax = 0.0f;
  for (int d = 0; d < D; ++d) {
    float v = fabsf((float)bf16_to_double(x[d]));
    if (v > amax) amax = v;
  }
  float sc = amax > 0.0f ? amax / 448.0f : 1.0f;
  *scale = sc;
  for (int d = 0; d < D; ++d) codes[d] = oracle_e4m3_encode((float)bf16_to_double(x[d]) / sc);
}

/*
 * Ring append into an FP8 ring (KV-cache quantisation, [tech analysis]
 * 内存使用效率, extended from the prefix to the ring; the format is this
 * library's reading): the new token's K and V rows of every head are quantised
 * one row at a time, since the ring is written one token at a time and a row is
 * the unit that is complete when written. Codes [B][H][n][D], scales [B][H][n]
 * for K and for V; wp / fill / slot_out advance as in oracle_append.
 * Pinned by: slots, wp and fill equal oracle_append's; every written row equals
 * the prefix quantiser (separately pinned) applied to that row as a one-row block.
 */
void oracle_append_fp8(int B, int H, int n, int D, uint8_t* rk8, uint8_t* rv8, float* rks, float* rvs,
                       const uint16_t* k_new, const uint16_t* v_new, int32_t* wp, int32_t* fill,
                       int32_t* slot_out) {
  for (int b = 0; b < B; ++b) {
    int32_t slot = wp[b];
    for (int h = 0; h < H; ++h) {
      int64_t row = ((int64_t)b * H + h) * n + slot;
      int64_t src = ((int64_t)b * H + h) * D;
      quantize_row(D, k_new + src, rk8 + row * D, rks + row);
      quantize_row(D, v_new + src, rv8 + row * D, rvs + row);
    }
    wp[b] = (slot + 1 == n) ? 0 : slot + 1;
    if (fill[b] < n) fill[b] = fill[b] + 1;
    if (slot_out) slot_out[b] = slot;
  }
}

/* The FP8 ring's valid slots (as push_ring), each row with its own scales. */
static void push_ring8(keylist* L, const uint8_t* rk8, const uint8_t* rv8, const float* rks, const float* rvs,
                       int64_t bh, int n, int D, int32_t wp, int32_t fill) {
  for (int32_t i = 0; i < fill; ++i) {
    int64_t row = bh * n + pos_mod((int64_t)wp - fill + i, n);
    keylist_push8(L, rk8 + row * D, rv8 + row * D, rks[row], rvs[row], 0.0);
  }
}

/*
 * R-SWA decode over an FP8 prefix (block scales) and an FP8 ring (row scales):
 * oracle_rswa_decode with every element read as code value * its scale.
 * Pinned by: on data on the E4M3 grid whose every block and row holds a 448
 * (unit scales) it equals oracle_rswa_decode of the same values exactly.
 */
void oracle_rswa_decode_fp8kv(int B, int H, int D, int n, int64_t cap, int blk, const uint16_t* q,
                              const uint8_t* pk8, const uint8_t* pv8, const float* kscale, const float* vscale,
                              const int32_t* prefix_len, const uint8_t* rk8, const uint8_t* rv8, const float* rks,
                              const float* rvs, const int32_t* wp, const int32_t* fill, double scale, double* out,
                              double* lse) {
  int64_t BH = (int64_t)B * H, nb_cap = (cap + blk - 1) / blk;
#pragma omp parallel
  {
    keylist L;
    keylist_init(&L, cap + n);
#pragma omp for schedule(dynamic, 1)
    for (int64_t bh = 0; bh < BH; ++bh) {
      int64_t b = bh / H;
      L.count = 0;
      for (int64_t j = 0; j < prefix_len[b]; ++j) {
        int64_t off = (bh * cap + j) * D, sc = bh * nb_cap + j / blk;
        keylist_push8(&L, pk8 + off, pv8 + off, kscale[sc], vscale[sc], 0.0);
      }
      push_ring8(&L, rk8, rv8, rks, rvs, bh, n, D, wp[b], fill[b]);
      attend(&L, q + bh * D, D, scale, out + bh * D, lse + bh);
    }
    keylist_free(&L);
  }
}

/* SR-SWA gathered decode over an FP8 prefix and an FP8 ring (same pins, against
 * oracle_srswa_decode). */
void oracle_srswa_decode_fp8kv(int B, int H, int D, int n, int64_t cap, int blk, const uint16_t* q,
                               const uint8_t* pk8, const uint8_t* pv8, const float* kscale, const float* vscale,
                               const int32_t* prefix_len, const int32_t* blk_idx, const double* blk_logp, int topk,
                               const uint8_t* rk8, const uint8_t* rv8, const float* rks, const float* rvs,
                               const int32_t* wp, const int32_t* fill, double scale, double* out, double* lse) {
  int64_t BH = (int64_t)B * H, nb_cap = (cap + blk - 1) / blk;
#pragma omp parallel
  {
    keylist L;
    keylist_init(&L, (int64_t)topk * blk + n);
#pragma omp for schedule(dynamic, 1)
    for (int64_t bh = 0; bh < BH; ++bh) {
      int64_t b = bh / H;
      int64_t m = prefix_len[b];
      L.count = 0;
      for (int k = 0; k < topk; ++k) {
        int64_t c = blk_idx[b * topk + k];
        double bias = blk_logp[b * topk + k];
        if (c < 0 || bias == -INFINITY) continue;
        int64_t t1 = (c + 1) * blk < m ? (c + 1) * blk : m;
        for (int64_t t = c * blk; t < t1; ++t) {
          int64_t off = (bh * cap + t) * D, sc = bh * nb_cap + c;
          keylist_push8(&L, pk8 + off, pv8 + off, kscale[sc], vscale[sc], bias);
        }
      }
      push_ring8(&L, rk8, rv8, rks, rvs, bh, n, D, wp[b], fill[b]);
      attend(&L, q + bh * D, D, scale, out + bh * D, lse + bh);
    }
    keylist_free(&L);
  }
}
