/*
 * s3r_oracle.c -- plain fp64 CPU oracle of the Speed3R dual-branch sparse global attention.
 *
 * TEST INFRASTRUCTURE, NOT PRODUCT CODE: it exists to check the CUDA library, and only the tests,
 * the smoke check and the benchmark's CPU-baseline leg use it. It is deliberately slow and direct:
 * every quantity is computed from its definition, in double precision, one row at a time, with no
 * tiling, fusion or reordering beyond what the definition states. Work is spread over threads by
 * (head, query block) only, which does not change any arithmetic.
 *
 * Source of the method: the gist.science summary of "Speed3R: Sparse Feed-forward 3D
 * Reconstruction Models" (arXiv 2603.08055), "Technische samenvatting" -> "Methodologie":
 *   §1 "Compressie-tak": spatial downsampling by average pooling; attention over the pooled
 *      tokens yields a score matrix that identifies the relevant regions;
 *   §1 "Selectie-tak": fine attention restricted to the top-k selection guided by those scores;
 *   §2 "Gated Aggregation": a learned gate mixes the two branch outputs per token;
 *   §4 "Efficient Kernel": top-k and softmax are computed together, so the scores are softmax
 *      probabilities.
 * Where the pages leave a step open, the reading taken is the plainest one the rest supports:
 * 1-D blocks of b consecutive tokens of the flattened sequence, the last block partial (or, as an
 * option, 2-D windows of each view's patch grid with the view's special tokens as a block of
 * their own: the "spatial downsampling" read literally); pooled
 * means divide by the count of valid tokens; scores are per head; probabilities are summed over
 * the rows of a query block that lie inside the sequence; ties in the top-k go to the lower block
 * index; two independent sigmoid gates, one per branch.
 *
 * Parity status of each function (what pins it, in tests/test_oracle_pins.py):
 *   s3r_ref_round_bf16  exhaustive comparison with the float -> bf16 definition on all halfway
 *                       and neighbouring cases; torch's bf16 cast on random values.
 *   s3r_ref_pool        closed forms (constant blocks, linear ramps, ragged tail).
 *   s3r_ref_cmp         uniform-key closed form, a hand-derived worked example (tests/golden),
 *                       row-probability sums, library attention (torch SDPA, fp64).
 *   s3r_ref_topk        brute force over every k-subset; torch.topk on tie-free rows; with forced
 *                       blocks, brute force over the subsets of the other blocks, and the forced
 *                       blocks' own scores have no effect.
 *   s3r_ref_sel         with forced blocks, dense attention when F + k = nb.
 *   2-D windows         every token in exactly one block, blocks are patch rectangles cut only
 *                       at the grid edges; one-patch-high windows reproduce the 1-D path bit for
 *                       bit; a ramp pools to its value at the window centre; selection equals
 *                       SDPA under the window mask; patches permuted within windows change
 *                       nothing.
 *   s3r_ref_sel         dense attention (torch SDPA, fp64) when k = nb; brute force per query.
 *   s3r_ref_combine     gate limits and the zero-logit midpoint.
 *   whole pipeline      composition of the pinned steps plus permutation invariances.
 *   s3r_ref_bwd         torch autograd of the forward restated in torch ops (whose output equals
 *                       this file's forward); a central finite difference along a random
 *                       direction; torch SDPA's own backward when the gates switch one branch
 *                       off (dense selection; attention over torch-pooled means); key gradients
 *                       summing to zero and value gradients conserving the gated mass; equal
 *                       values giving no query/key gradient.
 *   s3r_ref_bwd_keys    equal to the rows of s3r_ref_bwd's dk, dv for the listed blocks (1-D,
 *                       forced blocks, 2-D windows, ragged tail).
 * The backward (the path is trained end to end, arXiv abstract) holds the selection lists fixed,
 * since a top-k has no gradient, and passes the bf16 rounding of the pooled K/V straight through.
 */
#include "s3r_oracle.h"

#include <math.h>
#include <pthread.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

/* ------------------------------------------------------------------------------------------ */
/* scalar helpers                                                                              */
/* ------------------------------------------------------------------------------------------ */

/* bfloat16 bit pattern -> its exact value. A bf16 number is the upper half of an IEEE binary32. */
static double bf16_value(uint16_t bits) {
  uint32_t u = (uint32_t)bits << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

double s3r_ref_round_bf16(double x) {
  /* bfloat16: 8 significant bits, exponent range of binary32 (normal >= 2^-126, subnormal
   * quantum 2^-133). Round the exact double to the nearest representable value, ties to even. */
  if (x == 0.0 || !isfinite(x)) return x;
  int e;
  (void)frexp(x, &e); /* x = m * 2^e with 0.5 <= |m| < 1, so the leading bit weighs 2^(e-1) */
  int quantum_exp = (e - 1) - 7;             /* weight of the last of 8 significant bits */
  if (quantum_exp < -133) quantum_exp = -133; /* subnormal range: fixed quantum */
  double scaled = ldexp(x, -quantum_exp);     /* exact: only the exponent changes */
  double r = nearbyint(scaled);               /* default rounding mode = to nearest, ties even */
  double y = ldexp(r, quantum_exp);
  if (fabs(y) > 3.3895313892515355e38) y = copysign(INFINITY, x); /* above the largest bf16 */
  return y;
}

static double sigmoid(double x) { return 1.0 / (1.0 + exp(-x)); }

static int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

/* ------------------------------------------------------------------------------------------ */
/* a minimal parallel-for over independent tasks                                               */
/* ------------------------------------------------------------------------------------------ */

typedef void (*task_fn)(void* ctx, int64_t task);

typedef struct {
  task_fn fn;
  void* ctx;
  int64_t ntasks;
  int64_t next; /* accessed atomically */
} pool_job;

static void* pool_worker(void* arg) {
  pool_job* job = (pool_job*)arg;
  for (;;) {
    int64_t t = __atomic_fetch_add(&job->next, 1, __ATOMIC_RELAXED);
    if (t >= job->ntasks) break;
    job->fn(job->ctx, t);
  }
  return NULL;
}

int s3r_ref_hardware_threads(void) {
  long n = sysconf(_SC_NPROCESSORS_ONLN);
  return n > 0 ? (int)n : 1;
}

static void parallel_for(int64_t ntasks, int threads, task_fn fn, void* ctx) {
  pool_job job = {fn, ctx, ntasks, 0};
  if (threads <= 0) threads = s3r_ref_hardware_threads();
  if (threads > ntasks) threads = (int)(ntasks > 0 ? ntasks : 1);
  if (threads <= 1) {
    pool_worker(&job);
    return;
  }
  pthread_t* tid = (pthread_t*)malloc(sizeof(pthread_t) * (size_t)threads);
  int started = 0;
  for (int i = 0; i < threads; ++i) {
    if (pthread_create(&tid[i], NULL, pool_worker, &job) != 0) break;
    ++started;
  }
  if (started == 0) pool_worker(&job); /* could not start threads: run inline */
  for (int i = 0; i < started; ++i) pthread_join(tid[i], NULL);
  free(tid);
}

/* ------------------------------------------------------------------------------------------ */
/* argument checks shared by the entry points of this file                                     */
/* ------------------------------------------------------------------------------------------ */

static int check_geometry(const s3r_ref_params* p) {
  if (p->grid_h == 0) return 0; /* 1-D blocks */
  if (p->grid_h < 1 || p->grid_w < 1 || p->special < 0 || p->special > p->block) return -1;
  if (p->win_h < 1 || p->block % p->win_h != 0) return -1;
  const int64_t P = (int64_t)p->special + (int64_t)p->grid_h * p->grid_w;
  return p->L % P == 0 ? 0 : -1;
}

static int check_params(const s3r_ref_params* p) {
  if (!p) return -1;
  if (p->L < 1 || p->H < 1 || p->d < 1 || p->block < 1 || p->qblock < 1) return -1;
  return check_geometry(p);
}

/* ------------------------------------------------------------------------------------------ */
/* key-block geometry: which tokens each key block holds                                       */
/* ------------------------------------------------------------------------------------------ */

/* blocks of one view under 2-D windows: the special-token block, then the windows */
static int64_t blocks_per_view(const s3r_ref_params* p) {
  const int64_t win_w = p->block / p->win_h;
  const int64_t rows = ceil_div(p->grid_h, p->win_h), cols = ceil_div(p->grid_w, win_w);
  return (p->special > 0 ? 1 : 0) + rows * cols;
}

int64_t s3r_ref_num_blocks(const s3r_ref_params* p) {
  if (check_params(p)) return 0;
  if (p->grid_h == 0) return ceil_div(p->L, p->block);
  const int64_t P = (int64_t)p->special + (int64_t)p->grid_h * p->grid_w;
  return (p->L / P) * blocks_per_view(p);
}

int64_t s3r_ref_block_tokens(const s3r_ref_params* p, int64_t j, int64_t* out) {
  if (check_params(p) || !out || j < 0 || j >= s3r_ref_num_blocks(p)) return -1;
  int64_t n = 0;
  if (p->grid_h == 0) { /* b consecutive tokens, the last block cut at L */
    for (int64_t t = j * p->block; t < (j + 1) * p->block && t < p->L; ++t) out[n++] = t;
    return n;
  }
  const int64_t P = (int64_t)p->special + (int64_t)p->grid_h * p->grid_w;
  const int64_t per_view = blocks_per_view(p);
  const int64_t view = j / per_view;
  int64_t m = j % per_view; /* block within the view */
  const int64_t first = view * P;
  if (p->special > 0) {
    if (m == 0) { /* the view's camera / register tokens */
      for (int64_t t = 0; t < p->special; ++t) out[n++] = first + t;
      return n;
    }
    m -= 1;
  }
  /* window (wr, wc) of the view's patch grid: patch rows wr*win_h.., columns wc*win_w.. */
  const int64_t win_w = p->block / p->win_h;
  const int64_t cols = ceil_div(p->grid_w, win_w);
  const int64_t wr = m / cols, wc = m % cols;
  for (int64_t r = wr * p->win_h; r < (wr + 1) * p->win_h && r < p->grid_h; ++r)
    for (int64_t c = wc * win_w; c < (wc + 1) * win_w && c < p->grid_w; ++c)
      out[n++] = first + p->special + r * p->grid_w + c;
  return n;
}

/* Rows of the chosen query blocks: first row and count of each, and their concatenated offset. */
typedef struct {
  int64_t nq;
  int64_t* block;  /* query-block index */
  int64_t* first;  /* first sequence row of the block */
  int64_t* count;  /* valid rows of the block */
  int64_t* offset; /* offset of the block's rows in the concatenated row outputs */
  int64_t rows;    /* total rows */
} row_map;

static int row_map_make(const s3r_ref_params* p, const int64_t* qblocks, int64_t nq, row_map* m) {
  int64_t nqb = ceil_div(p->L, p->qblock);
  if (!qblocks) nq = nqb;
  if (nq < 0) return -1;
  m->nq = nq;
  m->block = (int64_t*)malloc(sizeof(int64_t) * (size_t)(nq + 1));
  m->first = (int64_t*)malloc(sizeof(int64_t) * (size_t)(nq + 1));
  m->count = (int64_t*)malloc(sizeof(int64_t) * (size_t)(nq + 1));
  m->offset = (int64_t*)malloc(sizeof(int64_t) * (size_t)(nq + 1));
  int64_t off = 0;
  for (int64_t i = 0; i < nq; ++i) {
    int64_t qb = qblocks ? qblocks[i] : i;
    if (qb < 0 || qb >= nqb) {
      free(m->block), free(m->first), free(m->count), free(m->offset);
      return -2;
    }
    int64_t first = qb * p->qblock;
    int64_t last = first + p->qblock < p->L ? first + p->qblock : p->L;
    m->block[i] = qb;
    m->first[i] = first;
    m->count[i] = last - first;
    m->offset[i] = off;
    off += last - first;
  }
  m->rows = off;
  return 0;
}

static void row_map_free(row_map* m) {
  free(m->block), free(m->first), free(m->count), free(m->offset);
}

/* ------------------------------------------------------------------------------------------ */
/* compression branch, step 1: block mean pooling                                              */
/* ------------------------------------------------------------------------------------------ */

typedef struct {
  const s3r_ref_params* p;
  const uint16_t* x;
  double* out;
} pool_ctx;

static void pool_task(void* vctx, int64_t j) {
  const pool_ctx* c = (const pool_ctx*)vctx;
  const s3r_ref_params* p = c->p;
  const int64_t HD = (int64_t)p->H * p->d;
  int64_t* tok = (int64_t*)malloc(sizeof(int64_t) * (size_t)p->block);
  const int64_t n = s3r_ref_block_tokens(p, j, tok);
  for (int64_t e = 0; e < HD; ++e) {
    double sum = 0.0;
    for (int64_t a = 0; a < n; ++a) sum += bf16_value(c->x[tok[a] * HD + e]);
    double mean = sum / (double)n;
    c->out[j * HD + e] = p->exact_pool ? mean : s3r_ref_round_bf16(mean);
  }
  free(tok);
}

int s3r_ref_pool(const s3r_ref_params* p, const uint16_t* x, double* out) {
  if (check_params(p) || !x || !out) return -1;
  pool_ctx c = {p, x, out};
  parallel_for(s3r_ref_num_blocks(p), p->threads, pool_task, &c);
  return 0;
}

/* ------------------------------------------------------------------------------------------ */
/* compression branch, step 2: attention over block summaries and the block score matrix       */
/* ------------------------------------------------------------------------------------------ */

typedef struct {
  const s3r_ref_params* p;
  const uint16_t* q;
  const double* kc;
  const double* vc;
  const row_map* rm;
  double* lse;
  double* o_cmp;
  double* scores;
} cmp_ctx;

static void cmp_task(void* vctx, int64_t task) {
  const cmp_ctx* c = (const cmp_ctx*)vctx;
  const s3r_ref_params* p = c->p;
  const row_map* rm = c->rm;
  const int64_t nb = s3r_ref_num_blocks(p);
  const int64_t H = p->H, d = p->d, HD = H * d;
  const int64_t h = task / rm->nq, i = task % rm->nq;
  double* s = (double*)malloc(sizeof(double) * (size_t)nb);
  double* score_row = c->scores ? c->scores + (h * rm->nq + i) * nb : NULL;
  if (score_row)
    for (int64_t j = 0; j < nb; ++j) score_row[j] = 0.0;

  for (int64_t r = 0; r < rm->count[i]; ++r) {
    const int64_t t = rm->first[i] + r;   /* sequence row */
    const int64_t out_r = rm->offset[i] + r;
    const uint16_t* qrow = c->q + t * HD + h * d;
    /* logits s_j = scale * <q, K~_j> for every block summary j */
    double m = -INFINITY;
    for (int64_t j = 0; j < nb; ++j) {
      const double* krow = c->kc + j * HD + h * d;
      double dot = 0.0;
      for (int64_t e = 0; e < d; ++e) dot += bf16_value(qrow[e]) * krow[e];
      s[j] = p->scale * dot;
      if (s[j] > m) m = s[j];
    }
    /* log-sum-exp over all nb summaries (no mask: the partial tail block is a normal summary) */
    double l = 0.0;
    for (int64_t j = 0; j < nb; ++j) l += exp(s[j] - m);
    const double lse = m + log(l);
    if (c->lse) c->lse[h * rm->rows + out_r] = lse;
    /* probabilities, the compressed output, and the per-query-block column sums (scores) */
    double* orow = c->o_cmp ? c->o_cmp + out_r * HD + h * d : NULL;
    if (orow)
      for (int64_t e = 0; e < d; ++e) orow[e] = 0.0;
    for (int64_t j = 0; j < nb; ++j) {
      const double pj = exp(s[j] - lse);
      if (orow) {
        const double* vrow = c->vc + j * HD + h * d;
        for (int64_t e = 0; e < d; ++e) orow[e] += pj * vrow[e];
      }
      if (score_row) score_row[j] += pj;
    }
  }
  free(s);
}

int s3r_ref_cmp(const s3r_ref_params* p, const uint16_t* q, const double* kc, const double* vc,
                const int64_t* qblocks, int64_t nq, double* lse, double* o_cmp, double* scores) {
  if (check_params(p) || !q || !kc || !vc) return -1;
  row_map rm;
  int rc = row_map_make(p, qblocks, nq, &rm);
  if (rc) return rc;
  cmp_ctx c = {p, q, kc, vc, &rm, lse, o_cmp, scores};
  parallel_for((int64_t)p->H * rm.nq, p->threads, cmp_task, &c);
  row_map_free(&rm);
  return 0;
}

/* ------------------------------------------------------------------------------------------ */
/* per-row top-k                                                                               */
/* ------------------------------------------------------------------------------------------ */

typedef struct {
  double score;
  int64_t index;
} scored;

/* order: larger score first; equal scores -> lower index first */
static int scored_cmp(const void* a, const void* b) {
  const scored* x = (const scored*)a;
  const scored* y = (const scored*)b;
  if (x->score > y->score) return -1;
  if (x->score < y->score) return 1;
  return (x->index > y->index) - (x->index < y->index);
}

typedef struct {
  int64_t n;
  int32_t k;
  int32_t forced;
  const double* scores;
  int32_t* idx;
  double* gap;
} topk_ctx;

static void topk_task(void* vctx, int64_t r) {
  const topk_ctx* c = (const topk_ctx*)vctx;
  int32_t* out = c->idx + r * ((int64_t)c->forced + c->k);
  /* the always-kept blocks open the list, in ascending order */
  for (int32_t f = 0; f < c->forced; ++f) out[f] = f;
  /* the other blocks compete on their scores */
  const int64_t m = c->n - c->forced;
  scored* a = (scored*)malloc(sizeof(scored) * (size_t)m);
  for (int64_t j = 0; j < m; ++j) {
    a[j].score = c->scores[r * c->n + c->forced + j];
    a[j].index = c->forced + j;
  }
  qsort(a, (size_t)m, sizeof(scored), scored_cmp);
  for (int32_t t = 0; t < c->k; ++t) out[c->forced + t] = (int32_t)a[t].index;
  if (c->gap) c->gap[r] = c->k < m ? a[c->k - 1].score - a[c->k].score : INFINITY;
  free(a);
}

int s3r_ref_topk(int64_t rows, int64_t n, int32_t k, int32_t forced, const double* scores,
                 int32_t* idx, double* gap) {
  if (rows < 0 || n < 1 || forced < 0 || k < 1 || k > n - forced || !scores || !idx) return -1;
  topk_ctx c = {n, k, forced, scores, idx, gap};
  parallel_for(rows, 0, topk_task, &c);
  return 0;
}

/* ------------------------------------------------------------------------------------------ */
/* selection branch: exact attention over the union of the selected key blocks                 */
/* ------------------------------------------------------------------------------------------ */

typedef struct {
  const s3r_ref_params* p;
  const uint16_t* q;
  const uint16_t* k;
  const uint16_t* v;
  const row_map* rm;
  const int32_t* idx;
  double* o_sel;
  int bad_index; /* set when an index is out of range */
} sel_ctx;

static void sel_task(void* vctx, int64_t task) {
  sel_ctx* c = (sel_ctx*)vctx;
  const s3r_ref_params* p = c->p;
  const row_map* rm = c->rm;
  const int64_t nb = s3r_ref_num_blocks(p);
  const int64_t H = p->H, d = p->d, HD = H * d;
  const int64_t h = task / rm->nq, i = task % rm->nq;
  const int32_t n_list = p->forced + p->topk; /* always-kept blocks, then the top-k */
  const int32_t* sel = c->idx + (h * rm->nq + i) * n_list;

  /* the token set T: every token of every selected block, each block once, tokens < L */
  char* chosen = (char*)calloc((size_t)nb, 1);
  int64_t* tokens = (int64_t*)malloc(sizeof(int64_t) * (size_t)n_list * (size_t)p->block);
  int64_t nt = 0;
  for (int32_t s = 0; s < n_list; ++s) {
    int64_t j = sel[s];
    if (j < 0 || j >= nb) {
      c->bad_index = 1;
      continue;
    }
    if (chosen[j]) continue;
    chosen[j] = 1;
    nt += s3r_ref_block_tokens(p, j, tokens + nt);
  }
  double* s = (double*)malloc(sizeof(double) * (size_t)(nt > 0 ? nt : 1));

  for (int64_t r = 0; r < rm->count[i]; ++r) {
    const int64_t t_q = rm->first[i] + r;
    const uint16_t* qrow = c->q + t_q * HD + h * d;
    double* orow = c->o_sel + (rm->offset[i] + r) * HD + h * d;
    double m = -INFINITY;
    for (int64_t a = 0; a < nt; ++a) {
      const uint16_t* krow = c->k + tokens[a] * HD + h * d;
      double dot = 0.0;
      for (int64_t e = 0; e < d; ++e) dot += bf16_value(qrow[e]) * bf16_value(krow[e]);
      s[a] = p->scale * dot;
      if (s[a] > m) m = s[a];
    }
    double l = 0.0;
    for (int64_t a = 0; a < nt; ++a) l += exp(s[a] - m);
    for (int64_t e = 0; e < d; ++e) orow[e] = 0.0;
    for (int64_t a = 0; a < nt; ++a) {
      const double w = exp(s[a] - m) / l;
      const uint16_t* vrow = c->v + tokens[a] * HD + h * d;
      for (int64_t e = 0; e < d; ++e) orow[e] += w * bf16_value(vrow[e]);
    }
  }
  free(s);
  free(tokens);
  free(chosen);
}

int s3r_ref_sel(const s3r_ref_params* p, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                const int64_t* qblocks, int64_t nq, const int32_t* idx, double* o_sel) {
  if (check_params(p) || !q || !k || !v || !idx || !o_sel || p->topk < 1 || p->forced < 0)
    return -1;
  row_map rm;
  int rc = row_map_make(p, qblocks, nq, &rm);
  if (rc) return rc;
  sel_ctx c = {p, q, k, v, &rm, idx, o_sel, 0};
  parallel_for((int64_t)p->H * rm.nq, p->threads, sel_task, &c);
  row_map_free(&rm);
  return c.bad_index ? -3 : 0;
}

/* ------------------------------------------------------------------------------------------ */
/* backward of the whole path (selection held fixed, pooled rounding passed straight through)  */
/* ------------------------------------------------------------------------------------------ */

typedef struct {
  const s3r_ref_params* p;
  const uint16_t *q, *k, *v;
  const double *kc, *vc;
  const float* gates;
  const int32_t* idx;
  const row_map* rm; /* the query blocks whose rows are differentiated */
  const double* dout;
  double *dq, *dk, *dv, *dgates; /* dk, dv NULL: row-local gradients only */
  int bad_index;                 /* set when an index is out of range */
} bwd_ctx;

/* One head: every chosen row's forward again, then its gradients; the pooled summaries'
 * gradients are gathered over the rows and spread back over their blocks' tokens at the end. */
static void bwd_task(void* vctx, int64_t h) {
  bwd_ctx* c = (bwd_ctx*)vctx;
  const s3r_ref_params* p = c->p;
  const row_map* rm = c->rm;
  const int64_t nb = s3r_ref_num_blocks(p);
  const int64_t H = p->H, d = p->d, HD = H * d;
  const int32_t n_list = p->forced + p->topk;
  double* sc = (double*)malloc(sizeof(double) * (size_t)nb);    /* compressed logits, then P */
  double* dkc = (double*)calloc((size_t)(nb * d), sizeof(double));
  double* dvc = (double*)calloc((size_t)(nb * d), sizeof(double));
  double* qv = (double*)malloc(sizeof(double) * (size_t)d);
  double* oc = (double*)malloc(sizeof(double) * (size_t)d);
  double* os = (double*)malloc(sizeof(double) * (size_t)d);
  double* doc = (double*)malloc(sizeof(double) * (size_t)d);
  double* dos = (double*)malloc(sizeof(double) * (size_t)d);
  char* chosen = (char*)malloc((size_t)nb);
  int64_t* tokens = (int64_t*)malloc(sizeof(int64_t) * (size_t)n_list * (size_t)p->block);
  double* ss = (double*)malloc(sizeof(double) * (size_t)n_list * (size_t)p->block);

  for (int64_t i = 0; i < rm->nq; ++i) {
    /* the query block's token set T, each selected block once */
    const int32_t* sel = c->idx + (h * rm->nq + i) * n_list;
    int64_t nt = 0;
    for (int64_t j = 0; j < nb; ++j) chosen[j] = 0;
    for (int32_t s = 0; s < n_list; ++s) {
      const int64_t j = sel[s];
      if (j < 0 || j >= nb) {
        c->bad_index = 1;
        continue;
      }
      if (chosen[j]) continue;
      chosen[j] = 1;
      nt += s3r_ref_block_tokens(p, j, tokens + nt);
    }
    for (int64_t rr = 0; rr < rm->count[i]; ++rr) {
      const int64_t r = rm->first[i] + rr, o = rm->offset[i] + rr; /* sequence row, output row */
      for (int64_t e = 0; e < d; ++e) qv[e] = bf16_value(c->q[r * HD + h * d + e]);
      /* compressed branch: P over all nb summaries and O_cmp */
      double m = -INFINITY;
      for (int64_t j = 0; j < nb; ++j) {
        double dot = 0.0;
        for (int64_t e = 0; e < d; ++e) dot += qv[e] * c->kc[j * HD + h * d + e];
        sc[j] = p->scale * dot;
        if (sc[j] > m) m = sc[j];
      }
      double l = 0.0;
      for (int64_t j = 0; j < nb; ++j) l += exp(sc[j] - m);
      for (int64_t e = 0; e < d; ++e) oc[e] = 0.0;
      for (int64_t j = 0; j < nb; ++j) {
        sc[j] = exp(sc[j] - m) / l;
        for (int64_t e = 0; e < d; ++e) oc[e] += sc[j] * c->vc[j * HD + h * d + e];
      }
      /* selection branch: P over the tokens of T and O_sel */
      double ms = -INFINITY;
      for (int64_t a = 0; a < nt; ++a) {
        double dot = 0.0;
        for (int64_t e = 0; e < d; ++e) dot += qv[e] * bf16_value(c->k[tokens[a] * HD + h * d + e]);
        ss[a] = p->scale * dot;
        if (ss[a] > ms) ms = ss[a];
      }
      double ls = 0.0;
      for (int64_t a = 0; a < nt; ++a) ls += exp(ss[a] - ms);
      for (int64_t e = 0; e < d; ++e) os[e] = 0.0;
      for (int64_t a = 0; a < nt; ++a) {
        ss[a] = exp(ss[a] - ms) / ls;
        for (int64_t e = 0; e < d; ++e) os[e] += ss[a] * bf16_value(c->v[tokens[a] * HD + h * d + e]);
      }
      /* gated aggregation: out = g0 O_cmp + g1 O_sel with g = sigmoid(logit) */
      const double g0 = sigmoid((double)c->gates[(r * H + h) * 2 + 0]);
      const double g1 = sigmoid((double)c->gates[(r * H + h) * 2 + 1]);
      const double* dy = c->dout + o * HD + h * d;
      double yc = 0.0, ys = 0.0;
      for (int64_t e = 0; e < d; ++e) {
        yc += dy[e] * oc[e];
        ys += dy[e] * os[e];
        doc[e] = g0 * dy[e];
        dos[e] = g1 * dy[e];
      }
      c->dgates[(o * H + h) * 2 + 0] = g0 * (1.0 - g0) * yc;
      c->dgates[(o * H + h) * 2 + 1] = g1 * (1.0 - g1) * ys;
      /* softmax backward: dS = P (dP - <dO, O>), dP = <dO, value>; dq = scale sum dS key,
       * dkey = scale dS q, dvalue = P dO */
      double* dqr = c->dq + o * HD + h * d;
      for (int64_t e = 0; e < d; ++e) dqr[e] = 0.0;
      double dc = 0.0, ds = 0.0;
      for (int64_t e = 0; e < d; ++e) dc += doc[e] * oc[e], ds += dos[e] * os[e];
      for (int64_t j = 0; j < nb; ++j) {
        double dp = 0.0;
        for (int64_t e = 0; e < d; ++e) dp += doc[e] * c->vc[j * HD + h * d + e];
        const double dsj = sc[j] * (dp - dc);
        for (int64_t e = 0; e < d; ++e) {
          dqr[e] += p->scale * dsj * c->kc[j * HD + h * d + e];
          dkc[j * d + e] += p->scale * dsj * qv[e];
          dvc[j * d + e] += sc[j] * doc[e];
        }
      }
      for (int64_t a = 0; a < nt; ++a) {
        const int64_t t = tokens[a];
        double dp = 0.0;
        for (int64_t e = 0; e < d; ++e) dp += dos[e] * bf16_value(c->v[t * HD + h * d + e]);
        const double dsa = ss[a] * (dp - ds);
        for (int64_t e = 0; e < d; ++e)
          dqr[e] += p->scale * dsa * bf16_value(c->k[t * HD + h * d + e]);
        if (c->dk)
          for (int64_t e = 0; e < d; ++e) {
            c->dk[t * HD + h * d + e] += p->scale * dsa * qv[e];
            c->dv[t * HD + h * d + e] += ss[a] * dos[e];
          }
      }
    }
  }
  /* pooling backward: each summary is the mean of its block's tokens */
  for (int64_t j = 0; c->dk && j < nb; ++j) {
    const int64_t n = s3r_ref_block_tokens(p, j, tokens);
    for (int64_t a = 0; a < n; ++a)
      for (int64_t e = 0; e < d; ++e) {
        c->dk[tokens[a] * HD + h * d + e] += dkc[j * d + e] / (double)n;
        c->dv[tokens[a] * HD + h * d + e] += dvc[j * d + e] / (double)n;
      }
  }
  free(sc), free(dkc), free(dvc), free(qv), free(oc), free(os), free(doc), free(dos);
  free(chosen), free(tokens), free(ss);
}

int s3r_ref_bwd(const s3r_ref_params* p, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                const double* kc, const double* vc, const float* gates, const int32_t* idx,
                const int64_t* qblocks, int64_t nq, const double* dout, double* dq, double* dk,
                double* dv, double* dgates) {
  if (check_params(p) || !q || !k || !v || !kc || !vc || !gates || !idx || !dout || !dq ||
      !dgates || p->topk < 1 || p->forced < 0)
    return -1;
  /* dk, dv sum over every query: all blocks and both arrays, or a sample and neither */
  if ((!dk) != (!dv) || (qblocks && dk) || (!qblocks && !dk)) return -1;
  row_map rm;
  int rc = row_map_make(p, qblocks, nq, &rm);
  if (rc) return rc;
  if (dk) {
    const int64_t n = p->L * p->H * p->d;
    for (int64_t e = 0; e < n; ++e) dk[e] = 0.0, dv[e] = 0.0;
  }
  bwd_ctx c = {p, q, k, v, kc, vc, gates, idx, &rm, dout, dq, dk, dv, dgates, 0};
  parallel_for(p->H, p->threads, bwd_task, &c); /* heads touch disjoint slices of every array */
  row_map_free(&rm);
  return c.bad_index ? -3 : 0;
}

/* ------------------------------------------------------------------------------------------ */
/* backward, key side only: dk, dv of the tokens of a few key blocks of one head               */
/* ------------------------------------------------------------------------------------------ */

/* The same gradients as s3r_ref_bwd, for one head and the tokens of the listed key blocks only,
 * so that they can be checked at sizes where the full backward is out of reach. A token t of
 * block j receives:
 *   from the compressed branch, through the pooled mean: (scale sum_r dS_rj q_r) / n_j for dk and
 *     (sum_r P_rj g0_r dout_r) / n_j for dv, summed over every row r of the sequence;
 *   from the selection branch: scale sum_r dS_rt q_r and sum_r P_rt g1_r dout_r, summed over the
 *     rows r of the query blocks whose lists hold block j.
 * Work is split over row chunks (compressed branch, partial sums added in chunk order) and over
 * the listed blocks (selection branch), which does not change the arithmetic of any term. */
typedef struct {
  const s3r_ref_params* p;
  const uint16_t *q, *k, *v;
  const double *kc, *vc;
  const float* gates;
  const int32_t* idx;
  const double* dout;
  int64_t h, nkb, chunk;
  const int64_t* kblocks;
  double *dkc_part, *dvc_part; /* [tasks][nkb][d] */
  double *dk, *dv;             /* [nkb][block][d] */
  int bad_index;
} bwdk_ctx;

/* the compressed branch over rows [task*chunk, ...): each row's P over all summaries and O_cmp,
 * then dS against the listed summaries */
static void bwdk_cmp_task(void* vctx, int64_t task) {
  bwdk_ctx* c = (bwdk_ctx*)vctx;
  const s3r_ref_params* p = c->p;
  const int64_t nb = s3r_ref_num_blocks(p);
  const int64_t H = p->H, d = p->d, HD = H * d, h = c->h;
  double* dkc = c->dkc_part + task * c->nkb * d;
  double* dvc = c->dvc_part + task * c->nkb * d;
  double* pr = (double*)malloc(sizeof(double) * (size_t)nb);
  double* qv = (double*)malloc(sizeof(double) * (size_t)d);
  double* oc = (double*)malloc(sizeof(double) * (size_t)d);
  double* doc = (double*)malloc(sizeof(double) * (size_t)d);
  for (int64_t e = 0; e < c->nkb * d; ++e) dkc[e] = 0.0, dvc[e] = 0.0;
  const int64_t r1 = (task + 1) * c->chunk < p->L ? (task + 1) * c->chunk : p->L;
  for (int64_t r = task * c->chunk; r < r1; ++r) {
    for (int64_t e = 0; e < d; ++e) qv[e] = bf16_value(c->q[r * HD + h * d + e]);
    double m = -INFINITY;
    for (int64_t j = 0; j < nb; ++j) {
      double dot = 0.0;
      for (int64_t e = 0; e < d; ++e) dot += qv[e] * c->kc[j * HD + h * d + e];
      pr[j] = p->scale * dot;
      if (pr[j] > m) m = pr[j];
    }
    double l = 0.0;
    for (int64_t j = 0; j < nb; ++j) l += exp(pr[j] - m);
    for (int64_t e = 0; e < d; ++e) oc[e] = 0.0;
    for (int64_t j = 0; j < nb; ++j) {
      pr[j] = exp(pr[j] - m) / l;
      for (int64_t e = 0; e < d; ++e) oc[e] += pr[j] * c->vc[j * HD + h * d + e];
    }
    const double g0 = sigmoid((double)c->gates[(r * H + h) * 2 + 0]);
    double dc = 0.0;
    for (int64_t e = 0; e < d; ++e) {
      doc[e] = g0 * c->dout[r * HD + h * d + e];
      dc += doc[e] * oc[e];
    }
    for (int64_t a = 0; a < c->nkb; ++a) {
      const int64_t j = c->kblocks[a];
      double dp = 0.0;
      for (int64_t e = 0; e < d; ++e) dp += doc[e] * c->vc[j * HD + h * d + e];
      const double dsj = pr[j] * (dp - dc);
      for (int64_t e = 0; e < d; ++e) {
        dkc[a * d + e] += p->scale * dsj * qv[e];
        dvc[a * d + e] += pr[j] * doc[e];
      }
    }
  }
  free(pr), free(qv), free(oc), free(doc);
}

/* the selection branch for listed block number a: every query block whose list holds it */
static void bwdk_sel_task(void* vctx, int64_t a) {
  bwdk_ctx* c = (bwdk_ctx*)vctx;
  const s3r_ref_params* p = c->p;
  const int64_t nb = s3r_ref_num_blocks(p), nqb = ceil_div(p->L, p->qblock);
  const int64_t H = p->H, d = p->d, HD = H * d, h = c->h, jt = c->kblocks[a];
  const int32_t n_list = p->forced + p->topk;
  char* chosen = (char*)malloc((size_t)nb);
  int64_t* tokens = (int64_t*)malloc(sizeof(int64_t) * (size_t)n_list * (size_t)p->block);
  int64_t* mine = (int64_t*)malloc(sizeof(int64_t) * (size_t)p->block);
  const int64_t n_mine = s3r_ref_block_tokens(p, jt, mine);
  double* ss = (double*)malloc(sizeof(double) * (size_t)n_list * (size_t)p->block);
  double* qv = (double*)malloc(sizeof(double) * (size_t)d);
  double* os = (double*)malloc(sizeof(double) * (size_t)d);
  double* dos = (double*)malloc(sizeof(double) * (size_t)d);
  double* dk = c->dk + a * p->block * d;
  double* dv = c->dv + a * p->block * d;
  for (int64_t i = 0; i < nqb; ++i) {
    const int32_t* sel = c->idx + (h * nqb + i) * n_list;
    int holds = 0;
    for (int32_t s = 0; s < n_list; ++s) holds |= sel[s] == jt;
    if (!holds) continue;
    int64_t nt = 0;
    for (int64_t j = 0; j < nb; ++j) chosen[j] = 0;
    for (int32_t s = 0; s < n_list; ++s) {
      const int64_t j = sel[s];
      if (j < 0 || j >= nb) {
        c->bad_index = 1;
        continue;
      }
      if (chosen[j]) continue;
      chosen[j] = 1;
      nt += s3r_ref_block_tokens(p, j, tokens + nt);
    }
    const int64_t r0 = i * p->qblock, r1 = r0 + p->qblock < p->L ? r0 + p->qblock : p->L;
    for (int64_t r = r0; r < r1; ++r) {
      for (int64_t e = 0; e < d; ++e) qv[e] = bf16_value(c->q[r * HD + h * d + e]);
      double ms = -INFINITY;
      for (int64_t t = 0; t < nt; ++t) {
        double dot = 0.0;
        for (int64_t e = 0; e < d; ++e) dot += qv[e] * bf16_value(c->k[tokens[t] * HD + h * d + e]);
        ss[t] = p->scale * dot;
        if (ss[t] > ms) ms = ss[t];
      }
      double ls = 0.0;
      for (int64_t t = 0; t < nt; ++t) ls += exp(ss[t] - ms);
      for (int64_t e = 0; e < d; ++e) os[e] = 0.0;
      for (int64_t t = 0; t < nt; ++t) {
        ss[t] = exp(ss[t] - ms) / ls;
        for (int64_t e = 0; e < d; ++e) os[e] += ss[t] * bf16_value(c->v[tokens[t] * HD + h * d + e]);
      }
      const double g1 = sigmoid((double)c->gates[(r * H + h) * 2 + 1]);
      double ds = 0.0;
      for (int64_t e = 0; e < d; ++e) {
        dos[e] = g1 * c->dout[r * HD + h * d + e];
        ds += dos[e] * os[e];
      }
      for (int64_t t = 0; t < nt; ++t) {
        int64_t slot = -1;
        for (int64_t u = 0; u < n_mine; ++u)
          if (mine[u] == tokens[t]) slot = u;
        if (slot < 0) continue;
        double dp = 0.0;
        for (int64_t e = 0; e < d; ++e) dp += dos[e] * bf16_value(c->v[tokens[t] * HD + h * d + e]);
        const double dst = ss[t] * (dp - ds);
        for (int64_t e = 0; e < d; ++e) {
          dk[slot * d + e] += p->scale * dst * qv[e];
          dv[slot * d + e] += ss[t] * dos[e];
        }
      }
    }
  }
  free(chosen), free(tokens), free(mine), free(ss), free(qv), free(os), free(dos);
}

int s3r_ref_bwd_keys(const s3r_ref_params* p, const uint16_t* q, const uint16_t* k,
                     const uint16_t* v, const double* kc, const double* vc, const float* gates,
                     const int32_t* idx, int32_t h, const int64_t* kblocks, int64_t nkb,
                     const double* dout, double* dk, double* dv) {
  if (check_params(p) || !q || !k || !v || !kc || !vc || !gates || !idx || !dout || !dk || !dv ||
      !kblocks || nkb < 1 || h < 0 || h >= p->H || p->topk < 1 || p->forced < 0)
    return -1;
  const int64_t nb = s3r_ref_num_blocks(p), d = p->d;
  for (int64_t a = 0; a < nkb; ++a)
    if (kblocks[a] < 0 || kblocks[a] >= nb) return -1;
  const int64_t chunk = 256, ntask = ceil_div(p->L, chunk);
  bwdk_ctx c = {p, q, k, v, kc, vc, gates, idx, dout, h, nkb, chunk, kblocks, NULL, NULL, dk, dv,
                0};
  c.dkc_part = (double*)malloc(sizeof(double) * (size_t)(ntask * nkb * d));
  c.dvc_part = (double*)malloc(sizeof(double) * (size_t)(ntask * nkb * d));
  for (int64_t e = 0; e < nkb * p->block * d; ++e) dk[e] = 0.0, dv[e] = 0.0;
  parallel_for(ntask, p->threads, bwdk_cmp_task, &c);
  parallel_for(nkb, p->threads, bwdk_sel_task, &c);
  /* pooling backward: each summary is the mean of its block's tokens */
  int64_t* tokens = (int64_t*)malloc(sizeof(int64_t) * (size_t)p->block);
  for (int64_t a = 0; a < nkb; ++a) {
    const int64_t n = s3r_ref_block_tokens(p, kblocks[a], tokens);
    for (int64_t e = 0; e < d; ++e) {
      double sk = 0.0, sv = 0.0;
      for (int64_t t = 0; t < ntask; ++t) {
        sk += c.dkc_part[(t * nkb + a) * d + e];
        sv += c.dvc_part[(t * nkb + a) * d + e];
      }
      for (int64_t u = 0; u < n; ++u) {
        dk[(a * p->block + u) * d + e] += sk / (double)n;
        dv[(a * p->block + u) * d + e] += sv / (double)n;
      }
    }
  }
  free(tokens), free(c.dkc_part), free(c.dvc_part);
  return c.bad_index ? -3 : 0;
}

/* ------------------------------------------------------------------------------------------ */
/* gated aggregation                                                                           */
/* ------------------------------------------------------------------------------------------ */

int s3r_ref_combine(int64_t n, int32_t H, int32_t d, const double* o_cmp, const double* o_sel,
                    const float* gates, double* out) {
  if (n < 0 || H < 1 || d < 1 || !o_cmp || !o_sel || !gates || !out) return -1;
  for (int64_t r = 0; r < n; ++r)
    for (int64_t h = 0; h < H; ++h) {
      const double g_cmp = sigmoid((double)gates[(r * H + h) * 2 + 0]);
      const double g_sel = sigmoid((double)gates[(r * H + h) * 2 + 1]);
      for (int64_t e = 0; e < d; ++e) {
        const int64_t at = (r * H + h) * d + e;
        out[at] = g_cmp * o_cmp[at] + g_sel * o_sel[at];
      }
    }
  return 0;
}
