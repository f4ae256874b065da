/*
 * s3r_oracle.h -- plain fp64 CPU oracle of the Speed3R dual-branch sparse global attention.
 *
 * TEST INFRASTRUCTURE, NOT PRODUCT CODE. Only the test-suite, the smoke check and the benchmark's
 * CPU-baseline leg load this library. It shares no code, header, table or helper with the CUDA
 * library under sparse_global_attention_s3r_b200/csrc.
 *
 * Method (Speed3R, "Technische samenvatting" -> "Methodologie" of the gist.science summary of
 * arXiv 2603.08055, §1 "Compressie-tak" / "Selectie-tak" and §2 "Gated Aggregation"):
 *   compression branch: K and V are mean-pooled over blocks of b tokens; every query attends to the
 *     block summaries; the softmax probabilities form the score matrix that ranks key blocks;
 *   selection branch: per query block, exact attention over the tokens of the top-k key blocks;
 *   gated aggregation: the two branch outputs are mixed by per-token, per-head sigmoid gates.
 *
 * Conventions (all arrays dense, row-major):
 *   Q, K, V      [L, H, d]   bf16, passed as their raw 16-bit patterns (uint16_t)
 *   pooled K/V   [nb, H, d]  double          nb  = ceil(L / block) for 1-D blocks, else the
 *                                           number of 2-D windows (see s3r_ref_params)
 *   gates        [L, H, 2]   float           [...,0] compression gate logit, [...,1] selection
 *   lse          [H, R]      double          R = rows of the chosen query blocks (see below)
 *   o_cmp, o_sel [R, H, d]   double
 *   scores       [H, nq, nb] double          nq = number of chosen query blocks
 *   idx          [H, nq, F + k] int32   F = forced blocks (0 unless the reference-frame variant)
 * A call may restrict the query side to a list of query-block indices ("sampled mode"); its row
 * outputs are then the rows of those blocks, concatenated in list order. A NULL list means every
 * query block 0 .. ceil(L / qblock) - 1.
 *
 * Every function returns 0 on success and a negative value on a bad argument; nothing is printed.
 */
#ifndef S3R_ORACLE_H
#define S3R_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct {
  int64_t L;        /* tokens in the flattened sequence (N views x P tokens per view), >= 1 */
  int32_t H;        /* heads */
  int32_t d;        /* head dimension */
  int32_t block;    /* b: key-block size of the pooling and of the selection unit */
  int32_t qblock;   /* rows per query block over which probabilities are summed */
  int32_t topk;     /* k: key blocks selected per query block, 1 <= k <= nb */
  double scale;     /* softmax scale applied to q.k in both branches */
  int32_t exact_pool; /* 0: pooled K/V are rounded to bf16 (RNE) like a tensor-core operand;
                         1: keep the exact fp64 mean (used by the closed-form checks) */
  int32_t threads;  /* worker threads, 0 = all online cores */
  int32_t forced;   /* F: key blocks 0 .. F-1 open every selection list (the VGGT variant keeps the
                       reference frame's tokens for every query); the top-k then picks k more
                       among blocks F .. nb-1, so a list holds F + k blocks. 0 = plain top-k. */
  /* Key-block geometry. grid_h == 0: 1-D blocks, block j = tokens [j*b, min((j+1)*b, L)).
   * grid_h > 0: 2-D windows on each view's patch grid ("spatial downsampling", Methodologie §1).
   * The sequence is N = L / P views of P = special + grid_h * grid_w tokens each: `special`
   * leading tokens (camera and register tokens), then the grid_h x grid_w patches in row-major
   * order. Each view contributes, in this order, one block holding its special tokens (when
   * special > 0) and the windows of win_h x (b / win_h) patches that tile its grid from the
   * top-left, row by row; windows at the right and bottom edges hold only the patches inside
   * the grid. Blocks are numbered view by view. Query blocks stay 64 consecutive tokens. */
  int32_t grid_h, grid_w, special, win_h;
} s3r_ref_params;

/* Number of key blocks nb of the geometry in p (0 if the geometry is invalid). */
int64_t s3r_ref_num_blocks(const s3r_ref_params* p);

/* Tokens of key block j in ascending order, written to out (room for p->block entries);
 * returns their count, or -1 for a bad argument. */
int64_t s3r_ref_block_tokens(const s3r_ref_params* p, int64_t j, int64_t* out);

/* Number of cores the oracle uses when params.threads == 0. */
int s3r_ref_hardware_threads(void);

/* Round a double to the nearest bfloat16 value (ties to even), returned as a double. */
double s3r_ref_round_bf16(double x);

/* Compression branch, step 1: block means of x over the tokens of each block.
 * out[j,h,c] = (1/n_j) sum_{t in block j} x[t,h,c], n_j = number of tokens of block j (1-D: the
 * tokens below L). */
int s3r_ref_pool(const s3r_ref_params* p, const uint16_t* x, double* out);

/* Compression branch, step 2: attention of each chosen query row to all nb block summaries,
 * and the block score matrix (sum of the row probabilities over each query block).
 * Any of lse, o_cmp, scores may be NULL. */
int s3r_ref_cmp(const s3r_ref_params* p, const uint16_t* q, const double* kc, const double* vc,
                const int64_t* qblocks, int64_t nq, double* lse, double* o_cmp, double* scores);

/* Per-row selection lists from a [rows, n] score matrix, F + k entries per row ([rows, F + k]):
 * first the forced blocks 0 .. F-1 in ascending order, then the k largest scores among columns
 * F .. n-1 in descending score order, equal scores by lower index. gap[r] = k-th largest minus
 * (k+1)-th largest of those columns (+inf when k == n - F). gap may be NULL. F = 0 is the plain
 * top-k. (Speed3R, "Methodologie" §3: for VGGT the reference-frame tokens are always kept while
 * the rest is sparsified.) */
int s3r_ref_topk(int64_t rows, int64_t n, int32_t k, int32_t forced, const double* scores,
                 int32_t* idx, double* gap);

/* Selection branch: exact softmax attention of each chosen query row over the tokens of the
 * F + k key blocks idx[h, i, :] of its query block (tokens >= L excluded; a block listed twice
 * counts once). */
int s3r_ref_sel(const s3r_ref_params* p, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                const int64_t* qblocks, int64_t nq, const int32_t* idx, double* o_sel);

/* Backward of the whole path (Speed3R is trained end to end, arXiv abstract): given dout =
 * dLoss/dout [L, H, d], the gradients dq, dk, dv [L, H, d] and dgates [L, H, 2] (all double, all
 * rows). The selection lists idx [H, nqb, F + k] are held fixed (no gradient flows through the
 * top-k), and the bf16 rounding of the pooled K/V is passed straight through: kc, vc are the
 * pooled values the forward used (s3r_ref_pool), and dK[t] += dKc[j] / n_j for the n_j tokens t
 * of block j (the same for V). Returns 0, -1 on bad parameters, -3 when idx holds an index
 * outside [0, nb).
 * qblocks (nullable): differentiate only the rows of these nq query blocks. idx is then
 * [H, nq, F + k] for them, dout, dq [R, H, d] and dgates [R, H, 2] hold their R rows
 * concatenated in list order, and dk, dv must be NULL: they sum over every query. With
 * qblocks NULL every array covers all L rows and dk, dv are required. */
int s3r_ref_bwd(const s3r_ref_params* p, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                const double* kc, const double* vc, const float* gates, const int32_t* idx,
                const int64_t* qblocks, int64_t nq, const double* dout, double* dq, double* dk,
                double* dv, double* dgates);

/* dk, dv of one head h for the tokens of nkb listed key blocks kblocks[], each in [0, nb): the
 * same gradients as s3r_ref_bwd (selection lists idx [H, nqb, F + k] held fixed, pooled rounding
 * passed straight through), computed from all L rows of q, gates [L, H, 2] and dout [L, H, d]
 * without forming the other blocks' gradients. dk, dv are [nkb, block, d]: row u of listed block
 * a is the u-th token of that block (ascending, as s3r_ref_block_tokens lists them); rows past
 * the block's token count are zero. Returns 0, -1 on bad arguments, -3 if idx held an index
 * outside [0, nb). */
int s3r_ref_bwd_keys(const s3r_ref_params* p, const uint16_t* q, const uint16_t* k,
                     const uint16_t* v, const double* kc, const double* vc, const float* gates,
                     const int32_t* idx, int32_t h, const int64_t* kblocks, int64_t nkb,
                     const double* dout, double* dk, double* dv);

/* Gated aggregation over n rows: out = sigmoid(g[...,0]) * o_cmp + sigmoid(g[...,1]) * o_sel. */
int s3r_ref_combine(int64_t n, int32_t H, int32_t d, const double* o_cmp, const double* o_sel,
                    const float* gates, double* out);

#ifdef __cplusplus
}
#endif
#endif
