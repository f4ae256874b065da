/*
 * s3r.h -- C ABI of the B200 (sm_100a) sparse global attention library, libs3r.so.
 *
 * The operation is the dual-branch global sparse attention of Speed3R ("Speed3R: Sparse
 * Feed-forward 3D Reconstruction Models", arXiv 2603.08055). Its pages describe it in prose only
 * (gist.science summary, "Technische samenvatting" -> "Methodologie"):
 *   §1 "Compressie-tak"  the compression branch pools the tokens spatially by averaging, attends
 *                        to the pooled tokens and produces a score matrix of relevant regions;
 *   §1 "Selectie-tak"    the selection branch runs fine-grained attention only on the tokens of
 *                        the top-k regions picked by those scores;
 *   §2 "Gated Aggregation" a learned gate per token mixes the outputs of the two branches;
 *   §4 "Efficient Kernel" top-k and softmax are computed together on chip.
 * The project README (github Visual-AI/speed3r, "Notice" 3) restricts the kernel to bf16/fp16.
 *
 * Definitions used by every entry point (h = head, all layouts dense row-major):
 *   L tokens of the flattened multi-view sequence (N views x P tokens per view), H heads, d = 64.
 *   Key block j = tokens [j*b, min((j+1)*b, L)), nb = ceil(L/b); the last block may be partial.
 *   Query block i = rows [64*i, min(64*i+64, L)), nqb = ceil(L/64).
 *   Pooled keys/values   Kc[j,h,:] = mean of K[t,h,:] over the valid tokens t of block j (same
 *                        for V), accumulated in fp32 and rounded once to bf16.
 *   Compressed logits    s[q,j] = scale * <Q[q,h,:], Kc[j,h,:]>, for all j < nb.
 *   lse[h,q]             = log sum_j exp(s[q,j])                       (natural log)
 *   P[q,j]               = exp(s[q,j] - lse[h,q])                      (fp32)
 *   O_cmp[q,h,:]         = sum_j P[q,j] * Vc[j,h,:]
 *   scores[h,i,j]        = sum over the valid rows q of query block i of P[q,j]
 *   idx[h,i,:]           = the selection list of query block i, F + topk entries: the forced
 *                          blocks 0 .. F-1 (F = params.forced, usually 0), then the topk block
 *                          indices j >= F with the largest scores[h,i,j], ties broken toward the
 *                          lower index
 *   O_sel[q,h,:]         = softmax-weighted sum of V[t,h,:] over the tokens t < L of the
 *                          blocks idx[h,i,:] of q's query block, weights softmax_t(scale*<Q,K[t]>)
 *   out[q,h,:]           = sigmoid(g[q,h,0]) * O_cmp[q,h,:] + sigmoid(g[q,h,1]) * O_sel[q,h,:]
 *
 * Conventions:
 *   - Every pointer argument is a DEVICE pointer of the current CUDA device, 16-byte aligned,
 *     to a dense row-major array; the caller owns every buffer. The library never allocates or
 *     frees device memory. Only s3r_read_device_status and s3r_last_device_error synchronise the
 *     stream (they read a word the stream's kernels write); every other call is asynchronous.
 *   - Calls are asynchronous on `stream` (NULL = the legacy default stream). The return value
 *     reports host-side validation and launch errors only; a call that returns an error has
 *     launched nothing, except S3R_ERR_CUDA which reports a failed launch.
 *   - Conditions detected on the device (a bounded wait that expired, an out-of-range index when
 *     S3R_FLAG_DEBUG_CHECKS is set) are OR-ed into the 32-bit word params->dev_status when it is
 *     non-NULL, and into the workspace's status word in s3r_sparse_attn_fwd. Read it with
 *     s3r_read_device_status (or s3r_last_device_error).
 *   - bf16 values are passed as their 16-bit patterns (s3r_bf16).
 *   - No C++ exception crosses this boundary. The functions are thread-safe. The global state is
 *     a launch counter and, for s3r_sparse_attn_fwd_static only, one device array per GPU with a
 *     per-device table of its address; calls of that entry point that overlap on the GPU race
 *     on the array (see its comment). Every other entry point works on caller buffers only.
 */
#ifndef S3R_H
#define S3R_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t s3r_bf16;            /* raw bfloat16 bit pattern */
typedef struct CUstream_st* s3r_stream; /* identical to cudaStream_t */

typedef enum {
  S3R_OK = 0,
  S3R_ERR_INVALID_ARG = 1, /* null/misaligned pointer, bad size, topk out of range */
  S3R_ERR_UNSUPPORTED = 2, /* a size this build does not implement (d, b, qblock, nb) */
  S3R_ERR_WORKSPACE = 3,   /* workspace missing or smaller than s3r_workspace_bytes() */
  S3R_ERR_CUDA = 4,        /* a CUDA runtime call or kernel launch failed */
  S3R_ERR_TIMEOUT = 5      /* reported via the device status word: a bounded wait expired */
} s3r_status;

/* Bits of the device status word. */
#define S3R_DEV_TIMEOUT 0x1u   /* a kernel gave up on a bounded wait and returned early */
#define S3R_DEV_BAD_INDEX 0x2u /* (debug checks) an idx entry was outside [0, nb) */

/* params.flags */
#define S3R_FLAG_DEBUG_CHECKS 0x1u /* validate idx on the device in s3r_sel_attn and
                                     s3r_sparse_attn_bwd */
#define S3R_FLAG_TEST_TIMEOUT 0x2u /* testing only: the tensor-core kernels (compressed branch,
                                      selection, the single fused kernel, and the backward's dq,
                                      dKc/dVc and dk/dv kernels) wait on a barrier that nothing
                                      signals, with a 1 ms limit, so their timeout paths run:
                                      S3R_DEV_TIMEOUT is set and the outputs are invalid */
#define S3R_FLAG_SINGLE_KERNEL 0x4u /* s3r_sparse_attn_fwd with topk <= 32: after pooling, one
                                       kernel per (query tile, head) runs the compressed branch,
                                       the top-k and the selection branch with the gated combine,
                                       keeping O_cmp (as bf16) and the lists on chip (2 launches);
                                       its stage S3R_STAGE_CMP then covers selection too */
#define S3R_FLAG_SAVE_FOR_BWD 0x8u  /* s3r_sparse_attn_fwd also keeps, in its workspace, what
                                       s3r_sparse_attn_bwd needs (O_cmp, O_sel, both branches'
                                       lse, the pooled K/V and their slot-order copies), so that
                                       a backward call given the same flag and the same workspace
                                       skips recomputing the forward. The workspace then grows
                                       (s3r_workspace_bytes reports it); S3R_FLAG_SINGLE_KERNEL
                                       is ignored (the 3-kernel path runs) */

#define S3R_FLAG_NVTX 0x10u         /* s3r_sparse_attn_fwd and s3r_sparse_attn_bwd push one NVTX
                                       range per stage ("s3r.pool", "s3r.cmp", ...), so profilers
                                       (ncu --nvtx, nsys) can attribute kernels to stages; off by
                                       default (the ranges cost host time only when a tool is
                                       attached) */

typedef struct {
  int64_t L;      /* tokens = N views * P tokens per view, >= 1 */
  int32_t H;      /* heads, >= 1 */
  int32_t d;      /* head dimension; this build implements d = 64 */
  int32_t block;  /* b, key-block size: 32, 64 or 128 */
  int32_t qblock; /* rows per query block for the score sums; must be 64 */
  int32_t topk;   /* k, blocks selected per query block, 1 <= k <= nb (k = nb: dense selection) */
  float scale;    /* softmax scale; <= 0 selects 1/sqrt(d) */
  uint32_t flags; /* S3R_FLAG_* */
  int32_t forced; /* F >= 0: key blocks 0 .. F-1 open every selection list without competing,
                     and topk more are chosen among blocks F .. nb-1 (topk <= nb - F). The VGGT
                     variant keeps the reference frame's tokens for every query ("Methodologie"
                     §3): with P tokens per view, F = ceil(P / b) (with 2-D windows: the
                     number of blocks of one view). 0 = plain top-k. */
  /* Key-block geometry. grid_h = 0: 1-D blocks, block j = tokens [j*b, min((j+1)*b, L)).
     grid_h > 0: 2-D windows on each view's patch grid ("Methodologie" §1: the compression branch
     downsamples spatially). The sequence is N = L / P views of P = special + grid_h * grid_w
     tokens: `special` leading tokens (camera, register), then the patches row by row. Each view
     contributes one block of its special tokens (if special > 0), then the windows of
     win_h x (b / win_h) patches tiling its grid from the top-left, row by row, cut at the
     right and bottom edges. Blocks are numbered view by view; query blocks stay 64 consecutive
     tokens. Requires 1 <= win_h, b % win_h == 0, 0 <= special <= b, L % P == 0. */
  int32_t grid_h, grid_w, special, win_h;
  uint32_t* dev_status; /* optional device word that receives S3R_DEV_* bits (may be NULL) */
  void* const* stage_events; /* optional: S3R_NUM_STAGES + 1 cudaEvent_t handles that
                                s3r_sparse_attn_fwd records on `stream` at the stage boundaries
                                (before stage 0, after each stage), for per-stage timing with
                                cudaEventElapsedTime; s3r_sparse_attn_bwd records
                                S3R_NUM_BWD_STAGES + 1 of them the same way; ignored by the
                                single-step entry points */
} s3r_params;

/* Stages of s3r_sparse_attn_fwd, in launch order (one kernel each). */
#define S3R_STAGE_POOL 0        /* K/V block pooling */
#define S3R_STAGE_CMP 1         /* compressed attention (lse pass, then O_cmp and block scores) */
#define S3R_STAGE_TOPK 2        /* per-query-block top-k; empty (no launch) when topk <= 32,
                                   where the compressed stage selects the blocks on the fly */
#define S3R_STAGE_SEL_COMBINE 3 /* selection attention fused with the gated combine */
#define S3R_NUM_STAGES 4

/* Stages of s3r_sparse_attn_bwd, in launch order. */
#define S3R_BWD_STAGE_RECOMPUTE 0 /* the forward again: pooling, both branches with their lse */
#define S3R_BWD_STAGE_PREP 1      /* D and gate gradients; the inverse of the selection lists and
                                     the token-side work order */
#define S3R_BWD_STAGE_DQ 2        /* dq of both branches (one kernel) */
#define S3R_BWD_STAGE_DKV_CMP 3   /* dKc, dVc of the block summaries */
#define S3R_BWD_STAGE_DKV_SEL 4   /* dk, dv of the selected tokens, plus dKc / n_j, dVc / n_j */
#define S3R_NUM_BWD_STAGES 5

/* Largest nb (key blocks) this build accepts; beyond it calls return S3R_ERR_UNSUPPORTED. */
#define S3R_MAX_BLOCKS 49152

/* Human-readable name of a status code (static string, never NULL). */
const char* s3r_status_string(s3r_status status);

/* Library version as major*10000 + minor*100 + patch. */
int s3r_version(void);

/* Number of kernels this process has launched through the library so far (monotonic). */
uint64_t s3r_kernel_launches(void);

/* Number of key blocks nb of the geometry in params (0 if params are invalid). */
int64_t s3r_num_key_blocks(const s3r_params* params);

/* Bytes of device workspace s3r_sparse_attn_fwd needs for these sizes (0 if params invalid). */
size_t s3r_workspace_bytes(const s3r_params* params);

/* Synchronise `stream`, copy the device status word at `dev_status` into *out and clear it.
 * Returns S3R_ERR_TIMEOUT if the S3R_DEV_TIMEOUT bit was set, S3R_OK otherwise. */
s3r_status s3r_read_device_status(uint32_t* dev_status, s3r_stream stream, uint32_t* out);

/* Device status word inside a workspace given to s3r_sparse_attn_fwd. */
uint32_t* s3r_workspace_status_word(void* workspace);

/* The same read as s3r_read_device_status, returning only the status: synchronise `stream`, read
 * and clear the 32-bit device word at flag_buf (params->dev_status, or a workspace's word), and
 * map its bits to a status: S3R_ERR_TIMEOUT if a bounded wait expired, S3R_ERR_INVALID_ARG if a
 * debug check found an index outside [0, nb), S3R_OK if neither. A NULL or misaligned flag_buf is
 * S3R_ERR_INVALID_ARG; a failed copy S3R_ERR_CUDA. */
s3r_status s3r_last_device_error(void* flag_buf, s3r_stream stream);

/* Compression branch, pooling ("Compressie-tak": average pooling).
 *   k, v         [L, H, d] bf16 (read)
 *   k_cmp, v_cmp [nb, H, d] bf16 (written): fp32 mean over the valid tokens, rounded to nearest
 *                even bf16. */
s3r_status s3r_compress_kv(const s3r_params* params, const s3r_bf16* k, const s3r_bf16* v,
                           s3r_bf16* k_cmp, s3r_bf16* v_cmp, s3r_stream stream);

/* Compression branch, attention to the block summaries and the score matrix
 * ("Compressie-tak": "scorematrix").
 *   q            [L, H, d] bf16;  k_cmp, v_cmp [nb, H, d] bf16 (read)
 *   o_cmp        [L, H, d] fp32   (written)
 *   lse          [H, L] fp32      (written, natural log)
 *   scores       [H, nqb, nb] fp32 (written)
 * Probabilities are formed in fp32 before the scores are summed; P is rounded to bf16 only as
 * the operand of the P*Vc product. */
s3r_status s3r_cmp_attn_and_score(const s3r_params* params, const s3r_bf16* q,
                                  const s3r_bf16* k_cmp, const s3r_bf16* v_cmp, float* o_cmp,
                                  float* lse, float* scores, s3r_stream stream);

/* Per-query-block top-k ("Selectie-tak": "Top-k selectie").
 *   scores [H, nqb, nb] fp32 (read), non-negative, not NaN
 *   idx    [H, nqb, forced + topk] int32 (written): blocks 0 .. forced-1, then the top-k of
 *          blocks forced .. nb-1. The set is exact: score bits compared as unsigned integers,
 *          equal scores broken toward the lower block index. For topk <= 2048 the top-k entries
 *          are ordered by descending score, ties by ascending index; for larger topk they are in
 *          ascending index order. */
s3r_status s3r_topk_blocks(const s3r_params* params, const float* scores, int32_t* idx,
                           s3r_stream stream);

/* Selection branch ("Selectie-tak": fine attention on the selected tokens).
 *   q, k, v [L, H, d] bf16 (read); idx [H, nqb, forced + topk] int32 (read): distinct block
 *           indices in [0, nb) per row (entries outside that range are skipped; with
 *           S3R_FLAG_DEBUG_CHECKS they also raise S3R_DEV_BAD_INDEX)
 *   o_sel   [L, H, d] fp32 (written)
 *   With 2-D windows narrower than 8 patches (b / win_h < 8) this entry point returns
 *   S3R_ERR_UNSUPPORTED; s3r_sparse_attn_fwd takes them. */
s3r_status s3r_sel_attn(const s3r_params* params, const s3r_bf16* q, const s3r_bf16* k,
                        const s3r_bf16* v, const int32_t* idx, float* o_sel, s3r_stream stream);

/* Gated aggregation (§2 "Gated Aggregation"), elementwise.
 *   o_cmp, o_sel [L, H, d] fp32 (read); gate_logits [L, H, 2] fp32 (read): [...,0] gates the
 *   compression branch, [...,1] the selection branch, each through its own sigmoid
 *   out          [L, H, d] bf16 (written, round to nearest even) */
s3r_status s3r_gate_combine(const s3r_params* params, const float* o_cmp, const float* o_sel,
                            const float* gate_logits, s3r_bf16* out, s3r_stream stream);

/* The whole path in one call: pooling, compressed attention and scores, top-k, selection
 * attention fused with the gated combine. For topk <= 32 the compressed-attention kernel keeps a
 * running top-k of every query block while it produces the scores, so the [H, nqb, nb] score
 * matrix is never written (3 kernel launches); larger topk materialise it in the workspace and run
 * s3r_topk_blocks' kernel (4 launches). Both select the same blocks.
 *   q, k, v     [L, H, d] bf16; gate_logits [L, H, 2] fp32 (read)
 *   out         [L, H, d] bf16 (written)
 *   idx_out     [H, nqb, forced + topk] int32 (written if not NULL)
 *   workspace   device buffer of at least s3r_workspace_bytes(params) bytes, 256-byte aligned;
 *               its contents on entry do not matter. */
s3r_status s3r_sparse_attn_fwd(const s3r_params* params, const s3r_bf16* q, const s3r_bf16* k,
                               const s3r_bf16* v, const float* gate_logits, s3r_bf16* out,
                               int32_t* idx_out, void* workspace, size_t workspace_bytes,
                               s3r_stream stream);

/* Backward of the whole path (Speed3R is trained end to end: arXiv abstract). Given the upstream
 * gradient dout of s3r_sparse_attn_fwd's output, the gradients of q, k, v and of the gate logits.
 * The selection lists are held fixed: a top-k passes no gradient, so idx is an input (the lists
 * the forward call wrote to idx_out for the same q, k, v). The bf16 rounding of the pooled K/V
 * passes the gradient unchanged: every token of key block j receives dKc[j] / n_j (n_j = its
 * token count), and likewise for V. Per head, with P = softmax(scale q K^T) of each branch and
 * dO = sigmoid(gate) dout:
 *   dS = P (dO V^T - <dO, O>),  dq = scale dS K,  dK = scale dS^T q,  dV = P^T dO
 * summed over both branches;  dgates[..., c] = sigmoid'(logit c) <dout, O_branch c>.
 * The call recomputes the forward (pooling, both branches with their softmax normalisers) in
 * the workspace, then runs the backward kernels; nothing is kept between calls.
 *   q, k, v     [L, H, d] bf16; gate_logits [L, H, 2] fp32; dout [L, H, d] bf16 (read)
 *   idx         [H, nqb, forced + topk] int32 (read): entries distinct within a list; entries
 *               outside [0, nb) contribute nothing (with S3R_FLAG_DEBUG_CHECKS they also raise
 *               S3R_DEV_BAD_INDEX)
 *   dq, dk, dv  [L, H, d] fp32 (written); dgates [L, H, 2] fp32 (written)
 *   workspace   device buffer of at least s3r_bwd_workspace_bytes(params) bytes, 256-byte aligned.
 * Returns S3R_ERR_UNSUPPORTED when H * nb * block exceeds 2^31 - 1 (row coordinates of the
 * slot-order K/V copies). The order in which query blocks add into one key block's dK, dV
 * follows an atomic fill and may differ between calls (fp32 rounding only). */
/* With S3R_FLAG_SAVE_FOR_BWD in params->flags, the backward reads the forward's saved tensors:
 * the workspace must be the one the forward call used, of at least s3r_bwd_workspace_bytes
 * bytes (its first s3r_workspace_bytes bytes are the forward's; pass the same buffer to both
 * calls), with the same q, k, v, gates and the idx the forward wrote. The call then starts at
 * S3R_BWD_STAGE_PREP (the recompute stage is empty). */
size_t s3r_bwd_workspace_bytes(const s3r_params* params);
s3r_status s3r_sparse_attn_bwd(const s3r_params* params, const s3r_bf16* q, const s3r_bf16* k,
                               const s3r_bf16* v, const float* gate_logits, const int32_t* idx,
                               const s3r_bf16* dout, float* dq, float* dk, float* dv,
                               float* dgates, void* workspace, size_t workspace_bytes,
                               s3r_stream stream);

/* Size of the scratch array built into the library for s3r_sparse_attn_fwd_static (32 MiB). */
#define S3R_STATIC_WORKSPACE_BYTES (32u << 20)

/* The whole path, like s3r_sparse_attn_fwd, for callers that cannot allocate device memory (for
 * example a host framework that owns all device memory and gives plugins no workspace, or a loop
 * that must not allocate once running). The paper has no counterpart; this is a deployment
 * variant. Instead of a caller-provided workspace it uses a fixed array of
 * S3R_STATIC_WORKSPACE_BYTES inside the library, present on every GPU that loads the library
 * until the process exits. It allocates nothing.
 *   Sizes whose workspace (s3r_workspace_bytes) exceeds S3R_STATIC_WORKSPACE_BYTES are rejected
 *   with S3R_ERR_WORKSPACE before anything is launched; other arguments as s3r_sparse_attn_fwd,
 *   with three more rules, each checked before any launch:
 *     - params->dev_status must be a device word of the caller (S3R_ERR_INVALID_ARG if NULL):
 *       the array's own status word is not visible to the caller, so an expired bounded wait
 *       is reported only there;
 *     - S3R_FLAG_SAVE_FOR_BWD is rejected with S3R_ERR_UNSUPPORTED: what it keeps would live in
 *       the shared array, which s3r_sparse_attn_bwd cannot be given and the next call overwrites;
 *     - `stream` (if not NULL) must belong to the current device (S3R_ERR_INVALID_ARG).
 *   The first call on a device looks up the array's device address on that device (the current
 *   one) and keeps it for the life of the process; make that first call before any stream
 *   capture. After a cudaDeviceReset of that device the kept address is stale: do not call this
 *   entry point on that device again in the same process.
 *   All calls share the one array per device and it keeps the last call's contents (the parts
 *   that must start at zero are cleared by every call). Calls whose executions overlap on the GPU
 *   (different streams, or different host threads) race on it: serialise them. */
s3r_status s3r_sparse_attn_fwd_static(const s3r_params* params, const s3r_bf16* q,
                                      const s3r_bf16* k, const s3r_bf16* v,
                                      const float* gate_logits, s3r_bf16* out, int32_t* idx_out,
                                      s3r_stream stream);

#ifdef __cplusplus
}
#endif
#endif /* S3R_H */
