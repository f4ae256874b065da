// internal.h -- launchers behind the C ABI of libs3r.so (not part of the public interface).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "geometry.cuh"
#include "s3r.h"

namespace s3r {

// Sizes of one call after validation; every count is derived here, never passed in.
struct Problem {
  int64_t L;        // tokens
  int H, d, b, qb;  // heads, head dim (64), key-block size, query-block rows (64)
  int k;            // top-k (blocks chosen by score)
  int F;            // leading key blocks kept in every selection list (0 = none)
  int nsel;         // selection list length F + k
  BlockGeo geo;     // which tokens each key block holds
  int64_t nb, nqb;  // key blocks, query blocks
  float scale;      // softmax scale
  float scale_log2; // scale * log2(e): logits in base-2 units
  uint32_t flags;
  uint32_t* status; // device status word or nullptr
};

// Each launcher enqueues one kernel on `st` and returns cudaGetLastError().
// kh, vh (nullable): head-major copies [H, nb*b, 64] of K and V written in the same pass.
cudaError_t launch_pool_kv(const Problem& p, const uint16_t* k, const uint16_t* v, uint16_t* kc,
                           uint16_t* vc, uint16_t* kh, uint16_t* vh, cudaStream_t st);
// Largest top-k the compressed-branch kernel selects on the fly (one key per lane of a warp).
constexpr int kFusedTopkMax = 32;

// Compression branch in one launch (both passes): O_cmp, and any of lse, scores (the block score
// matrix) and idx (the per-query-block top-k, topk <= kFusedTopkMax), each may be null.
cudaError_t launch_cmp_attn_tc(const Problem& p, const uint16_t* q, const uint16_t* kc,
                               const uint16_t* vc, float* lse, float* o_cmp, float* scores,
                               int32_t* idx, cudaStream_t st);
// The single fused kernel (topk <= kFusedTopkMax): the compressed branch with the streamed
// top-k, then, in the same CTA, the selection branch on the head-major K/V copies kh, vh and the
// gated combine into out; idx (nullable) receives the selection lists.
cudaError_t launch_fused_tc(const Problem& p, const uint16_t* q, const uint16_t* kc,
                            const uint16_t* vc, const uint16_t* kh, const uint16_t* vh,
                            const float* gates, uint16_t* out, int32_t* idx, cudaStream_t st);
cudaError_t launch_topk(const Problem& p, const float* scores, int32_t* idx, cudaStream_t st);
// o_sel != nullptr: write the selection output (fp32). out != nullptr: fuse the gated combine,
// reading o_cmp and gates and writing out (bf16). Either or both. lse (nullable): [H, L] natural log of each row's
// softmax normaliser over its selected tokens.
// k, v: [L, H, 64] token-major, or (head_major) the [H, nb*b, 64] copies of launch_pool_kv.
cudaError_t launch_sel_attn(const Problem& p, const uint16_t* q, const uint16_t* k,
                            const uint16_t* v, bool head_major, const int32_t* idx, float* o_sel,
                            const float* o_cmp, const float* gates, uint16_t* out,
                            cudaStream_t st, float* lse = nullptr);
cudaError_t launch_gate_combine(const Problem& p, const float* o_cmp, const float* o_sel,
                                const float* gates, uint16_t* out, cudaStream_t st);

// Backward of the whole path (bwd.cu). The caller has run the pooling (kc, vc and the slot-order
// copies kh, vh), the compressed branch (o_cmp, lse_c) and the selection branch (o_sel, lse_s)
// on the same inputs and selection lists idx.
struct BwdLayout {
  int64_t Lp;        // rows of the statistics planes: L rounded up to whole 128-row tiles
  int64_t per_head;  // entries of one head's selection lists: nqb * nsel
  int cpb;           // 64-slot groups per key block (token-side kernel)
  int64_t G;         // groups per head: nb * cpb
  int kv_chunks;     // pieces the dKc/dVc kernel's walk over the queries is split into
  int64_t kv_chunk_steps;  // 64-query steps of one piece
};
BwdLayout bwd_layout(const Problem& p);
struct BwdBuffers {
  const uint16_t *q, *dout, *kc, *vc, *kh, *vh;  // bf16
  const float *gates, *o_cmp, *o_sel, *lse_c, *lse_s;
  const int32_t* idx;     // [H, nqb, nsel]
  float* stats;           // [6][H][Lp] scratch
  float *dkc, *dvc;       // [nb, H, 64] scratch
  float* dkv_part;        // [2][kv_chunks][nb, H, 64] scratch, null when kv_chunks == 1
  int32_t *cnt, *cursor;  // [H, nb] scratch
  int32_t* off;           // [H, nb + 1] scratch
  int32_t* ent;           // [H, per_head] scratch
  int32_t* order;         // [H * G] scratch: token-side items, longest list first
  int32_t *hist, *hcur;   // [nqb + 1] scratch
  int32_t* hoff;          // [nqb + 2] scratch
  float *dq, *dk, *dv;    // [L, H, 64] outputs
  float* dgates;          // [L, H, 2] output
};
// ev (nullable): the call's stage events; records events 2..5 (see S3R_BWD_STAGE_*).
cudaError_t launch_bwd(const Problem& p, const BwdBuffers& b, cudaStream_t st, void* const* ev);

void count_launch();

// NVTX ranges around the stages of the whole-path calls, when S3R_FLAG_NVTX is set.
void stage_range_push(const Problem& p, const char* name);
void stage_range_pop(const Problem& p);

// Workspace bytes of the fused path (0 if params are invalid), and the fused path itself on a
// caller-provided workspace (returns an s3r_status value).
size_t fused_workspace_bytes(const s3r_params* params);
int fused_forward(const s3r_params* params, const uint16_t* q, const uint16_t* k,
                  const uint16_t* v, const float* gate_logits, uint16_t* out, int32_t* idx_out,
                  void* workspace, size_t workspace_bytes, cudaStream_t stream);

}  // namespace s3r
