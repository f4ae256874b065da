// api.cu -- the extern "C" entry points of libs3r.so: argument validation, the workspace layout
// of the fused call, and the launch sequence. The operation and its conventions are defined in
// include/s3r.h.
#include <atomic>
#include <climits>
#include <cmath>

#include <nvtx3/nvToolsExt.h>

#include "internal.h"
#include "s3r.h"

namespace s3r {

static std::atomic<uint64_t> g_launches{0};
void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

void stage_range_push(const Problem& p, const char* name) {
  if (p.flags & S3R_FLAG_NVTX) nvtxRangePushA(name);
}
void stage_range_pop(const Problem& p) {
  if (p.flags & S3R_FLAG_NVTX) nvtxRangePop();
}

size_t topk_smem_bytes(int64_t nb);

namespace {

bool aligned16(const void* p) { return p && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

s3r_status derive(const s3r_params* prm, Problem* out) {
  if (!prm) return S3R_ERR_INVALID_ARG;
  if (prm->L < 1 || prm->H < 1 || prm->H > 65535 || prm->topk < 1) return S3R_ERR_INVALID_ARG;
  if (std::isnan(prm->scale) || std::isinf(prm->scale)) return S3R_ERR_INVALID_ARG;
  if (prm->d != 64) return S3R_ERR_UNSUPPORTED;
  if (prm->block != 32 && prm->block != 64 && prm->block != 128) return S3R_ERR_UNSUPPORTED;
  if (prm->qblock != 64) return S3R_ERR_UNSUPPORTED;
  Problem p{};
  p.L = prm->L;
  p.H = prm->H;
  p.d = prm->d;
  p.b = prm->block;
  p.qb = prm->qblock;
  p.k = prm->topk;
  p.F = prm->forced;
  p.nsel = p.F + p.k;
  BlockGeo& g = p.geo;
  g.L = p.L;
  g.b = p.b;
  if (prm->grid_h == 0) {
    p.nb = (p.L + p.b - 1) / p.b;
  } else {  // 2-D windows: check the geometry, count the blocks of a view
    if (prm->grid_h < 1 || prm->grid_w < 1 || prm->special < 0 || prm->special > p.b ||
        prm->win_h < 1 || p.b % prm->win_h != 0)
      return S3R_ERR_INVALID_ARG;
    g.two_d = 1;
    g.special = prm->special;
    g.gh = prm->grid_h;
    g.gw = prm->grid_w;
    g.wh = prm->win_h;
    const int ww = p.b / g.wh;  // a power of 2, as b is
    while ((1 << g.lww) < ww) ++g.lww;
    g.P = static_cast<int64_t>(g.special) + static_cast<int64_t>(g.gh) * g.gw;
    if (p.L % g.P != 0) return S3R_ERR_INVALID_ARG;
    g.cols = (g.gw + ww - 1) / ww;
    const int64_t per_view =
        (g.special > 0 ? 1 : 0) + static_cast<int64_t>((g.gh + g.wh - 1) / g.wh) * g.cols;
    if (per_view > S3R_MAX_BLOCKS) return S3R_ERR_UNSUPPORTED;
    g.per_view = static_cast<int>(per_view);
    p.nb = (p.L / g.P) * per_view;
  }
  p.nqb = (p.L + p.qb - 1) / p.qb;
  if (p.nb > S3R_MAX_BLOCKS) return S3R_ERR_UNSUPPORTED;
  if (p.F < 0 || p.k > p.nb - p.F) return S3R_ERR_INVALID_ARG;
  p.scale = prm->scale > 0.f ? prm->scale : 1.0f / std::sqrt(static_cast<float>(p.d));
  p.scale_log2 = static_cast<float>(static_cast<double>(p.scale) * 1.4426950408889634);
  p.flags = prm->flags;
  p.status = prm->dev_status;
  if (p.status && (reinterpret_cast<uintptr_t>(p.status) & 3u)) return S3R_ERR_INVALID_ARG;
  *out = p;
  return S3R_OK;
}

s3r_status launched(cudaError_t e) { return e == cudaSuccess ? S3R_OK : S3R_ERR_CUDA; }

// Workspace of the fused call, every region 256-byte aligned:
//   status word | Kc [nb,H,d] bf16 | Vc | Kh [H,nb*b,d] bf16 | Vh | O_cmp [L,H,d] f32
//   | scores [H,nqb,nb] f32 | idx [H,nqb,forced+k] i32
//   [with S3R_FLAG_SAVE_FOR_BWD: | O_sel [L,H,d] f32 | lse_c, lse_s [H,L] f32]
// Kh, Vh are head-major copies of K and V written by the pooling pass, from which the selection
// branch gathers each selected block as contiguous rows.
// The score matrix is only materialised when k > kFusedTopkMax; otherwise the compressed-branch
// kernel selects the top-k on the fly and the scores region is empty.
struct Workspace {
  size_t status, kc, vc, kh, vh, o_cmp, scores, idx, o_sel, lse_c, lse_s, total;
};

size_t round256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// The head-major copies are addressed with 32-bit TMA row coordinates (H * nb*b rows); beyond
// that the selection branch gathers from K and V themselves.
bool use_head_major(const Problem& p) {
  return static_cast<int64_t>(p.H) * p.nb * p.b <= INT32_MAX;
}

Workspace layout(const Problem& p) {
  Workspace w{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off += round256(bytes);
    return at;
  };
  const size_t HD = static_cast<size_t>(p.H) * p.d;
  w.status = take(4);
  w.kc = take(static_cast<size_t>(p.nb) * HD * 2);
  w.vc = take(static_cast<size_t>(p.nb) * HD * 2);
  const size_t copy = use_head_major(p) ? static_cast<size_t>(p.nb) * p.b * HD * 2 : 0;
  w.kh = take(copy);
  w.vh = take(copy);
  w.o_cmp = take(static_cast<size_t>(p.L) * HD * 4);
  w.scores = take(p.k > kFusedTopkMax ? static_cast<size_t>(p.H) * p.nqb * p.nb * 4 : 0);
  w.idx = take(static_cast<size_t>(p.H) * p.nqb * p.nsel * 4);
  if (p.flags & S3R_FLAG_SAVE_FOR_BWD) {  // what the backward reads instead of recomputing
    w.o_sel = take(static_cast<size_t>(p.L) * HD * 4);
    w.lse_c = take(static_cast<size_t>(p.H) * p.L * 4);
    w.lse_s = take(static_cast<size_t>(p.H) * p.L * 4);
  }
  w.total = off;
  return w;
}

// Workspace of the backward call, every region 256-byte aligned:
//   status | Kc | Vc | Kh | Vh (as the forward) | O_cmp, O_sel [L,H,d] f32 | lse_c, lse_s [H,L]
//   | statistics [6][H][Lp] f32 | dKc, dVc [nb,H,d] f32 | dKc, dVc partial sums of the pieces of
//   the summaries' walk over the queries [2][C][nb,H,d] f32 (C > 1 only) | cnt, cursor [H,nb] | off [H,nb+1]
//   | ent [H,nqb*nsel] | order [H*G] | hist, hcur [nqb+1] | hoff [nqb+2] i32
struct BwdWorkspace {
  size_t status, kc, vc, kh, vh, o_cmp, o_sel, lse_c, lse_s, stats, dkc, dvc, dkv_part, cnt,
      cursor, off, ent, order, hist, hcur, hoff, total;
};

BwdWorkspace bwd_ws_layout(const Problem& p) {
  BwdWorkspace w{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off += round256(bytes);
    return at;
  };
  const BwdLayout bl = bwd_layout(p);
  const size_t HD = static_cast<size_t>(p.H) * p.d;
  const size_t H = static_cast<size_t>(p.H);
  if (p.flags & S3R_FLAG_SAVE_FOR_BWD) {  // the forward's workspace, with its saved tensors, first
    const Workspace f = layout(p);
    w.status = f.status, w.kc = f.kc, w.vc = f.vc, w.kh = f.kh, w.vh = f.vh;
    w.o_cmp = f.o_cmp, w.o_sel = f.o_sel, w.lse_c = f.lse_c, w.lse_s = f.lse_s;
    off = f.total;
  } else {
    w.status = take(4);
    w.kc = take(static_cast<size_t>(p.nb) * HD * 2);
    w.vc = take(static_cast<size_t>(p.nb) * HD * 2);
    w.kh = take(static_cast<size_t>(p.nb) * p.b * HD * 2);
    w.vh = take(static_cast<size_t>(p.nb) * p.b * HD * 2);
    w.o_cmp = take(static_cast<size_t>(p.L) * HD * 4);
    w.o_sel = take(static_cast<size_t>(p.L) * HD * 4);
    w.lse_c = take(H * p.L * 4);
    w.lse_s = take(H * p.L * 4);
  }
  w.stats = take(6 * H * bl.Lp * 4);
  w.dkc = take(static_cast<size_t>(p.nb) * HD * 4);
  w.dvc = take(static_cast<size_t>(p.nb) * HD * 4);
  w.dkv_part = bl.kv_chunks > 1 ? take(2 * static_cast<size_t>(bl.kv_chunks) * p.nb * HD * 4) : 0;
  w.cnt = take(H * p.nb * 4);
  w.cursor = take(H * p.nb * 4);
  w.off = take(H * (p.nb + 1) * 4);
  w.ent = take(H * bl.per_head * 4);
  w.order = take(H * bl.G * 4);
  w.hist = take((p.nqb + 1) * 4);
  w.hcur = take((p.nqb + 1) * 4);
  w.hoff = take((p.nqb + 2) * 4);
  w.total = off;
  return w;
}

}  // namespace

size_t fused_workspace_bytes(const s3r_params* params) {
  Problem p;
  if (derive(params, &p) != S3R_OK) return 0;
  return layout(p).total;
}

// The whole path on a caller-provided workspace; shared by the fused entry points.
int fused_forward(const s3r_params* params, const uint16_t* q, const uint16_t* k,
                  const uint16_t* v, const float* gate_logits, uint16_t* out, int32_t* idx_out,
                  void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  Problem p;
  s3r_status st = derive(params, &p);
  if (st != S3R_OK) return st;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(gate_logits) ||
      !aligned16(out) || (idx_out && !aligned16(idx_out)))
    return S3R_ERR_INVALID_ARG;
  const bool save = (p.flags & S3R_FLAG_SAVE_FOR_BWD) != 0;
  if (save && !use_head_major(p)) return S3R_ERR_UNSUPPORTED;
  const Workspace w = layout(p);
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) || workspace_bytes < w.total)
    return S3R_ERR_WORKSPACE;
  uint8_t* base = static_cast<uint8_t*>(workspace);
  uint32_t* status = reinterpret_cast<uint32_t*>(base + w.status);
  float* o_sel = save ? reinterpret_cast<float*>(base + w.o_sel) : nullptr;
  float* lse_c = save ? reinterpret_cast<float*>(base + w.lse_c) : nullptr;
  float* lse_s = save ? reinterpret_cast<float*>(base + w.lse_s) : nullptr;
  if (!p.status) p.status = status;
  uint16_t* kc = reinterpret_cast<uint16_t*>(base + w.kc);
  uint16_t* vc = reinterpret_cast<uint16_t*>(base + w.vc);
  const bool hm = use_head_major(p);
  uint16_t* kh = hm ? reinterpret_cast<uint16_t*>(base + w.kh) : nullptr;
  uint16_t* vh = hm ? reinterpret_cast<uint16_t*>(base + w.vh) : nullptr;
  float* o_cmp = reinterpret_cast<float*>(base + w.o_cmp);
  float* scores = reinterpret_cast<float*>(base + w.scores);
  int32_t* idx = idx_out ? idx_out : reinterpret_cast<int32_t*>(base + w.idx);

  void* const* ev = params->stage_events;
  auto mark = [&](int i) {
    return ev ? cudaEventRecord(static_cast<cudaEvent_t>(ev[i]), stream) : cudaSuccess;
  };
  if (cudaMemsetAsync(status, 0, 4, stream) != cudaSuccess) return S3R_ERR_CUDA;
  if (mark(0) != cudaSuccess) return S3R_ERR_CUDA;
  // one stage: NVTX range, launch, event
  auto stage = [&](const char* name, int ev_after, auto&& launch) -> s3r_status {
    stage_range_push(p, name);
    const s3r_status r = launched(launch());
    stage_range_pop(p);
    if (r != S3R_OK) return r;
    return mark(ev_after) == cudaSuccess ? S3R_OK : S3R_ERR_CUDA;
  };
  if ((st = stage("s3r.pool", 1, [&] { return launch_pool_kv(p, k, v, kc, vc, kh, vh, stream); })) !=
      S3R_OK)
    return st;
  const bool fused_topk = p.k <= kFusedTopkMax;
  if ((p.flags & S3R_FLAG_SINGLE_KERNEL) && fused_topk && hm && !save) {
    st = stage("s3r.fused", 2, [&] {
      return launch_fused_tc(p, q, kc, vc, kh, vh, gate_logits, out, idx_out, stream);
    });
    if (st != S3R_OK) return st;
    for (int i = 3; i <= 4; ++i)
      if (mark(i) != cudaSuccess) return S3R_ERR_CUDA;
    return S3R_OK;
  }
  if ((st = stage("s3r.cmp", 2, [&] {
         return launch_cmp_attn_tc(p, q, kc, vc, lse_c, o_cmp, fused_topk ? nullptr : scores,
                                   fused_topk ? idx : nullptr, stream);
       })) != S3R_OK)
    return st;
  if ((st = stage("s3r.topk", 3, [&] {
         return fused_topk ? cudaSuccess : launch_topk(p, scores, idx, stream);
       })) != S3R_OK)
    return st;
  return stage("s3r.sel_combine", 4, [&] {
    return launch_sel_attn(p, q, hm ? kh : k, hm ? vh : v, hm, idx, o_sel, o_cmp, gate_logits, out,
                           stream, lse_s);
  });
}

}  // namespace s3r

using namespace s3r;

extern "C" {

const char* s3r_status_string(s3r_status s) {
  switch (s) {
    case S3R_OK: return "S3R_OK";
    case S3R_ERR_INVALID_ARG: return "S3R_ERR_INVALID_ARG";
    case S3R_ERR_UNSUPPORTED: return "S3R_ERR_UNSUPPORTED";
    case S3R_ERR_WORKSPACE: return "S3R_ERR_WORKSPACE";
    case S3R_ERR_CUDA: return "S3R_ERR_CUDA";
    case S3R_ERR_TIMEOUT: return "S3R_ERR_TIMEOUT";
  }
  return "S3R_ERR_UNKNOWN";
}

int s3r_version(void) { return 100; }

uint64_t s3r_kernel_launches(void) { return g_launches.load(std::memory_order_relaxed); }

size_t s3r_workspace_bytes(const s3r_params* params) { return fused_workspace_bytes(params); }

int64_t s3r_num_key_blocks(const s3r_params* params) {
  Problem p;
  return derive(params, &p) == S3R_OK ? p.nb : 0;
}

uint32_t* s3r_workspace_status_word(void* workspace) {
  return static_cast<uint32_t*>(workspace);  // the status word is the first region
}

s3r_status s3r_read_device_status(uint32_t* dev_status, s3r_stream stream, uint32_t* out) {
  if (!dev_status || !out || (reinterpret_cast<uintptr_t>(dev_status) & 3u)) return S3R_ERR_INVALID_ARG;
  uint32_t v = 0;
  if (cudaMemcpyAsync(&v, dev_status, 4, cudaMemcpyDeviceToHost, stream) != cudaSuccess)
    return S3R_ERR_CUDA;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return S3R_ERR_CUDA;
  if (cudaMemsetAsync(dev_status, 0, 4, stream) != cudaSuccess) return S3R_ERR_CUDA;
  *out = v;
  return (v & S3R_DEV_TIMEOUT) ? S3R_ERR_TIMEOUT : S3R_OK;
}

s3r_status s3r_last_device_error(void* flag_buf, s3r_stream stream) {
  uint32_t bits = 0;
  const s3r_status st = s3r_read_device_status(static_cast<uint32_t*>(flag_buf), stream, &bits);
  if (st == S3R_ERR_INVALID_ARG || st == S3R_ERR_CUDA) return st;
  if (bits & S3R_DEV_TIMEOUT) return S3R_ERR_TIMEOUT;
  if (bits & S3R_DEV_BAD_INDEX) return S3R_ERR_INVALID_ARG;
  return S3R_OK;
}

s3r_status s3r_compress_kv(const s3r_params* params, const s3r_bf16* k, const s3r_bf16* v,
                           s3r_bf16* k_cmp, s3r_bf16* v_cmp, s3r_stream stream) {
  Problem p;
  s3r_status st = derive(params, &p);
  if (st != S3R_OK) return st;
  if (!aligned16(k) || !aligned16(v) || !aligned16(k_cmp) || !aligned16(v_cmp))
    return S3R_ERR_INVALID_ARG;
  return launched(launch_pool_kv(p, k, v, k_cmp, v_cmp, nullptr, nullptr, stream));
}

s3r_status s3r_cmp_attn_and_score(const s3r_params* params, const s3r_bf16* q,
                                  const s3r_bf16* k_cmp, const s3r_bf16* v_cmp, float* o_cmp,
                                  float* lse, float* scores, s3r_stream stream) {
  Problem p;
  s3r_status st = derive(params, &p);
  if (st != S3R_OK) return st;
  if (!aligned16(q) || !aligned16(k_cmp) || !aligned16(v_cmp) || !aligned16(o_cmp) ||
      !aligned16(lse) || !aligned16(scores))
    return S3R_ERR_INVALID_ARG;
  return launched(launch_cmp_attn_tc(p, q, k_cmp, v_cmp, lse, o_cmp, scores, nullptr, stream));
}

s3r_status s3r_topk_blocks(const s3r_params* params, const float* scores, int32_t* idx,
                           s3r_stream stream) {
  Problem p;
  s3r_status st = derive(params, &p);
  if (st != S3R_OK) return st;
  if (!aligned16(scores) || !aligned16(idx)) return S3R_ERR_INVALID_ARG;
  return launched(launch_topk(p, scores, idx, stream));
}

s3r_status s3r_sel_attn(const s3r_params* params, const s3r_bf16* q, const s3r_bf16* k,
                        const s3r_bf16* v, const int32_t* idx, float* o_sel, s3r_stream stream) {
  Problem p;
  s3r_status st = derive(params, &p);
  if (st != S3R_OK) return st;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(idx) || !aligned16(o_sel))
    return S3R_ERR_INVALID_ARG;
  // gathered straight from K and V, a window row is one TMA box; a 128-byte-swizzled box must
  // cover whole 8-row (1024-byte) swizzle atoms, so windows narrower than 8 patches are not
  // gathered this way (the fused call, which gathers from its slot-ordered copies, takes them)
  if (p.geo.two_d && (1 << p.geo.lww) < 8) return S3R_ERR_UNSUPPORTED;
  return launched(launch_sel_attn(p, q, k, v, false, idx, o_sel, nullptr, nullptr, nullptr, stream));
}

s3r_status s3r_gate_combine(const s3r_params* params, const float* o_cmp, const float* o_sel,
                            const float* gate_logits, s3r_bf16* out, s3r_stream stream) {
  Problem p;
  s3r_status st = derive(params, &p);
  if (st != S3R_OK) return st;
  if (!aligned16(o_cmp) || !aligned16(o_sel) || !aligned16(gate_logits) || !aligned16(out))
    return S3R_ERR_INVALID_ARG;
  return launched(launch_gate_combine(p, o_cmp, o_sel, gate_logits, out, stream));
}

size_t s3r_bwd_workspace_bytes(const s3r_params* params) {
  Problem p;
  if (derive(params, &p) != S3R_OK) return 0;
  return bwd_ws_layout(p).total;
}

s3r_status s3r_sparse_attn_bwd(const s3r_params* params, const s3r_bf16* q, const s3r_bf16* k,
                               const s3r_bf16* v, const float* gate_logits, const int32_t* idx,
                               const s3r_bf16* dout, float* dq, float* dk, float* dv,
                               float* dgates, void* workspace, size_t workspace_bytes,
                               s3r_stream stream) {
  Problem p;
  s3r_status st = derive(params, &p);
  if (st != S3R_OK) return st;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(gate_logits) ||
      !aligned16(idx) || !aligned16(dout) || !aligned16(dq) || !aligned16(dk) ||
      !aligned16(dv) || !aligned16(dgates))
    return S3R_ERR_INVALID_ARG;
  if (!use_head_major(p)) return S3R_ERR_UNSUPPORTED;
  const BwdWorkspace w = bwd_ws_layout(p);
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) || workspace_bytes < w.total)
    return S3R_ERR_WORKSPACE;
  uint8_t* base = static_cast<uint8_t*>(workspace);
  auto f32 = [&](size_t at) { return reinterpret_cast<float*>(base + at); };
  auto i32 = [&](size_t at) { return reinterpret_cast<int32_t*>(base + at); };
  auto b16 = [&](size_t at) { return reinterpret_cast<uint16_t*>(base + at); };
  uint32_t* status = reinterpret_cast<uint32_t*>(base + w.status);
  if (!p.status) p.status = status;
  void* const* ev = params->stage_events;
  if (cudaMemsetAsync(status, 0, 4, stream) != cudaSuccess) return S3R_ERR_CUDA;
  if (ev && cudaEventRecord(static_cast<cudaEvent_t>(ev[0]), stream) != cudaSuccess)
    return S3R_ERR_CUDA;
  // the forward again, keeping what the backward needs (unless the forward call saved it)
  if (!(p.flags & S3R_FLAG_SAVE_FOR_BWD)) {
    stage_range_push(p, "s3r.bwd.recompute");
    if ((st = launched(launch_pool_kv(p, k, v, b16(w.kc), b16(w.vc), b16(w.kh), b16(w.vh),
                                      stream))) != S3R_OK)
      return st;
    if ((st = launched(launch_cmp_attn_tc(p, q, b16(w.kc), b16(w.vc), f32(w.lse_c), f32(w.o_cmp),
                                          nullptr, nullptr, stream))) != S3R_OK)
      return st;
    if ((st = launched(launch_sel_attn(p, q, b16(w.kh), b16(w.vh), true, idx, f32(w.o_sel),
                                       nullptr, nullptr, nullptr, stream, f32(w.lse_s)))) != S3R_OK)
      return st;
    stage_range_pop(p);
  }
  if (ev && cudaEventRecord(static_cast<cudaEvent_t>(ev[1]), stream) != cudaSuccess)
    return S3R_ERR_CUDA;
  BwdBuffers b{q, dout, b16(w.kc), b16(w.vc), b16(w.kh), b16(w.vh), gate_logits, f32(w.o_cmp),
               f32(w.o_sel), f32(w.lse_c), f32(w.lse_s), idx, f32(w.stats), f32(w.dkc),
               f32(w.dvc), bwd_layout(p).kv_chunks > 1 ? f32(w.dkv_part) : nullptr, i32(w.cnt),
               i32(w.cursor), i32(w.off), i32(w.ent), i32(w.order), i32(w.hist), i32(w.hcur),
               i32(w.hoff), dq, dk, dv, dgates};
  return launched(launch_bwd(p, b, stream, ev));
}

s3r_status s3r_sparse_attn_fwd(const s3r_params* params, const s3r_bf16* q, const s3r_bf16* k,
                               const s3r_bf16* v, const float* gate_logits, s3r_bf16* out,
                               int32_t* idx_out, void* workspace, size_t workspace_bytes,
                               s3r_stream stream) {
  return static_cast<s3r_status>(s3r::fused_forward(params, q, k, v, gate_logits, out, idx_out,
                                                     workspace, workspace_bytes, stream));
}

}  // extern "C"
