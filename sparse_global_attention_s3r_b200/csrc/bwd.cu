// bwd.cu -- backward of the whole path on the sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// Speed3R (arXiv abstract: the sparse attention is trained end to end; gist.science summary,
// "Methodologie" §1 compression and selection branches, §2 gated aggregation). With the selection
// lists held fixed (a top-k passes no gradient) and the bf16 rounding of the pooled K/V passed
// straight through, each branch is softmax attention and its gradient is the usual one:
//   P = exp(s - lse), dP = dO V^T, dS = P (dP - D) with D = <dO, O> per row,
//   dQ = scale dS K, dK = scale dS^T Q, dV = P^T dO,
// with dO = sigmoid(g) dout for the branch's gate g (folded in per query: dP = g (dout V^T),
// D = g <dout, O>, and P^T dO = (g P)^T dout). The compressed branch's dKc, dVc then reach every
// token of block j divided by its count n_j.
//
// Kernels (one stream, no host synchronisation):
//   bwd_prep_kernel    per (row, head): D and the gate gradients from dout, O_cmp, O_sel; the
//                      per-query statistics (lse in base 2, sigmoid gates, D) of both branches
//                      in [6][H][Lp] planes, padded to whole 128-row tiles (pad: lse = +inf)
//   csr_*_kernel       the inverse of the selection lists: for each (head, key block) the query
//                      blocks that selected it (counts, per-head prefix sums, atomic fill; the
//                      order inside a list follows the fill)
//   order_*_kernel     the token-side items (head, 64-slot group) by decreasing list length, a
//                      counting sort on the length
//   bwd_q_kernel       Q-outer, one CTA per 128 query rows (two query blocks) and head: walks
//                      the nb summaries in 64-column steps, then the selected tokens in steps of
//                      32 slots per query block (block-diagonal 128 x 64, like the forward
//                      selection kernel); S = Q K^T and dP' = dout V^T on the tensor cores, dS in
//                      fp32 -> bf16 to TMEM, dQ += dS K with dS as the TMEM operand; writes dq
//   bwd_kv_kernel      KV-outer, one CTA per 128 key rows and head, 64 query columns per step:
//                      S^T = K Q^T, dP'^T = V dout^T, then (g P)^T and dS^T are written in place
//                      over S^T and dP'^T as bf16 and dV += (gP)^T dout, dK += dS^T Q.
//                      <false>: the 128 rows are block summaries, every query is a column
//                      (writes dKc, dVc); the walk over the queries may be split into pieces
//                      (grid z) whose partial sums dkv_reduce_kernel adds in piece order;
//                      <true>: rows are two 64-slot groups of key blocks
//                      (neighbours in the longest-first order, of any heads), each walking the
//                      query blocks that selected its block, 32 rows of one per step
//                      (block-diagonal); writes dk, dv per token and adds the pooled gradients
//                      dKc[j] / n_j.
// Roles (320 threads): warp 0 TMA producer, warp 1 TMEM owner + MMA issuer, warps 2-9 softmax
// (warp w reads TMEM lane quadrant w%4 and column half (w-2)/4). Every wait is bounded in time
// and watches a CTA abort flag (S3R_DEV_TIMEOUT on expiry).
#include <climits>
#include <cmath>

#include "s3r.h"
#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"
#include "tma_host.h"

namespace s3r {
namespace {

using namespace sm100;

constexpr float kLog2e = 1.4426950408889634f;
constexpr int kThreads = 320;
constexpr int kStages = 4;
constexpr uint32_t kIdescN64 = idesc_bf16_f32(128, 64, 0, 0);   // A, B K-major, N = 64
constexpr uint32_t kIdescMN = idesc_bf16_f32(128, 64, 0, 1);    // A TMEM, B MN-major, N = 64
// statistics planes of the [6][H][Lp] array
enum { kLse2C = 0, kLse2S = 1, kGC = 2, kGS = 3, kDC = 4, kDS = 5 };

// untiled bulk copy global -> shared (16-byte aligned addresses, size a multiple of 16)
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes,
                                          uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n" ::
          "r"(dst),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}

__device__ __forceinline__ void raise_abort(volatile int* abort, uint32_t* status) {
  *abort = 1;
  set_status(status, S3R_DEV_TIMEOUT);
}

__device__ __forceinline__ float bf16_lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t u) { return __uint_as_float(u & 0xffff0000u); }

// bits 0..31: columns c0 .. c0+31 below n
__device__ __forceinline__ uint32_t below_bits(int64_t c0, int64_t n) {
  const int64_t v = n - c0;
  return v >= 32 ? 0xffffffffu : v <= 0 ? 0u : ((1u << v) - 1u);
}

// Tokens held by key block j.
__device__ __forceinline__ int block_count(const BlockGeo& g, int64_t j) {
  const BlockOrigin bo = block_origin(g, j);
  if (g.b <= 64) return __popcll(slot_bits(g, bo, 0, g.b));
  return __popcll(slot_bits(g, bo, 0, 64)) + __popcll(slot_bits(g, bo, 64, 64));
}

// ------------------------------------------------------------------------------------------
// prep: per (row, head) D and the gate gradients; the statistics planes
// ------------------------------------------------------------------------------------------
// 16 lanes per (row, head), 4 channels each.
__global__ void bwd_prep_kernel(const uint16_t* __restrict__ dout, const float* __restrict__ o_cmp,
                                const float* __restrict__ o_sel, const float* __restrict__ gates,
                                const float* __restrict__ lse_c, const float* __restrict__ lse_s,
                                float* __restrict__ stats, float* __restrict__ dgates, int64_t L,
                                int64_t Lp, int H) {
  const int64_t gid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t pair = gid >> 4;
  const int sub = threadIdx.x & 15;
  if (pair >= Lp * H) return;  // whole 16-lane groups leave together
  const int64_t row = pair / H;
  const int h = static_cast<int>(pair - row * H);
  const int64_t plane = static_cast<int64_t>(H) * Lp;
  float* st = stats + static_cast<int64_t>(h) * Lp + row;
  if (row >= L) {  // padding rows: no probability mass, no gradient
    if (sub == 0) {
      st[kLse2C * plane] = INFINITY;
      st[kLse2S * plane] = INFINITY;
      st[kGC * plane] = 0.f;
      st[kGS * plane] = 0.f;
      st[kDC * plane] = 0.f;
      st[kDS * plane] = 0.f;
    }
    return;
  }
  const int64_t at = (row * H + h) * 64 + sub * 4;
  const uint2 dr = *reinterpret_cast<const uint2*>(dout + at);
  const float4 oc = *reinterpret_cast<const float4*>(o_cmp + at);
  const float4 os = *reinterpret_cast<const float4*>(o_sel + at);
  const float d0 = bf16_lo(dr.x), d1 = bf16_hi(dr.x), d2 = bf16_lo(dr.y), d3 = bf16_hi(dr.y);
  float yc = d0 * oc.x + d1 * oc.y + d2 * oc.z + d3 * oc.w;
  float ys = d0 * os.x + d1 * os.y + d2 * os.z + d3 * os.w;
  const unsigned mask = 0xffffu << (threadIdx.x & 16);
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) {
    yc += __shfl_xor_sync(mask, yc, o, 16);
    ys += __shfl_xor_sync(mask, ys, o, 16);
  }
  if (sub == 0) {
    const float2 gl = *reinterpret_cast<const float2*>(gates + (row * H + h) * 2);
    const float gc = 1.f / (1.f + expf(-gl.x));
    const float gs = 1.f / (1.f + expf(-gl.y));
    *reinterpret_cast<float2*>(dgates + (row * H + h) * 2) =
        make_float2(gc * (1.f - gc) * yc, gs * (1.f - gs) * ys);
    // a row with no valid key (lse = -inf) has no probability mass: +inf makes every P zero
    const float lc = lse_c[static_cast<int64_t>(h) * L + row];
    const float ls = lse_s[static_cast<int64_t>(h) * L + row];
    st[kLse2C * plane] = lc == -INFINITY ? INFINITY : lc * kLog2e;
    st[kLse2S * plane] = ls == -INFINITY ? INFINITY : ls * kLog2e;
    st[kGC * plane] = gc;
    st[kGS * plane] = gs;
    st[kDC * plane] = gc * yc;
    st[kDS * plane] = gs * ys;
  }
}

// ------------------------------------------------------------------------------------------
// the inverse of the selection lists (per head, CSR over key blocks)
// ------------------------------------------------------------------------------------------
// Every list entry passes through here once: an entry outside [0, nb) is skipped (its block
// gets no gradient from that query block) and, with S3R_FLAG_DEBUG_CHECKS, raises
// S3R_DEV_BAD_INDEX in the status word.
__global__ void csr_count_kernel(const int32_t* __restrict__ idx, int32_t* __restrict__ cnt,
                                 int64_t per_head, int64_t total, int64_t nb, uint32_t flags,
                                 uint32_t* status) {
  for (int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; e < total;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t h = e / per_head;
    const int32_t j = idx[e];
    if (j >= 0 && j < nb)
      atomicAdd(cnt + h * nb + j, 1);
    else if ((flags & S3R_FLAG_DEBUG_CHECKS) && status)
      set_status(status, S3R_DEV_BAD_INDEX);
  }
}

// one CTA of 1024 threads per head: off[h][j] = sum of cnt[h][0..j-1], off[h][nb] = total
__global__ void __launch_bounds__(1024) csr_scan_kernel(const int32_t* __restrict__ cnt,
                                                        int32_t* __restrict__ off,
                                                        int32_t* __restrict__ cursor, int64_t nb) {
  __shared__ int32_t warp_sum[32];
  const int64_t h = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t chunk = (nb + 1023) / 1024;
  const int64_t lo = tid * chunk < nb ? tid * chunk : nb;
  const int64_t hi = lo + chunk < nb ? lo + chunk : nb;
  const int32_t* c = cnt + h * nb;
  int32_t sum = 0;
  for (int64_t j = lo; j < hi; ++j) sum += c[j];
  int32_t incl = sum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int32_t t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  if (lane == 31) warp_sum[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int32_t w = warp_sum[lane];
    int32_t wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t t = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += t;
    }
    warp_sum[lane] = wi - w;  // exclusive prefix of the warps
  }
  __syncthreads();
  int32_t run = warp_sum[warp] + incl - sum;
  int32_t* o = off + h * (nb + 1);
  for (int64_t j = lo; j < hi; ++j) {
    o[j] = run;
    cursor[h * nb + j] = run;
    run += c[j];
  }
  if (tid == 1023) o[nb] = run;
}

__global__ void csr_fill_kernel(const int32_t* __restrict__ idx, int32_t* __restrict__ cursor,
                                int32_t* __restrict__ ent, int64_t per_head, int64_t total,
                                int64_t nb, int nsel) {
  for (int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; e < total;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t h = e / per_head;
    const int32_t i = static_cast<int32_t>((e - h * per_head) / nsel);
    const int32_t j = idx[e];
    if (j >= 0 && j < nb) ent[h * per_head + atomicAdd(cursor + h * nb + j, 1)] = i;
  }
}

// The token-side items (head, 64-slot group) in order of decreasing list length: a counting sort
// on bin nqb - min(len, nqb), so that a CTA pairs two groups of about equal length and the long
// lists start first.
__device__ __forceinline__ int64_t item_bin(const int32_t* off, int64_t item, int64_t G,
                                            int64_t nb, int cpb, int64_t nqb) {
  const int64_t h = item / G, j = (item - h * G) / cpb;
  const int64_t len = off[h * (nb + 1) + j + 1] - off[h * (nb + 1) + j];
  return nqb - (len < nqb ? len : nqb);
}

__global__ void order_count_kernel(const int32_t* __restrict__ off, int32_t* __restrict__ hist,
                                   int64_t n_items, int64_t G, int64_t nb, int cpb, int64_t nqb) {
  for (int64_t it = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; it < n_items;
       it += static_cast<int64_t>(gridDim.x) * blockDim.x)
    atomicAdd(hist + item_bin(off, it, G, nb, cpb, nqb), 1);
}

__global__ void order_fill_kernel(const int32_t* __restrict__ off, int32_t* __restrict__ cursor,
                                  int32_t* __restrict__ order, int64_t n_items, int64_t G,
                                  int64_t nb, int cpb, int64_t nqb) {
  for (int64_t it = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; it < n_items;
       it += static_cast<int64_t>(gridDim.x) * blockDim.x)
    order[atomicAdd(cursor + item_bin(off, it, G, nb, cpb, nqb), 1)] = static_cast<int32_t>(it);
}

// ------------------------------------------------------------------------------------------
// Q-outer: dq of both branches
// ------------------------------------------------------------------------------------------
namespace q_outer {
constexpr uint32_t kQBytes = 128 * 128;                 // 128 rows x 64 bf16
constexpr uint32_t kStageBytes = 2 * 64 * 128;          // K tile + V tile of 64 rows
constexpr uint32_t kOffQ = 0, kOffDO = kQBytes, kOffRing = 2 * kQBytes;
constexpr uint32_t kOffBars = kOffRing + kStages * kStageBytes;
constexpr uint32_t kColS = 0, kColDP = 64, kColDQ = 128, kColDS = 192, kTmemCols = 256;
struct __align__(8) Bars {
  uint64_t q_full;
  uint64_t kv_full[kStages], kv_empty[kStages];
  uint64_t s_full, s_empty, ds_full, ds_empty, o_full, drain;
  uint64_t never;  // never signalled: waited on only under S3R_FLAG_TEST_TIMEOUT
};
constexpr uint32_t kOffMisc = kOffBars + sizeof(Bars);
constexpr uint32_t kSmemBytes = kOffMisc + 16 + 1024;
}  // namespace q_outer

struct BwdQArgs {
  const int32_t* idx;  // [H, nqb, nsel]
  const float* stats;  // [6][H][Lp]
  float* dq;           // [L, H, 64]
  int64_t L, Lp, nb, nqb, kv_rows;  // kv_rows = nb*b: rows of one head in the slot-order copies
  BlockGeo geo;
  int H, b, lb, nsel, n_cmp, n_sel;
  float scale, scale_log2;
  uint32_t* status;
  uint64_t limit_ns;
  uint32_t flags;
};

__device__ __forceinline__ int64_t list_block(const int32_t* list, int s, int n, int64_t nb,
                                              bool& ok) {
  if (s >= n) {
    ok = false;
    return 0;
  }
  const int64_t j = list[s];
  ok = j >= 0 && j < nb;
  return ok ? j : 0;
}

__global__ void __launch_bounds__(kThreads, 2)
    bwd_q_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmO,
                 const __grid_constant__ CUtensorMap tmKc, const __grid_constant__ CUtensorMap tmVc,
                 const __grid_constant__ CUtensorMap tmKh, const __grid_constant__ CUtensorMap tmVh,
                 const BwdQArgs a) {
  using namespace q_outer;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_s = smem_addr(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_s & 1023u)) & 1023u);
  const uint32_t sbase = smem_addr(smem);
  Bars* bars = reinterpret_cast<Bars*>(smem + kOffBars);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + kOffMisc);
  volatile int* abort = reinterpret_cast<volatile int*>(smem + kOffMisc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.y;
  const int64_t qt = blockIdx.x;
  const int64_t q0 = qt * 128;
  const uint64_t lim = a.limit_ns;
  const int nsteps = a.n_cmp + a.n_sel;
  const int32_t* glist[2];
  for (int qb = 0; qb < 2; ++qb) {
    const int64_t i = qt * 2 + qb < a.nqb ? qt * 2 + qb : qt * 2;
    glist[qb] = a.idx + (static_cast<int64_t>(h) * a.nqb + i) * a.nsel;
  }

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bars->kv_full[s], 1);
      mbar_init(&bars->kv_empty[s], 1);
    }
    mbar_init(&bars->s_full, 1);
    mbar_init(&bars->s_empty, 8);
    mbar_init(&bars->ds_full, 8);
    mbar_init(&bars->ds_empty, 1);
    mbar_init(&bars->o_full, 1);
    mbar_init(&bars->drain, 1);
    mbar_init(&bars->never, 1);
    *abort = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmO);
    prefetch_tmap(&tmKc);
    prefetch_tmap(&tmVc);
    prefetch_tmap(&tmKh);
    prefetch_tmap(&tmVh);
  }
  if (warp == 1) tmem_alloc(tmem_holder, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_holder;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      bool ok = true;
      int issued = 0;
      mbar_arrive_expect_tx(&bars->q_full, 2 * kQBytes);
      tma_load_2d(sbase + kOffQ, &tmQ, h * 64, static_cast<int32_t>(q0), &bars->q_full);
      tma_load_2d(sbase + kOffDO, &tmO, h * 64, static_cast<int32_t>(q0), &bars->q_full);
      for (int t = 0; t < nsteps; ++t) {
        const int stage = t % kStages;
        if (!mbar_wait(&bars->kv_empty[stage], ((t / kStages) & 1) ^ 1, abort, lim)) {
          ok = false;
          break;
        }
        const uint32_t sk = sbase + kOffRing + stage * kStageBytes;
        mbar_arrive_expect_tx(&bars->kv_full[stage], kStageBytes);
        if (t < a.n_cmp) {  // 64 block summaries (rows past nb read as zeros)
          tma_load_2d(sk, &tmKc, h * 64, t * 64, &bars->kv_full[stage]);
          tma_load_2d(sk + kStageBytes / 2, &tmVc, h * 64, t * 64, &bars->kv_full[stage]);
        } else {  // 32 slots of each query block's list, from the slot-order copies
          const int pos = (t - a.n_cmp) * 32;
          for (int qb = 0; qb < 2; ++qb) {
            bool valid;
            const int64_t j = list_block(glist[qb], pos >> a.lb, a.nsel, a.nb, valid);
            const int32_t y =
                static_cast<int32_t>(h * a.kv_rows + j * a.b + (pos & (a.b - 1)));
            tma_load_2d(sk + qb * 4096, &tmKh, 0, y, &bars->kv_full[stage]);
            tma_load_2d(sk + kStageBytes / 2 + qb * 4096, &tmVh, 0, y, &bars->kv_full[stage]);
          }
        }
        issued = t + 1;
      }
      if (!ok) {
        raise_abort(abort, a.status);
        int dummy = 0;
        mbar_wait(&bars->q_full, 0, &dummy, lim);
        for (int t = issued - 1; t >= 0 && t >= issued - kStages; --t)
          mbar_wait(&bars->kv_full[t % kStages], (t / kStages) & 1, &dummy, lim);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      bool ok = mbar_wait(&bars->q_full, 0, abort, lim);
      tc_fence_after();
      const uint64_t dqd = desc_sw128(sbase + kOffQ), dod = desc_sw128(sbase + kOffDO);
      auto sdp = [&](int t) -> bool {
        const int stage = t % kStages;
        if (!mbar_wait(&bars->kv_full[stage], (t / kStages) & 1, abort, lim)) return false;
        if (!mbar_wait(&bars->s_empty, (t & 1) ^ 1, abort, lim)) return false;
        tc_fence_after();
        const uint32_t sk = sbase + kOffRing + stage * kStageBytes;
        const uint64_t dk = desc_sw128(sk), dv = desc_sw128(sk + kStageBytes / 2);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) mma_ss(tbase + kColS, dqd + 2 * ks, dk + 2 * ks, kIdescN64, ks > 0);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) mma_ss(tbase + kColDP, dod + 2 * ks, dv + 2 * ks, kIdescN64, ks > 0);
        tc_commit(&bars->s_full);
        return true;
      };
      auto dsk = [&](int t) -> bool {
        const int stage = t % kStages;
        if (!mbar_wait(&bars->ds_full, t & 1, abort, lim)) return false;
        tc_fence_after();
        const uint64_t dk = desc_sw128(sbase + kOffRing + stage * kStageBytes);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)  // 64 keys in steps of 16: 16 rows x 128 B = 2048 B
          mma_ts(tbase + kColDQ, tbase + kColDS + ks * 8, dk + 128 * ks, kIdescMN,
                 (t > 0 || ks > 0) ? 1u : 0u);
        tc_commit(&bars->kv_empty[stage]);
        tc_commit(&bars->ds_empty);
        return true;
      };
      for (int t = 0; ok && t < nsteps; ++t) {
        if (!(ok = sdp(t))) break;
        if (t > 0 && !(ok = dsk(t - 1))) break;
      }
      if (ok) ok = dsk(nsteps - 1);
      if (ok) {
        tc_commit(&bars->o_full);
      } else {
        raise_abort(abort, a.status);
        int dummy = 0;
        tc_commit(&bars->drain);
        mbar_wait(&bars->drain, 0, &dummy, lim);
      }
    }
  } else {
    // ------------------------------------------------------------------ softmax warps
    const int qd = warp & 3;           // TMEM lane quadrant: rows 32qd .. 32qd+31
    const int half = (warp - 2) >> 2;  // columns 32half .. 32half+31 of each step
    const int qb = qd >> 1;            // the query block of these rows
    const int64_t grow = q0 + qd * 32 + lane;
    const uint32_t tl = tbase + (static_cast<uint32_t>(qd * 32) << 16);
    const int64_t plane = static_cast<int64_t>(a.H) * a.Lp;
    const float* st = a.stats + static_cast<int64_t>(h) * a.Lp + grow;
    const float lse2c = st[kLse2C * plane], lse2s = st[kLse2S * plane];
    const float gc = st[kGC * plane], gs = st[kGS * plane];
    const float dc = st[kDC * plane], ds_ = st[kDS * plane];
    const float sl2 = a.scale_log2;
    const int32_t* list = glist[qb];
    bool ok = true;
    if (a.flags & S3R_FLAG_TEST_TIMEOUT) ok = mbar_wait(&bars->never, 0, abort, lim);
    for (int t = 0; ok && t < nsteps; ++t) {
      if (!(ok = mbar_wait(&bars->s_full, t & 1, abort, lim))) break;
      tc_fence_after();
      const bool sel = t >= a.n_cmp;
      uint32_t packed[16];
      if (!sel || half == qb) {
        uint32_t rs0[16], rs1[16], rp0[16], rp1[16];
        tmem_ld32x16(tl + kColS + 32 * half, rs0);
        tmem_ld32x16(tl + kColS + 32 * half + 16, rs1);
        tmem_ld32x16(tl + kColDP + 32 * half, rp0);
        tmem_ld32x16(tl + kColDP + 32 * half + 16, rp1);
        tmem_wait_ld_n<16>(rs0);
        tmem_wait_ld_n<16>(rs1);
        tmem_wait_ld_n<16>(rp0);
        tmem_wait_ld_n<16>(rp1);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->s_empty);
        uint32_t bits;
        float lse2, g, dd;
        if (!sel) {
          bits = below_bits(static_cast<int64_t>(t) * 64 + 32 * half, a.nb);
          lse2 = lse2c, g = gc, dd = dc;
        } else {
          const int pos = (t - a.n_cmp) * 32;
          bool okb;
          const int64_t j = list_block(list, pos >> a.lb, a.nsel, a.nb, okb);
          bits = okb ? static_cast<uint32_t>(
                           slot_bits(a.geo, block_origin(a.geo, j), pos & (a.b - 1), 32))
                     : 0u;
          lse2 = lse2s, g = gs, dd = ds_;
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          float d2[2];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int c = 2 * i + e;
            const uint32_t sv = c < 16 ? rs0[c] : rs1[c - 16];
            const uint32_t pv = c < 16 ? rp0[c] : rp1[c - 16];
            const float p = ((bits >> c) & 1u)
                                ? exp2_approx(fmaf(__uint_as_float(sv), sl2, -lse2))
                                : 0.f;
            d2[e] = p * fmaf(g, __uint_as_float(pv), -dd);
          }
          packed[i] = pack_bf16(d2[0], d2[1]);
        }
      } else {  // the other query block's columns: dS = 0 for these rows
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->s_empty);
#pragma unroll
        for (int i = 0; i < 16; ++i) packed[i] = 0u;
      }
      if (!(ok = mbar_wait(&bars->ds_empty, (t & 1) ^ 1, abort, lim))) break;
      tc_fence_after();
      tmem_st32x16(tl + kColDS + 16 * half, packed);
      tmem_wait_st_keep16(packed);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->ds_full);
    }
    if (ok && (ok = mbar_wait(&bars->o_full, 0, abort, lim))) {
      tc_fence_after();
      uint32_t r0[16], r1[16];
      tmem_ld32x16(tl + kColDQ + 32 * half, r0);
      tmem_ld32x16(tl + kColDQ + 32 * half + 16, r1);
      tmem_wait_ld_n<16>(r0);
      tmem_wait_ld_n<16>(r1);
      if (grow < a.L) {
        float4* dst = reinterpret_cast<float4*>(a.dq + (grow * a.H + h) * 64 + 32 * half);
        const float sc = a.scale;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          dst[j] = make_float4(__uint_as_float(r0[4 * j]) * sc, __uint_as_float(r0[4 * j + 1]) * sc,
                               __uint_as_float(r0[4 * j + 2]) * sc,
                               __uint_as_float(r0[4 * j + 3]) * sc);
          dst[4 + j] =
              make_float4(__uint_as_float(r1[4 * j]) * sc, __uint_as_float(r1[4 * j + 1]) * sc,
                          __uint_as_float(r1[4 * j + 2]) * sc, __uint_as_float(r1[4 * j + 3]) * sc);
        }
      }
    }
    if (!ok) raise_abort(abort, a.status);
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tbase, kTmemCols);
}

// ------------------------------------------------------------------------------------------
// KV-outer: dKc, dVc (kSel = false) or the token dk, dv (kSel = true)
// ------------------------------------------------------------------------------------------
namespace kv_outer {
constexpr uint32_t kKBytes = 128 * 128;            // 128 key rows x 64 bf16
constexpr uint32_t kQTile = 64 * 128;              // 64 query rows x 64 bf16
constexpr uint32_t kStatBytes = 3 * 64 * 4;        // lse2, g, D of 64 query columns
constexpr uint32_t kStageBytes = 17 * 1024;        // Q | dout | statistics, 1024-aligned
constexpr uint32_t kOffK = 0, kOffV = kKBytes, kOffRing = 2 * kKBytes;
constexpr uint32_t kOffBars = kOffRing + kStages * kStageBytes;
constexpr uint32_t kColS = 0, kColDP = 64, kColDV = 128, kColDK = 192, kTmemCols = 256;
struct __align__(8) Bars {
  uint64_t kv_full;
  uint64_t st_full[kStages], st_empty[kStages];
  uint64_t s_full, p_full, mma_done, o_full, drain;
  uint64_t never;  // never signalled: waited on only under S3R_FLAG_TEST_TIMEOUT
};
constexpr uint32_t kOffMisc = kOffBars + sizeof(Bars);
constexpr uint32_t kSmemBytes = kOffMisc + 16 + 1024;
static_assert(2 * kQTile + kStatBytes <= kStageBytes, "stage layout");
}  // namespace kv_outer

struct BwdKVArgs {
  const float* stats;   // [6][H][Lp]
  const int32_t* off;   // kSel: [H][nb+1] list offsets
  const int32_t* ent;   // kSel: [H][per_head] query blocks
  const int32_t* order; // kSel: the H*G (head, group) items, longest list first
  const float* dkc;     // kSel: pooled gradients [nb, H, 64] (already scaled)
  const float* dvc;
  float* out_k;         // !kSel: dKc [nb, H, 64]; kSel: dk [L, H, 64]
  float* out_v;
  int64_t L, Lp, nb, nqb, kv_rows, per_head, G;  // kSel: G groups per head
  int64_t chunk_steps;  // !kSel: 64-query steps of one piece of the walk (blockIdx.z = piece)
  int64_t part_stride;  // !kSel: elements between the pieces' outputs (0: one piece)
  BlockGeo geo;
  int H, b, cpb;        // cpb: 64-slot groups per key block
  float scale, scale_log2;
  uint32_t* status;
  uint64_t limit_ns;
  uint32_t flags;
};

template <bool kSel>
__global__ void __launch_bounds__(kThreads, 2)
    bwd_kv_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                  const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmO,
                  const BwdKVArgs a) {
  using namespace kv_outer;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_s = smem_addr(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_s & 1023u)) & 1023u);
  const uint32_t sbase = smem_addr(smem);
  Bars* bars = reinterpret_cast<Bars*>(smem + kOffBars);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + kOffMisc);
  volatile int* abort = reinterpret_cast<volatile int*>(smem + kOffMisc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.y;
  const uint64_t lim = a.limit_ns;
  const int64_t plane = static_cast<int64_t>(a.H) * a.Lp;
  // kSel: the CTA's two 64-slot groups (items 2x, 2x+1 of the longest-first order, each of its
  // own head), their key blocks and query-block lists
  int64_t gj[2] = {0, 0};
  int go[2] = {0, 0}, glen[2] = {0, 0}, hg[2] = {h, h};
  bool gvalid[2] = {false, false};
  int64_t gbase[2] = {0, 0};
  int nsteps;
  if constexpr (kSel) {
    const int64_t n_items = a.G * a.H;
    for (int grp = 0; grp < 2; ++grp) {
      const int64_t item = 2 * static_cast<int64_t>(blockIdx.x) + grp;
      gvalid[grp] = item < n_items;
      const int64_t it = a.order[gvalid[grp] ? item : 2 * static_cast<int64_t>(blockIdx.x)];
      hg[grp] = static_cast<int>(it / a.G);
      const int64_t g = it - static_cast<int64_t>(hg[grp]) * a.G;
      gj[grp] = g / a.cpb;
      go[grp] = static_cast<int>(g - gj[grp] * a.cpb) * 64;
      if (gvalid[grp]) {
        const int32_t* o = a.off + static_cast<int64_t>(hg[grp]) * (a.nb + 1) + gj[grp];
        gbase[grp] = o[0];
        glen[grp] = o[1] - o[0];
      }
    }
    nsteps = 2 * (glen[0] > glen[1] ? glen[0] : glen[1]);
  } else {  // piece blockIdx.z of the walk over the queries
    const int64_t all = (a.L + 63) / 64, t0 = static_cast<int64_t>(blockIdx.z) * a.chunk_steps;
    nsteps = static_cast<int>(all - t0 < a.chunk_steps ? all - t0 : a.chunk_steps);
  }
  const int64_t qt0 = kSel ? 0 : static_cast<int64_t>(blockIdx.z) * a.chunk_steps;

  if (threadIdx.x == 0) {
    mbar_init(&bars->kv_full, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bars->st_full[s], 1);
      mbar_init(&bars->st_empty[s], 1);
    }
    mbar_init(&bars->s_full, 1);
    mbar_init(&bars->p_full, 8);
    mbar_init(&bars->mma_done, 1);
    mbar_init(&bars->o_full, 1);
    mbar_init(&bars->drain, 1);
    mbar_init(&bars->never, 1);
    *abort = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmO);
  }
  if (warp == 1) tmem_alloc(tmem_holder, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_holder;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      bool ok = true;
      int issued = 0;
      mbar_arrive_expect_tx(&bars->kv_full, 2 * kKBytes);
      if constexpr (kSel) {  // 64 slots of each group from the slot-order copies
        for (int grp = 0; grp < 2; ++grp) {
          const int32_t y = static_cast<int32_t>(hg[grp] * a.kv_rows + gj[grp] * a.b + go[grp]);
          tma_load_2d(sbase + kOffK + grp * (kKBytes / 2), &tmK, 0, y, &bars->kv_full);
          tma_load_2d(sbase + kOffV + grp * (kKBytes / 2), &tmV, 0, y, &bars->kv_full);
        }
      } else {  // 128 block summaries (rows past nb read as zeros)
        const int32_t y = static_cast<int32_t>(blockIdx.x) * 128;
        tma_load_2d(sbase + kOffK, &tmK, h * 64, y, &bars->kv_full);
        tma_load_2d(sbase + kOffV, &tmV, h * 64, y, &bars->kv_full);
      }
      for (int t = 0; t < nsteps; ++t) {
        const int stage = t % kStages;
        if (!mbar_wait(&bars->st_empty[stage], ((t / kStages) & 1) ^ 1, abort, lim)) {
          ok = false;
          break;
        }
        const uint32_t sq = sbase + kOffRing + stage * kStageBytes;
        uint64_t* full = &bars->st_full[stage];
        mbar_arrive_expect_tx(full, 2 * kQTile + kStatBytes);
        if constexpr (kSel) {  // rows (t%2)*32 .. +32 of the (t/2)-th query block of each list
          const int u = t >> 1;
          for (int grp = 0; grp < 2; ++grp) {
            const int hh = hg[grp];
            const int64_t i = u < glen[grp]
                                  ? a.ent[static_cast<int64_t>(hh) * a.per_head + gbase[grp] + u]
                                  : 0;
            const int64_t row0 = i * 64 + (t & 1) * 32;
            tma_load_2d(sq + grp * (kQTile / 2), &tmQ, hh * 64, static_cast<int32_t>(row0), full);
            tma_load_2d(sq + kQTile + grp * (kQTile / 2), &tmO, hh * 64,
                        static_cast<int32_t>(row0), full);
            const float* s0 = a.stats + static_cast<int64_t>(hh) * a.Lp + row0;
            const uint32_t sd = sq + 2 * kQTile + grp * 384;
            bulk_load(sd, s0 + kLse2S * plane, 128, full);
            bulk_load(sd + 128, s0 + kGS * plane, 128, full);
            bulk_load(sd + 256, s0 + kDS * plane, 128, full);
          }
        } else {  // 64 consecutive queries
          const int64_t row0 = (qt0 + t) * 64;
          tma_load_2d(sq, &tmQ, h * 64, static_cast<int32_t>(row0), full);
          tma_load_2d(sq + kQTile, &tmO, h * 64, static_cast<int32_t>(row0), full);
          const float* s0 = a.stats + static_cast<int64_t>(h) * a.Lp + row0;
          const uint32_t sd = sq + 2 * kQTile;
          bulk_load(sd, s0 + kLse2C * plane, 256, full);
          bulk_load(sd + 256, s0 + kGC * plane, 256, full);
          bulk_load(sd + 512, s0 + kDC * plane, 256, full);
        }
        issued = t + 1;
      }
      if (!ok) {
        raise_abort(abort, a.status);
        int dummy = 0;
        mbar_wait(&bars->kv_full, 0, &dummy, lim);
        for (int t = issued - 1; t >= 0 && t >= issued - kStages; --t)
          mbar_wait(&bars->st_full[t % kStages], (t / kStages) & 1, &dummy, lim);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      bool ok = mbar_wait(&bars->kv_full, 0, abort, lim);
      tc_fence_after();
      const uint64_t dkd = desc_sw128(sbase + kOffK), dvd = desc_sw128(sbase + kOffV);
      for (int t = 0; ok && t < nsteps; ++t) {
        const int stage = t % kStages;
        if (!(ok = mbar_wait(&bars->st_full[stage], (t / kStages) & 1, abort, lim))) break;
        // P and dS of the previous step live in place over S and dP: their products must
        // have completed before S and dP are written again
        if (t > 0 && !(ok = mbar_wait(&bars->mma_done, (t - 1) & 1, abort, lim))) break;
        tc_fence_after();
        const uint32_t sq = sbase + kOffRing + stage * kStageBytes;
        const uint64_t dq = desc_sw128(sq), dob = desc_sw128(sq + kQTile);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) mma_ss(tbase + kColS, dkd + 2 * ks, dq + 2 * ks, kIdescN64, ks > 0);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) mma_ss(tbase + kColDP, dvd + 2 * ks, dob + 2 * ks, kIdescN64, ks > 0);
        tc_commit(&bars->s_full);
        if (!(ok = mbar_wait(&bars->p_full, t & 1, abort, lim))) break;
        tc_fence_after();
        // 64 query columns in steps of 16: the bf16 (gP)^T / dS^T of column half w sit in TMEM
        // columns 32w .. 32w+15 of their region; the B rows advance 16 x 128 B = 2048 B
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
          const uint32_t col = (ks >> 1) * 32 + (ks & 1) * 8;
          mma_ts(tbase + kColDV, tbase + kColS + col, dob + 128 * ks, kIdescMN,
                 (t > 0 || ks > 0) ? 1u : 0u);
        }
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
          const uint32_t col = (ks >> 1) * 32 + (ks & 1) * 8;
          mma_ts(tbase + kColDK, tbase + kColDP + col, dq + 128 * ks, kIdescMN,
                 (t > 0 || ks > 0) ? 1u : 0u);
        }
        tc_commit(&bars->st_empty[stage]);
        tc_commit(&bars->mma_done);
      }
      if (ok) {
        tc_commit(&bars->o_full);
      } else {
        raise_abort(abort, a.status);
        int dummy = 0;
        tc_commit(&bars->drain);
        mbar_wait(&bars->drain, 0, &dummy, lim);
      }
    }
  } else {
    // ------------------------------------------------------------------ softmax warps
    const int qd = warp & 3;
    const int half = (warp - 2) >> 2;
    const int row = qd * 32 + lane;
    const uint32_t tl = tbase + (static_cast<uint32_t>(qd * 32) << 16);
    const int grp = qd >> 1;  // kSel: the group of these rows; column half `half` is group half
    const bool diag = !kSel || half == grp;
    const float sl2 = a.scale_log2;
    bool ok = true;
    if (a.flags & S3R_FLAG_TEST_TIMEOUT) ok = mbar_wait(&bars->never, 0, abort, lim);
    for (int t = 0; ok && t < nsteps; ++t) {
      const int stage = t % kStages;
      if (!(ok = mbar_wait(&bars->s_full, t & 1, abort, lim))) break;
      tc_fence_after();
      uint32_t pk[16], dk[16];
      if (diag && (!kSel || (t >> 1) < glen[half])) {
        const float* sst =
            reinterpret_cast<const float*>(smem + kOffRing + stage * kStageBytes + 2 * kQTile);
        // column c of this half: lse2, g, D of its query
        const float* s_l = kSel ? sst + half * 96 : sst + 32 * half;
        const float* s_g = kSel ? s_l + 32 : s_l + 64;
        const float* s_d = kSel ? s_l + 64 : s_l + 128;
#pragma unroll
        for (int part = 0; part < 2; ++part) {
          uint32_t rs[16], rp[16];
          tmem_ld32x16(tl + kColS + 32 * half + 16 * part, rs);
          tmem_ld32x16(tl + kColDP + 32 * half + 16 * part, rp);
          tmem_wait_ld_n<16>(rs);
          tmem_wait_ld_n<16>(rp);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            float pg[2], d2[2];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const int c = 16 * part + 2 * i + e;
              const float p =
                  exp2_approx(fmaf(__uint_as_float(rs[2 * i + e]), sl2, -s_l[c]));
              pg[e] = p * s_g[c];
              d2[e] = p * fmaf(s_g[c], __uint_as_float(rp[2 * i + e]), -s_d[c]);
            }
            pk[8 * part + i] = pack_bf16(pg[0], pg[1]);
            dk[8 * part + i] = pack_bf16(d2[0], d2[1]);
          }
        }
      } else {  // off-diagonal block, or a list that has run out: no contribution
#pragma unroll
        for (int i = 0; i < 16; ++i) pk[i] = 0u, dk[i] = 0u;
      }
      // in place: the 16 packed columns overwrite the first 16 of this half's 32 (already read)
      tmem_st32x16(tl + kColS + 32 * half, pk);
      tmem_st32x16(tl + kColDP + 32 * half, dk);
      tmem_wait_st_keep16(pk);
      tmem_wait_st_keep16(dk);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->p_full);
    }
    if (ok && (ok = mbar_wait(&bars->o_full, 0, abort, lim))) {
      tc_fence_after();
      uint32_t rk0[16], rk1[16], rv0[16], rv1[16];
      if (nsteps > 0) {
        tmem_ld32x16(tl + kColDK + 32 * half, rk0);
        tmem_ld32x16(tl + kColDK + 32 * half + 16, rk1);
        tmem_ld32x16(tl + kColDV + 32 * half, rv0);
        tmem_ld32x16(tl + kColDV + 32 * half + 16, rv1);
        tmem_wait_ld_n<16>(rk0);
        tmem_wait_ld_n<16>(rk1);
        tmem_wait_ld_n<16>(rv0);
        tmem_wait_ld_n<16>(rv1);
      } else {  // a key block nobody selected
#pragma unroll
        for (int i = 0; i < 16; ++i) rk0[i] = rk1[i] = rv0[i] = rv1[i] = 0u;
      }
      const float sc = a.scale;
      auto kval = [&](int c) { return __uint_as_float(c < 16 ? rk0[c] : rk1[c - 16]) * sc; };
      auto vval = [&](int c) { return __uint_as_float(c < 16 ? rv0[c] : rv1[c - 16]); };
      if constexpr (kSel) {
        const int o = go[grp] + (row & 63);
        if (gvalid[grp] && (row & 63) < a.b && o < a.b) {
          const int64_t j = gj[grp];
          const int64_t tok = slot_token(a.geo, j, o);
          if (tok >= 0) {
            const float inv = 1.f / static_cast<float>(block_count(a.geo, j));
            const int64_t src = (j * a.H + hg[grp]) * 64 + 32 * half;
            const int64_t dst = (tok * a.H + hg[grp]) * 64 + 32 * half;
            const float4* pk4 = reinterpret_cast<const float4*>(a.dkc + src);
            const float4* pv4 = reinterpret_cast<const float4*>(a.dvc + src);
            float4* k4 = reinterpret_cast<float4*>(a.out_k + dst);
            float4* v4 = reinterpret_cast<float4*>(a.out_v + dst);
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              const float4 ck = pk4[q], cv = pv4[q];
              k4[q] = make_float4(kval(4 * q) + ck.x * inv, kval(4 * q + 1) + ck.y * inv,
                                  kval(4 * q + 2) + ck.z * inv, kval(4 * q + 3) + ck.w * inv);
              v4[q] = make_float4(vval(4 * q) + cv.x * inv, vval(4 * q + 1) + cv.y * inv,
                                  vval(4 * q + 2) + cv.z * inv, vval(4 * q + 3) + cv.w * inv);
            }
          }
        }
      } else {
        const int64_t j = static_cast<int64_t>(blockIdx.x) * 128 + row;
        if (j < a.nb) {
          const int64_t dst =
              static_cast<int64_t>(blockIdx.z) * a.part_stride + (j * a.H + h) * 64 + 32 * half;
          float4* k4 = reinterpret_cast<float4*>(a.out_k + dst);
          float4* v4 = reinterpret_cast<float4*>(a.out_v + dst);
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            k4[q] = make_float4(kval(4 * q), kval(4 * q + 1), kval(4 * q + 2), kval(4 * q + 3));
            v4[q] = make_float4(vval(4 * q), vval(4 * q + 1), vval(4 * q + 2), vval(4 * q + 3));
          }
        }
      }
    }
    if (!ok) raise_abort(abort, a.status);
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tbase, kTmemCols);
}

// dKc, dVc = the sum of the pieces' partial sums, added in piece order (part: [2][chunks][n/4])
__global__ void dkv_reduce_kernel(const float4* __restrict__ part, float4* __restrict__ dkc,
                                  float4* __restrict__ dvc, int64_t n4, int chunks) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < 2 * n4;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t which = i >= n4 ? 1 : 0, j = i - which * n4;
    const float4* src = part + which * chunks * n4 + j;
    float4 s = src[0];
    for (int c = 1; c < chunks; ++c) {
      const float4 x = src[c * n4];
      s = make_float4(s.x + x.x, s.y + x.y, s.z + x.z, s.w + x.w);
    }
    (which ? dvc : dkc)[j] = s;
  }
}

template <typename K>
cudaError_t prepare(K kernel, uint32_t smem) {
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                              cudaSharedmemCarveoutMaxShared);
}

}  // namespace

BwdLayout bwd_layout(const Problem& p) {
  BwdLayout w{};
  w.Lp = (p.L + 127) / 128 * 128;
  w.per_head = p.nqb * p.nsel;
  w.cpb = p.b > 64 ? p.b / 64 : 1;
  w.G = p.nb * w.cpb;
  // The dKc/dVc kernel runs one CTA per 128 summaries and head, each walking every query. When
  // those CTAs fill the last wave of a B200 (148 SMs x 2 resident CTAs) poorly, the walk is split
  // into c pieces of at least 32 steps: the smallest c up to 16 whose waves are at least 95 %
  // full, else the one that fills them best. The pieces' partial sums are added in order.
  const int64_t tiles = (p.nb + 127) / 128 * p.H, steps = (p.L + 63) / 64;
  constexpr int64_t kResident = 2 * 148;
  int best = 1;
  int64_t best_num = 0, best_den = 1;  // fill of the best c so far, as a fraction
  for (int c = 1; c <= 16 && (c == 1 || (steps + c - 1) / c >= 32); ++c) {
    const int64_t ctas = c * tiles, waves = (ctas + kResident - 1) / kResident;
    const int64_t num = ctas, den = waves * kResident;  // fill = ctas / (waves * resident)
    if (100 * num >= 95 * den) {
      best = c;
      break;
    }
    if (num * best_den > best_num * den) best = c, best_num = num, best_den = den;
  }
  w.kv_chunk_steps = (steps + best - 1) / best;
  w.kv_chunks = static_cast<int>((steps + w.kv_chunk_steps - 1) / w.kv_chunk_steps);
  return w;
}

cudaError_t launch_bwd(const Problem& p, const BwdBuffers& B, cudaStream_t st,
                       void* const* ev) {
  const BwdLayout w = bwd_layout(p);
  auto mark = [&](int i) {
    return ev ? cudaEventRecord(static_cast<cudaEvent_t>(ev[i]), st) : cudaSuccess;
  };
  const int64_t kv_rows = p.nb * p.b;
  if (static_cast<int64_t>(p.H) * kv_rows > INT32_MAX) return cudaErrorInvalidValue;
  const uint64_t lim = (p.flags & S3R_FLAG_TEST_TIMEOUT) ? 1000000ull : 2000000000ull;
  cudaError_t e;
  stage_range_push(p, "s3r.bwd.prep");
  // D, gate gradients, statistics planes
  {
    const int64_t threads = w.Lp * p.H * 16;
    const int64_t blocks = (threads + 255) / 256;
    bwd_prep_kernel<<<static_cast<unsigned>(blocks), 256, 0, st>>>(
        B.dout, B.o_cmp, B.o_sel, B.gates, B.lse_c, B.lse_s, B.stats, B.dgates, p.L, w.Lp, p.H);
    count_launch();
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  // inverse selection lists
  {
    const int64_t total = p.H * w.per_head;
    const unsigned blocks = static_cast<unsigned>((total + 255) / 256 < 4096 ? (total + 255) / 256 : 4096);
    if ((e = cudaMemsetAsync(B.cnt, 0, sizeof(int32_t) * p.H * p.nb, st)) != cudaSuccess) return e;
    csr_count_kernel<<<blocks, 256, 0, st>>>(B.idx, B.cnt, w.per_head, total, p.nb, p.flags,
                                             p.status);
    count_launch();
    csr_scan_kernel<<<p.H, 1024, 0, st>>>(B.cnt, B.off, B.cursor, p.nb);
    count_launch();
    csr_fill_kernel<<<blocks, 256, 0, st>>>(B.idx, B.cursor, B.ent, w.per_head, total, p.nb,
                                            p.nsel);
    count_launch();
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    // the token-side items, longest list first
    const int64_t n_items = w.G * p.H;
    const unsigned ob = static_cast<unsigned>((n_items + 255) / 256 < 4096 ? (n_items + 255) / 256 : 4096);
    if ((e = cudaMemsetAsync(B.hist, 0, sizeof(int32_t) * (p.nqb + 1), st)) != cudaSuccess) return e;
    order_count_kernel<<<ob, 256, 0, st>>>(B.off, B.hist, n_items, w.G, p.nb, w.cpb, p.nqb);
    count_launch();
    csr_scan_kernel<<<1, 1024, 0, st>>>(B.hist, B.hoff, B.hcur, p.nqb + 1);
    count_launch();
    order_fill_kernel<<<ob, 256, 0, st>>>(B.off, B.hcur, B.order, n_items, w.G, p.nb, w.cpb,
                                          p.nqb);
    count_launch();
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  stage_range_pop(p);
  if ((e = mark(2)) != cudaSuccess) return e;
  stage_range_push(p, "s3r.bwd.dq");
  // dq
  {
    CUtensorMap tq, to, tkc, tvc, tkh, tvh;
    if (!make_tmap_head_rows(&tq, B.q, p.L, p.H, 128) ||
        !make_tmap_head_rows(&to, B.dout, p.L, p.H, 128) ||
        !make_tmap_head_rows(&tkc, B.kc, p.nb, p.H, 64) ||
        !make_tmap_head_rows(&tvc, B.vc, p.nb, p.H, 64) ||
        !make_tmap_rows64(&tkh, B.kh, p.H * kv_rows, 32) ||
        !make_tmap_rows64(&tvh, B.vh, p.H * kv_rows, 32))
      return cudaErrorInvalidValue;
    if ((e = prepare(bwd_q_kernel, q_outer::kSmemBytes)) != cudaSuccess) return e;
    const int lb = p.b == 32 ? 5 : p.b == 64 ? 6 : 7;
    BwdQArgs a{B.idx, B.stats, B.dq, p.L, w.Lp, p.nb, p.nqb, kv_rows, p.geo, p.H, p.b, lb,
               p.nsel, static_cast<int>((p.nb + 63) / 64), static_cast<int>(p.nsel * p.b / 32),
               p.scale, p.scale_log2, p.status, lim, p.flags};
    dim3 grid(static_cast<unsigned>((p.L + 127) / 128), p.H);
    bwd_q_kernel<<<grid, kThreads, q_outer::kSmemBytes, st>>>(tq, to, tkc, tvc, tkh, tvh, a);
    count_launch();
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  stage_range_pop(p);
  if ((e = mark(3)) != cudaSuccess) return e;
  stage_range_push(p, "s3r.bwd.dkv_cmp");
  // dKc, dVc, then the token dk, dv (with the pooled gradients spread over each block)
  {
    CUtensorMap tkc, tvc, tq, to;
    if (!make_tmap_head_rows(&tkc, B.kc, p.nb, p.H, 128) ||
        !make_tmap_head_rows(&tvc, B.vc, p.nb, p.H, 128) ||
        !make_tmap_head_rows(&tq, B.q, p.L, p.H, 64) ||
        !make_tmap_head_rows(&to, B.dout, p.L, p.H, 64))
      return cudaErrorInvalidValue;
    if ((e = prepare(bwd_kv_kernel<false>, kv_outer::kSmemBytes)) != cudaSuccess) return e;
    // with several pieces, each writes its partial sums to the scratch, added in order below
    const int64_t n = p.nb * p.H * 64;
    const bool pieces = w.kv_chunks > 1;
    if (pieces && !B.dkv_part) return cudaErrorInvalidValue;
    float* out_k = pieces ? B.dkv_part : B.dkc;
    float* out_v = pieces ? B.dkv_part + w.kv_chunks * n : B.dvc;
    BwdKVArgs a{B.stats, nullptr, nullptr, nullptr, nullptr, nullptr, out_k, out_v, p.L, w.Lp,
                p.nb, p.nqb, kv_rows, w.per_head, 0, w.kv_chunk_steps, pieces ? n : 0, p.geo, p.H,
                p.b, 1, p.scale, p.scale_log2, p.status, lim, p.flags};
    dim3 grid(static_cast<unsigned>((p.nb + 127) / 128), p.H, w.kv_chunks);
    bwd_kv_kernel<false><<<grid, kThreads, kv_outer::kSmemBytes, st>>>(tkc, tvc, tq, to, a);
    count_launch();
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if (pieces) {
      const int64_t n4 = n / 4;
      const int64_t blocks = (2 * n4 + 255) / 256;
      dkv_reduce_kernel<<<static_cast<unsigned>(blocks < 8192 ? blocks : 8192), 256, 0, st>>>(
          reinterpret_cast<const float4*>(B.dkv_part), reinterpret_cast<float4*>(B.dkc),
          reinterpret_cast<float4*>(B.dvc), n4, w.kv_chunks);
      count_launch();
      if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
  }
  stage_range_pop(p);
  if ((e = mark(4)) != cudaSuccess) return e;
  stage_range_push(p, "s3r.bwd.dkv_sel");
  {
    CUtensorMap tkh, tvh, tq, to;
    if (!make_tmap_rows64(&tkh, B.kh, p.H * kv_rows, 64) ||
        !make_tmap_rows64(&tvh, B.vh, p.H * kv_rows, 64) ||
        !make_tmap_head_rows(&tq, B.q, p.L, p.H, 32) ||
        !make_tmap_head_rows(&to, B.dout, p.L, p.H, 32))
      return cudaErrorInvalidValue;
    if ((e = prepare(bwd_kv_kernel<true>, kv_outer::kSmemBytes)) != cudaSuccess) return e;
    BwdKVArgs a{B.stats, B.off, B.ent, B.order, B.dkc, B.dvc, B.dk, B.dv, p.L, w.Lp, p.nb,
                p.nqb, kv_rows, w.per_head, w.G, 0, 0, p.geo, p.H, p.b, w.cpb, p.scale,
                p.scale_log2, p.status, lim, p.flags};
    dim3 grid(static_cast<unsigned>((w.G * p.H + 1) / 2), 1);
    bwd_kv_kernel<true><<<grid, kThreads, kv_outer::kSmemBytes, st>>>(tkh, tvh, tq, to, a);
    count_launch();
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  stage_range_pop(p);
  return mark(5);
}

}  // namespace s3r
