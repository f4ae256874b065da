// sel_attn_tc.cu -- selection branch on the sm_100a tensor cores (tcgen05 + TMEM + TMA),
// optionally fused with the gated aggregation.
//
// Speed3R (gist.science summary, "Methodologie" §1 "Selectie-tak"): fine-grained attention only
// on the tokens of the top-k key blocks chosen by the compression branch; §2 "Gated Aggregation":
// a per-token gate mixes the two branch outputs (two independent sigmoid gates here).
//
// One CTA = two 64-row query blocks of one head (a 128-row tile, one TMEM lane per row). The k
// selected blocks of a query block form a list of k*b tokens, walked in steps of 64 tokens. Each
// step gathers, with 2-D TMA boxes straight from K/V [L, H, 64] (or their head-major copies), the
// next 64 tokens of each of the two query blocks into one 128-token K tile and V tile (rows past L
// read as zeros). K and V tiles have rings and barriers of their own: a K tile is released as soon
// as its Q K^T has completed, and the K gathers run kKLead steps ahead of the V gathers, so the
// next steps' keys are in flight while P V still holds the V ring. Then
//   S = Q K^T       tcgen05.mma, M=128 x N=128: rows of query block 0 only use columns 0-63 (its
//                   tokens), rows of block 1 columns 64-127
//   O += P V        tcgen05.mma with bf16 P as the TMEM operand; the P columns of the other
//                   block's tokens are zero (written once), so the product stays block-diagonal
// The MMA work is twice what a 64-row tile would need, in exchange for the 128-lane layouts.
// Softmax: two warps per TMEM lane quadrant, each holding 16 rows of one query block, 2 rows x 16
// columns per thread with the 16x256b load shape (a row lies in one warp, so its maximum and sum
// need only the quad's shuffles); the reference max of a row is fixed at the first step and
// moves (with O and the row sum rescaled in TMEM once the previous product has completed) only if
// a logit exceeds it by 32 in base-2 units, so the bf16 P stays below 2^32.
// Roles (320 threads): warp 0 TMA producer, warp 1 TMEM owner + MMA issuer, warps 2-9 softmax
// (warp w holds rows 16*((w-2)/4) .. +15 of lane quadrant w%4). TMEM: S (128 cols) | O (64) |
// P (64 = 128 keys).
// Every wait is bounded in time and watches a CTA abort flag (S3R_DEV_TIMEOUT on expiry).
#include <climits>

#include "s3r.h"
#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"
#include "tma_host.h"

namespace s3r {
namespace {

using namespace sm100;

constexpr int kBM = 128;                 // rows: two 64-row query blocks
constexpr int kStep = 64;                // tokens per query block per step
#ifndef S3R_SEL_K_STAGES
#define S3R_SEL_K_STAGES 3
#endif
#ifndef S3R_SEL_K_LEAD
#define S3R_SEL_K_LEAD 2
#endif
constexpr int kStagesK = S3R_SEL_K_STAGES;  // K tile ring depth
constexpr int kStagesV = 2;                 // V tile ring depth
constexpr int kKLead = S3R_SEL_K_LEAD;      // steps by which the K gathers run ahead of V's
static_assert(kKLead >= 0 && kKLead < kStagesK + 2, "a lead the rings cannot hold deadlocks");
constexpr int kThreads = 320;            // 10 warps
constexpr int kSoftmaxThreads = 256;
constexpr uint32_t kQBytes = kBM * 128;  // 16 KB
constexpr uint32_t kTileBytes = 2 * kStep * 128;  // 128 tokens x 128 B = 16 KB (K or V)
constexpr uint32_t kColS = 0, kColO = 128, kColP = 192, kTmemCols = 256;
constexpr uint32_t kIdescQK = idesc_bf16_f32(kBM, 2 * kStep, 0, 0);  // Q K-major, K K-major
constexpr uint32_t kIdescPV = idesc_bf16_f32(kBM, 64, 0, 1);          // P TMEM, V MN-major
constexpr float kMoveRef = 32.f;  // base-2 margin before a row's reference max moves
constexpr int kIdxCache = 256;    // selection lists up to this length are staged in shared memory

struct __align__(8) Bars {
  uint64_t q_full;
  uint64_t k_full[kStagesK], k_empty[kStagesK];  // K tile of a step: freed once Q K^T completed
  uint64_t v_full[kStagesV], v_empty[kStagesV];  // V tile: freed once P V completed
  uint64_t s_full, s_empty;
  uint64_t p_full, p_empty;
  uint64_t o_full, drain;
  uint64_t never;  // never signalled: waited on only under S3R_FLAG_TEST_TIMEOUT
};

constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffK = kQBytes;                          // K tile of stage s at +s*16K
constexpr uint32_t kOffV = kOffK + kStagesK * kTileBytes;    // V tile of stage s at +s*16K
constexpr uint32_t kOffIdx = kOffV + kStagesV * kTileBytes;  // [2][kIdxCache] int32
constexpr uint32_t kOffBars = kOffIdx + 2 * kIdxCache * 4;
constexpr uint32_t kOffMisc = kOffBars + sizeof(Bars);
constexpr uint32_t kSmemUsed = kOffMisc + 16;
// more than a third of an SM's shared memory: at most two CTAs per SM, so TMEM always fits
constexpr uint32_t kSmemBytes = (kSmemUsed + 1024 > 80 * 1024 ? kSmemUsed + 1024 : 80 * 1024);

struct SelArgs {
  const int32_t* idx;  // [H, nqb, topk] (topk here = list length: forced blocks + top-k)
  float* o_sel;        // [L, H, 64] fp32, or null for the fused combine
  const float* o_cmp;  // [L, H, 64] fp32 (fused combine)
  const float* gates;  // [L, H, 2]  fp32 (fused combine)
  uint16_t* out;       // [L, H, 64] bf16 (fused combine)
  int64_t L, nb, nqb;
  BlockGeo geo;      // which tokens each key block holds
  int box;           // K/V rows per TMA box: a run of consecutive tokens (or copy rows)
  int head_major;    // K/V are the [H, nb*b, 64] copies in slot order
  int kv_xh, kv_yh;  // K/V box of head h, token tok at (h*kv_xh, h*kv_yh + tok): token-major
                     // [L, H, 64] is (64, 0), the head-major [H, nb*b, 64] copy is (0, nb*b)
  int H, b, lb, topk, nsteps;  // lb = log2(b)
  float scale_log2;
  uint32_t flags;
  uint32_t* status;
  uint64_t limit_ns;
  float* lse;  // [H, L] natural log of each row's softmax normaliser, or null
};

__device__ __forceinline__ void raise_abort(volatile int* abort, uint32_t* status) {
  *abort = 1;
  set_status(status, S3R_DEV_TIMEOUT);
}

// Block index of entry s of a selection list, clamped into range (out-of-range entries are
// loaded as block 0 and masked).
__device__ __forceinline__ int64_t sel_block(const int32_t* list, int s, int k, int64_t nb,
                                             bool& ok) {
  if (s >= k) {
    ok = false;
    return 0;
  }
  const int64_t j = list[s];
  ok = j >= 0 && j < nb;
  return ok ? j : 0;
}

// two CTAs of 10 warps per SM: at most 96 registers a thread
__global__ void __launch_bounds__(kThreads, 2)
    sel_attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ,
                       const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const SelArgs a) {
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
  const int64_t q0 = qt * kBM;
  const uint64_t lim = a.limit_ns;
  const int ns = a.nsteps;
  // the two query blocks' selection lists (a missing second block reuses the first one's)
  const int32_t* glist[2];
  int32_t* slist = reinterpret_cast<int32_t*>(smem + kOffIdx);
  const bool cached = a.topk <= kIdxCache;
  for (int qb = 0; qb < 2; ++qb) {
    const int64_t i = qt * 2 + qb < a.nqb ? qt * 2 + qb : qt * 2;
    glist[qb] = a.idx + (static_cast<int64_t>(h) * a.nqb + i) * a.topk;
    if (cached)
      for (int s = threadIdx.x; s < a.topk; s += kThreads) slist[qb * kIdxCache + s] = glist[qb][s];
  }
  const int32_t* list_of[2] = {cached ? slist : glist[0], cached ? slist + kIdxCache : glist[1]};

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    for (int s = 0; s < kStagesK; ++s) {
      mbar_init(&bars->k_full[s], 1);
      mbar_init(&bars->k_empty[s], 1);
    }
    for (int s = 0; s < kStagesV; ++s) {
      mbar_init(&bars->v_full[s], 1);
      mbar_init(&bars->v_empty[s], 1);
    }
    mbar_init(&bars->s_full, 1);
    mbar_init(&bars->s_empty, kSoftmaxThreads / 32);
    mbar_init(&bars->p_full, kSoftmaxThreads / 32);
    mbar_init(&bars->p_empty, 1);
    mbar_init(&bars->o_full, 1);
    mbar_init(&bars->drain, 1);
    mbar_init(&bars->never, 1);
    *abort = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
  }
  if (warp == 1) tmem_alloc(tmem_holder, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_holder;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer (gather)
    if (lane == 0) {
      bool ok = true;
      int issued_k = 0, issued_v = 0;
      mbar_arrive_expect_tx(&bars->q_full, kQBytes);
      tma_load_2d(sbase + kOffQ, &tmQ, h * 64, static_cast<int32_t>(q0), &bars->q_full);
      const int box = a.box;
      // the step's boxes of K (v = 0) or V (v = 1) into the stage's tile
      auto gather = [&](int t, int v, uint32_t dst, uint64_t* bar) {
        for (int qb = 0; qb < 2; ++qb) {
          const int32_t* list = list_of[qb];
          for (int part = 0; part < kStep / box; ++part) {
            // position of this box in the query block's slot list: block j, slot o
            const int pos = t * kStep + part * box;
            bool valid;
            const int64_t j = sel_block(list, pos >> a.lb, a.topk, a.nb, valid);
            const int o = pos & (a.b - 1);
            // the copy's slot row, or the 1-D token (past L reads zeros); a 2-D window's run of
            // box slots lies in one patch row, so it is box consecutive tokens from its first
            // (a run whose first slot holds no token holds none: any row will do, it is masked)
            int64_t row = j * a.b + o;
            if (!a.head_major && a.geo.two_d) {
              const int64_t tk = slot_token(a.geo, j, o);
              row = tk >= 0 ? tk : 0;
            }
            const uint32_t row_off = (qb * kStep + part * box) * 128;
            const int32_t x = h * a.kv_xh, y = static_cast<int32_t>(h * a.kv_yh + row);
            tma_load_2d(dst + row_off, v ? &tmV : &tmK, x, y, bar);
          }
        }
      };
      // K of step u, then V of step u - kKLead: the K tiles run ahead, since Q K^T needs them a
      // whole softmax earlier than P V needs the V tiles
      for (int u = 0; u < ns + kKLead; ++u) {
        if (u < ns) {
          const int sk = u % kStagesK;
          if (!mbar_wait(&bars->k_empty[sk], ((u / kStagesK) & 1) ^ 1, abort, lim)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&bars->k_full[sk], kTileBytes);
          gather(u, 0, sbase + kOffK + sk * kTileBytes, &bars->k_full[sk]);
          issued_k = u + 1;
        }
        const int t = u - kKLead;
        if (t >= 0 && t < ns) {
          const int sv = t % kStagesV;
          if (!mbar_wait(&bars->v_empty[sv], ((t / kStagesV) & 1) ^ 1, abort, lim)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&bars->v_full[sv], kTileBytes);
          gather(t, 1, sbase + kOffV + sv * kTileBytes, &bars->v_full[sv]);
          issued_v = t + 1;
        }
      }
      if (!ok) {
        raise_abort(abort, a.status);
        int dummy = 0;
        mbar_wait(&bars->q_full, 0, &dummy, lim);
        for (int t = issued_k - 1; t >= 0 && t >= issued_k - kStagesK; --t)
          mbar_wait(&bars->k_full[t % kStagesK], (t / kStagesK) & 1, &dummy, lim);
        for (int t = issued_v - 1; t >= 0 && t >= issued_v - kStagesV; --t)
          mbar_wait(&bars->v_full[t % kStagesV], (t / kStagesV) & 1, &dummy, lim);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      bool ok = mbar_wait(&bars->q_full, 0, abort, lim);
      tc_fence_after();
      const uint64_t dq = desc_sw128(sbase + kOffQ);
      auto qk = [&](int t) -> bool {
        const int stage = t % kStagesK;
        if (!mbar_wait(&bars->k_full[stage], (t / kStagesK) & 1, abort, lim)) return false;
        if (!mbar_wait(&bars->s_empty, (t & 1) ^ 1, abort, lim)) return false;
        tc_fence_after();
        const uint64_t dk = desc_sw128(sbase + kOffK + stage * kTileBytes);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
          mma_ss(tbase + kColS, dq + 2 * ks, dk + 2 * ks, kIdescQK, ks > 0);
        tc_commit(&bars->s_full);
        tc_commit(&bars->k_empty[stage]);
        return true;
      };
      auto pv = [&](int t) -> bool {
        const int stage = t % kStagesV;
        if (!mbar_wait(&bars->p_full, t & 1, abort, lim)) return false;
        if (!mbar_wait(&bars->v_full[stage], (t / kStagesV) & 1, abort, lim)) return false;
        tc_fence_after();
        const uint64_t dv = desc_sw128(sbase + kOffV + stage * kTileBytes);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)  // 128 keys in steps of 16: 16 rows x 128 B = 2048 B
          mma_ts(tbase + kColO, tbase + kColP + ks * 8, dv + 128 * ks, kIdescPV,
                 (t > 0 || ks > 0) ? 1u : 0u);
        tc_commit(&bars->v_empty[stage]);
        tc_commit(&bars->p_empty);
        return true;
      };
      for (int t = 0; ok && t < ns; ++t) {
        if (!(ok = qk(t))) break;
        if (t > 0 && !(ok = pv(t - 1))) break;
      }
      if (ok) ok = pv(ns - 1);
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
    // warp w holds rows 16*sub .. 16*sub+15 of TMEM lane quadrant w%4 (sub = (w-2)/4), so that
    // each row lies in one warp: 2 rows x 16 columns per thread with the 16x256b load shape
    const int g = warp & 3;                   // TMEM lane quadrant: rows 32g .. 32g+31
    const int sub = (warp - 2) >> 2;          // which 16 of them
    const int qb = g >> 1;                    // which of the two query blocks these rows belong to
    const int tq = lane & 3;
    const uint32_t tl = tbase + (static_cast<uint32_t>(g * 32 + sub * 16) << 16);
    const float sl2 = a.scale_log2;
    const int32_t* list = list_of[qb];
    bool ok = true;

    {  // the other query block's P columns of these rows stay zero for the whole kernel
      const uint32_t z[16] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
      tmem_st16x256_x4(tl + kColP + (1 - qb) * 32, z);
      tmem_wait_st_keep16(z);
    }

    // value v[i][c]: row tr + 8i of the warp's 16 rows, column c of this thread within the
    // step's 64 columns of the query block: 32*(c/8) + 8*((c%8)/2) + 2*tq + c%2
    auto col_of = [&](int c) { return 32 * (c >> 3) + 8 * ((c & 7) >> 1) + 2 * tq + (c & 1); };
    float mr[2], l[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) mr[i] = -INFINITY, l[i] = 0.f;
    if (a.flags & S3R_FLAG_TEST_TIMEOUT) ok = mbar_wait(&bars->never, 0, abort, lim);

    for (int t = 0; ok && t < ns; ++t) {
      if (!(ok = mbar_wait(&bars->s_full, t & 1, abort, lim))) break;
      tc_fence_after();
      uint32_t r[2][16];
      tmem_ld16x256_x4(tl + kColS + qb * 64, r[0]);
      tmem_ld16x256_x4(tl + kColS + qb * 64 + 32, r[1]);
      tmem_wait_ld_n<16>(r[0]);
      tmem_wait_ld_n<16>(r[1]);
      tc_fence_before();
      __syncwarp();  // one arrival per warp: its lanes' TMEM loads have all completed
      if (lane == 0) mbar_arrive(&bars->s_empty);
      float v[2][16];
#pragma unroll
      for (int hh = 0; hh < 2; ++hh)
#pragma unroll
        for (int rep = 0; rep < 4; ++rep)
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int c = hh * 8 + 2 * rep + e;
            v[0][c] = __uint_as_float(r[hh][4 * rep + e]);
            v[1][c] = __uint_as_float(r[hh][4 * rep + 2 + e]);
          }
      // columns whose slot holds no token: past the list, an out-of-range index, past L, or
      // outside a view's patch grid. A 64-slot step spans at most two selected blocks (b >= 32).
      {
        const int p0 = t * kStep;
        const int s_lo = p0 >> a.lb, s_hi = (p0 + kStep - 1) >> a.lb;
        bool ok_lo, ok_hi;
        const int64_t j_lo = sel_block(list, s_lo, a.topk, a.nb, ok_lo);
        const int64_t j_hi = sel_block(list, s_hi, a.topk, a.nb, ok_hi);
        if ((a.flags & S3R_FLAG_DEBUG_CHECKS) && lane == 0 &&
            ((!ok_lo && s_lo < a.topk) || (!ok_hi && s_hi < a.topk)))
          set_status(a.status, S3R_DEV_BAD_INDEX);
        const BlockOrigin bo_lo = block_origin(a.geo, j_lo), bo_hi = block_origin(a.geo, j_hi);
        // the same for the whole warp; false only on a list's last step or at a cut block
        const bool all_valid =
            ok_lo && ok_hi && origin_full(a.geo, bo_lo) && origin_full(a.geo, bo_hi);
        if (!all_valid) {
          // bit p: slot p0 + p of the list holds a token (b >= 64: one block covers the step;
          // b = 32: two blocks, 32 slots each)
          uint64_t bits;
          if (a.b >= kStep) {
            bits = ok_lo ? slot_bits(a.geo, bo_lo, p0 & (a.b - 1), kStep) : 0ull;
          } else {
            bits = (ok_lo ? slot_bits(a.geo, bo_lo, 0, 32) : 0ull) |
                   ((ok_hi ? slot_bits(a.geo, bo_hi, 0, 32) : 0ull) << 32);
          }
#pragma unroll
          for (int c = 0; c < 16; ++c)
            if (!((bits >> col_of(c)) & 1ull)) v[0][c] = v[1][c] = -INFINITY;
        }
      }
      // row maxima of this step (the quad's 4 threads hold the same rows)
      float tmax[2];
      bool move = false;
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        float m = fmax3(fmax3(v[i][0], v[i][1], v[i][2]), fmax3(v[i][3], v[i][4], v[i][5]),
                        fmax3(v[i][6], v[i][7], v[i][8]));
        m = fmax3(m, fmax3(v[i][9], v[i][10], v[i][11]), fmax3(v[i][12], v[i][13], v[i][14]));
        m = fmaxf(m, v[i][15]);
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
        tmax[i] = m;
        move |= m * sl2 > mr[i] * sl2 + kMoveRef;  // true on the first step with a valid column
      }
      // P(t) may overwrite the P buffer (and O may be rescaled) once P*V of step t-1 completed
      if (!(ok = mbar_wait(&bars->p_empty, (t & 1) ^ 1, abort, lim))) break;
      if (__any_sync(0xffffffffu, move)) {  // rare after the first step: move references
        float f[2];
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          const float mn = tmax[i] * sl2 > mr[i] * sl2 + kMoveRef ? tmax[i] : mr[i];
          f[i] = mr[i] == -INFINITY ? 0.f : exp2_approx((mr[i] - mn) * sl2);
          l[i] *= f[i];
          mr[i] = mn;
        }
        if (t > 0) {  // the warp's O rows times the factor of their row, in the same layout
          tc_fence_after();
#pragma unroll 1
          for (int hh = 0; hh < 2; ++hh) {
            uint32_t o[16];
            tmem_ld16x256_x4(tl + kColO + 32 * hh, o);
            tmem_wait_ld_n<16>(o);
#pragma unroll
            for (int rep = 0; rep < 4; ++rep)
#pragma unroll
              for (int e = 0; e < 2; ++e) {
                o[4 * rep + e] = __float_as_uint(__uint_as_float(o[4 * rep + e]) * f[0]);
                o[4 * rep + 2 + e] = __float_as_uint(__uint_as_float(o[4 * rep + 2 + e]) * f[1]);
              }
            tmem_st16x256_x4(tl + kColO + 32 * hh, o);
            tmem_wait_st_keep16(o);
          }
        }
      }
      // P = exp2(v * sl2 - ref * sl2), its row sums, and bf16 P for the tensor cores, one half of
      // the columns at a time. 16x128b store layout: repetition rep covers TMEM columns
      // 4rep..4rep+3 (keys 8rep.. of the half), lane tr -> register 2rep, lane tr+8 -> 2rep+1;
      // value columns (hh*8 + 2rep, +1) are exactly keys 32hh + 8rep + 2tq + {0,1}.
      float off[2];
#pragma unroll
      for (int i = 0; i < 2; ++i) off[i] = mr[i] == -INFINITY ? 0.f : -mr[i] * sl2;
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        uint32_t a0[8];
#pragma unroll
        for (int rep = 0; rep < 4; ++rep) {
          const int c = hh * 8 + 2 * rep;
          float e[2][2];
#pragma unroll
          for (int i = 0; i < 2; ++i) {
            const float2 x = __ffma2_rn(make_float2(v[i][c], v[i][c + 1]), make_float2(sl2, sl2),
                                        make_float2(off[i], off[i]));
            e[i][0] = exp2_approx(x.x);
            e[i][1] = exp2_approx(x.y);
            l[i] += e[i][0] + e[i][1];
          }
          a0[2 * rep] = pack_bf16(e[0][0], e[0][1]);
          a0[2 * rep + 1] = pack_bf16(e[1][0], e[1][1]);
        }
        // keys 64*qb + 32*hh .. : TMEM columns 32*qb + 16*hh of the P region
        tmem_st16x128_x4(tl + kColP + qb * 32 + hh * 16, a0);
        tmem_wait_st_keep8(a0);
      }
      tc_fence_before();
      __syncwarp();  // one arrival per warp: its lanes' TMEM stores have all completed
      if (lane == 0) mbar_arrive(&bars->p_full);
    }

    // finish: O / l per row, then write O_sel or the combine. The 32x32b load gives lane = row
    // of the quadrant; this warp writes the rows it owns (lanes 16*sub .. 16*sub+15).
    if (ok && (ok = mbar_wait(&bars->o_full, 0, abort, lim))) {
      float lsum[2];
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        float s = l[i];
        s += __shfl_xor_sync(0xffffffffu, s, 1);
        s += __shfl_xor_sync(0xffffffffu, s, 2);
        lsum[i] = s;
      }
      // row `lane` of the quadrant is held by lane 4*(lane%8) of warp sub = lane/16, as i = (lane/8)%2
      const int src = 4 * (lane & 7);
      const bool hi = (lane >> 3) & 1;
      const float s0 = __shfl_sync(0xffffffffu, lsum[0], src);
      const float s1 = __shfl_sync(0xffffffffu, lsum[1], src);
      const float rs = hi ? s1 : s0;
      const float inv = rs > 0.f ? 1.f / rs : 0.f;
      const bool mine = (lane >> 4) == sub;
      const int64_t row = q0 + g * 32 + lane;
      if (a.lse) {  // lse = (reference max * scale * log2 e + log2 of the row sum) * ln 2
        const float m0 = __shfl_sync(0xffffffffu, mr[0], src);
        const float m1 = __shfl_sync(0xffffffffu, mr[1], src);
        const float mrow = hi ? m1 : m0;
        if (mine && row < a.L)
          a.lse[static_cast<int64_t>(h) * a.L + row] =
              rs > 0.f ? (mrow * sl2 + log2f(rs)) * kLn2 : -INFINITY;
      }
      tc_fence_after();
      const uint32_t tq0 = tbase + (static_cast<uint32_t>(g * 32) << 16);
      uint32_t o[2][32];
      tmem_ld32(tq0 + kColO, o[0]);
      tmem_ld32(tq0 + kColO + 32, o[1]);
      tmem_wait_ld_regs(o[0]);
      tmem_wait_ld_regs(o[1]);
      if (mine && row < a.L) {
        const int64_t at = (row * a.H + h) * 64;
        if (a.o_sel) {
          float4* dst = reinterpret_cast<float4*>(a.o_sel + at);
#pragma unroll
          for (int j = 0; j < 16; ++j)
            dst[j] = make_float4(__uint_as_float(o[j >> 3][(4 * j) & 31]) * inv,
                                 __uint_as_float(o[j >> 3][(4 * j + 1) & 31]) * inv,
                                 __uint_as_float(o[j >> 3][(4 * j + 2) & 31]) * inv,
                                 __uint_as_float(o[j >> 3][(4 * j + 3) & 31]) * inv);
        }
        if (a.out) {
          const float2 gl = *reinterpret_cast<const float2*>(a.gates + (row * a.H + h) * 2);
          const float gc = 1.f / (1.f + expf(-gl.x));
          const float gs = 1.f / (1.f + expf(-gl.y));
          const float4* oc = reinterpret_cast<const float4*>(a.o_cmp + at);
          uint4* dst = reinterpret_cast<uint4*>(a.out + at);
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const float4 c0 = oc[2 * j], c1 = oc[2 * j + 1];
            const uint32_t* os = &o[j >> 2][(8 * j) & 31];
            uint4 w;
            w.x = pack_bf16(gc * c0.x + gs * (__uint_as_float(os[0]) * inv),
                            gc * c0.y + gs * (__uint_as_float(os[1]) * inv));
            w.y = pack_bf16(gc * c0.z + gs * (__uint_as_float(os[2]) * inv),
                            gc * c0.w + gs * (__uint_as_float(os[3]) * inv));
            w.z = pack_bf16(gc * c1.x + gs * (__uint_as_float(os[4]) * inv),
                            gc * c1.y + gs * (__uint_as_float(os[5]) * inv));
            w.w = pack_bf16(gc * c1.z + gs * (__uint_as_float(os[6]) * inv),
                            gc * c1.w + gs * (__uint_as_float(os[7]) * inv));
            dst[j] = w;
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

}  // namespace

cudaError_t launch_sel_attn(const Problem& p, const uint16_t* q, const uint16_t* k,
                            const uint16_t* v, bool head_major, const int32_t* idx, float* o_sel,
                            const float* o_cmp, const float* gates, uint16_t* out,
                            cudaStream_t st, float* lse) {
  // rows per K/V box: a run of slots that are consecutive rows in memory (32 for b = 32, else
  // 64; gathers of 2-D windows from K and V themselves: one window row, at most 64)
  int box = p.b < kStep ? p.b : kStep;
  if (!head_major && p.geo.two_d && (1 << p.geo.lww) < box) box = 1 << p.geo.lww;
  if (box < 8) return cudaErrorInvalidValue;  // whole 1024-byte swizzle atoms only
  const int64_t Lp = p.nb * p.b;
  if (head_major && p.H * Lp > INT32_MAX) return cudaErrorInvalidValue;  // TMA coordinates
  CUtensorMap tq, tk, tv;
  const bool maps =
      make_tmap_head_rows(&tq, q, p.L, p.H, kBM) &&
      (head_major ? make_tmap_rows64(&tk, k, p.H * Lp, box) && make_tmap_rows64(&tv, v, p.H * Lp, box)
                  : make_tmap_head_rows(&tk, k, p.L, p.H, box) &&
                        make_tmap_head_rows(&tv, v, p.L, p.H, box));
  if (!maps) return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(sel_attn_tc_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e != cudaSuccess) return e;
  // two CTAs of about 85 KB each: ask for the largest shared-memory carveout
  e = cudaFuncSetAttribute(sel_attn_tc_kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                           cudaSharedmemCarveoutMaxShared);
  if (e != cudaSuccess) return e;
  const int64_t ntok = static_cast<int64_t>(p.nsel) * p.b;
  const int lb = p.b == 32 ? 5 : p.b == 64 ? 6 : 7;
  SelArgs a{idx, o_sel, o_cmp, gates, out, p.L, p.nb, p.nqb, p.geo, box, head_major ? 1 : 0,
            head_major ? 0 : 64, head_major ? static_cast<int>(Lp) : 0, p.H, p.b, lb, p.nsel,
            static_cast<int>((ntok + kStep - 1) / kStep), p.scale_log2, p.flags, p.status,
            (p.flags & S3R_FLAG_TEST_TIMEOUT) ? 1000000ull : 2000000000ull, lse};
  dim3 grid(static_cast<unsigned>((p.L + kBM - 1) / kBM), p.H);
  sel_attn_tc_kernel<<<grid, kThreads, kSmemBytes, st>>>(tq, tk, tv, a);
  count_launch();
  return cudaGetLastError();
}

}  // namespace s3r
