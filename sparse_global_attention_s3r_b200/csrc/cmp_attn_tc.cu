// cmp_attn_tc.cu -- compression branch on the sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// Speed3R (gist.science summary, "Methodologie" §1 "Compressie-tak"): every query attends to the
// mean-pooled block summaries, and the softmax probabilities form a score matrix that ranks the
// key blocks; §4 "Efficient Kernel": the full score matrix is never materialised.
//
// Exact scores need normalised probabilities, so one launch makes two passes over the nb block
// summaries of its 128-row query tile (two 64-row query blocks) and one head:
//   pass A: S = Q Kc^T (tcgen05.mma into TMEM), running sum of exp2 -> lse per row
//   pass B: S again; P = exp2(S*scale*log2e - lse2) in fp32; the column sums of the fp32 P over
//           each 64-row query block are that block's scores; bf16(P) is stored to TMEM and
//           O_cmp += P Vc runs on the tensor cores with P as the TMEM operand.
// Q is placed in TMEM once, so both products read their A operand from TMEM and shared memory
// only serves the Kc/Vc tiles (a 128x64x16 MMA with A in shared memory would re-read 4 KB of Q
// per instruction and be limited by shared-memory bandwidth).
// Roles (384 threads, 12 warps):
//   warp 0      TMA producer: Kc (pass A) or Kc+Vc (pass B) 64-key tiles into a ring of
//               128-byte-swizzled shared-memory tiles
//   warp 1      TMEM owner (256 columns) and the single-thread tcgen05.mma issuer
//   warps 2-9   softmax: warp w reads TMEM lane quadrant w%4 (32 rows) and column half
//               (w-2)/4 (32 of the tile's 64 columns). With the 16x256b load shape a thread
//               holds 4 rows x 8 columns, so a column sum is 3 in-thread adds plus 3 shuffle
//               levels; P goes back with the matching 16x128b store shape.
//   warps 10-11 one per query block of the tile: add the two row-quadrant partial column sums;
//               write the scores and/or keep the query block's running top-k (k <= 32) in
//               registers: lane i holds the i-th largest key (score bits << 32 | ~block index),
//               a tile's candidates are tested against the k-th key with one ballot and the
//               winners are inserted by a warp-wide ordered shift, so the score matrix never
//               exists; blocks below `forced` never compete
// TMEM columns: S[2] (64 fp32 each) | O (64 fp32) | Q (64 bf16 = 32) | P (64 bf16 = 32).
// Every wait is an mbarrier wait bounded in time that also watches a CTA abort flag; on expiry
// the kernel records S3R_DEV_TIMEOUT, drains its in-flight copies and MMAs, frees TMEM and exits.
#include "s3r.h"
#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"
#include "tma_host.h"

namespace s3r {
namespace {

using namespace sm100;

constexpr int kBM = 128;       // query rows per CTA (TMEM lanes)
constexpr int kBN = 64;        // block summaries per tile
constexpr int kStages = 5;     // shared-memory ring depth
constexpr int kSoftmaxWarps = 8;
constexpr int kThreads = (4 + kSoftmaxWarps) * 32;  // producer, MMA, softmax x8, scores x2
constexpr int kScoreWarp = 2 + kSoftmaxWarps;
constexpr int kSoftmaxThreads = kSoftmaxWarps * 32;
constexpr uint32_t kKVBytes = kBN * 128;  // 8 KB
constexpr uint32_t kColS = 0, kColO = 128, kColQ = 192, kColP = 224, kTmemCols = 256;
constexpr uint32_t kIdescQK = idesc_bf16_f32(kBM, kBN, 0, 0);  // A=Q (TMEM), B=Kc K-major
constexpr uint32_t kIdescPV = idesc_bf16_f32(kBM, 64, 0, 1);   // A=P (TMEM), B=Vc MN-major
constexpr int kRed = 8;  // depth of the ring of per-tile partial column sums
// pass A keeps a per-row reference max from the first tile; a row sum beyond 2^64 (or inf/nan)
// means a later logit exceeded it by a lot, and only then is the reference moved
constexpr float kSumLimit = 1.8446744073709552e19f;

// Tuning: how many of a thread's 4 column pairs per row take the FMA-pipe polynomial 2^x instead
// of MUFU.EX2, in pass A and in pass B. MUFU.EX2 sustains 16 per clock per SM and the FMA pipe
// could evaluate about as many polynomials, but this kernel is latency-bound rather than
// MUFU-bound (measured at 1000 views: 0/0 -> 285 ms, 0/1 -> 292 ms, 1/1 -> 309 ms), so both
// default to 0.
#ifndef S3R_CMP_POLY_A
#define S3R_CMP_POLY_A 0
#endif
#ifndef S3R_CMP_POLY_B
#define S3R_CMP_POLY_B 0
#endif

struct __align__(8) Bars {
  uint64_t q_ready;  // every softmax thread has stored its part of Q into TMEM
  uint64_t kv_full[kStages], kv_empty[kStages];
  uint64_t s_full[2], s_empty[2];
  uint64_t p_full, p_empty;
  uint64_t red_full[kRed], red_empty[kRed];
  uint64_t stat;  // both column halves' row statistics of pass A are in shared memory
  uint64_t o_full, drain;
  uint64_t never;  // never signalled: waited on only under S3R_FLAG_TEST_TIMEOUT
};

constexpr uint32_t kOffKV = 0;                                 // stage s: K at +2s*8K, V +8K
constexpr uint32_t kOffRed = kOffKV + kStages * 2 * kKVBytes;  // [kRed][4 quadrant][64] f32
constexpr uint32_t kOffStat = kOffRed + kRed * 4 * 64 * 4;     // [2 halves][128 rows] float2
constexpr uint32_t kOffBars = kOffStat + 2 * 128 * 8;
constexpr uint32_t kOffMisc = kOffBars + sizeof(Bars);  // tmem base, abort flag
constexpr uint32_t kSmemUsed = kOffMisc + 16;
// At most two CTAs share an SM (shared memory), so two 256-column TMEM allocations always fit.
constexpr uint32_t kSmemBytes = (kSmemUsed + 1024 > 80 * 1024 ? kSmemUsed + 1024 : 80 * 1024);

struct CmpArgs {
  const uint16_t* q;  // [L, H, 64]
  float* lse;         // [H, L] natural log, may be null
  float* o_cmp;       // [L, H, 64]
  float* scores;      // [H, nqb, nb], may be null
  int32_t* idx;       // [H, nqb, forced + topk] selection lists (topk <= 32), may be null
  int topk;
  int forced;         // blocks 0 .. forced-1 open every list and do not compete
  int64_t L, nb, nqb;
  int H;
  float scale_log2;
  uint32_t* status;
  uint64_t limit_ns;
  uint32_t flags;
};

// Offer one candidate key c per lane to the warp's sorted list (lane i holds the i-th largest
// key; lanes 0..k-1 are the current top-k). Keys are unique. Candidates above the k-th key are
// inserted one at a time by an ordered shift. The threshold is not re-read between insertions:
// a candidate that an earlier one pushed below the k-th key lands at a position >= k (or drops
// off the end), which leaves the top-k unchanged, so each insertion costs three collectives.
__device__ __forceinline__ void topk_offer(uint64_t& mine, uint64_t c, int k, int lane) {
  const uint64_t thr = __shfl_sync(0xffffffffu, mine, k - 1);
  unsigned pending = __ballot_sync(0xffffffffu, c > thr);
  while (pending) {
    const int src = __ffs(pending) - 1;
    pending &= pending - 1;
    const uint64_t cand = __shfl_sync(0xffffffffu, c, src);
    const int pos = __popc(__ballot_sync(0xffffffffu, mine > cand));
    const uint64_t up = __shfl_up_sync(0xffffffffu, mine, 1);
    if (lane > pos) mine = up;
    if (lane == pos) mine = cand;
  }
}

__device__ __forceinline__ void raise_abort(volatile int* abort, uint32_t* status) {
  *abort = 1;
  set_status(status, S3R_DEV_TIMEOUT);
}

// Split the 16 registers of a 16x256b.x4 load at row offset 0 and the 16 at row offset 16 into
// v[i][c]: row i in {tr, tr+8, tr+16, tr+24}, column c in 0..7 = 8*(c/2) + 2*(lane%4) + c%2.
__device__ __forceinline__ void unpack_rows(const uint32_t (&a)[16], const uint32_t (&b)[16],
                                            float (&v)[4][8]) {
#pragma unroll
  for (int r = 0; r < 4; ++r)
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      v[0][2 * r + e] = __uint_as_float(a[4 * r + e]);
      v[1][2 * r + e] = __uint_as_float(a[4 * r + 2 + e]);
      v[2][2 * r + e] = __uint_as_float(b[4 * r + e]);
      v[3][2 * r + e] = __uint_as_float(b[4 * r + 2 + e]);
    }
}

// sum over the 8 values of v of exp2(v * sl2 + off); the first `npoly` column pairs use the
// FMA-pipe polynomial, the others MUFU.EX2
template <int npoly>
__device__ __forceinline__ float exp2_sum8(const float (&v)[8], float sl2, float off) {
  float2 acc = make_float2(0.f, 0.f);
#pragma unroll
  for (int c = 0; c < 8; c += 2) {
    const float2 x = __ffma2_rn(make_float2(v[c], v[c + 1]), make_float2(sl2, sl2),
                                make_float2(off, off));
    if (c / 2 < npoly)
      acc = __fadd2_rn(acc, exp2_poly5x2(x));
    else
      acc = __fadd2_rn(acc, make_float2(exp2_approx(x.x), exp2_approx(x.y)));
  }
  return acc.x + acc.y;
}

__device__ __forceinline__ float max8(const float (&v)[8]) {
  return fmax3(fmax3(v[0], v[1], v[2]), fmax3(v[3], v[4], v[5]), fmaxf(v[6], v[7]));
}

__global__ void __launch_bounds__(kThreads, 2)
    cmp_attn_tc_kernel(const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const CmpArgs a) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_s = smem_addr(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_s & 1023u)) & 1023u);  // 1024-byte aligned base
  const uint32_t sbase = smem_addr(smem);
  Bars* bars = reinterpret_cast<Bars*>(smem + kOffBars);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + kOffMisc);
  volatile int* abort = reinterpret_cast<volatile int*>(smem + kOffMisc + 4);
  float* red = reinterpret_cast<float*>(smem + kOffRed);
  float2* stat = reinterpret_cast<float2*>(smem + kOffStat);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.y;
  const int64_t qtile = blockIdx.x;
  const int64_t q0 = qtile * kBM;
  const int nt = static_cast<int>((a.nb + kBN - 1) / kBN);
  const uint64_t lim = a.limit_ns;

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_ready, kSoftmaxThreads);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bars->kv_full[s], 1);
      mbar_init(&bars->kv_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars->s_full[b], 1);
      mbar_init(&bars->s_empty[b], kSoftmaxWarps);
    }
    mbar_init(&bars->p_full, kSoftmaxWarps);
    mbar_init(&bars->p_empty, 1);
    for (int r = 0; r < kRed; ++r) {
      mbar_init(&bars->red_full[r], kSoftmaxWarps);
      mbar_init(&bars->red_empty[r], 2);  // one arrival per score warp
    }
    mbar_init(&bars->stat, kSoftmaxWarps);
    mbar_init(&bars->o_full, 1);
    mbar_init(&bars->drain, 1);
    mbar_init(&bars->never, 1);
    *abort = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
  }
  if (warp == 1) tmem_alloc(tmem_holder, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_holder;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int issued = 0;
      bool ok = true;
      for (int u = 0; u < 2 * nt; ++u) {
        const int stage = u % kStages, n = u / kStages;
        if (!mbar_wait(&bars->kv_empty[stage], (n & 1) ^ 1, abort, lim)) {
          ok = false;
          break;
        }
        const bool pass_b = u >= nt;
        const int t = pass_b ? u - nt : u;
        const uint32_t sk = sbase + kOffKV + stage * 2 * kKVBytes;
        mbar_arrive_expect_tx(&bars->kv_full[stage], pass_b ? 2 * kKVBytes : kKVBytes);
        tma_load_2d(sk, &tmK, h * 64, t * kBN, &bars->kv_full[stage]);
        if (pass_b) tma_load_2d(sk + kKVBytes, &tmV, h * 64, t * kBN, &bars->kv_full[stage]);
        issued = u + 1;
      }
      if (!ok) {
        raise_abort(abort, a.status);
        // let the copies already issued land before this CTA's shared memory is released
        int dummy = 0;
        for (int u = issued - 1; u >= 0 && u >= issued - kStages; --u)
          mbar_wait(&bars->kv_full[u % kStages], (u / kStages) & 1, &dummy, lim);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      bool ok = mbar_wait(&bars->q_ready, 0, abort, lim);
      tc_fence_after();
      auto qk = [&](int u, int c) -> bool {  // S[c&1] = Q Kc^T for ring use u
        const int stage = u % kStages;
        if (!mbar_wait(&bars->kv_full[stage], (u / kStages) & 1, abort, lim)) return false;
        const int b = c & 1;
        if (!mbar_wait(&bars->s_empty[b], ((c >> 1) & 1) ^ 1, abort, lim)) return false;
        tc_fence_after();
        const uint64_t dk = desc_sw128(sbase + kOffKV + stage * 2 * kKVBytes);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)  // 16 of d per step: 8 TMEM columns of Q, 32 B of Kc rows
          mma_ts(tbase + kColS + b * kBN, tbase + kColQ + ks * 8, dk + 2 * ks, kIdescQK, ks > 0);
        return true;
      };
      auto pv = [&](int t) -> bool {  // O += P Vc for pass-B tile t
        const int u = nt + t, stage = u % kStages;
        if (!mbar_wait(&bars->p_full, t & 1, abort, lim)) return false;
        tc_fence_after();
        const uint64_t dv = desc_sw128(sbase + kOffKV + stage * 2 * kKVBytes + kKVBytes);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)  // 16 keys per step: 16 rows x 128 B = 2048 B
          mma_ts(tbase + kColO, tbase + kColP + ks * 8, dv + 128 * ks, kIdescPV,
                 (t > 0 || ks > 0) ? 1u : 0u);
        tc_commit(&bars->kv_empty[stage]);
        tc_commit(&bars->p_empty);
        return true;
      };
      for (int t = 0; ok && t < nt; ++t) {  // pass A
        if (!(ok = qk(t, t))) break;
        tc_commit(&bars->kv_empty[t % kStages]);
        tc_commit(&bars->s_full[t & 1]);
      }
      for (int t = 0; ok && t < nt; ++t) {  // pass B: QK of tile t overlaps softmax of t-1
        if (!(ok = qk(nt + t, nt + t))) break;
        tc_commit(&bars->s_full[(nt + t) & 1]);
        if (t > 0 && !(ok = pv(t - 1))) break;
      }
      if (ok) ok = pv(nt - 1);
      if (ok) {
        tc_commit(&bars->o_full);
      } else {
        raise_abort(abort, a.status);
        int dummy = 0;
        tc_commit(&bars->drain);  // every MMA issued so far has finished once this arrives
        mbar_wait(&bars->drain, 0, &dummy, lim);
      }
    }
  } else if (warp < kScoreWarp) {
    // ------------------------------------------------------------------ softmax warps
    const int g = warp & 3;             // TMEM lane quadrant this warp may access
    const int half = (warp - 2) >> 2;   // which 32 of the tile's 64 columns (and of Q's d)
    const int tq = lane & 3, tr = lane >> 2;
    const uint32_t tl0 = tbase + (static_cast<uint32_t>(g * 32) << 16);
    const uint32_t tl16 = tbase + (static_cast<uint32_t>(g * 32 + 16) << 16);
    const float sl2 = a.scale_log2;
    // column (within the tile) of value column c of this thread
    auto col_of = [&](int c) { return half * 32 + 8 * (c >> 1) + 2 * tq + (c & 1); };
    bool ok = true;

    {  // Q row (this lane's row, this warp's 32 of d) into TMEM, the A operand of Q Kc^T
      const int64_t row = q0 + g * 32 + lane;
      uint32_t qv[16];
      if (row < a.L) {
        const uint4* src = reinterpret_cast<const uint4*>(a.q + (row * a.H + h) * 64 + half * 32);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint4 x = __ldg(src + j);
          qv[4 * j] = x.x, qv[4 * j + 1] = x.y, qv[4 * j + 2] = x.z, qv[4 * j + 3] = x.w;
        }
      } else {
#pragma unroll
        for (int j = 0; j < 16; ++j) qv[j] = 0u;
      }
      tmem_st32x16(tl0 + kColQ + half * 16, qv);
      tmem_wait_st_keep16(qv);
      tc_fence_before();
      mbar_arrive(&bars->q_ready);
    }
    if (a.flags & S3R_FLAG_TEST_TIMEOUT) ok = mbar_wait(&bars->never, 0, abort, lim);

    // pass A: per row a reference max (raw logits) and the sum of exp2 relative to it
    float mr[4], l[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) mr[i] = -INFINITY, l[i] = 0.f;
    for (int t = 0; ok && t < nt; ++t) {
      const int b = t & 1;
      if (!(ok = mbar_wait(&bars->s_full[b], (t >> 1) & 1, abort, lim))) break;
      tc_fence_after();
      uint32_t ra[16], rb[16];
      tmem_ld16x256_x4(tl0 + kColS + b * kBN + half * 32, ra);
      tmem_ld16x256_x4(tl16 + kColS + b * kBN + half * 32, rb);
      tmem_wait_ld_n<16>(ra);
      tmem_wait_ld_n<16>(rb);
      tc_fence_before();
      __syncwarp();  // one arrival per warp: its lanes' TMEM loads have all completed
      if (lane == 0) mbar_arrive(&bars->s_empty[b]);
      float v[4][8];
      unpack_rows(ra, rb, v);
      if (static_cast<int64_t>(t + 1) * kBN > a.nb) {  // ragged last tile
        const int64_t valid = a.nb - static_cast<int64_t>(t) * kBN;
#pragma unroll
        for (int c = 0; c < 8; ++c)
          if (col_of(c) >= valid) v[0][c] = v[1][c] = v[2][c] = v[3][c] = -INFINITY;
      }
      if (t == 0) {  // first tile: its row maxima become the reference (-inf if all masked)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          mr[i] = max8(v[i]);
          l[i] = mr[i] == -INFINITY ? 0.f : exp2_sum8<S3R_CMP_POLY_A>(v[i], sl2, -mr[i] * sl2);
        }
        continue;
      }
      // later tiles (tile 0 was full, so every reference is finite): straight-line sums for the
      // four rows, one combined check for the rare row whose sum left the safe range
      float sum[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) sum[i] = l[i] + exp2_sum8<S3R_CMP_POLY_A>(v[i], sl2, -mr[i] * sl2);
      const bool safe = (sum[0] <= kSumLimit) & (sum[1] <= kSumLimit) & (sum[2] <= kSumLimit) &
                        (sum[3] <= kSumLimit);
      if (safe) {
#pragma unroll
        for (int i = 0; i < 4; ++i) l[i] = sum[i];
      } else {  // a logit far above its reference: move the reference, redo this tile's sum
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float mn = fmaxf(mr[i], max8(v[i]));
          l[i] = l[i] * exp2_approx((mr[i] - mn) * sl2) + exp2_sum8<S3R_CMP_POLY_A>(v[i], sl2, -mn * sl2);
          mr[i] = mn;
        }
      }
    }
    // combine the statistics of the 4 threads of a quad and of the two column halves
    float lse2[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
#pragma unroll
      for (int o = 1; o <= 2; o <<= 1) {
        const float m2 = __shfl_xor_sync(0xffffffffu, mr[i], o);
        const float l2 = __shfl_xor_sync(0xffffffffu, l[i], o);
        const float mn = fmaxf(mr[i], m2);
        const float w1 = mr[i] == -INFINITY ? 0.f : exp2_approx((mr[i] - mn) * sl2);
        const float w2 = m2 == -INFINITY ? 0.f : exp2_approx((m2 - mn) * sl2);
        l[i] = l[i] * w1 + l2 * w2;
        mr[i] = mn;
      }
      if (tq == 0) stat[half * 128 + g * 32 + tr + 8 * i] = make_float2(mr[i], l[i]);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&bars->stat);
    if (ok) ok = mbar_wait(&bars->stat, 0, abort, lim);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int rl = g * 32 + tr + 8 * i;
      const float2 s0 = stat[rl], s1 = stat[128 + rl];
      const float mn = fmaxf(s0.x, s1.x);  // finite: column 0 is valid for every row
      const float w0 = s0.x == -INFINITY ? 0.f : exp2_approx((s0.x - mn) * sl2);
      const float w1 = s1.x == -INFINITY ? 0.f : exp2_approx((s1.x - mn) * sl2);
      const int64_t row = q0 + rl;
      lse2[i] = row < a.L ? mn * sl2 + log2f(s0.y * w0 + s1.y * w1) : INFINITY;
      if (ok && a.lse && half == 0 && tq == 0 && row < a.L)
        a.lse[static_cast<int64_t>(h) * a.L + row] = lse2[i] * kLn2;
    }

    // pass B: probabilities, column sums, P to TMEM for the P*Vc product
    for (int t = 0; ok && t < nt; ++t) {
      const int c2 = nt + t, b = c2 & 1;
      if (!(ok = mbar_wait(&bars->s_full[b], (c2 >> 1) & 1, abort, lim))) break;
      tc_fence_after();
      uint32_t ra[16], rb[16];
      tmem_ld16x256_x4(tl0 + kColS + b * kBN + half * 32, ra);
      tmem_ld16x256_x4(tl16 + kColS + b * kBN + half * 32, rb);
      tmem_wait_ld_n<16>(ra);
      tmem_wait_ld_n<16>(rb);
      tc_fence_before();
      __syncwarp();  // one arrival per warp: its lanes' TMEM loads have all completed
      if (lane == 0) mbar_arrive(&bars->s_empty[b]);
      float v[4][8];
      unpack_rows(ra, rb, v);
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int c = 0; c < 8; c += 2) {
          const float2 x = __ffma2_rn(make_float2(v[i][c], v[i][c + 1]), make_float2(sl2, sl2),
                                      make_float2(-lse2[i], -lse2[i]));
          if (c / 2 < S3R_CMP_POLY_B) {
            const float2 e = exp2_poly5x2(x);
            v[i][c] = e.x;
            v[i][c + 1] = e.y;
          } else {
            v[i][c] = exp2_approx(x.x);
            v[i][c + 1] = exp2_approx(x.y);
          }
        }
      if (static_cast<int64_t>(t + 1) * kBN > a.nb) {  // ragged last tile: P = 0 past nb
        const int64_t valid = a.nb - static_cast<int64_t>(t) * kBN;
#pragma unroll
        for (int c = 0; c < 8; ++c)
          if (col_of(c) >= valid) v[0][c] = v[1][c] = v[2][c] = v[3][c] = 0.f;
      }
      // bf16 P for the tensor cores, in the 16x128b store layout (same columns as the load)
      uint32_t p0[8], p1[8];
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        p0[2 * r] = pack_bf16(v[0][2 * r], v[0][2 * r + 1]);
        p0[2 * r + 1] = pack_bf16(v[1][2 * r], v[1][2 * r + 1]);
        p1[2 * r] = pack_bf16(v[2][2 * r], v[2][2 * r + 1]);
        p1[2 * r + 1] = pack_bf16(v[3][2 * r], v[3][2 * r + 1]);
      }
      // column sums of the fp32 P: the thread's 4 rows, then the 8 row groups of the warp
      float cs[8];
#pragma unroll
      for (int c = 0; c < 8; c += 2) {
        const float2 s01 = __fadd2_rn(make_float2(v[0][c], v[0][c + 1]),
                                      make_float2(v[1][c], v[1][c + 1]));
        const float2 s23 = __fadd2_rn(make_float2(v[2][c], v[2][c + 1]),
                                      make_float2(v[3][c], v[3][c + 1]));
        const float2 s = __fadd2_rn(s01, s23);
        cs[c] = s.x;
        cs[c + 1] = s.y;
      }
#pragma unroll
      for (int w = 4; w >= 1; w >>= 1) {  // lane bits 4, 3, 2 (the row group tr)
        const bool upper = lane & (w << 2);
#pragma unroll
        for (int i = 0; i < w; ++i) {
          const float send = upper ? cs[i] : cs[i + w];
          const float keep = upper ? cs[i + w] : cs[i];
          cs[i] = keep + __shfl_xor_sync(0xffffffffu, send, w << 2);
        }
      }
      // cs[0] is now the 32-row sum of value column c = tr of this lane
      const int par = t % kRed;
      if (!(ok = mbar_wait(&bars->red_empty[par], ((t / kRed) & 1) ^ 1, abort, lim))) break;
      red[(par * 4 + g) * 64 + col_of(tr)] = cs[0];
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->red_full[par]);
      // the single P buffer is free once the P*Vc product of tile t-1 has completed
      if (!(ok = mbar_wait(&bars->p_empty, (t & 1) ^ 1, abort, lim))) break;
      tmem_st16x128_x4(tl0 + kColP + half * 16, p0);
      tmem_st16x128_x4(tl16 + kColP + half * 16, p1);
      tmem_wait_st_keep8(p0);
      tmem_wait_st_keep8(p1);
      tc_fence_before();
      __syncwarp();  // one arrival per warp: its lanes' TMEM stores have all completed
      if (lane == 0) mbar_arrive(&bars->p_full);
    }
    if (ok && (ok = mbar_wait(&bars->o_full, 0, abort, lim))) {
      tc_fence_after();
      uint32_t o[32];
      tmem_ld32(tl0 + kColO + half * 32, o);
      tmem_wait_ld_regs(o);
      const int64_t row = q0 + g * 32 + lane;
      if (row < a.L) {
        float4* dst = reinterpret_cast<float4*>(a.o_cmp + (row * a.H + h) * 64 + half * 32);
#pragma unroll
        for (int j = 0; j < 8; ++j)
          dst[j] = make_float4(__uint_as_float(o[4 * j]), __uint_as_float(o[4 * j + 1]),
                               __uint_as_float(o[4 * j + 2]), __uint_as_float(o[4 * j + 3]));
      }
    }
    if (!ok) raise_abort(abort, a.status);
  } else {
    // ------------------------------------------------------------------ scores / top-k
    // one warp per query block of the tile, so the two running lists grow in parallel
    const int qb = warp - kScoreWarp;
    const int64_t i = qtile * 2 + qb;
    float* dst = a.scores && i < a.nqb ? a.scores + (static_cast<int64_t>(h) * a.nqb + i) * a.nb
                                       : nullptr;
    uint64_t best = 0ull;  // below every real key
    bool ok = true;
    for (int t = 0; t < nt; ++t) {
      const int par = t % kRed;
      if (!mbar_wait(&bars->red_full[par], (t / kRed) & 1, abort, lim)) {
        if (lane == 0) raise_abort(abort, a.status);
        ok = false;
        break;
      }
      float sc[2];
#pragma unroll
      for (int hc = 0; hc < 2; ++hc) {
        const int cc = hc * 32 + lane;
        sc[hc] = red[(par * 4 + 2 * qb) * 64 + cc] + red[(par * 4 + 2 * qb + 1) * 64 + cc];
      }
      __syncwarp();  // the ring slot is read: hand it back before the (slower) list updates
      if (lane == 0) mbar_arrive(&bars->red_empty[par]);
      if (i >= a.nqb) continue;
#pragma unroll
      for (int hc = 0; hc < 2; ++hc) {
        const int64_t col = static_cast<int64_t>(t) * kBN + hc * 32 + lane;
        if (dst && col < a.nb) dst[col] = sc[hc];
        if (a.idx) {
          const uint64_t key = col < a.nb && col >= a.forced
                                   ? (static_cast<uint64_t>(__float_as_uint(sc[hc])) << 32) |
                                         static_cast<uint32_t>(~static_cast<uint32_t>(col))
                                   : 0ull;
          topk_offer(best, key, a.topk, lane);
        }
      }
    }
    if (ok && a.idx && i < a.nqb) {
      int32_t* list = a.idx + (static_cast<int64_t>(h) * a.nqb + i) * (a.forced + a.topk);
      for (int f = lane; f < a.forced; f += 32) list[f] = f;
      if (lane < a.topk)
        list[a.forced + lane] = static_cast<int32_t>(~static_cast<uint32_t>(best & 0xFFFFFFFFull));
    }
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tbase, kTmemCols);
}

}  // namespace

cudaError_t launch_cmp_attn_tc(const Problem& p, const uint16_t* q, const uint16_t* kc,
                               const uint16_t* vc, float* lse, float* o_cmp, float* scores,
                               int32_t* idx, cudaStream_t st) {
  if (idx && p.k > kFusedTopkMax) return cudaErrorInvalidValue;
  CUtensorMap tk, tv;
  if (!make_tmap_head_rows(&tk, kc, p.nb, p.H, kBN) || !make_tmap_head_rows(&tv, vc, p.nb, p.H, kBN))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(cmp_attn_tc_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e != cudaSuccess) return e;
  CmpArgs a{q, lse, o_cmp, scores, idx, p.k, p.F, p.L, p.nb, p.nqb, p.H, p.scale_log2, p.status,
            (p.flags & S3R_FLAG_TEST_TIMEOUT) ? 1000000ull : 2000000000ull, p.flags};
  dim3 grid(static_cast<unsigned>((p.L + kBM - 1) / kBM), p.H);
  cmp_attn_tc_kernel<<<grid, kThreads, kSmemBytes, st>>>(tk, tv, a);
  count_launch();
  return cudaGetLastError();
}

}  // namespace s3r
