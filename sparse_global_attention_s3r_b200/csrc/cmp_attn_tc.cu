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
// The kernel is a template on kFused. cmp_attn_tc_kernel<false> is the compressed branch alone
// (O_cmp, lse, scores and/or the top-k to global memory). cmp_attn_tc_kernel<true> is the single
// fused kernel: after pass B the same warps run the selection branch for the CTA's two query
// blocks on the streamed top-k (fused_selection) and write the gated combine; O_cmp is parked in
// shared memory as bf16 and the selection's ring reuses the Kc/Vc ring.
// Every wait is an mbarrier wait bounded in time that also watches a CTA abort flag; on expiry
// the kernel records S3R_DEV_TIMEOUT, drains its in-flight copies and MMAs, frees TMEM and exits.
#include <climits>

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

// barriers of the selection phase of the single fused kernel
struct __align__(8) Bars2 {
  uint64_t lists_ready;  // both score warps have posted their lists (and read their last sums)
  uint64_t ocmp_read;    // every softmax warp has read O_cmp out of TMEM
  uint64_t q2_full;
  uint64_t kv2_full[2], kv2_empty[2];
  uint64_t s2_full, s2_empty;
  uint64_t p2_full, p2_empty;
  uint64_t o2_full;
  uint64_t pair[4];  // per lane quadrant: both column halves have posted their row statistics
};

constexpr uint32_t kOffKV = 0;                                 // stage s: K at +2s*8K, V +8K
constexpr uint32_t kOffRed = kOffKV + kStages * 2 * kKVBytes;  // [kRed][4 quadrant][64] f32
constexpr uint32_t kOffStat = kOffRed + kRed * 4 * 64 * 4;     // [2 halves][128 rows] float2
constexpr uint32_t kOffBars = kOffStat + 2 * 128 * 8;

// The single fused kernel runs the selection branch in the same CTA once the compressed branch
// is done. Its gathered K/V ring and Q tile take the Kc/Vc ring's 80 KB; O_cmp (bf16) takes the
// partial-sum and statistics area; then come the row-statistics exchange, the top-k lists and
// the barriers. Two CTAs still share an SM.
constexpr int kSelStep = 64;    // slots of each query block per selection step
constexpr int kSelStages = 2;   // gathered K/V ring depth
constexpr uint32_t kSelTileBytes = 2 * kSelStep * 128;  // 128 tokens x 128 B: one K or V tile
constexpr uint32_t kOffKV2 = 0;  // stage s: K tile at 2s*16K, V tile at +16K
constexpr uint32_t kOffQ2 = kOffKV2 + kSelStages * 2 * kSelTileBytes;
constexpr uint32_t kQ2Bytes = kBM * 128;
static_assert(kOffQ2 + kQ2Bytes <= kOffRed, "the selection ring and Q tile fit the Kc/Vc ring");
constexpr uint32_t kOffOcmp = kOffRed;  // [128 rows][64] bf16
constexpr uint32_t kOcmpBytes = kBM * 64 * 2;
static_assert(kOcmpBytes >= kOffBars - kOffRed, "O_cmp covers the partial sums and statistics");
constexpr uint32_t kOffXch = kOffOcmp + kOcmpBytes;        // [2 parity][2 half][128 rows] f32
constexpr uint32_t kOffLists = kOffXch + 2 * 2 * 128 * 4;  // [2 query blocks][32] int32
constexpr uint32_t kOffBarsF = kOffLists + 2 * 32 * 4;
constexpr uint32_t kColS2 = 0, kColO2 = 128, kColP2 = 192;  // selection TMEM: S | O_sel | P
constexpr uint32_t kIdescQK2 = idesc_bf16_f32(kBM, 2 * kSelStep, 0, 0);  // Q smem, K K-major
constexpr float kMoveRef = 32.f;  // base-2 margin before a selection row's reference max moves

template <bool kFused>
constexpr uint32_t bars_offset() { return kFused ? kOffBarsF : kOffBars; }
template <bool kFused>
constexpr uint32_t misc_offset() {  // tmem base, abort flag
  return bars_offset<kFused>() + sizeof(Bars) + (kFused ? sizeof(Bars2) : 0);
}
// At most two CTAs share an SM (shared memory), so two 256-column TMEM allocations always fit.
template <bool kFused>
constexpr uint32_t smem_bytes() {
  return misc_offset<kFused>() + 16 + 1024 > 80 * 1024 ? misc_offset<kFused>() + 16 + 1024
                                                       : 80 * 1024;
}

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
  // the selection phase of the single fused kernel
  const float* gates;  // [L, H, 2] fp32
  uint16_t* out;       // [L, H, 64] bf16
  BlockGeo geo;        // which tokens each key block holds
  int64_t Lp;          // rows of one head in the head-major K/V copies (nb * b)
  int b, lb, nsel, nsteps2;  // block size, log2(b), list length forced + topk, 64-slot steps
};

// Block index of entry s of a query block's selection list in the fused kernel: the forced
// blocks 0 .. forced-1, then the streamed top-k held in shared memory; past the list, invalid.
__device__ __forceinline__ int64_t fused_sel_block(const int32_t* topk_list, int s, int forced,
                                                   int nsel, int64_t nb, bool& ok) {
  if (s >= nsel) {
    ok = false;
    return 0;
  }
  const int64_t j = s < forced ? s : topk_list[s - forced];
  ok = j >= 0 && j < nb;
  return ok ? j : 0;
}

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

// The selection phase of the single fused kernel for one softmax warp. Two warps per TMEM lane
// quadrant (32 rows of one query block) each take 32 of a step's 64 columns, 4 rows x 8 columns
// per thread with the 16x256b load shape. The two halves swap their row maxima every step (and
// their row sums at the end) through shared memory on a bounded per-quadrant mbarrier. A row's
// reference max is fixed at its first step with a valid column and moves (with O_sel and the row
// sum rescaled once the previous product has completed) only if a logit exceeds it by 32 in
// base-2 units, so bf16 P stays below 2^32. Ends with the gated combine of O_cmp (parked in
// shared memory as bf16) and O_sel, written as bf16. False if a wait gave up.
__device__ __forceinline__ bool fused_selection(const CmpArgs& a, int h, int64_t q0, int g,
                                                int half, int lane, uint32_t tbase,
                                                uint8_t* smem, const int32_t* lists, Bars2* b2,
                                                volatile int* abort, uint64_t lim) {
  const int qb = g >> 1;
  const int tq = lane & 3, tr = lane >> 2;
  const uint32_t tl0 = tbase + (static_cast<uint32_t>(g * 32) << 16);
  const uint32_t tl16 = tbase + (static_cast<uint32_t>(g * 32 + 16) << 16);
  const float sl2 = a.scale_log2;
  const int32_t* list = lists + qb * 32;
  float* xch = reinterpret_cast<float*>(smem + kOffXch);  // [parity][half][row]

  {  // the other query block's P columns of these rows stay zero for the whole phase
    const uint32_t z[16] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
    tmem_st32x16(tl0 + kColP2 + (1 - qb) * 32 + half * 16, z);
    tmem_wait_st_keep16(z);
  }
  // value v[i][c]: row tr + 8i of the quadrant, column 32*half + 8*(c/2) + 2*tq + c%2 of the
  // step's 64 columns of the query block
  auto col_of = [&](int c) { return half * 32 + 8 * (c >> 1) + 2 * tq + (c & 1); };
  // post this warp's values for rows tr + 8i (one thread per quad) and return the other half's
  auto exchange = [&](const float (&mine)[4], float (&theirs)[4], int phase) -> bool {
    float* buf = xch + (phase & 1) * 256;
    if (tq == 0) {
#pragma unroll
      for (int i = 0; i < 4; ++i) buf[half * 128 + g * 32 + tr + 8 * i] = mine[i];
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&b2->pair[g]);
    if (!mbar_wait(&b2->pair[g], phase & 1, abort, lim)) return false;
#pragma unroll
    for (int i = 0; i < 4; ++i) theirs[i] = buf[(1 - half) * 128 + g * 32 + tr + 8 * i];
    return true;
  };
  float mr[4], l[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) mr[i] = -INFINITY, l[i] = 0.f;

  for (int t = 0; t < a.nsteps2; ++t) {
    if (!mbar_wait(&b2->s2_full, t & 1, abort, lim)) return false;
    tc_fence_after();
    uint32_t r0[16], r1[16];
    tmem_ld16x256_x4(tl0 + kColS2 + qb * 64 + half * 32, r0);
    tmem_ld16x256_x4(tl16 + kColS2 + qb * 64 + half * 32, r1);
    tmem_wait_ld_n<16>(r0);
    tmem_wait_ld_n<16>(r1);
    tc_fence_before();
    __syncwarp();  // one arrival per warp: its lanes' TMEM loads have all completed
    if (lane == 0) mbar_arrive(&b2->s2_empty);
    float v[4][8];
    unpack_rows(r0, r1, v);
    {  // columns whose slot holds no token (a 64-slot step spans at most two blocks, b >= 32)
      const int p0 = t * kSelStep;
      const int s_lo = p0 >> a.lb, s_hi = (p0 + kSelStep - 1) >> a.lb;
      bool ok_lo, ok_hi;
      const int64_t j_lo = fused_sel_block(list, s_lo, a.forced, a.nsel, a.nb, ok_lo);
      const int64_t j_hi = fused_sel_block(list, s_hi, a.forced, a.nsel, a.nb, ok_hi);
      const BlockOrigin bo_lo = block_origin(a.geo, j_lo), bo_hi = block_origin(a.geo, j_hi);
      const bool all_valid =
          ok_lo && ok_hi && origin_full(a.geo, bo_lo) && origin_full(a.geo, bo_hi);
      if (!all_valid) {
        uint64_t bits;
        if (a.b >= kSelStep) {
          bits = ok_lo ? slot_bits(a.geo, bo_lo, p0 & (a.b - 1), kSelStep) : 0ull;
        } else {
          bits = (ok_lo ? slot_bits(a.geo, bo_lo, 0, 32) : 0ull) |
                 ((ok_hi ? slot_bits(a.geo, bo_hi, 0, 32) : 0ull) << 32);
        }
#pragma unroll
        for (int c = 0; c < 8; ++c)
          if (!((bits >> col_of(c)) & 1ull)) v[0][c] = v[1][c] = v[2][c] = v[3][c] = -INFINITY;
      }
    }
    // row maxima of this step over both column halves
    float tmax[4], other[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float m = max8(v[i]);
      m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
      m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
      tmax[i] = m;
    }
    if (!exchange(tmax, other, t)) return false;
    bool move = false;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      tmax[i] = fmaxf(tmax[i], other[i]);
      move |= tmax[i] * sl2 > mr[i] * sl2 + kMoveRef;  // true on the first step with a valid column
    }
    // P(t) may overwrite the P buffer (and O_sel be rescaled) once P*V of step t-1 completed
    if (!mbar_wait(&b2->p2_empty, (t & 1) ^ 1, abort, lim)) return false;
    if (__any_sync(0xffffffffu, move)) {
      float f[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float mn = tmax[i] * sl2 > mr[i] * sl2 + kMoveRef ? tmax[i] : mr[i];
        f[i] = mr[i] == -INFINITY ? 0.f : exp2_approx((mr[i] - mn) * sl2);
        l[i] *= f[i];
        mr[i] = mn;
      }
      if (t > 0) {  // this half's O_sel columns of the warp's rows (lane = row) times the factor
        const int src = 4 * (lane & 7);  // a thread of the quad that holds row `lane`
        const float f0 = __shfl_sync(0xffffffffu, f[0], src);
        const float f1 = __shfl_sync(0xffffffffu, f[1], src);
        const float f2 = __shfl_sync(0xffffffffu, f[2], src);
        const float f3 = __shfl_sync(0xffffffffu, f[3], src);
        const int which = lane >> 3;
        const float fr = which == 0 ? f0 : which == 1 ? f1 : which == 2 ? f2 : f3;
        tc_fence_after();
#pragma unroll 1
        for (int q4 = 0; q4 < 2; ++q4) {
          uint32_t o[16];
          tmem_ld32x16(tl0 + kColO2 + half * 32 + 16 * q4, o);
          tmem_wait_ld_n<16>(o);
#pragma unroll
          for (int j = 0; j < 16; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * fr);
          tmem_st32x16(tl0 + kColO2 + half * 32 + 16 * q4, o);
          tmem_wait_st_keep16(o);
        }
      }
    }
    // P = exp2(v * sl2 - ref * sl2), its row sums, and bf16 P in the 16x128b store layout:
    // repetition rep covers TMEM columns 4rep..4rep+3 of this half's 16, lane tr -> register
    // 2rep, lane tr+8 -> 2rep+1; value columns (2rep, 2rep+1) are keys 32half + 8rep + 2tq + {0,1}
    float off[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) off[i] = mr[i] == -INFINITY ? 0.f : -mr[i] * sl2;
    uint32_t a0[8], a1[8];
#pragma unroll
    for (int rep = 0; rep < 4; ++rep) {
      const int c = 2 * rep;
      float e[4][2];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 x = __ffma2_rn(make_float2(v[i][c], v[i][c + 1]), make_float2(sl2, sl2),
                                    make_float2(off[i], off[i]));
        e[i][0] = exp2_approx(x.x);
        e[i][1] = exp2_approx(x.y);
        l[i] += e[i][0] + e[i][1];
      }
      a0[2 * rep] = pack_bf16(e[0][0], e[0][1]);
      a0[2 * rep + 1] = pack_bf16(e[1][0], e[1][1]);
      a1[2 * rep] = pack_bf16(e[2][0], e[2][1]);
      a1[2 * rep + 1] = pack_bf16(e[3][0], e[3][1]);
    }
    tmem_st16x128_x4(tl0 + kColP2 + qb * 32 + half * 16, a0);
    tmem_st16x128_x4(tl16 + kColP2 + qb * 32 + half * 16, a1);
    tmem_wait_st_keep8(a0);
    tmem_wait_st_keep8(a1);
    tc_fence_before();
    __syncwarp();  // one arrival per warp: its lanes' TMEM stores have all completed
    if (lane == 0) mbar_arrive(&b2->p2_full);
  }

  // row sums over both halves, then O_sel / l on this half's 32 columns (lane = row), combined
  float lsum[4], lother[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float s = l[i];
    s += __shfl_xor_sync(0xffffffffu, s, 1);
    s += __shfl_xor_sync(0xffffffffu, s, 2);
    lsum[i] = s;
  }
  if (!exchange(lsum, lother, a.nsteps2)) return false;
  if (!mbar_wait(&b2->o2_full, 0, abort, lim)) return false;
  const int src = 4 * (lane & 7);
  float tot[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) tot[i] = lsum[i] + lother[i];
  const float s0 = __shfl_sync(0xffffffffu, tot[0], src);
  const float s1 = __shfl_sync(0xffffffffu, tot[1], src);
  const float s2 = __shfl_sync(0xffffffffu, tot[2], src);
  const float s3 = __shfl_sync(0xffffffffu, tot[3], src);
  const int which = lane >> 3;
  const float rs = which == 0 ? s0 : which == 1 ? s1 : which == 2 ? s2 : s3;
  const float inv = rs > 0.f ? 1.f / rs : 0.f;
  tc_fence_after();
  uint32_t o[32];
  tmem_ld32(tl0 + kColO2 + half * 32, o);
  tmem_wait_ld_regs(o);
  const int64_t row = q0 + g * 32 + lane;
  if (row < a.L) {
    const int64_t at = (row * a.H + h) * 64 + half * 32;
    const float2 gl = *reinterpret_cast<const float2*>(a.gates + (row * a.H + h) * 2);
    const float gc = 1.f / (1.f + expf(-gl.x));
    const float gs = 1.f / (1.f + expf(-gl.y));
    const uint4* oc = reinterpret_cast<const uint4*>(smem + kOffOcmp) + (g * 32 + lane) * 8 + half * 4;
    uint4* dst = reinterpret_cast<uint4*>(a.out + at);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint4 c = oc[j];
      const uint32_t cw[4] = {c.x, c.y, c.z, c.w};
      uint32_t w[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float c_lo = __uint_as_float(cw[e] << 16), c_hi = __uint_as_float(cw[e] & 0xFFFF0000u);
        w[e] = pack_bf16(gc * c_lo + gs * (__uint_as_float(o[8 * j + 2 * e]) * inv),
                         gc * c_hi + gs * (__uint_as_float(o[8 * j + 2 * e + 1]) * inv));
      }
      dst[j] = make_uint4(w[0], w[1], w[2], w[3]);
    }
  }
  return true;
}

// kFused: after the compressed branch, the same CTA runs the selection branch for its two query
// blocks on the streamed top-k lists and writes the gated combine; tmQ2, tmK2, tmV2 (the Q tile,
// and the head-major K/V copies) are used only then.
template <bool kFused>
__global__ void __launch_bounds__(kThreads, 2)
    cmp_attn_tc_kernel(const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV,
                       const __grid_constant__ CUtensorMap tmQ2,
                       const __grid_constant__ CUtensorMap tmK2,
                       const __grid_constant__ CUtensorMap tmV2, const CmpArgs a) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_s = smem_addr(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_s & 1023u)) & 1023u);  // 1024-byte aligned base
  const uint32_t sbase = smem_addr(smem);
  Bars* bars = reinterpret_cast<Bars*>(smem + bars_offset<kFused>());
  Bars2* b2 = reinterpret_cast<Bars2*>(smem + bars_offset<kFused>() + sizeof(Bars));
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + misc_offset<kFused>());
  volatile int* abort = reinterpret_cast<volatile int*>(smem + misc_offset<kFused>() + 4);
  float* red = reinterpret_cast<float*>(smem + kOffRed);
  float2* stat = reinterpret_cast<float2*>(smem + kOffStat);
  int32_t* lists = reinterpret_cast<int32_t*>(smem + kOffLists);  // fused: [2][32] top-k

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
    if constexpr (kFused) {
      mbar_init(&b2->lists_ready, 2);
      mbar_init(&b2->ocmp_read, kSoftmaxWarps);
      mbar_init(&b2->q2_full, 1);
      for (int s = 0; s < kSelStages; ++s) {
        mbar_init(&b2->kv2_full[s], 1);
        mbar_init(&b2->kv2_empty[s], 1);
      }
      mbar_init(&b2->s2_full, 1);
      mbar_init(&b2->s2_empty, kSoftmaxWarps);
      mbar_init(&b2->p2_full, kSoftmaxWarps);
      mbar_init(&b2->p2_empty, 1);
      mbar_init(&b2->o2_full, 1);
      for (int g = 0; g < 4; ++g) mbar_init(&b2->pair[g], 2);
    }
    *abort = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
    if constexpr (kFused) {
      prefetch_tmap(&tmQ2);
      prefetch_tmap(&tmK2);
      prefetch_tmap(&tmV2);
    }
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
      if constexpr (kFused) {
        // selection: once every compressed-branch product has completed (the Kc/Vc ring is
        // free) and the lists are posted, load the Q tile and gather the selected blocks' K/V
        // rows from the head-major copies, 64 slots of each query block per step
        if (ok) ok = mbar_wait(&bars->o_full, 0, abort, lim);
        if (ok) ok = mbar_wait(&b2->lists_ready, 0, abort, lim);
        int issued2 = 0;
        bool q_issued = false;
        if (ok) {
          mbar_arrive_expect_tx(&b2->q2_full, kQ2Bytes);
          tma_load_2d(sbase + kOffQ2, &tmQ2, h * 64, static_cast<int32_t>(q0), &b2->q2_full);
          q_issued = true;
          const int box = a.b < kSelStep ? a.b : kSelStep;  // rows per box: one run of slots
          for (int t = 0; t < a.nsteps2; ++t) {
            const int stage = t % kSelStages;
            if (!mbar_wait(&b2->kv2_empty[stage], ((t / kSelStages) & 1) ^ 1, abort, lim)) {
              ok = false;
              break;
            }
            const uint32_t sk = sbase + kOffKV2 + stage * 2 * kSelTileBytes;
            mbar_arrive_expect_tx(&b2->kv2_full[stage], 2 * kSelTileBytes);
            for (int qb = 0; qb < 2; ++qb) {
              for (int part = 0; part < kSelStep / box; ++part) {
                const int pos = t * kSelStep + part * box;
                bool valid;  // an entry past the list loads block 0 and is masked
                const int64_t j = fused_sel_block(lists + qb * 32, pos >> a.lb, a.forced, a.nsel,
                                                  a.nb, valid);
                const int64_t row = j * a.b + (pos & (a.b - 1));  // slot row of the copy
                const uint32_t row_off = (qb * kSelStep + part * box) * 128;
                const int32_t y = static_cast<int32_t>(h * a.Lp + row);
                tma_load_2d(sk + row_off, &tmK2, 0, y, &b2->kv2_full[stage]);
                tma_load_2d(sk + kSelTileBytes + row_off, &tmV2, 0, y, &b2->kv2_full[stage]);
              }
            }
            issued2 = t + 1;
          }
        }
        if (!ok) {
          raise_abort(abort, a.status);
          int dummy = 0;
          if (q_issued) mbar_wait(&b2->q2_full, 0, &dummy, lim);
          for (int t = issued2 - 1; t >= 0 && t >= issued2 - kSelStages; --t)
            mbar_wait(&b2->kv2_full[t % kSelStages], (t / kSelStages) & 1, &dummy, lim);
        }
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
      if (ok) tc_commit(&bars->o_full);
      if constexpr (kFused) {
        // selection: S = Q K^T (M=128 x N=128, Q from shared memory: its TMEM columns now hold
        // P) and O_sel += P V, with O_sel where O_cmp was once the softmax warps have read it
        if (ok) ok = mbar_wait(&b2->q2_full, 0, abort, lim);
        if (ok) ok = mbar_wait(&b2->ocmp_read, 0, abort, lim);
        tc_fence_after();
        const uint64_t dq = desc_sw128(sbase + kOffQ2);
        auto qk2 = [&](int t) -> bool {
          const int stage = t % kSelStages;
          if (!mbar_wait(&b2->kv2_full[stage], (t / kSelStages) & 1, abort, lim)) return false;
          if (!mbar_wait(&b2->s2_empty, (t & 1) ^ 1, abort, lim)) return false;
          tc_fence_after();
          const uint64_t dk = desc_sw128(sbase + kOffKV2 + stage * 2 * kSelTileBytes);
#pragma unroll
          for (int ks = 0; ks < 4; ++ks)
            mma_ss(tbase + kColS2, dq + 2 * ks, dk + 2 * ks, kIdescQK2, ks > 0);
          tc_commit(&b2->s2_full);
          return true;
        };
        auto pv2 = [&](int t) -> bool {
          const int stage = t % kSelStages;
          if (!mbar_wait(&b2->p2_full, t & 1, abort, lim)) return false;
          tc_fence_after();
          const uint64_t dv =
              desc_sw128(sbase + kOffKV2 + stage * 2 * kSelTileBytes + kSelTileBytes);
#pragma unroll
          for (int ks = 0; ks < 8; ++ks)  // 128 keys in steps of 16: 16 rows x 128 B = 2048 B
            mma_ts(tbase + kColO2, tbase + kColP2 + ks * 8, dv + 128 * ks, kIdescPV,
                   (t > 0 || ks > 0) ? 1u : 0u);
          tc_commit(&b2->kv2_empty[stage]);
          tc_commit(&b2->p2_empty);
          return true;
        };
        for (int t = 0; ok && t < a.nsteps2; ++t) {
          if (!(ok = qk2(t))) break;
          if (t > 0 && !(ok = pv2(t - 1))) break;
        }
        if (ok) ok = pv2(a.nsteps2 - 1);
        if (ok) tc_commit(&b2->o2_full);
      }
      if (!ok) {
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
      if constexpr (kFused) {
        // O_cmp has left TMEM (the selection accumulates there next); once the score warps
        // have read their last partial sums it is parked, in bf16, over that area: this thread
        // writes and later reads back row g*32 + lane, columns half*32 ..
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&b2->ocmp_read);
        if ((ok = mbar_wait(&b2->lists_ready, 0, abort, lim))) {
          uint4* dst = reinterpret_cast<uint4*>(smem + kOffOcmp) + (g * 32 + lane) * 8 + half * 4;
#pragma unroll
          for (int j = 0; j < 4; ++j)
            dst[j] = make_uint4(
                pack_bf16(__uint_as_float(o[8 * j]), __uint_as_float(o[8 * j + 1])),
                pack_bf16(__uint_as_float(o[8 * j + 2]), __uint_as_float(o[8 * j + 3])),
                pack_bf16(__uint_as_float(o[8 * j + 4]), __uint_as_float(o[8 * j + 5])),
                pack_bf16(__uint_as_float(o[8 * j + 6]), __uint_as_float(o[8 * j + 7])));
        }
      } else {
        const int64_t row = q0 + g * 32 + lane;
        if (row < a.L) {
          float4* dst = reinterpret_cast<float4*>(a.o_cmp + (row * a.H + h) * 64 + half * 32);
#pragma unroll
          for (int j = 0; j < 8; ++j)
            dst[j] = make_float4(__uint_as_float(o[4 * j]), __uint_as_float(o[4 * j + 1]),
                                 __uint_as_float(o[4 * j + 2]), __uint_as_float(o[4 * j + 3]));
        }
      }
    }
    if constexpr (kFused) {
      if (ok) ok = fused_selection(a, h, q0, g, half, lane, tbase, smem, lists, b2, abort, lim);
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
    if constexpr (kFused) {  // the top-k part of the list, for this CTA's selection phase
      if (lane < a.topk)
        lists[qb * 32 + lane] = static_cast<int32_t>(~static_cast<uint32_t>(best & 0xFFFFFFFFull));
      __syncwarp();
      if (lane == 0) mbar_arrive(&b2->lists_ready);  // also after a timeout: waiters stop sooner
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
  constexpr uint32_t smem = smem_bytes<false>();
  cudaError_t e = cudaFuncSetAttribute(cmp_attn_tc_kernel<false>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  CmpArgs a{q, lse, o_cmp, scores, idx, p.k, p.F, p.L, p.nb, p.nqb, p.H, p.scale_log2, p.status,
            (p.flags & S3R_FLAG_TEST_TIMEOUT) ? 1000000ull : 2000000000ull, p.flags};
  dim3 grid(static_cast<unsigned>((p.L + kBM - 1) / kBM), p.H);
  cmp_attn_tc_kernel<false><<<grid, kThreads, smem, st>>>(tk, tv, tk, tk, tk, a);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_fused_tc(const Problem& p, const uint16_t* q, const uint16_t* kc,
                            const uint16_t* vc, const uint16_t* kh, const uint16_t* vh,
                            const float* gates, uint16_t* out, int32_t* idx, cudaStream_t st) {
  const int64_t Lp = p.nb * p.b;
  if (p.k > kFusedTopkMax || p.H * Lp > INT32_MAX) return cudaErrorInvalidValue;
  const int box = p.b < kSelStep ? p.b : kSelStep;
  CUtensorMap tk, tv, tq2, tk2, tv2;
  if (!make_tmap_head_rows(&tk, kc, p.nb, p.H, kBN) || !make_tmap_head_rows(&tv, vc, p.nb, p.H, kBN) ||
      !make_tmap_head_rows(&tq2, q, p.L, p.H, kBM) || !make_tmap_rows64(&tk2, kh, p.H * Lp, box) ||
      !make_tmap_rows64(&tv2, vh, p.H * Lp, box))
    return cudaErrorInvalidValue;
  constexpr uint32_t smem = smem_bytes<true>();
  cudaError_t e = cudaFuncSetAttribute(cmp_attn_tc_kernel<true>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const int lb = p.b == 32 ? 5 : p.b == 64 ? 6 : 7;
  const int64_t ntok = static_cast<int64_t>(p.nsel) * p.b;
  CmpArgs a{q, nullptr, nullptr, nullptr, idx, p.k, p.F, p.L, p.nb, p.nqb, p.H, p.scale_log2,
            p.status, (p.flags & S3R_FLAG_TEST_TIMEOUT) ? 1000000ull : 2000000000ull, p.flags,
            gates, out, p.geo, Lp, p.b, lb, p.nsel,
            static_cast<int>((ntok + kSelStep - 1) / kSelStep)};
  dim3 grid(static_cast<unsigned>((p.L + kBM - 1) / kBM), p.H);
  cmp_attn_tc_kernel<true><<<grid, kThreads, smem, st>>>(tk, tv, tq2, tk2, tv2, a);
  count_launch();
  return cudaGetLastError();
}

}  // namespace s3r
