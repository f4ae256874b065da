// cmp_attn_tc.cu -- compression branch on the sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// Speed3R (gist.science summary, "Methodologie" §1 "Compressie-tak"): every query attends to the
// mean-pooled block summaries, and the softmax probabilities form a score matrix that ranks the
// key blocks; §4 "Efficient Kernel": the full score matrix is never materialised.
//
// Exact scores need normalised probabilities, so one launch makes two passes over the nb block
// summaries of its 128-row query tile (two 64-row query blocks) and one head:
//   pass A: S = Q Kc^T (tcgen05.mma into TMEM), online max / sum  -> lse per row (registers)
//   pass B: S again; P = exp2(S*scale*log2e - lse2) in fp32; the column sums of the fp32 P over
//           each 64-row query block are that block's scores; bf16(P) is stored to TMEM and
//           O_cmp += P Vc runs on the tensor cores with P as the TMEM operand.
// Roles (224 threads):
//   warp 0     TMA producer: Q once, then Kc (pass A) or Kc+Vc (pass B) 64-key tiles into a
//              4-stage ring of 128-byte-swizzled shared-memory tiles
//   warp 1     TMEM owner (256 columns) and the single-thread tcgen05.mma issuer
//   warps 2-5  softmax: one query row per thread (TMEM lane), column sums by shuffle halving
//   warp 6     sums the two warps' partial column sums of each query block, writes scores
// TMEM: S[2] (64 fp32 columns each), P[2] (64 bf16 = 32 columns each), O (64 fp32 columns).
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

constexpr int kBM = 128;      // query rows per CTA (TMEM lanes)
constexpr int kBN = 64;       // block summaries per tile
constexpr int kStages = 4;    // shared-memory ring depth
constexpr int kThreads = 224; // 7 warps
constexpr uint32_t kQBytes = kBM * 128;   // 16 KB
constexpr uint32_t kKVBytes = kBN * 128;  // 8 KB
constexpr uint32_t kColS = 0, kColP = 128, kColO = 192, kTmemCols = 256;
constexpr uint32_t kIdescQK = idesc_bf16_f32(kBM, kBN, 0, 0);  // A=Q K-major, B=Kc K-major
constexpr uint32_t kIdescPV = idesc_bf16_f32(kBM, 64, 0, 1);   // A=P (TMEM), B=Vc MN-major

struct __align__(8) Bars {
  uint64_t q_full;
  uint64_t kv_full[kStages], kv_empty[kStages];
  uint64_t s_full[2], s_empty[2];
  uint64_t p_full[2], p_empty[2];
  uint64_t red_full[2], red_empty[2];
  uint64_t o_full, drain;
  uint64_t never;  // never signalled: waited on only under S3R_FLAG_TEST_TIMEOUT
};

constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffKV = kQBytes;                              // stage s: K at +2s*8K, V +8K
constexpr uint32_t kOffRed = kOffKV + kStages * 2 * kKVBytes;     // [2][4][64] floats
constexpr uint32_t kOffBars = kOffRed + 2 * 4 * 64 * 4;
constexpr uint32_t kOffMisc = kOffBars + sizeof(Bars);            // tmem base, abort flag
constexpr uint32_t kSmemUsed = kOffMisc + 16;
// Request enough that at most two CTAs share an SM, so two 256-column TMEM allocations always fit.
constexpr uint32_t kSmemBytes = (kSmemUsed + 1024 > 80 * 1024 ? kSmemUsed + 1024 : 80 * 1024);

struct CmpArgs {
  float* lse;     // [H, L] natural log, may be null
  float* o_cmp;   // [L, H, 64]
  float* scores;  // [H, nqb, nb]
  int64_t L, nb, nqb;
  int H;
  float scale_log2;
  uint32_t* status;
  uint64_t limit_ns;
  uint32_t flags;
};

__device__ __forceinline__ void raise_abort(volatile int* abort, uint32_t* status) {
  *abort = 1;
  set_status(status, S3R_DEV_TIMEOUT);
}

__global__ void __launch_bounds__(kThreads, 2)
    cmp_attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ,
                       const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const CmpArgs a) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_s = smem_addr(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_s & 1023u)) & 1023u);  // 1024-byte aligned base
  const uint32_t sbase = smem_addr(smem);
  Bars* bars = reinterpret_cast<Bars*>(smem + kOffBars);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + kOffMisc);
  volatile int* abort = reinterpret_cast<volatile int*>(smem + kOffMisc + 4);
  float* red = reinterpret_cast<float*>(smem + kOffRed);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.y;
  const int64_t qtile = blockIdx.x;
  const int64_t q0 = qtile * kBM;
  const int nt = static_cast<int>((a.nb + kBN - 1) / kBN);
  const uint64_t lim = a.limit_ns;

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bars->kv_full[s], 1);
      mbar_init(&bars->kv_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars->s_full[b], 1);
      mbar_init(&bars->s_empty[b], 128);
      mbar_init(&bars->p_full[b], 128);
      mbar_init(&bars->p_empty[b], 1);
      mbar_init(&bars->red_full[b], 4);
      mbar_init(&bars->red_empty[b], 1);
    }
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
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int issued = 0;
      bool ok = true;
      mbar_arrive_expect_tx(&bars->q_full, kQBytes);
      tma_load_2d(sbase + kOffQ, &tmQ, h * 64, static_cast<int32_t>(q0), &bars->q_full);
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
        mbar_wait(&bars->q_full, 0, &dummy, lim);
        for (int u = issued - 1; u >= 0 && u >= issued - kStages; --u)
          mbar_wait(&bars->kv_full[u % kStages], (u / kStages) & 1, &dummy, lim);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      bool ok = mbar_wait(&bars->q_full, 0, abort, lim);
      tc_fence_after();
      const uint64_t dq = desc_sw128(sbase + kOffQ);
      auto qk = [&](int u, int c) -> bool {  // S[c&1] = Q Kc^T for ring use u
        const int stage = u % kStages;
        if (!mbar_wait(&bars->kv_full[stage], (u / kStages) & 1, abort, lim)) return false;
        const int b = c & 1;
        if (!mbar_wait(&bars->s_empty[b], ((c >> 1) & 1) ^ 1, abort, lim)) return false;
        tc_fence_after();
        const uint64_t dk = desc_sw128(sbase + kOffKV + stage * 2 * kKVBytes);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
          mma_ss(tbase + kColS + b * kBN, dq + 2 * ks, dk + 2 * ks, kIdescQK, ks > 0);
        return true;
      };
      auto pv = [&](int t) -> bool {  // O += P[t&1] Vc for pass-B tile t
        const int u = nt + t, stage = u % kStages, pb = t & 1;
        if (!mbar_wait(&bars->p_full[pb], (t >> 1) & 1, abort, lim)) return false;
        tc_fence_after();
        const uint64_t dv = desc_sw128(sbase + kOffKV + stage * 2 * kKVBytes + kKVBytes);
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)  // 16 keys per step: 16 rows x 128 B = 2048 B
          mma_ts(tbase + kColO, tbase + kColP + pb * 32 + ks * 8, dv + 128 * ks, kIdescPV,
                 (t > 0 || ks > 0) ? 1u : 0u);
        tc_commit(&bars->kv_empty[stage]);
        tc_commit(&bars->p_empty[pb]);
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
  } else if (warp <= 5) {
    // ------------------------------------------------------------------ softmax warps
    const int g = warp & 3;  // TMEM lane quadrant this warp may access
    const int row_local = g * 32 + lane;
    const int64_t row = q0 + row_local;
    const bool row_ok = row < a.L;
    const uint32_t tl = tbase + (static_cast<uint32_t>(g * 32) << 16);
    const float sl2 = a.scale_log2;
    bool ok = true;
    if (a.flags & S3R_FLAG_TEST_TIMEOUT) ok = mbar_wait(&bars->never, 0, abort, lim);

    // pass A: online max / sum over all nb summaries
    float m = -INFINITY, l = 0.f;
    for (int t = 0; ok && t < nt; ++t) {
      const int b = t & 1;
      if (!(ok = mbar_wait(&bars->s_full[b], (t >> 1) & 1, abort, lim))) break;
      tc_fence_after();
      uint32_t r0[32], r1[32];
      tmem_ld32(tl + kColS + b * kBN, r0);
      tmem_ld32(tl + kColS + b * kBN + 32, r1);
      tmem_wait_ld_regs(r0);
      tmem_wait_ld_regs(r1);
      tc_fence_before();
      mbar_arrive(&bars->s_empty[b]);
      const int64_t valid = a.nb - static_cast<int64_t>(t) * kBN;  // columns < valid are real
      float x[64];
      float tmax = -INFINITY;
#pragma unroll
      for (int j = 0; j < 64; ++j) {
        const float s = __uint_as_float(j < 32 ? r0[j] : r1[j - 32]);
        x[j] = j < valid ? s * sl2 : -INFINITY;
        tmax = fmaxf(tmax, x[j]);
      }
      const float mn = fmaxf(m, tmax);  // finite: the first column of every tile is real
      l *= exp2_approx(m - mn);
      m = mn;
#pragma unroll
      for (int j = 0; j < 64; ++j) l += exp2_approx(x[j] - m);
    }
    const float lse2 = row_ok ? m + log2f(l) : INFINITY;
    if (ok && a.lse && row_ok) a.lse[static_cast<int64_t>(h) * a.L + row] = lse2 * kLn2;

    // pass B: probabilities, column sums, P to TMEM for the P*Vc product
    for (int t = 0; ok && t < nt; ++t) {
      const int c = nt + t, b = c & 1;
      if (!(ok = mbar_wait(&bars->s_full[b], (c >> 1) & 1, abort, lim))) break;
      tc_fence_after();
      uint32_t r[2][32];
      tmem_ld32(tl + kColS + b * kBN, r[0]);
      tmem_ld32(tl + kColS + b * kBN + 32, r[1]);
      tmem_wait_ld_regs(r[0]);
      tmem_wait_ld_regs(r[1]);
      tc_fence_before();
      mbar_arrive(&bars->s_empty[b]);
      const int64_t valid = a.nb - static_cast<int64_t>(t) * kBN;
      const int par = t & 1;
      if (!(ok = mbar_wait(&bars->red_empty[par], ((t >> 1) & 1) ^ 1, abort, lim))) break;
      uint32_t pk[32];
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        float p[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const float s = __uint_as_float(r[half][j]);
          p[j] = (half * 32 + j) < valid ? exp2_approx(fmaf(s, sl2, -lse2)) : 0.f;
        }
#pragma unroll
        for (int j = 0; j < 16; ++j) pk[half * 16 + j] = pack_bf16(p[2 * j], p[2 * j + 1]);
        // column sums over the warp's 32 rows: recursive halving leaves column `lane` here
#pragma unroll
        for (int w = 16; w >= 1; w >>= 1) {
          const bool upper = lane & w;
#pragma unroll
          for (int i = 0; i < w; ++i) {
            const float send = upper ? p[i] : p[i + w];
            const float keep = upper ? p[i + w] : p[i];
            p[i] = keep + __shfl_xor_sync(0xffffffffu, send, w);
          }
        }
        red[(par * 4 + g) * 64 + half * 32 + lane] = p[0];
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->red_full[par]);
      const int pb = t & 1;
      if (!(ok = mbar_wait(&bars->p_empty[pb], ((t >> 1) & 1) ^ 1, abort, lim))) break;
      tmem_st32(tl + kColP + pb * 32, pk);
      tmem_wait_st_regs(pk);
      tc_fence_before();
      mbar_arrive(&bars->p_full[pb]);
    }
    if (ok && (ok = mbar_wait(&bars->o_full, 0, abort, lim))) {
      tc_fence_after();
      uint32_t o0[32], o1[32];
      tmem_ld32(tl + kColO, o0);
      tmem_ld32(tl + kColO + 32, o1);
      tmem_wait_ld_regs(o0);
      tmem_wait_ld_regs(o1);
      if (row_ok) {
        float4* dst = reinterpret_cast<float4*>(a.o_cmp + (row * a.H + h) * 64);
#pragma unroll
        for (int j = 0; j < 8; ++j)
          dst[j] = make_float4(__uint_as_float(o0[4 * j]), __uint_as_float(o0[4 * j + 1]),
                               __uint_as_float(o0[4 * j + 2]), __uint_as_float(o0[4 * j + 3]));
#pragma unroll
        for (int j = 0; j < 8; ++j)
          dst[8 + j] = make_float4(__uint_as_float(o1[4 * j]), __uint_as_float(o1[4 * j + 1]),
                                   __uint_as_float(o1[4 * j + 2]), __uint_as_float(o1[4 * j + 3]));
      }
    }
    if (!ok) raise_abort(abort, a.status);
  } else {
    // ------------------------------------------------------------------ score writer
    for (int t = 0; t < nt; ++t) {
      const int par = t & 1;
      if (!mbar_wait(&bars->red_full[par], (t >> 1) & 1, abort, lim)) {
        if (lane == 0) raise_abort(abort, a.status);
        break;
      }
#pragma unroll
      for (int qb = 0; qb < 2; ++qb) {
        const int64_t i = qtile * 2 + qb;
        if (i >= a.nqb) continue;
        float* dst = a.scores + (static_cast<int64_t>(h) * a.nqb + i) * a.nb;
#pragma unroll
        for (int hc = 0; hc < 2; ++hc) {
          const int cc = hc * 32 + lane;
          const int64_t col = static_cast<int64_t>(t) * kBN + cc;
          if (col < a.nb)
            dst[col] = red[(par * 4 + 2 * qb) * 64 + cc] + red[(par * 4 + 2 * qb + 1) * 64 + cc];
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->red_empty[par]);
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
                               cudaStream_t st) {
  CUtensorMap tq, tk, tv;
  if (!make_tmap_head_rows(&tq, q, p.L, p.H, kBM) || !make_tmap_head_rows(&tk, kc, p.nb, p.H, kBN) ||
      !make_tmap_head_rows(&tv, vc, p.nb, p.H, kBN))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(cmp_attn_tc_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e != cudaSuccess) return e;
  CmpArgs a{lse, o_cmp, scores, p.L, p.nb, p.nqb, p.H, p.scale_log2, p.status,
            (p.flags & S3R_FLAG_TEST_TIMEOUT) ? 1000000ull : 2000000000ull, p.flags};
  dim3 grid(static_cast<unsigned>((p.L + kBM - 1) / kBM), p.H);
  cmp_attn_tc_kernel<<<grid, kThreads, kSmemBytes, st>>>(tq, tk, tv, a);
  count_launch();
  return cudaGetLastError();
}

}  // namespace s3r
