// cmp_attn.cu -- compression branch: attention of every query to the nb block summaries, and the
// block score matrix.
//
// Speed3R (gist.science summary, "Methodologie" §1 "Compressie-tak"): attention over the pooled
// tokens produces a score matrix that identifies the relevant regions; §4 "Efficient Kernel": the
// scores are softmax probabilities and are never materialised as a full [L, nb] matrix.
//
// Exact scores need normalised probabilities, hence two passes over the nb summaries:
//   pass A  lse[q]   = log sum_j exp(s[q,j])                  (online max / sum)
//   pass B  P[q,j]   = exp(s[q,j] - lse[q])  in fp32
//           O_cmp[q] = sum_j bf16(P[q,j]) * Vc[j]             (tensor cores, fp32 accumulate)
//           score[i,j] = sum over the 64 rows q of block i of the fp32 P[q,j]
// One CTA = one 64-row query block of one head (4 warps x 16 rows), which is exactly the row set
// a score sums over, so the column sums never leave the CTA. Key tiles of 64 summaries are
// double-buffered in shared memory with cp.async; logits and P*V use mma.sync m16n8k16 (bf16 in,
// fp32 accumulate). Column sums: in-thread add of the two rows a thread holds, a recursive-halving
// shuffle reduction over the 8 row groups of the warp (14 shuffles for 64 columns), then a
// 4-warp sum through shared memory.
#include "common.cuh"
#include "internal.h"

namespace s3r {
namespace {

constexpr int kThreads = 128;  // 4 warps x 16 query rows
constexpr int kTile = 64;      // rows of a Q tile and keys of a K/V tile (64 x 64 bf16 = 8 KB)
constexpr int kTileBytes = kTile * 128;

// cp.async a [64, 64] bf16 tile (rows r0.. of a [nrows, H, 64] tensor, head h) into swizzled smem.
// Rows at or beyond nrows are zero-filled without being read.
__device__ __forceinline__ void load_tile(uint32_t sbase, const uint16_t* __restrict__ g,
                                          int64_t r0, int64_t nrows, int HD, int h) {
#pragma unroll
  for (int c = threadIdx.x; c < kTile * 8; c += kThreads) {
    const int row = c >> 3, ch = c & 7;
    const int64_t r = r0 + row;
    const bool ok = r < nrows;
    const uint16_t* src = g + (ok ? r : 0) * HD + h * 64 + ch * 8;
    cp_async_16(sbase + swz128(row, ch), src, ok);
  }
}

// A fragments of this warp's 16 query rows for the 4 k-steps of d = 64.
__device__ __forceinline__ void load_q_frags(uint32_t sQ, int warp, int lane, uint32_t qf[4][4]) {
  const int mi = lane >> 3, r = lane & 7;
#pragma unroll
  for (int ks = 0; ks < 4; ++ks) {
    const int row = warp * 16 + (mi & 1) * 8 + r;
    const int ch = 2 * ks + (mi >> 1);
    ldsm_x4(sQ + swz128(row, ch), qf[ks][0], qf[ks][1], qf[ks][2], qf[ks][3]);
  }
}

// s[nt][c] = Q K^T for the warp's 16 rows x 64 keys of the tile at sK (fp32).
// Element (nt, c): row g + 8*(c>>1), key nt*8 + 2*(lane&3) + (c&1), with g = lane>>2.
__device__ __forceinline__ void qk_tile(uint32_t sK, int lane, const uint32_t qf[4][4],
                                        float s[8][4]) {
#pragma unroll
  for (int nt = 0; nt < 8; ++nt) s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
  const int mi = lane >> 3, r = lane & 7;
#pragma unroll
  for (int ks = 0; ks < 4; ++ks) {
#pragma unroll
    for (int np = 0; np < 4; ++np) {
      const int key = np * 16 + (mi >> 1) * 8 + r;
      const int ch = 2 * ks + (mi & 1);
      uint32_t b0, b1, b2, b3;
      ldsm_x4(sK + swz128(key, ch), b0, b1, b2, b3);
      mma16816(s[2 * np], qf[ks], b0, b1);
      mma16816(s[2 * np + 1], qf[ks], b2, b3);
    }
  }
}

// ---------------------------------------------------------------------------------------------
// pass A: lse
// ---------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(kThreads)
    cmp_lse_kernel(const uint16_t* __restrict__ q, const uint16_t* __restrict__ kc,
                   float* __restrict__ lse, int64_t L, int H, int64_t nb, float scale_log2) {
  __shared__ __align__(128) uint8_t smem[3 * kTileBytes];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.y;
  const int64_t q0 = static_cast<int64_t>(blockIdx.x) * kTile;
  const int HD = H * 64;
  const uint32_t sQ = smem_addr(smem);
  const uint32_t sK0 = sQ + kTileBytes;
  const int ntiles = static_cast<int>((nb + kTile - 1) / kTile);

  load_tile(sQ, q, q0, L, HD, h);
  load_tile(sK0, kc, 0, nb, HD, h);
  cp_async_commit();

  float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.f, 0.f};
  uint32_t qf[4][4];
  const int tq = lane & 3;

  for (int t = 0; t < ntiles; ++t) {
    if (t + 1 < ntiles) {
      load_tile(sK0 + ((t + 1) & 1) * kTileBytes, kc, static_cast<int64_t>(t + 1) * kTile, nb, HD, h);
      cp_async_commit();
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    if (t == 0) load_q_frags(sQ, warp, lane, qf);

    float s[8][4];
    qk_tile(sK0 + (t & 1) * kTileBytes, lane, qf, s);
    const int64_t col0 = static_cast<int64_t>(t) * kTile + 2 * tq;
    float tmax[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const bool ok = col0 + nt * 8 + (c & 1) < nb;
        s[nt][c] = ok ? s[nt][c] * scale_log2 : -INFINITY;
        tmax[c >> 1] = fmaxf(tmax[c >> 1], s[nt][c]);
      }
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      tmax[r] = fmaxf(tmax[r], __shfl_xor_sync(0xffffffffu, tmax[r], 1));
      tmax[r] = fmaxf(tmax[r], __shfl_xor_sync(0xffffffffu, tmax[r], 2));
      const float mn = fmaxf(m[r], tmax[r]);  // finite: every tile has a valid column
      l[r] *= exp2_approx(m[r] - mn);
      m[r] = mn;
    }
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int c = 0; c < 4; ++c) l[c >> 1] += exp2_approx(s[nt][c] - m[c >> 1]);
    __syncthreads();
  }

  const int g = lane >> 2;
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    l[r] += __shfl_xor_sync(0xffffffffu, l[r], 1);
    l[r] += __shfl_xor_sync(0xffffffffu, l[r], 2);
    const int64_t row = q0 + warp * 16 + g + 8 * r;
    if (tq == 0 && row < L) lse[static_cast<int64_t>(h) * L + row] = (m[r] + log2f(l[r])) * kLn2;
  }
}

// ---------------------------------------------------------------------------------------------
// pass B: O_cmp and scores
// ---------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(kThreads)
    cmp_pv_score_kernel(const uint16_t* __restrict__ q, const uint16_t* __restrict__ kc,
                        const uint16_t* __restrict__ vc, const float* __restrict__ lse,
                        float* __restrict__ o_cmp, float* __restrict__ scores, int64_t L, int H,
                        int64_t nb, int64_t nqb, float scale_log2) {
  __shared__ __align__(128) uint8_t smem[5 * kTileBytes];
  __shared__ float red[4][kTile];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.y;
  const int64_t qb = blockIdx.x;
  const int64_t q0 = qb * kTile;
  const int HD = H * 64;
  const uint32_t sQ = smem_addr(smem);
  const uint32_t sKV = sQ + kTileBytes;  // stage s: K at sKV + 2s*T, V at sKV + (2s+1)*T
  const int ntiles = static_cast<int>((nb + kTile - 1) / kTile);

  load_tile(sQ, q, q0, L, HD, h);
  load_tile(sKV, kc, 0, nb, HD, h);
  load_tile(sKV + kTileBytes, vc, 0, nb, HD, h);
  cp_async_commit();

  const int g = lane >> 2, tq = lane & 3;
  // lse in base-2 units per owned row; rows past the end get +inf so that their P is 0
  float lse2[2];
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int64_t row = q0 + warp * 16 + g + 8 * r;
    lse2[r] = row < L ? lse[static_cast<int64_t>(h) * L + row] * kLog2e : INFINITY;
  }

  float o[8][4];
#pragma unroll
  for (int nt = 0; nt < 8; ++nt) o[nt][0] = o[nt][1] = o[nt][2] = o[nt][3] = 0.f;
  uint32_t qf[4][4];
  float* score_row = scores + (static_cast<int64_t>(h) * nqb + qb) * nb;

  for (int t = 0; t < ntiles; ++t) {
    if (t + 1 < ntiles) {
      const uint32_t st = sKV + ((t + 1) & 1) * 2 * kTileBytes;
      load_tile(st, kc, static_cast<int64_t>(t + 1) * kTile, nb, HD, h);
      load_tile(st + kTileBytes, vc, static_cast<int64_t>(t + 1) * kTile, nb, HD, h);
      cp_async_commit();
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    if (t == 0) load_q_frags(sQ, warp, lane, qf);
    const uint32_t sK = sKV + (t & 1) * 2 * kTileBytes;
    const uint32_t sV = sK + kTileBytes;

    float s[8][4];
    qk_tile(sK, lane, qf, s);
    const int64_t col0 = static_cast<int64_t>(t) * kTile + 2 * tq;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const bool ok = col0 + nt * 8 + (c & 1) < nb;
        s[nt][c] = ok ? exp2_approx(fmaf(s[nt][c], scale_log2, -lse2[c >> 1])) : 0.f;
      }

    // column sums of the fp32 probabilities over the warp's 16 rows (recursive halving)
    float v[16];
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      v[2 * nt] = s[nt][0] + s[nt][2];
      v[2 * nt + 1] = s[nt][1] + s[nt][3];
    }
    const bool b4 = lane & 16, b3 = lane & 8, b2 = lane & 4;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float send = b4 ? v[i] : v[i + 8];
      const float keep = b4 ? v[i + 8] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float send = b3 ? v[i] : v[i + 4];
      const float keep = b3 ? v[i + 4] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
    }
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const float send = b2 ? v[i] : v[i + 2];
      const float keep = b2 ? v[i + 2] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
    }
    // lane now holds the sums of columns g*8 + 2*tq + {0, 1}
    red[warp][g * 8 + 2 * tq] = v[0];
    red[warp][g * 8 + 2 * tq + 1] = v[1];

    // O += bf16(P) * Vc
    uint32_t pa[4][4];
#pragma unroll
    for (int ks = 0; ks < 4; ++ks) {
      pa[ks][0] = pack_bf16(s[2 * ks][0], s[2 * ks][1]);
      pa[ks][1] = pack_bf16(s[2 * ks][2], s[2 * ks][3]);
      pa[ks][2] = pack_bf16(s[2 * ks + 1][0], s[2 * ks + 1][1]);
      pa[ks][3] = pack_bf16(s[2 * ks + 1][2], s[2 * ks + 1][3]);
    }
    const int mi = lane >> 3, r8 = lane & 7;
#pragma unroll
    for (int ks = 0; ks < 4; ++ks)
#pragma unroll
      for (int dp = 0; dp < 4; ++dp) {
        const int key = ks * 16 + (mi & 1) * 8 + r8;
        const int ch = 2 * dp + (mi >> 1);
        uint32_t b0, b1, b2_, b3_;
        ldsm_x4_t(sV + swz128(key, ch), b0, b1, b2_, b3_);
        mma16816(o[2 * dp], pa[ks], b0, b1);
        mma16816(o[2 * dp + 1], pa[ks], b2_, b3_);
      }

    __syncthreads();  // red[] complete; every warp is done with this K/V stage
    if (threadIdx.x < kTile) {
      const int64_t col = static_cast<int64_t>(t) * kTile + threadIdx.x;
      if (col < nb)
        score_row[col] = (red[0][threadIdx.x] + red[1][threadIdx.x]) +
                         (red[2][threadIdx.x] + red[3][threadIdx.x]);
    }
    __syncthreads();  // red[] may be rewritten by the next tile
  }

#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int64_t row = q0 + warp * 16 + g + 8 * r;
    if (row >= L) continue;
    float* dst = o_cmp + row * HD + h * 64 + 2 * tq;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
      *reinterpret_cast<float2*>(dst + nt * 8) = make_float2(o[nt][2 * r], o[nt][2 * r + 1]);
  }
}

}  // namespace

cudaError_t launch_cmp_lse(const Problem& p, const uint16_t* q, const uint16_t* kc, float* lse,
                           cudaStream_t st) {
  dim3 grid(static_cast<unsigned>(p.nqb), p.H);
  cmp_lse_kernel<<<grid, kThreads, 0, st>>>(q, kc, lse, p.L, p.H, p.nb, p.scale_log2);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_cmp_pv_score(const Problem& p, const uint16_t* q, const uint16_t* kc,
                                const uint16_t* vc, const float* lse, float* o_cmp, float* scores,
                                cudaStream_t st) {
  dim3 grid(static_cast<unsigned>(p.nqb), p.H);
  cmp_pv_score_kernel<<<grid, kThreads, 0, st>>>(q, kc, vc, lse, o_cmp, scores, p.L, p.H, p.nb,
                                                 p.nqb, p.scale_log2);
  count_launch();
  return cudaGetLastError();
}

}  // namespace s3r
