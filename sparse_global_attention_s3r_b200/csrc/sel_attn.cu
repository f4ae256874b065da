// sel_attn.cu -- selection branch: exact attention over the tokens of the top-k key blocks,
// optionally fused with the gated aggregation.
//
// Speed3R (gist.science summary, "Methodologie" §1 "Selectie-tak"): fine-grained attention only on
// the tokens selected by the compression branch's top-k; §2 "Gated Aggregation": a per-token gate
// mixes the two branch outputs (here two independent sigmoid gates, one per branch).
//
// One CTA = one 64-row query block of one head (4 warps x 16 rows). The k selected blocks form a
// list of k*b key tokens, walked in tiles of 64: each tile row is gathered from K/V [L, H, 64] with
// cp.async (16-byte chunks, zero-fill for tokens at or past L, for padding past k*b and for
// out-of-range indices, which are also masked to -inf). Logits and P*V use mma.sync m16n8k16
// (bf16 in, fp32 accumulate) with an online softmax in base-2 units. The epilogue either writes
// O_sel (fp32) or reads O_cmp and the gate logits and writes the combined output in bf16.
#include "s3r.h"
#include "common.cuh"
#include "internal.h"

namespace s3r {
namespace {

constexpr int kThreads = 128;
constexpr int kTile = 64;
constexpr int kTileBytes = kTile * 128;

struct SelArgs {
  const uint16_t* q;
  const uint16_t* k;
  const uint16_t* v;
  const int32_t* idx;
  float* o_sel;
  const float* o_cmp;
  const float* gates;
  uint16_t* out;
  int64_t L, nb, nqb;
  int H, b, topk;
  float scale_log2;
  uint32_t flags;
  uint32_t* status;
};

// Gather tile t of the selected-token list of (h, query block) into stage buffers sK/sV.
// Thread pair (2r, 2r+1) fetches key row r: 4 chunks of K and 4 of V each.
__device__ __forceinline__ void gather_tile(const SelArgs& a, const int32_t* sel, int h, int t,
                                            uint32_t sK, uint32_t sV, uint8_t* valid) {
  const int r = threadIdx.x >> 1, half = threadIdx.x & 1;
  const int64_t ntok = static_cast<int64_t>(a.topk) * a.b;
  const int64_t pos = static_cast<int64_t>(t) * kTile + r;
  bool ok = false;
  int64_t tok = 0;
  if (pos < ntok) {
    const int64_t j = __ldg(sel + pos / a.b);
    if (j >= 0 && j < a.nb) {
      tok = j * a.b + pos % a.b;
      ok = tok < a.L;
    } else if ((a.flags & S3R_FLAG_DEBUG_CHECKS) && half == 0 && pos % a.b == 0) {
      set_status(a.status, S3R_DEV_BAD_INDEX);
    }
  }
  const int HD = a.H * 64;
  const uint16_t* ks = a.k + tok * HD + h * 64;
  const uint16_t* vs = a.v + tok * HD + h * 64;
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const int ch = half * 4 + c;
    cp_async_16(sK + swz128(r, ch), ks + ch * 8, ok);
    cp_async_16(sV + swz128(r, ch), vs + ch * 8, ok);
  }
  if (half == 0) valid[r] = ok ? 1 : 0;
}

__global__ void __launch_bounds__(kThreads) sel_attn_kernel(const SelArgs a) {
  __shared__ __align__(128) uint8_t smem[5 * kTileBytes];
  __shared__ uint8_t valid[2][kTile];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.y;
  const int64_t qb = blockIdx.x;
  const int64_t q0 = qb * kTile;
  const int HD = a.H * 64;
  const uint32_t sQ = smem_addr(smem);
  const uint32_t sKV = sQ + kTileBytes;
  const int32_t* sel = a.idx + (static_cast<int64_t>(h) * a.nqb + qb) * a.topk;
  const int ntiles = static_cast<int>((static_cast<int64_t>(a.topk) * a.b + kTile - 1) / kTile);

  // Q tile (rows past L zero-filled)
#pragma unroll
  for (int c = threadIdx.x; c < kTile * 8; c += kThreads) {
    const int row = c >> 3, ch = c & 7;
    const int64_t rr = q0 + row;
    const bool ok = rr < a.L;
    cp_async_16(sQ + swz128(row, ch), a.q + (ok ? rr : 0) * HD + h * 64 + ch * 8, ok);
  }
  gather_tile(a, sel, h, 0, sKV, sKV + kTileBytes, valid[0]);
  cp_async_commit();

  const int g = lane >> 2, tq = lane & 3;
  float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.f, 0.f};
  float o[8][4];
#pragma unroll
  for (int nt = 0; nt < 8; ++nt) o[nt][0] = o[nt][1] = o[nt][2] = o[nt][3] = 0.f;
  uint32_t qf[4][4];
  const int mi = lane >> 3, r8 = lane & 7;

  for (int t = 0; t < ntiles; ++t) {
    if (t + 1 < ntiles) {
      const uint32_t st = sKV + ((t + 1) & 1) * 2 * kTileBytes;
      gather_tile(a, sel, h, t + 1, st, st + kTileBytes, valid[(t + 1) & 1]);
      cp_async_commit();
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    if (t == 0) {
#pragma unroll
      for (int ks = 0; ks < 4; ++ks) {
        const int row = warp * 16 + (mi & 1) * 8 + r8;
        ldsm_x4(sQ + swz128(row, 2 * ks + (mi >> 1)), qf[ks][0], qf[ks][1], qf[ks][2], qf[ks][3]);
      }
    }
    const uint32_t sK = sKV + (t & 1) * 2 * kTileBytes;
    const uint32_t sV = sK + kTileBytes;
    const uint8_t* vld = valid[t & 1];

    float s[8][4];
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
#pragma unroll
    for (int ks = 0; ks < 4; ++ks)
#pragma unroll
      for (int np = 0; np < 4; ++np) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4(sK + swz128(np * 16 + (mi >> 1) * 8 + r8, 2 * ks + (mi & 1)), b0, b1, b2, b3);
        mma16816(s[2 * np], qf[ks], b0, b1);
        mma16816(s[2 * np + 1], qf[ks], b2, b3);
      }

    float tmax[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const bool ok = vld[nt * 8 + 2 * tq + (c & 1)];
        s[nt][c] = ok ? s[nt][c] * a.scale_log2 : -INFINITY;
        tmax[c >> 1] = fmaxf(tmax[c >> 1], s[nt][c]);
      }
    float base[2], alpha[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      tmax[r] = fmaxf(tmax[r], __shfl_xor_sync(0xffffffffu, tmax[r], 1));
      tmax[r] = fmaxf(tmax[r], __shfl_xor_sync(0xffffffffu, tmax[r], 2));
      const float mn = fmaxf(m[r], tmax[r]);
      base[r] = mn == -INFINITY ? 0.f : mn;  // nothing valid yet: keep every weight at 0
      alpha[r] = exp2_approx(m[r] - base[r]);
      m[r] = mn;
      l[r] *= alpha[r];
    }
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        s[nt][c] = exp2_approx(s[nt][c] - base[c >> 1]);
        l[c >> 1] += s[nt][c];
        o[nt][c] *= alpha[c >> 1];
      }

    uint32_t pa[4][4];
#pragma unroll
    for (int ks = 0; ks < 4; ++ks) {
      pa[ks][0] = pack_bf16(s[2 * ks][0], s[2 * ks][1]);
      pa[ks][1] = pack_bf16(s[2 * ks][2], s[2 * ks][3]);
      pa[ks][2] = pack_bf16(s[2 * ks + 1][0], s[2 * ks + 1][1]);
      pa[ks][3] = pack_bf16(s[2 * ks + 1][2], s[2 * ks + 1][3]);
    }
#pragma unroll
    for (int ks = 0; ks < 4; ++ks)
#pragma unroll
      for (int dp = 0; dp < 4; ++dp) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(sV + swz128(ks * 16 + (mi & 1) * 8 + r8, 2 * dp + (mi >> 1)), b0, b1, b2, b3);
        mma16816(o[2 * dp], pa[ks], b0, b1);
        mma16816(o[2 * dp + 1], pa[ks], b2, b3);
      }
    __syncthreads();  // this stage may be overwritten by the next prefetch
  }

#pragma unroll
  for (int r = 0; r < 2; ++r) {
    l[r] += __shfl_xor_sync(0xffffffffu, l[r], 1);
    l[r] += __shfl_xor_sync(0xffffffffu, l[r], 2);
    const int64_t row = q0 + warp * 16 + g + 8 * r;
    if (row >= a.L) continue;
    const float inv = l[r] > 0.f ? 1.f / l[r] : 0.f;
    const int64_t at = row * HD + h * 64 + 2 * tq;
    if (a.o_sel) {
#pragma unroll
      for (int nt = 0; nt < 8; ++nt)
        *reinterpret_cast<float2*>(a.o_sel + at + nt * 8) =
            make_float2(o[nt][2 * r] * inv, o[nt][2 * r + 1] * inv);
    } else {
      const float2 gl = *reinterpret_cast<const float2*>(a.gates + (row * a.H + h) * 2);
      const float gc = 1.f / (1.f + expf(-gl.x));
      const float gs = 1.f / (1.f + expf(-gl.y));
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        const float2 oc = *reinterpret_cast<const float2*>(a.o_cmp + at + nt * 8);
        const float x0 = gc * oc.x + gs * (o[nt][2 * r] * inv);
        const float x1 = gc * oc.y + gs * (o[nt][2 * r + 1] * inv);
        *reinterpret_cast<uint32_t*>(a.out + at + nt * 8) = pack_bf16(x0, x1);
      }
    }
  }
}

}  // namespace

cudaError_t launch_sel_attn(const Problem& p, const uint16_t* q, const uint16_t* k,
                            const uint16_t* v, const int32_t* idx, float* o_sel,
                            const float* o_cmp, const float* gates, uint16_t* out,
                            cudaStream_t st) {
  SelArgs a{q, k, v, idx, o_sel, o_cmp, gates, out, p.L, p.nb, p.nqb, p.H, p.b, p.k,
            p.scale_log2, p.flags, p.status};
  dim3 grid(static_cast<unsigned>(p.nqb), p.H);
  sel_attn_kernel<<<grid, kThreads, 0, st>>>(a);
  count_launch();
  return cudaGetLastError();
}

}  // namespace s3r
