// pool.cu -- compression branch, block mean pooling of K and V.
//
// Speed3R (gist.science summary, "Methodologie" §1 "Compressie-tak"): the compression branch
// downsamples the tokens by average pooling. Blocks are b consecutive tokens of the flattened
// sequence; the last block holds only its valid tokens and is divided by their count.
//
// HBM-streaming kernel: one thread owns one 16-byte column chunk (8 bf16) of a [L, H*d] row and
// walks the b token rows of its block, so a warp reads 512 contiguous bytes per row and every
// token row is read exactly once. Blocks follow the block <-> token map of geometry.cuh (1-D runs,
// or 2-D windows of a view's patch grid and the view's special tokens). fp32 accumulation, one IEEE division by the valid
// count, round-to-nearest-even to bf16. Algorithmic traffic: 2 * (L + nb) * H * d * 2 bytes.
// Optionally the same pass also writes head-major copies Kh, Vh [H, nb*b, 64] of K and V in slot
// order (slot o of block j at row j*b + o; slots without a token are zero), so that the selection
// branch can gather a selected block of one head as b contiguous 128-byte rows rather than rows
// H*128 bytes apart; that adds 2 * nb*b * H*d * 2 bytes of writes.
#include "common.cuh"
#include "internal.h"

namespace s3r {
namespace {

constexpr int kPoolThreads = 128;

__device__ __forceinline__ void add_bf16x8(float acc[8], const uint4& x) {
  const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    acc[2 * e] += __uint_as_float(w[e] << 16);
    acc[2 * e + 1] += __uint_as_float(w[e] & 0xFFFF0000u);
  }
}

// Sum the n rows of a contiguous run of tokens (row t at p + t*chunks) into acc, copying each to
// the head-major row t (hp + t*8, if hp) and zeroing the copy's rows n .. b-1.
__device__ __forceinline__ void pool_run(const uint4* p, int chunks, int n, int b, uint4* hp,
                                         float (&acc)[8]) {
  int t = 0;
  for (; t + 8 <= n; t += 8) {  // 8 independent 16-byte loads in flight per thread
    uint4 x[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) x[u] = __ldg(p + static_cast<int64_t>(t + u) * chunks);
    if (hp) {
#pragma unroll
      for (int u = 0; u < 8; ++u) hp[(t + u) * 8] = x[u];
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) add_bf16x8(acc, x[u]);
  }
  for (; t < n; ++t) {
    const uint4 x = __ldg(p + static_cast<int64_t>(t) * chunks);
    if (hp) hp[t * 8] = x;
    add_bf16x8(acc, x);
  }
  if (hp)
    for (; t < b; ++t) hp[t * 8] = make_uint4(0u, 0u, 0u, 0u);  // slots past L
}

__global__ void __launch_bounds__(kPoolThreads)
    pool_kv_kernel(const uint16_t* __restrict__ k, const uint16_t* __restrict__ v,
                   uint16_t* __restrict__ kc, uint16_t* __restrict__ vc,
                   uint16_t* __restrict__ kh, uint16_t* __restrict__ vh, const BlockGeo g,
                   int64_t Lp, int HD) {
  const uint16_t* src = blockIdx.z ? v : k;
  uint16_t* dst = blockIdx.z ? vc : kc;
  uint16_t* hm = blockIdx.z ? vh : kh;  // head-major copy [H, Lp, 64] or null
  const int chunk = blockIdx.x * kPoolThreads + threadIdx.x;  // 16-byte chunk within a row
  const int chunks = HD / 8;
  if (chunk >= chunks) return;
  const int64_t j = blockIdx.y;
  const int b = g.b;
  const BlockOrigin bo = block_origin(g, j);
  // head chunk >> 3, 16-byte piece chunk & 7 of its 128-byte row; rows are 8 uint4 apart
  uint4* hp = hm ? reinterpret_cast<uint4*>(hm + ((chunk >> 3) * Lp + j * b) * 64) + (chunk & 7)
                 : nullptr;
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  int n = 0;  // tokens in the block
  if (bo.kind == 0) {
    n = static_cast<int>(min(static_cast<int64_t>(b), g.L - bo.first));
    pool_run(reinterpret_cast<const uint4*>(src + bo.first * HD) + chunk, chunks, n, b, hp, acc);
  } else {  // a window or a view's special tokens: token of each slot from the geometry
    const uint4* p = reinterpret_cast<const uint4*>(src) + chunk;
    for (int o0 = 0; o0 < b; o0 += 8) {
      int64_t tok[8];
      uint4 x[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) tok[u] = origin_token(g, bo, o0 + u);
#pragma unroll
      for (int u = 0; u < 8; ++u)
        x[u] = tok[u] >= 0 ? __ldg(p + tok[u] * chunks) : make_uint4(0u, 0u, 0u, 0u);
      if (hp) {
#pragma unroll
        for (int u = 0; u < 8; ++u) hp[(o0 + u) * 8] = x[u];
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        add_bf16x8(acc, x[u]);  // a slot without a token adds zeros
        n += tok[u] >= 0;
      }
    }
  }

  const float fn = static_cast<float>(n);
  uint4 o;
  o.x = pack_bf16(acc[0] / fn, acc[1] / fn);
  o.y = pack_bf16(acc[2] / fn, acc[3] / fn);
  o.z = pack_bf16(acc[4] / fn, acc[5] / fn);
  o.w = pack_bf16(acc[6] / fn, acc[7] / fn);
  reinterpret_cast<uint4*>(dst + j * HD)[chunk] = o;
}

}  // namespace

cudaError_t launch_pool_kv(const Problem& p, const uint16_t* k, const uint16_t* v, uint16_t* kc,
                           uint16_t* vc, uint16_t* kh, uint16_t* vh, cudaStream_t st) {
  const int HD = p.H * p.d;
  dim3 grid((HD / 8 + kPoolThreads - 1) / kPoolThreads, static_cast<unsigned>(p.nb), 2);
  pool_kv_kernel<<<grid, kPoolThreads, 0, st>>>(k, v, kc, vc, kh, vh, p.geo, p.nb * p.b, HD);
  count_launch();
  return cudaGetLastError();
}

}  // namespace s3r
