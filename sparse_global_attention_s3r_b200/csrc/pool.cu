// pool.cu -- compression branch, block mean pooling of K and V.
//
// Speed3R (gist.science summary, "Methodologie" §1 "Compressie-tak"): the compression branch
// downsamples the tokens by average pooling. Blocks are b consecutive tokens of the flattened
// sequence; the last block holds only its valid tokens and is divided by their count.
//
// HBM-streaming kernel: one thread owns one 16-byte column chunk (8 bf16) of a [L, H*d] row and
// walks the b rows of its block, so a warp reads 512 contiguous bytes per row and the block's
// whole [b, H*d] slab is read exactly once. fp32 accumulation, one IEEE division by the valid
// count, round-to-nearest-even to bf16. Algorithmic traffic: 2 * (L + nb) * H * d * 2 bytes.
// Optionally the same pass also writes head-major copies Kh, Vh [H, nb*b, 64] of K and V (rows
// past L zero), so that the selection branch can gather a selected block of one head as b
// contiguous 128-byte rows rather than rows H*128 bytes apart; that adds 2 * nb*b * H*d * 2 bytes
// of writes.
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

__global__ void __launch_bounds__(kPoolThreads)
    pool_kv_kernel(const uint16_t* __restrict__ k, const uint16_t* __restrict__ v,
                   uint16_t* __restrict__ kc, uint16_t* __restrict__ vc,
                   uint16_t* __restrict__ kh, uint16_t* __restrict__ vh, int64_t L, int64_t Lp,
                   int HD, int b) {
  const uint16_t* src = blockIdx.z ? v : k;
  uint16_t* dst = blockIdx.z ? vc : kc;
  uint16_t* hm = blockIdx.z ? vh : kh;  // head-major copy [H, Lp, 64] or null
  const int chunk = blockIdx.x * kPoolThreads + threadIdx.x;  // 16-byte chunk within a row
  const int chunks = HD / 8;
  if (chunk >= chunks) return;
  const int64_t j = blockIdx.y;
  const int64_t t0 = j * b;
  const int n = static_cast<int>(min(static_cast<int64_t>(b), L - t0));
  const uint4* p = reinterpret_cast<const uint4*>(src + t0 * HD) + chunk;
  // head chunk >> 3, 16-byte piece chunk & 7 of its 128-byte row; rows are 8 uint4 apart
  uint4* hp = hm ? reinterpret_cast<uint4*>(hm + ((chunk >> 3) * Lp + t0) * 64) + (chunk & 7)
                 : nullptr;

  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
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
    for (; t < b; ++t) hp[t * 8] = make_uint4(0u, 0u, 0u, 0u);  // padding rows of the last block

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
  pool_kv_kernel<<<grid, kPoolThreads, 0, st>>>(k, v, kc, vc, kh, vh, p.L, p.nb * p.b, HD, p.b);
  count_launch();
  return cudaGetLastError();
}

}  // namespace s3r
