// combine.cu -- gated aggregation of the two branch outputs.
//
// Speed3R (gist.science summary, "Methodologie" §2 "Gated Aggregation"): the outputs of the
// compression and selection branches are merged by a learned per-token gate. The gate logits are
// inputs here, two per (token, head): out = sigmoid(g0) * O_cmp + sigmoid(g1) * O_sel.
//
// Elementwise, HBM-bound: each thread reads 8 fp32 of each branch (2 x 16-byte loads each) and the
// two logits of its (token, head), and writes 8 bf16 (one 16-byte store).
// Algorithmic traffic: L*H*d*(4 + 4 + 2) + L*H*2*4 bytes.
#include "common.cuh"
#include "internal.h"

namespace s3r {
namespace {

constexpr int kThreads = 256;

__global__ void __launch_bounds__(kThreads)
    gate_combine_kernel(const float* __restrict__ o_cmp, const float* __restrict__ o_sel,
                        const float* __restrict__ gates, uint16_t* __restrict__ out,
                        int64_t groups) {
  const int64_t gi = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x;  // 8 elements
  if (gi >= groups) return;
  const int64_t rh = gi >> 3;  // (token, head) pair: 64 elements = 8 groups
  const float2 gl = __ldg(reinterpret_cast<const float2*>(gates) + rh);
  const float gc = 1.f / (1.f + expf(-gl.x));
  const float gs = 1.f / (1.f + expf(-gl.y));
  const float4* pc = reinterpret_cast<const float4*>(o_cmp) + gi * 2;
  const float4* ps = reinterpret_cast<const float4*>(o_sel) + gi * 2;
  const float4 c0 = __ldg(pc), c1 = __ldg(pc + 1), s0 = __ldg(ps), s1 = __ldg(ps + 1);
  uint4 o;
  o.x = pack_bf16(gc * c0.x + gs * s0.x, gc * c0.y + gs * s0.y);
  o.y = pack_bf16(gc * c0.z + gs * s0.z, gc * c0.w + gs * s0.w);
  o.z = pack_bf16(gc * c1.x + gs * s1.x, gc * c1.y + gs * s1.y);
  o.w = pack_bf16(gc * c1.z + gs * s1.z, gc * c1.w + gs * s1.w);
  reinterpret_cast<uint4*>(out)[gi] = o;
}

}  // namespace

cudaError_t launch_gate_combine(const Problem& p, const float* o_cmp, const float* o_sel,
                                const float* gates, uint16_t* out, cudaStream_t st) {
  const int64_t groups = p.L * p.H * (p.d / 8);
  const int64_t blocks = (groups + kThreads - 1) / kThreads;
  gate_combine_kernel<<<static_cast<unsigned>(blocks), kThreads, 0, st>>>(o_cmp, o_sel, gates, out,
                                                                         groups);
  count_launch();
  return cudaGetLastError();
}

}  // namespace s3r
