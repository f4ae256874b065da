// common.cuh -- small device helpers shared by the kernels of libs3r.so (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace s3r {

constexpr float kLn2 = 0.6931471805599453f;

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// two floats -> packed bf16x2 (round to nearest even); `lo` lands in the low half
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// 2^x through the hardware approximation (MUFU.EX2); 2^-inf = +0.
__device__ __forceinline__ float exp2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
  return y;
}

// 2^x for two values on the FMA pipe (no MUFU), for x < 128, at the accuracy of MUFU.EX2.
// Round-to-nearest range reduction x = n + f, f in [-1/2, 1/2] (Cody-Waite with one constant):
// adding 1.5 * 2^23 + 127 rounds x to an integer and leaves the biased exponent 127 + n in the low
// bits of the sum. A degree-5 minimax polynomial fitted for this library approximates 2^f
// (relative error 7.5e-8 in exact arithmetic, 2.1e-7 evaluated with fp32 FMAs). One multiply
// scales it by 2^n, whose bit pattern is those low bits shifted into the exponent field. x is
// clamped below at -127, where that pattern is +0: the result is +0 for x below about -126.5,
// close to where MUFU.EX2 with flush-to-zero returns 0 (x < -126).
__device__ __forceinline__ float2 exp2_poly5x2(float2 x) {
  constexpr float kMagic = 12583039.0f;  // 1.5 * 2^23 + 127
  x.x = fmaxf(x.x, -127.f);
  x.y = fmaxf(x.y, -127.f);
  const float2 t = __fadd2_rn(x, make_float2(kMagic, kMagic));
  const float2 n = __fadd2_rn(t, make_float2(-kMagic, -kMagic));
  const float2 f = __ffma2_rn(n, make_float2(-1.f, -1.f), x);
  float2 p = __ffma2_rn(make_float2(1.327647199e-03f, 1.327647199e-03f), f,
                        make_float2(9.675541334e-03f, 9.675541334e-03f));
  p = __ffma2_rn(p, f, make_float2(5.550713273e-02f, 5.550713273e-02f));
  p = __ffma2_rn(p, f, make_float2(2.402211972e-01f, 2.402211972e-01f));
  p = __ffma2_rn(p, f, make_float2(6.931469671e-01f, 6.931469671e-01f));
  p = __ffma2_rn(p, f, make_float2(1.000000072e+00f, 1.000000072e+00f));
  const float2 s = make_float2(__uint_as_float(__float_as_uint(t.x) << 23),
                               __uint_as_float(__float_as_uint(t.y) << 23));
  return __fmul2_rn(p, s);
}

// max(a, b, c) in one instruction (sm_100 three-input max)
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;\n" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

__device__ __forceinline__ void set_status(uint32_t* status, uint32_t bits) {
  if (status) atomicOr(status, bits);
}

}  // namespace s3r
