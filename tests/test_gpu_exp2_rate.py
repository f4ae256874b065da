"""The exp2 rate behind the compressed branch's secondary roofline: MUFU.EX2 per clock per SM.

The compressed branch evaluates two exponentials per (query, block summary) pair, so its speed is
set by the unit that evaluates them. bench.py states that unit's rate as 16 exp2 per clock per SM
(4 sub-partitions x 4 lanes). This test measures it on the device: one CTA per SM runs
independent chains of ex2.approx.ftz.f32 and times them with the SM's own cycle counter, so the
figure is per clock and does not depend on the clock the GPU happens to run at. The kernel is a
measurement probe compiled here with NVRTC, not part of the library.
"""
import ctypes

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

SRC = r"""
extern "C" __global__ void ex2_rate(float* out, long long* cycles, int iters) {
  extern __shared__ float pad[];  // sized so that only one CTA fits an SM
  float a[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) a[c] = -0.5f - 0.01f * c - 1e-6f * threadIdx.x;
  __syncthreads();
  const long long t0 = clock64();
  for (int i = 0; i < iters; ++i) {
#pragma unroll
    for (int c = 0; c < 8; ++c)  // a <- -2^a: bounded (fixed point near -0.64), one MUFU op each
      asm volatile("ex2.approx.ftz.f32 %0, %0;\n neg.f32 %0, %0;" : "+f"(a[c]));
  }
  __syncthreads();
  const long long t1 = clock64();
  float s = 0.f;
#pragma unroll
  for (int c = 0; c < 8; ++c) s += a[c];
  out[blockIdx.x * blockDim.x + threadIdx.x] = s + pad[0] * 0.f;
  if (threadIdx.x == 0) cycles[blockIdx.x] = t1 - t0;
}
"""


def _check(err, what):
    code = err[0] if isinstance(err, tuple) else err
    assert int(code) == 0, f"{what}: {code}"


def test_mufu_ex2_rate_is_16_per_clock_per_sm():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from cuda.bindings import driver as cu
    from cuda.bindings import nvrtc

    torch.cuda.init()
    dev = torch.device("cuda")
    torch.zeros(1, device=dev)  # the primary context is current from here on
    err, prog = nvrtc.nvrtcCreateProgram(SRC.encode(), b"ex2_rate.cu", 0, [], [])
    _check(err, "nvrtcCreateProgram")
    opts = [b"--gpu-architecture=sm_100a"]
    (err,) = nvrtc.nvrtcCompileProgram(prog, len(opts), opts)
    if int(err) != 0:
        _, n = nvrtc.nvrtcGetProgramLogSize(prog)
        log = b" " * n
        nvrtc.nvrtcGetProgramLog(prog, log)
        pytest.fail(log.decode(errors="replace"))
    err, n = nvrtc.nvrtcGetCUBINSize(prog)
    _check(err, "nvrtcGetCUBINSize")
    cubin = b" " * n
    _check(nvrtc.nvrtcGetCUBIN(prog, cubin), "nvrtcGetCUBIN")
    err, mod = cu.cuModuleLoadData(cubin)
    _check(err, "cuModuleLoadData")
    err, fn = cu.cuModuleGetFunction(mod, b"ex2_rate")
    _check(err, "cuModuleGetFunction")

    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    threads, iters = 1024, 4096
    smem = 150 * 1024  # more than half an SM's shared memory: one CTA per SM
    _check(cu.cuFuncSetAttribute(
        fn, cu.CUfunction_attribute.CU_FUNC_ATTRIBUTE_MAX_DYNAMIC_SHARED_SIZE_BYTES, smem),
        "cuFuncSetAttribute")
    out = torch.empty(sms * threads, dtype=torch.float32, device=dev)
    cycles = torch.zeros(sms, dtype=torch.int64, device=dev)
    args = [ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(cycles.data_ptr()),
            ctypes.c_int(iters)]
    argp = (ctypes.c_void_p * 3)(*[ctypes.addressof(a) for a in args])
    stream = cu.CUstream(torch.cuda.current_stream().cuda_stream)
    rates = []
    for _ in range(3):  # the first launch warms the clocks up
        _check(cu.cuLaunchKernel(fn, sms, 1, 1, threads, 1, 1, smem, stream, ctypes.addressof(argp),
                                 0), "cuLaunchKernel")
        torch.cuda.synchronize()
        c = cycles.cpu().numpy().astype(np.float64)
        rates.append(threads * iters * 8 / np.median(c))
    cu.cuModuleUnload(mod)
    assert torch.isfinite(out).all()
    rate = max(rates)
    print(f"MUFU.EX2: {rate:.2f} per clock per SM (median over {sms} SMs, best of 3 launches)")
    assert 14.4 <= rate <= 16.5, rate
