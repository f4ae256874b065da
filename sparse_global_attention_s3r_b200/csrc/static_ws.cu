// static_ws.cu -- s3r_sparse_attn_fwd_static: the whole sparse-attention path with its scratch
// memory taken from a fixed array inside this library instead of a caller-provided workspace.
//
// Some callers cannot allocate device memory: a host framework that owns all device memory
// through its own allocator and gives plugins no workspace, or a latency-critical loop that must
// not allocate once it is running. For them this entry point uses the file-scope array below,
// which exists on every GPU that loads the library and stays allocated until the process exits.
// It allocates nothing itself: no cudaMalloc, no cudaFree, no allocating library call.
#include <mutex>

#include "internal.h"
#include "s3r.h"

namespace s3r {
namespace {

// The scratch memory. In host code this name is only a host-side handle for the symbol, not a
// device address: the address on each device comes from cudaGetSymbolAddress.
static __device__ __align__(256) uint8_t g_static_workspace[S3R_STATIC_WORKSPACE_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
void* g_address[kMaxDevices] = {};  // device address of g_static_workspace, per device ordinal

// Device address of the array on the current device, looked up on first use per device (with
// that device current, as the lookup requires). Null if the lookup fails.
void* static_workspace_on_current_device() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (!g_address[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_static_workspace) != cudaSuccess) return nullptr;
    g_address[dev] = ptr;
  }
  return g_address[dev];
}

}  // namespace
}  // namespace s3r

extern "C" s3r_status s3r_sparse_attn_fwd_static(const s3r_params* params, const s3r_bf16* q,
                                                 const s3r_bf16* k, const s3r_bf16* v,
                                                 const float* gate_logits, s3r_bf16* out,
                                                 int32_t* idx_out, s3r_stream stream) {
  const size_t need = s3r::fused_workspace_bytes(params);
  if (need == 0)  // invalid sizes: report the argument error without touching the device
    return static_cast<s3r_status>(
        s3r::fused_forward(params, q, k, v, gate_logits, out, idx_out, nullptr, 0, stream));
  if (need > S3R_STATIC_WORKSPACE_BYTES) return S3R_ERR_WORKSPACE;
  // What a saving forward keeps for the backward would live in the shared array, which the
  // caller cannot hand to s3r_sparse_attn_bwd and the next call overwrites.
  if (params->flags & S3R_FLAG_SAVE_FOR_BWD) return S3R_ERR_UNSUPPORTED;
  // The array's own status word is not visible to the caller, so device-side conditions (an
  // expired bounded wait) must go to a word the caller can read.
  if (!params->dev_status) return S3R_ERR_INVALID_ARG;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return S3R_ERR_CUDA;
  if (stream) {  // the array's address is the current device's: the stream must run there
    int stream_dev = -1;
    if (cudaStreamGetDevice(stream, &stream_dev) != cudaSuccess || stream_dev != dev)
      return S3R_ERR_INVALID_ARG;
  }
  void* ws = s3r::static_workspace_on_current_device();
  if (!ws) return S3R_ERR_CUDA;
  return static_cast<s3r_status>(s3r::fused_forward(params, q, k, v, gate_logits, out, idx_out,
                                                     ws, S3R_STATIC_WORKSPACE_BYTES, stream));
}
