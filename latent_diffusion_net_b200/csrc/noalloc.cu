// sd_time_embed_noalloc: the time-embedding MLP without a caller workspace.
//
// Some callers cannot hand this library a workspace: code running where
// allocating device memory is forbidden or unsafe, such as the enqueue step of a
// plugin inside another inference engine (which owns every allocation and
// forbids its plugins from calling cudaMalloc), or a latency-critical loop where
// cudaMalloc/cudaFree would synchronise the device. For them this entry point
// keeps its intermediate vectors (the sinusoid phi(t) and the hidden layer) in
// a fixed file-scope device array instead of a workspace. The caller still
// passes the packed weights and the output buffer.
//
// The array holds kNoAllocMaxDim floats for phi and kNoAllocMaxDim for the
// hidden layer (32 KiB); every GPU that loads this library keeps it resident
// until the process exits. Both vectors are fully rewritten by every call before
// they are read, so nothing has to be cleared between calls.
#include <cuda_runtime.h>
#include <string.h>

#include <mutex>

#include "kernels.cuh"
#include "sd_api.h"

namespace {

constexpr int kNoAllocMaxDim = 4096;
constexpr int kMaxDevices = 64;

// File-scope scratch: [0, kNoAllocMaxDim) = phi(t), [kNoAllocMaxDim, 2*kNoAllocMaxDim) = hidden.
static __device__ __align__(256) float g_time_scratch[2 * kNoAllocMaxDim];

std::mutex g_mu;
float* g_scratch_ptr[kMaxDevices];

// Device address of g_time_scratch on the current device. In host code the
// symbol name is only a host-side stand-in, so the address is looked up once per
// device with that device current.
sd_status scratch_ptr(float** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SD_ERR_LAUNCH;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_time_scratch) != cudaSuccess || !p) {
      (void)cudaGetLastError();
      return SD_ERR_LAUNCH;
    }
    g_scratch_ptr[dev] = static_cast<float*>(p);
  }
  *out = g_scratch_ptr[dev];
  return SD_OK;
}

// Byte offsets of the four tensors in the packed time-MLP buffer: each tensor
// starts on a 256-byte boundary, in table order (lin1.weight, lin1.bias,
// lin2.weight, lin2.bias).
inline int64_t align256(int64_t x) { return (x + 255) & ~int64_t(255); }

}  // namespace

extern "C" sd_status sd_time_embed_noalloc(const sd_time_cfg* cfg, const void* packed_w, float timestep,
                                           float* temb_out, sd_stream_t stream) {
  if (!cfg) return SD_ERR_NULL_ARG;
  if (cfg->proj_dim <= 0 || cfg->proj_dim % 16 || cfg->temb_dim <= 0 || cfg->temb_dim % 8) return SD_ERR_BAD_SHAPE;
  if (cfg->proj_dim > kNoAllocMaxDim || cfg->temb_dim > kNoAllocMaxDim) return SD_ERR_UNSUPPORTED;
  if (!packed_w || !temb_out) return SD_ERR_NULL_ARG;
  if ((reinterpret_cast<uintptr_t>(packed_w) & 15) || (reinterpret_cast<uintptr_t>(temb_out) & 15))
    return SD_ERR_MISALIGNED;
  int dev = 0, major = 0, minor = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SD_ERR_LAUNCH;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
    return SD_ERR_LAUNCH;
  if (major != 10 || minor != 0) return SD_ERR_NOT_SM100;
  float* scratch = nullptr;
  sd_status s = scratch_ptr(&scratch);
  if (s != SD_OK) return s;
  float* phi = scratch;
  float* hid = scratch + kNoAllocMaxDim;

  const int P = cfg->proj_dim, T = cfg->temb_dim;
  const uint8_t* base = static_cast<const uint8_t*>(packed_w);
  const int64_t l1w = 0;
  const int64_t l1b = align256(l1w + (int64_t)T * P * 2);
  const int64_t l2w = align256(l1b + (int64_t)T * 2);
  const int64_t l2b = align256(l2w + (int64_t)T * T * 2);
  cudaStream_t st = static_cast<cudaStream_t>(stream);

  if (sdk::launch_sinusoid(timestep, P, phi, st) != 0) return SD_ERR_LAUNCH;
  sdk::GemvBatch b;
  memset(&b, 0, sizeof(b));
  b.njobs = 1;
  b.K = P;
  b.silu_out = 1;
  b.x = phi;
  b.job[0] = {reinterpret_cast<const __nv_bfloat16*>(base + l1w), reinterpret_cast<const __nv_bfloat16*>(base + l1b),
              hid, T};
  if (sdk::launch_gemv(b, st) != 0) return SD_ERR_LAUNCH;
  b.K = T;
  b.silu_out = 0;
  b.x = hid;
  b.job[0] = {reinterpret_cast<const __nv_bfloat16*>(base + l2w), reinterpret_cast<const __nv_bfloat16*>(base + l2b),
              temb_out, T};
  if (sdk::launch_gemv(b, st) != 0) return SD_ERR_LAUNCH;
  return SD_OK;
}
