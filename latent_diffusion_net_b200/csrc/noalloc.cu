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

#include "kernels.cuh"
#include "profile.h"
#include "sd_api.h"
#include "weights.h"

namespace {

constexpr int kNoAllocMaxDim = 4096;

// File-scope scratch: [0, kNoAllocMaxDim) = phi(t), [kNoAllocMaxDim, 2*kNoAllocMaxDim) = hidden.
static __device__ __align__(256) float g_time_scratch[2 * kNoAllocMaxDim];

// Device address of g_time_scratch on the current device. In host code the
// symbol name is only a host-side stand-in, so the address is asked for with
// the device current, on every call: the query is a host call that allocates
// nothing, and a fresh answer stays right after a device reset reloads the module.
sd_status scratch_ptr(float** out) {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_time_scratch) != cudaSuccess || !p) {
    (void)cudaGetLastError();
    return SD_ERR_LAUNCH;
  }
  *out = static_cast<float*>(p);
  return SD_OK;
}

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
  // packed offsets from the same weight table sd_time_embed uses (host only)
  sdw::Table tab;
  const sdw::TimeW tw = sdw::add_time(tab, "time", P, T);
  const int64_t l1w = tw.l1w, l1b = tw.l1b, l2w = tw.l2w, l2b = tw.l2b;
  cudaStream_t st = static_cast<cudaStream_t>(stream);

  {
    sdp::Scope sc("sinusoid", sdp::F_OTHER, 0, 4.0 * P, st);
    if (sdk::launch_sinusoid(timestep, P, phi, st) != 0) return SD_ERR_LAUNCH;
  }
  sdk::GemvBatch b;
  memset(&b, 0, sizeof(b));
  b.njobs = 1;
  b.K = P;
  b.silu_out = 1;
  b.x = phi;
  b.job[0] = {reinterpret_cast<const __nv_bfloat16*>(base + l1w), reinterpret_cast<const __nv_bfloat16*>(base + l1b),
              hid, T};
  {
    sdp::Scope sc("gemv", sdp::F_GEMV, 2.0 * T * P, 2.0 * T * P, st);
    if (sdk::launch_gemv(b, st) != 0) return SD_ERR_LAUNCH;
  }
  b.K = T;
  b.silu_out = 0;
  b.x = hid;
  b.job[0] = {reinterpret_cast<const __nv_bfloat16*>(base + l2w), reinterpret_cast<const __nv_bfloat16*>(base + l2b),
              temb_out, T};
  {
    sdp::Scope sc("gemv", sdp::F_GEMV, 2.0 * T * T, 2.0 * T * T, st);
    if (sdk::launch_gemv(b, st) != 0) return SD_ERR_LAUNCH;
  }
  return SD_OK;
}
