// Normalisation kernels, HBM-bound, 16-byte vector loads.
//
// GroupNorm (GSC unit; ResnetBlock2D and Transformer2DModel panels, section 4 of
// the SD2.1 page): 32 groups of C/32 consecutive channels, statistics over
// (C/32) x H x W, biased variance, then scale/shift and optionally SiLU. The
// input may be the channel concatenation of two NHWC tensors (skip connections
// of the up path) and is never materialised: a vector of 8 channels is read
// from whichever source holds it.
//
// The transformer's LayerNorms are folded into the GEMMs they feed (gemm_tc.cu
// row statistics), so no LayerNorm kernel exists.
#include "common.cuh"
#include "kernels.cuh"

namespace sdk {

// ------------------------------------------------------------------ GroupNorm (+SiLU)
// Two kernels, both fully parallel (no CTA waits for another):
//   gn_stats: each CTA sums x and x^2 per group over a contiguous pixel range
//     in FP32 and adds the sums to per-group accumulators as 64-bit fixed-point
//     integers (x scaled by 2^24, x^2 by 2^18). Integer addition is associative,
//     so the totals do not depend on the order in which CTAs arrive.
//   gn_apply: every CTA turns the accumulators into mean and rstd (FP64), folds
//     them with gamma/beta into a per-channel scale and shift, and normalises
//     (+SiLU) a grid-stride share of the tensor.
constexpr double kSumScale = 16777216.0;  // 2^24
constexpr double kSqScale = 262144.0;     // 2^18

__device__ __forceinline__ long long to_fixed(float v, double scale) {
  double d = (double)v * scale;
  d = fmin(fmax(d, -4.0e18), 4.0e18);
  return __double2ll_rn(d);
}

__global__ void gn_stats_kernel(const __nv_bfloat16* __restrict__ x0, int C0, const __nv_bfloat16* __restrict__ x1,
                                int C1, int HW, int G, int ppi, unsigned long long* __restrict__ acc) {
  extern __shared__ float4 red[];  // [blockDim.x]
  pdl_wait();
  pdl_trigger();
  const int C = C0 + C1;
  const int V = C >> 3;
  const int cpg = C / G;
  const int t = threadIdx.x;
  const int v = t % V;
  const int pi = t / V;
  const int c = v * 8;
  const int ga = c / cpg;
  const int split = (ga + 1) * cpg - c;  // channels c .. c+split-1 belong to ga, the rest to ga+1
  const int chunk = (HW + gridDim.x - 1) / gridDim.x;
  const int p0 = blockIdx.x * chunk;
  const int p1 = min(HW, p0 + chunk);
  const __nv_bfloat16* base;
  int ld;
  if (c < C0) {
    base = x0 + c;
    ld = C0;
  } else {
    base = x1 + (c - C0);
    ld = C1;
  }
  float sa = 0.f, qa = 0.f, sb = 0.f, qb = 0.f;
  auto accum = [&](const uint4 w) {
    const float f[8] = {bf16lo(w.x), bf16hi(w.x), bf16lo(w.y), bf16hi(w.y),
                        bf16lo(w.z), bf16hi(w.z), bf16lo(w.w), bf16hi(w.w)};
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (j < split) {
        sa += f[j];
        qa = fmaf(f[j], f[j], qa);
      } else {
        sb += f[j];
        qb = fmaf(f[j], f[j], qb);
      }
    }
  };
  if (pi < ppi) {
    int p = p0 + pi;
    for (; p + 3 * ppi < p1; p += 4 * ppi) {
      const uint4 w0 = __ldg(reinterpret_cast<const uint4*>(base + (size_t)p * ld));
      const uint4 w1 = __ldg(reinterpret_cast<const uint4*>(base + (size_t)(p + ppi) * ld));
      const uint4 w2 = __ldg(reinterpret_cast<const uint4*>(base + (size_t)(p + 2 * ppi) * ld));
      const uint4 w3 = __ldg(reinterpret_cast<const uint4*>(base + (size_t)(p + 3 * ppi) * ld));
      accum(w0);
      accum(w1);
      accum(w2);
      accum(w3);
    }
    for (; p < p1; p += ppi) accum(__ldg(reinterpret_cast<const uint4*>(base + (size_t)p * ld)));
  }
  red[t] = make_float4(sa, qa, sb, qb);
  __syncthreads();
  if (t < G) {
    const int g = t;
    const int vlo = (g * cpg) / 8;
    const int vhi = min(V - 1, ((g + 1) * cpg - 1) / 8);
    float s = 0.f, q = 0.f;
    for (int pp = 0; pp < ppi; ++pp) {
      for (int vv = vlo; vv <= vhi; ++vv) {
        const float4 r = red[pp * V + vv];
        if ((vv * 8) / cpg == g) {
          s += r.x;
          q += r.y;
        } else {
          s += r.z;
          q += r.w;
        }
      }
    }
    atomicAdd(&acc[2 * g], (unsigned long long)to_fixed(s, kSumScale));
    atomicAdd(&acc[2 * g + 1], (unsigned long long)to_fixed(q, kSqScale));
  }
}

__global__ void gn_apply_kernel(const __nv_bfloat16* __restrict__ x0, int C0, const __nv_bfloat16* __restrict__ x1,
                                int C1, int HW, int G, float eps, const unsigned long long* __restrict__ acc,
                                const __nv_bfloat16* __restrict__ gamma, const __nv_bfloat16* __restrict__ beta,
                                int silu, __nv_bfloat16* __restrict__ y) {
  extern __shared__ float2 ab[];  // [C] scale, shift
  __shared__ float2 gstat[64];
  pdl_wait();
  pdl_trigger();
  const int C = C0 + C1;
  const int cpg = C / G;
  if (threadIdx.x < G) {
    const double cnt = (double)HW * cpg;
    const double mean = (double)(long long)acc[2 * threadIdx.x] / kSumScale / cnt;
    double var = (double)(long long)acc[2 * threadIdx.x + 1] / kSqScale / cnt - mean * mean;
    if (var < 0.0) var = 0.0;
    gstat[threadIdx.x] = make_float2((float)mean, (float)(1.0 / sqrt(var + (double)eps)));
  }
  __syncthreads();
  for (int c = threadIdx.x; c < C; c += blockDim.x) {
    const float2 st = gstat[c / cpg];
    const float a = st.y * __bfloat162float(gamma[c]);
    ab[c] = make_float2(a, __bfloat162float(beta[c]) - st.x * a);
  }
  __syncthreads();
  const int V = C >> 3;
  const size_t total = (size_t)HW * V;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < total; i += (size_t)gridDim.x * blockDim.x) {
    const int p = (int)(i / V);
    const int c = (int)(i % V) * 8;
    const __nv_bfloat16* src = (c < C0) ? (x0 + (size_t)p * C0 + c) : (x1 + (size_t)p * C1 + (c - C0));
    const uint4 w = *reinterpret_cast<const uint4*>(src);
    float f[8] = {bf16lo(w.x), bf16hi(w.x), bf16lo(w.y), bf16hi(w.y),
                  bf16lo(w.z), bf16hi(w.z), bf16lo(w.w), bf16hi(w.w)};
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float2 s = ab[c + j];
      float o = fmaf(f[j], s.x, s.y);
      if (silu) o = __fdividef(o, 1.0f + __expf(-o));
      f[j] = o;
    }
    *reinterpret_cast<uint4*>(y + (size_t)p * C + c) =
        make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]), pack_bf16x2(f[4], f[5]), pack_bf16x2(f[6], f[7]));
  }
}

// Single-pass GroupNorm: every CTA copies its contiguous pixel range of [x0 | x1]
// into shared memory while summing it (the statistics of gn_stats_kernel, same
// fixed-point accumulators), then all CTAs meet at a grid-wide barrier (an
// arrival counter polled with a bounded wait), read the final sums and
// normalise their shared-memory copy. The tensor is read once and written once,
// in one launch. The grid never exceeds the CTAs that can be resident at once:
// each CTA waits in griddepcontrol.wait for the previous kernel, which then
// leaves the whole GPU to this grid, and this kernel lets its dependents launch
// only after the barrier, so every CTA is resident before any waits on the others.
__global__ void gn_fused_kernel(const __nv_bfloat16* __restrict__ x0, int C0, const __nv_bfloat16* __restrict__ x1,
                                int C1, int HW, int G, int ppi, float eps, const __nv_bfloat16* __restrict__ gamma,
                                const __nv_bfloat16* __restrict__ beta, int silu, __nv_bfloat16* __restrict__ y,
                                unsigned long long* __restrict__ acc, unsigned int* counter, int* err) {
  extern __shared__ __align__(16) uint8_t gsm[];
  __shared__ float2 gstat[64];
  __shared__ int give_up;
  const int C = C0 + C1;
  const int V = C >> 3;
  const int cpg = C / G;
  const int t = threadIdx.x;
  const int v = t % V;
  const int pi = t / V;
  const int c = v * 8;
  const int chunk = (HW + gridDim.x - 1) / gridDim.x;
  const int p0 = blockIdx.x * chunk;
  const int p1 = min(HW, p0 + chunk);
  float4* red = reinterpret_cast<float4*>(gsm);                                   // [blockDim.x]
  uint4* slice = reinterpret_cast<uint4*>(gsm + (size_t)blockDim.x * sizeof(float4));  // [chunk][V]
  pdl_wait();
  const int ga = c / cpg;
  const int split = (ga + 1) * cpg - c;  // channels c .. c+split-1 belong to ga, the rest to ga+1
  const __nv_bfloat16* base;
  int ld;
  if (c < C0) {
    base = x0 + c;
    ld = C0;
  } else {
    base = x1 + (c - C0);
    ld = C1;
  }
  float sa = 0.f, qa = 0.f, sb = 0.f, qb = 0.f;
  auto accum = [&](const uint4 w) {
    const float f[8] = {bf16lo(w.x), bf16hi(w.x), bf16lo(w.y), bf16hi(w.y),
                        bf16lo(w.z), bf16hi(w.z), bf16lo(w.w), bf16hi(w.w)};
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (j < split) {
        sa += f[j];
        qa = fmaf(f[j], f[j], qa);
      } else {
        sb += f[j];
        qb = fmaf(f[j], f[j], qb);
      }
    }
  };
  if (pi < ppi) {
    // four independent loads in flight per thread before any is used
    int p = p0 + pi;
    for (; p + 3 * ppi < p1; p += 4 * ppi) {
      uint4 w[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) w[u] = __ldcg(reinterpret_cast<const uint4*>(base + (size_t)(p + u * ppi) * ld));
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        slice[(size_t)(p + u * ppi - p0) * V + v] = w[u];
        accum(w[u]);
      }
    }
    for (; p < p1; p += ppi) {
      const uint4 w = __ldcg(reinterpret_cast<const uint4*>(base + (size_t)p * ld));
      slice[(size_t)(p - p0) * V + v] = w;
      accum(w);
    }
  }
  red[t] = make_float4(sa, qa, sb, qb);
  if (t == 0) give_up = 0;
  __syncthreads();
  if (t < G) {
    const int g = t;
    const int vlo = (g * cpg) / 8;
    const int vhi = min(V - 1, ((g + 1) * cpg - 1) / 8);
    float s = 0.f, q = 0.f;
    for (int pp = 0; pp < ppi; ++pp) {
      for (int vv = vlo; vv <= vhi; ++vv) {
        const float4 r = red[pp * V + vv];
        if ((vv * 8) / cpg == g) {
          s += r.x;
          q += r.y;
        } else {
          s += r.z;
          q += r.w;
        }
      }
    }
    atomicAdd(&acc[2 * g], (unsigned long long)to_fixed(s, kSumScale));
    atomicAdd(&acc[2 * g + 1], (unsigned long long)to_fixed(q, kSqScale));
  }
  __syncthreads();
  if (t == 0) {
    // grid-wide barrier: the statistics of every CTA are in acc once all have arrived
    __threadfence();
    atomicAdd(counter, 1u);
    uint32_t n = 0;
    unsigned int seen;
    do {
      asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(seen) : "l"(counter) : "memory");
      if (seen >= gridDim.x) break;
      __nanosleep(64);
    } while (++n < kSpinLimit);
    if (seen < gridDim.x) {
      give_up = 1;
      atomicOr(err, ERR_MBAR_TIMEOUT);
    }
  }
  __syncthreads();
  pdl_trigger();
  if (give_up) return;
  if (t < G) {
    const double cnt = (double)HW * cpg;
    const double mean = (double)(long long)__ldcg(&acc[2 * t]) / kSumScale / cnt;
    double var = (double)(long long)__ldcg(&acc[2 * t + 1]) / kSqScale / cnt - mean * mean;
    if (var < 0.0) var = 0.0;
    gstat[t] = make_float2((float)mean, (float)(1.0 / sqrt(var + (double)eps)));
  }
  __syncthreads();
  if (pi >= ppi) return;
  float a[8], b[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const float2 stt = gstat[(c + j) / cpg];
    a[j] = stt.y * __bfloat162float(gamma[c + j]);
    b[j] = __bfloat162float(beta[c + j]) - stt.x * a[j];
  }
  for (int p = p0 + pi; p < p1; p += ppi) {
    const uint4 w = slice[(size_t)(p - p0) * V + v];
    float f[8] = {bf16lo(w.x), bf16hi(w.x), bf16lo(w.y), bf16hi(w.y),
                  bf16lo(w.z), bf16hi(w.z), bf16lo(w.w), bf16hi(w.w)};
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      float o = fmaf(f[j], a[j], b[j]);
      if (silu) o = __fdividef(o, 1.0f + __expf(-o));
      f[j] = o;
    }
    *reinterpret_cast<uint4*>(y + (size_t)p * C + c) =
        make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]), pack_bf16x2(f[4], f[5]), pack_bf16x2(f[6], f[7]));
  }
}

constexpr int kFusedSmemLimit = 200 * 1024;

// Pixels handled side by side by one CTA of the single-pass kernel: as many as
// keep the CTA at most 1024 threads, so that each SM has many loads in flight.
static int fused_ppi(int V) { return V >= 1024 ? 1 : 1024 / V; }

static size_t fused_smem(int C, int HW, int num_sms) {
  const int V = C / 8;
  const int chunk = (HW + num_sms - 1) / num_sms;
  return (size_t)V * fused_ppi(V) * sizeof(float4) + (size_t)chunk * C * 2;
}

int groupnorm_plan_launches(int C, int HW, int num_sms) {
  return fused_smem(C, HW, num_sms) <= (size_t)kFusedSmemLimit ? 1 : 2;
}

int launch_groupnorm(const __nv_bfloat16* x0, int C0, const __nv_bfloat16* x1, int C1, int HW, int G, float eps,
                     const __nv_bfloat16* gamma, const __nv_bfloat16* beta, int silu, __nv_bfloat16* y,
                     unsigned long long* acc, unsigned int* counter, int num_sms, cudaStream_t st, int* err) {
  {
    // single pass when every CTA's pixel range fits in shared memory
    const int C = C0 + C1;
    const int V = C / 8;
    const int ppi = fused_ppi(V);
    const int threads = V * ppi;
    if (threads < G || threads > 1024 || G > 64) return -1;
    static bool attr_set = false;  // benign race: the attribute value is identical for every caller
    int nblk = num_sms;
    const size_t smem = fused_smem(C, HW, num_sms);
    if (counter && err && smem <= (size_t)kFusedSmemLimit) {
      if (!attr_set) {
        if (cudaFuncSetAttribute(gn_fused_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kFusedSmemLimit) !=
            cudaSuccess)
          return (int)cudaGetLastError();
        attr_set = true;
      }
      int occ = 0;
      if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, gn_fused_kernel, threads, smem) == cudaSuccess &&
          occ >= 1) {
        const int chunk_n = (HW + nblk - 1) / nblk;
        nblk = (HW + chunk_n - 1) / chunk_n;  // no CTA without pixels
        return (int)launch_pdl(gn_fused_kernel, dim3(nblk), dim3(threads), smem, st, x0, C0, x1, C1, HW, G, ppi, eps,
                               gamma, beta, silu, y, acc, counter, err);
      }
      (void)cudaGetLastError();
    }
  }
  const int C = C0 + C1;
  const int V = C / 8;
  const int ppi = V >= 256 ? 1 : 256 / V;
  const int threads = V * ppi;
  if (threads < G || threads > 1024 || G > 64) return -1;
  int nblk = HW / (ppi * 8);  // about 8 pixels per thread
  if (nblk < 1) nblk = 1;
  if (nblk > 2 * num_sms) nblk = 2 * num_sms;
  cudaError_t e = launch_pdl(gn_stats_kernel, dim3(nblk), dim3(threads), threads * sizeof(float4), st, x0, C0, x1, C1,
                             HW, G, ppi, acc);
  if (e != cudaSuccess) return (int)e;
  const size_t total = (size_t)HW * V;
  int blocks = (int)((total + 255) / 256);
  if (blocks > 2 * num_sms) blocks = 2 * num_sms;
  return (int)launch_pdl(gn_apply_kernel, dim3(blocks), dim3(256), C * sizeof(float2), st, x0, C0, x1, C1, HW, G, eps,
                         (const unsigned long long*)acc, gamma, beta, silu, y);
}

}  // namespace sdk
