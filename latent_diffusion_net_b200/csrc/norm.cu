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

int launch_groupnorm(const __nv_bfloat16* x0, int C0, const __nv_bfloat16* x1, int C1, int HW, int G, float eps,
                     const __nv_bfloat16* gamma, const __nv_bfloat16* beta, int silu, __nv_bfloat16* y,
                     unsigned long long* acc, int num_sms, cudaStream_t st) {
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
