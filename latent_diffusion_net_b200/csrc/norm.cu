// Normalisation kernels, HBM-bound, 16-byte vector loads.
//
// GroupNorm (GSC unit; ResnetBlock2D and Transformer2DModel panels, section 4 of
// the SD2.1 page): 32 groups of C/32 consecutive channels, statistics over
// (C/32) x H x W, biased variance, then scale/shift and optionally SiLU. The
// input may be the channel concatenation of two NHWC tensors (skip connections
// of the up path) and is never materialised: a vector of 8 channels is read
// from whichever source holds it.
//
// LayerNorm (BasicTransformer Block bullet of the tutorial page): per token
// over C, biased variance, then scale/shift.
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

// ------------------------------------------------------------------ LayerNorm
// T lanes per token (T = 4..32, a power of two), each lane holding at most 8
// 16-byte vectors of the row in registers; two-pass mean/variance.
constexpr int kLnMaxVec = 8;

__global__ void ln_kernel(const __nv_bfloat16* __restrict__ x, int N, int C, int T,
                          const __nv_bfloat16* __restrict__ gamma, const __nv_bfloat16* __restrict__ beta, float eps,
                          __nv_bfloat16* __restrict__ y) {
  pdl_wait();
  pdl_trigger();
  const int gtid = blockIdx.x * blockDim.x + threadIdx.x;
  const int tok = gtid / T;
  const int sub = gtid % T;
  const bool active = tok < N;
  const int V = C >> 3;
  const __nv_bfloat16* row = x + (size_t)(active ? tok : 0) * C;
  uint4 buf[kLnMaxVec];
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < kLnMaxVec; ++i) {
    const int v = sub + T * i;
    if (active && v < V) {
      buf[i] = *reinterpret_cast<const uint4*>(row + v * 8);
      s += bf16lo(buf[i].x) + bf16hi(buf[i].x) + bf16lo(buf[i].y) + bf16hi(buf[i].y) + bf16lo(buf[i].z) +
           bf16hi(buf[i].z) + bf16lo(buf[i].w) + bf16hi(buf[i].w);
    }
  }
  for (int o = T >> 1; o; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  const float mean = s / C;
  float q = 0.f;
#pragma unroll
  for (int i = 0; i < kLnMaxVec; ++i) {
    const int v = sub + T * i;
    if (active && v < V) {
      const float f[8] = {bf16lo(buf[i].x), bf16hi(buf[i].x), bf16lo(buf[i].y), bf16hi(buf[i].y),
                          bf16lo(buf[i].z), bf16hi(buf[i].z), bf16lo(buf[i].w), bf16hi(buf[i].w)};
#pragma unroll
      for (int j = 0; j < 8; ++j) q = fmaf(f[j] - mean, f[j] - mean, q);
    }
  }
  for (int o = T >> 1; o; o >>= 1) q += __shfl_xor_sync(0xffffffffu, q, o);
  const float rstd = rsqrtf(q / C + eps);
  if (!active) return;
  __nv_bfloat16* out = y + (size_t)tok * C;
#pragma unroll
  for (int i = 0; i < kLnMaxVec; ++i) {
    const int v = sub + T * i;
    if (v < V) {
      const int c = v * 8;
      const uint4 gw = __ldg(reinterpret_cast<const uint4*>(gamma + c));
      const uint4 bw = __ldg(reinterpret_cast<const uint4*>(beta + c));
      const float f[8] = {bf16lo(buf[i].x), bf16hi(buf[i].x), bf16lo(buf[i].y), bf16hi(buf[i].y),
                          bf16lo(buf[i].z), bf16hi(buf[i].z), bf16lo(buf[i].w), bf16hi(buf[i].w)};
      const float g[8] = {bf16lo(gw.x), bf16hi(gw.x), bf16lo(gw.y), bf16hi(gw.y),
                          bf16lo(gw.z), bf16hi(gw.z), bf16lo(gw.w), bf16hi(gw.w)};
      const float b[8] = {bf16lo(bw.x), bf16hi(bw.x), bf16lo(bw.y), bf16hi(bw.y),
                          bf16lo(bw.z), bf16hi(bw.z), bf16lo(bw.w), bf16hi(bw.w)};
      float o[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) o[j] = fmaf((f[j] - mean) * rstd, g[j], b[j]);
      *reinterpret_cast<uint4*>(out + c) =
          make_uint4(pack_bf16x2(o[0], o[1]), pack_bf16x2(o[2], o[3]), pack_bf16x2(o[4], o[5]), pack_bf16x2(o[6], o[7]));
    }
  }
}

// ------------------------------------------------------------------ launchers

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

int launch_layernorm(const __nv_bfloat16* x, int N, int C, const __nv_bfloat16* gamma, const __nv_bfloat16* beta,
                     float eps, __nv_bfloat16* y, cudaStream_t st) {
  const int V = C / 8;
  int T = 4;
  while (T < 32 && (V + T - 1) / T > kLnMaxVec) T <<= 1;
  if ((V + T - 1) / T > kLnMaxVec) return -1;
  const int threads = 256;
  const long total = (long)N * T;
  const int blocks = (int)((total + threads - 1) / threads);
  return (int)launch_pdl(ln_kernel, dim3(blocks), dim3(threads), 0, st, x, N, C, T, gamma, beta, eps, y);
}

}  // namespace sdk
