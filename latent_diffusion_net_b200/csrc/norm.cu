// Normalisation kernels, HBM-bound, 16-byte vector loads.
//
// GroupNorm (GSC unit; ResnetBlock2D and Transformer2DModel panels, section 4 of
// the SD2.1 page): 32 groups of C/32 consecutive channels, statistics over
// (C/32) x H x W, biased variance. The input may be the channel concatenation
// of two NHWC tensors (skip connections of the up path) and is never
// materialised: a vector of 8 channels is read from whichever source holds it.
//
// LayerNorm (BasicTransformer Block bullet of the tutorial page): per token
// over C, biased variance.
#include "common.cuh"
#include "kernels.cuh"

namespace sdk {

// ------------------------------------------------------------------ GroupNorm statistics
// Pass 1: each CTA sums x and x^2 per group over a contiguous pixel range
// (FP32 per thread over a few hundred elements). The partial sums of every
// CTA land in `partial`; the last CTA to finish (atomic ticket) reduces them in
// a fixed order in FP64 and writes (mean, rstd) per group. No CTA ever waits
// for another, and the result does not depend on scheduling order.
__global__ void gn_stats_kernel(const __nv_bfloat16* __restrict__ x0, int C0, const __nv_bfloat16* __restrict__ x1,
                                int C1, int HW, int G, int ppi, float eps, float2* __restrict__ partial,
                                unsigned int* __restrict__ counter, float2* __restrict__ stats) {
  extern __shared__ float4 red[];  // [blockDim.x]
  __shared__ bool is_last;
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
  const int split = (ga + 1) * cpg - c;  // channels c .. c+split-1 belong to ga
  const int chunk = (HW + gridDim.x - 1) / gridDim.x;
  const int p0 = blockIdx.x * chunk;
  const int p1 = min(HW, p0 + chunk);
  float sa = 0.f, qa = 0.f, sb = 0.f, qb = 0.f;
  if (pi < ppi) {
    const __nv_bfloat16* base;
    int ld;
    if (c < C0) {
      base = x0 + c;
      ld = C0;
    } else {
      base = x1 + (c - C0);
      ld = C1;
    }
    auto acc = [&](const uint4 w) {
      const float f[8] = {bf16lo(w.x), bf16hi(w.x), bf16lo(w.y), bf16hi(w.y),
                          bf16lo(w.z), bf16hi(w.z), bf16lo(w.w), bf16hi(w.w)};
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (j < split) {
          sa += f[j];
          qa += f[j] * f[j];
        } else {
          sb += f[j];
          qb += f[j] * f[j];
        }
      }
    };
    int p = p0 + pi;
    // four independent 16-byte loads in flight per thread
    for (; p + 3 * ppi < p1; p += 4 * ppi) {
      const uint4 w0 = __ldg(reinterpret_cast<const uint4*>(base + (size_t)p * ld));
      const uint4 w1 = __ldg(reinterpret_cast<const uint4*>(base + (size_t)(p + ppi) * ld));
      const uint4 w2 = __ldg(reinterpret_cast<const uint4*>(base + (size_t)(p + 2 * ppi) * ld));
      const uint4 w3 = __ldg(reinterpret_cast<const uint4*>(base + (size_t)(p + 3 * ppi) * ld));
      acc(w0);
      acc(w1);
      acc(w2);
      acc(w3);
    }
    for (; p < p1; p += ppi) acc(__ldg(reinterpret_cast<const uint4*>(base + (size_t)p * ld)));
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
        const int gav = (vv * 8) / cpg;
        if (gav == g) {
          s += r.x;
          q += r.y;
        } else {
          s += r.z;
          q += r.w;
        }
      }
    }
    partial[(size_t)blockIdx.x * G + g] = make_float2(s, q);
  }
  __threadfence();
  __syncthreads();
  if (t == 0) {
    const unsigned int ticket = atomicAdd(counter, 1u);
    is_last = (ticket == gridDim.x - 1);
  }
  __syncthreads();
  if (is_last) {
    __threadfence();
    // thread t sums the partials of group t % G over blocks r, r + R, ... (r = t / G)
    // in FP64; the R slices are then added in a fixed order.
    double* dred = reinterpret_cast<double*>(red);  // reuses the CTA's reduction buffer
    const int R = blockDim.x / G;
    const int g = t % G;
    const int r = t / G;
    double s = 0.0, q = 0.0;
    if (r < R) {
#pragma unroll 8
      for (int b = r; b < (int)gridDim.x; b += R) {
        const float2 pr = __ldcg(&partial[(size_t)b * G + g]);
        s += pr.x;
        q += pr.y;
      }
    }
    __syncthreads();
    if (r < R) {
      dred[2 * (r * G + g)] = s;
      dred[2 * (r * G + g) + 1] = q;
    }
    __syncthreads();
    if (t < G) {
      double ss = 0.0, qq = 0.0;
      for (int rr = 0; rr < R; ++rr) {
        ss += dred[2 * (rr * G + t)];
        qq += dred[2 * (rr * G + t) + 1];
      }
      const double n = (double)HW * cpg;
      const double mean = ss / n;
      double var = qq / n - mean * mean;
      if (var < 0.0) var = 0.0;
      stats[t] = make_float2((float)mean, (float)(1.0 / sqrt(var + (double)eps)));
    }
    if (t == 0) *counter = 0u;
  }
}

// ------------------------------------------------------------------ GroupNorm apply (+SiLU)
// y[p, c] = act((x[p, c] - mean_g) * rstd_g * gamma_c + beta_c) for the
// concatenation of two sources, written as one dense NHWC tensor.
__global__ void gn_apply_kernel(const __nv_bfloat16* __restrict__ x0, int C0, const __nv_bfloat16* __restrict__ x1,
                                int C1, int HW, int G, const float2* __restrict__ stats,
                                const __nv_bfloat16* __restrict__ gamma, const __nv_bfloat16* __restrict__ beta,
                                int silu, __nv_bfloat16* __restrict__ y) {
  extern __shared__ float2 ab[];  // per channel (scale, shift)
  pdl_wait();
  pdl_trigger();
  const int C = C0 + C1;
  const int cpg = C / G;
  for (int c = threadIdx.x; c < C; c += blockDim.x) {
    const float2 st = stats[c / cpg];
    const float a = st.y * __bfloat162float(gamma[c]);
    ab[c] = make_float2(a, __bfloat162float(beta[c]) - st.x * a);
  }
  __syncthreads();
  const int V = C >> 3;
  const size_t total = (size_t)HW * V;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < total; i += (size_t)gridDim.x * blockDim.x) {
    const int p = (int)(i / V);
    const int v = (int)(i % V);
    const int c = v * 8;
    const __nv_bfloat16* src = (c < C0) ? (x0 + (size_t)p * C0 + c) : (x1 + (size_t)p * C1 + (c - C0));
    const uint4 w = *reinterpret_cast<const uint4*>(src);
    float f[8] = {bf16lo(w.x), bf16hi(w.x), bf16lo(w.y), bf16hi(w.y),
                  bf16lo(w.z), bf16hi(w.z), bf16lo(w.w), bf16hi(w.w)};
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float2 s = ab[c + j];
      float o = fmaf(f[j], s.x, s.y);
      if (silu) o = silu_f(o);
      f[j] = o;
    }
    *reinterpret_cast<uint4*>(y + (size_t)p * C + c) =
        make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]), pack_bf16x2(f[4], f[5]), pack_bf16x2(f[6], f[7]));
  }
}

// ------------------------------------------------------------------ LayerNorm
// One warp per token; the row stays in registers (C <= 2048).
constexpr int kLnMaxVecPerLane = 8;

__global__ void ln_kernel(const __nv_bfloat16* __restrict__ x, int N, int C, const __nv_bfloat16* __restrict__ gamma,
                          const __nv_bfloat16* __restrict__ beta, float eps, __nv_bfloat16* __restrict__ y) {
  pdl_wait();
  pdl_trigger();
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= N) return;
  const int V = C >> 3;
  const __nv_bfloat16* row = x + (size_t)warp * C;
  uint4 buf[kLnMaxVecPerLane];
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < kLnMaxVecPerLane; ++i) {
    const int v = lane + 32 * i;
    if (v < V) {
      buf[i] = *reinterpret_cast<const uint4*>(row + v * 8);
      s += bf16lo(buf[i].x) + bf16hi(buf[i].x) + bf16lo(buf[i].y) + bf16hi(buf[i].y) + bf16lo(buf[i].z) +
           bf16hi(buf[i].z) + bf16lo(buf[i].w) + bf16hi(buf[i].w);
    }
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  const float mean = s / C;
  float q = 0.f;
#pragma unroll
  for (int i = 0; i < kLnMaxVecPerLane; ++i) {
    const int v = lane + 32 * i;
    if (v < V) {
      const float f[8] = {bf16lo(buf[i].x), bf16hi(buf[i].x), bf16lo(buf[i].y), bf16hi(buf[i].y),
                          bf16lo(buf[i].z), bf16hi(buf[i].z), bf16lo(buf[i].w), bf16hi(buf[i].w)};
#pragma unroll
      for (int j = 0; j < 8; ++j) q += (f[j] - mean) * (f[j] - mean);
    }
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) q += __shfl_xor_sync(0xffffffffu, q, o);
  const float rstd = rsqrtf(q / C + eps);
  __nv_bfloat16* out = y + (size_t)warp * C;
#pragma unroll
  for (int i = 0; i < kLnMaxVecPerLane; ++i) {
    const int v = lane + 32 * i;
    if (v < V) {
      const int c = v * 8;
      const uint4 gw = *reinterpret_cast<const uint4*>(gamma + c);
      const uint4 bw = *reinterpret_cast<const uint4*>(beta + c);
      const float f[8] = {bf16lo(buf[i].x), bf16hi(buf[i].x), bf16lo(buf[i].y), bf16hi(buf[i].y),
                          bf16lo(buf[i].z), bf16hi(buf[i].z), bf16lo(buf[i].w), bf16hi(buf[i].w)};
      const float g[8] = {bf16lo(gw.x), bf16hi(gw.x), bf16lo(gw.y), bf16hi(gw.y),
                          bf16lo(gw.z), bf16hi(gw.z), bf16lo(gw.w), bf16hi(gw.w)};
      const float b[8] = {bf16lo(bw.x), bf16hi(bw.x), bf16lo(bw.y), bf16hi(bw.y),
                          bf16lo(bw.z), bf16hi(bw.z), bf16lo(bw.w), bf16hi(bw.w)};
      float o[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) o[j] = (f[j] - mean) * rstd * g[j] + b[j];
      *reinterpret_cast<uint4*>(out + c) =
          make_uint4(pack_bf16x2(o[0], o[1]), pack_bf16x2(o[2], o[3]), pack_bf16x2(o[4], o[5]), pack_bf16x2(o[6], o[7]));
    }
  }
}

// ------------------------------------------------------------------ launchers

int gn_stats_blocks(int HW, int C, int num_sms) {
  const int V = C / 8;
  const int ppi = V >= 256 ? 1 : 256 / V;
  // about 8 pixels per thread, at most two CTAs per SM
  int nblk = HW / (ppi * 8);
  if (nblk < 1) nblk = 1;
  if (nblk > 2 * num_sms) nblk = 2 * num_sms;
  return nblk;
}

int launch_gn_stats(const __nv_bfloat16* x0, int C0, const __nv_bfloat16* x1, int C1, int HW, int G, float eps,
                    float2* partial, unsigned int* counter, float2* stats, int num_sms, cudaStream_t st) {
  const int C = C0 + C1;
  const int V = C / 8;
  const int ppi = V >= 256 ? 1 : 256 / V;
  const int threads = V * ppi;
  const int nblk = gn_stats_blocks(HW, C, num_sms);
  return (int)launch_pdl(gn_stats_kernel, dim3(nblk), dim3(threads), threads * sizeof(float4), st, x0, C0, x1, C1, HW,
                         G, ppi, eps, partial, counter, stats);
}

int launch_gn_apply(const __nv_bfloat16* x0, int C0, const __nv_bfloat16* x1, int C1, int HW, int G,
                    const float2* stats, const __nv_bfloat16* gamma, const __nv_bfloat16* beta, int silu,
                    __nv_bfloat16* y, int num_sms, cudaStream_t st) {
  const int C = C0 + C1;
  const size_t total = (size_t)HW * (C / 8);
  int blocks = (int)((total + 255) / 256);
  if (blocks > num_sms * 8) blocks = num_sms * 8;
  return (int)launch_pdl(gn_apply_kernel, dim3(blocks), dim3(256), C * sizeof(float2), st, x0, C0, x1, C1, HW, G,
                         stats, gamma, beta, silu, y);
}

int launch_layernorm(const __nv_bfloat16* x, int N, int C, const __nv_bfloat16* gamma, const __nv_bfloat16* beta,
                     float eps, __nv_bfloat16* y, cudaStream_t st) {
  const int warps_per_block = 8;
  const int blocks = (N + warps_per_block - 1) / warps_per_block;
  return (int)launch_pdl(ln_kernel, dim3(blocks), dim3(warps_per_block * 32), 0, st, x, N, C, gamma, beta, eps, y);
}

}  // namespace sdk
