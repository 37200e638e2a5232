// Reverse-diffusion sampling around the denoiser: noise schedules, the DDPM and
// DDIM updates with classifier-free guidance fused into one elementwise kernel,
// and a stream-ordered loop of denoiser passes and updates.
//
// Sources: SD/SDXL tutorial page (bfzx365.com), DDPM paragraphs (forward step,
// linear schedule 0.0001 -> 0.02 over 1000 steps, the reverse-step formula with
// sigma_t^2 = beta_t, the sampling loop from step T down); the cosine schedule
// that page names is the one of Nichol and Dhariwal (2021); the DDIM step
// (eta = 0) follows Song, Meng and Ermon (2021); guidance is the classifier-free
// combination eps_u + s (eps_c - eps_u).
#include <cuda_runtime.h>
#include <math.h>
#include <string.h>

#include "common.cuh"
#include "profile.h"
#include "sd_api.h"

namespace {

typedef __nv_bfloat16 bf16;

// x' = a x + b eps + c z
struct StepCoef {
  float a, b, c;
};

// One reverse step, one latent element per thread: guidance, update of the FP32
// state, BF16 copy into the next denoiser input. The first thread also folds
// the denoiser passes' device error words into the loop's own.
__global__ void sampler_step_kernel(float* __restrict__ x, const bf16* __restrict__ ec, const bf16* __restrict__ eu,
                                    const float* __restrict__ z, bf16* __restrict__ xb, int64_t n, int out_ch, int ld,
                                    float guidance, StepCoef k, const int* err_a, const int* err_b, int* err_out) {
  sdk::pdl_wait();
  sdk::pdl_trigger();
  if (err_out && blockIdx.x == 0 && threadIdx.x == 0) {
    const int e = (err_a ? *err_a : 0) | (err_b ? *err_b : 0);
    if (e) atomicOr(err_out, e);
  }
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    float e = __bfloat162float(ec[i]);
    if (eu) {
      const float u = __bfloat162float(eu[i]);
      e = fmaf(guidance, e - u, u);
    }
    float v = fmaf(k.a, x[i], k.b * e);
    if (z) v = fmaf(k.c, z[i], v);
    x[i] = v;
    if (xb) xb[(i / out_ch) * ld + (i % out_ch)] = __float2bfloat16_rn(v);
  }
}

// Denoiser input [x (BF16) | cond] per pixel.
__global__ void assemble_input_kernel(const float* __restrict__ x, const bf16* __restrict__ cond, int64_t hw,
                                      int out_ch, int in_ch, bf16* __restrict__ y) {
  sdk::pdl_wait();
  sdk::pdl_trigger();
  const int64_t total = hw * in_ch;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t p = i / in_ch;
    const int c = (int)(i % in_ch);
    y[i] = c < out_ch ? __float2bfloat16_rn(x[p * out_ch + c]) : cond[p * (in_ch - out_ch) + (c - out_ch)];
  }
}

int grid_for(int64_t n) {
  const int64_t b = (n + 255) / 256;
  return (int)(b < 148 * 8 ? (b > 0 ? b : 1) : 148 * 8);
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

// Update coefficients of one step (double precision on the host).
sd_status step_coef(int kind, double ab_t, double ab_p, StepCoef* k) {
  if (!(ab_t > 0.0 && ab_t < 1.0 && ab_p >= ab_t && ab_p <= 1.0)) return SD_ERR_BAD_SHAPE;
  if (kind == SD_SAMPLER_DDPM) {
    const double alpha = ab_t / ab_p;  // 1 - beta_t
    const double beta = 1.0 - alpha;
    k->a = (float)(1.0 / sqrt(alpha));
    k->b = (float)(-beta / (sqrt(1.0 - ab_t) * sqrt(alpha)));
    k->c = (float)sqrt(beta);
    return SD_OK;
  }
  if (kind == SD_SAMPLER_DDIM) {
    k->a = (float)(sqrt(ab_p) / sqrt(ab_t));
    k->b = (float)(sqrt(1.0 - ab_p) - sqrt(ab_p) * sqrt(1.0 - ab_t) / sqrt(ab_t));
    k->c = 0.f;
    return SD_OK;
  }
  return SD_ERR_UNSUPPORTED;
}

sd_status launch_step(const sd_sampler_cfg* cfg, float* x, const void* ec, const void* eu, const float* z, void* xb,
                      const int* err_a, const int* err_b, int* err_out, cudaStream_t st) {
  StepCoef k;
  sd_status s = step_coef(cfg->kind, cfg->alpha_bar_t, cfg->alpha_bar_prev, &k);
  if (s != SD_OK) return s;
  sdp::Scope sc("sampler_step", sdp::F_OTHER, 0, cfg->n * (4.0 + 4.0 + 2.0 + (eu ? 2.0 : 0.0) + (z ? 4.0 : 0.0)), st);
  const cudaError_t e = sdk::launch_pdl(sampler_step_kernel, dim3(grid_for(cfg->n)), dim3(256), 0, st, x,
                                        static_cast<const bf16*>(ec), static_cast<const bf16*>(eu),
                                        cfg->kind == SD_SAMPLER_DDPM ? z : nullptr, static_cast<bf16*>(xb), cfg->n,
                                        cfg->out_ch, cfg->ld, cfg->guidance, k, err_a, err_b, err_out);
  return e == cudaSuccess ? SD_OK : SD_ERR_LAUNCH;
}

constexpr size_t kHeader = 256;
size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

struct DenoisePlan {
  size_t unet_ws, off_ws_a, off_ws_b, off_ec, off_eu, off_in, total;
};

DenoisePlan plan_denoise(const sd_unet_cfg* cfg, size_t unet_ws) {
  DenoisePlan p;
  const size_t hw = (size_t)cfg->height * cfg->width;
  p.unet_ws = align256(unet_ws);
  p.off_ws_a = kHeader;
  p.off_ws_b = p.off_ws_a + p.unet_ws;
  p.off_ec = p.off_ws_b + p.unet_ws;
  p.off_eu = p.off_ec + align256(hw * cfg->out_channels * 2);
  p.off_in = p.off_eu + align256(hw * cfg->out_channels * 2);
  p.total = p.off_in + align256(hw * cfg->in_channels * 2);
  return p;
}

}  // namespace

extern "C" {

sd_status sd_schedule(int32_t kind, int32_t T, double beta_start, double beta_end, double* ac) {
  if (!ac) return SD_ERR_NULL_ARG;
  if (T < 1 || T > 100000) return SD_ERR_BAD_SHAPE;
  double prod = 1.0;
  if (kind == SD_SCHED_LINEAR) {
    if (!(beta_start > 0.0 && beta_end < 1.0 && beta_start <= beta_end)) return SD_ERR_BAD_SHAPE;
    for (int i = 0; i < T; ++i) {
      const double beta = T == 1 ? beta_start : beta_start + (beta_end - beta_start) * i / (T - 1);
      prod *= 1.0 - beta;
      ac[i] = prod;
    }
    return SD_OK;
  }
  if (kind == SD_SCHED_COSINE) {
    const double s = 0.008, half_pi = 1.5707963267948966;
    auto f = [&](int t) {
      const double c = cos(((double)t / T + s) / (1.0 + s) * half_pi);
      return c * c;
    };
    for (int t = 1; t <= T; ++t) {
      double beta = 1.0 - f(t) / f(t - 1);
      if (beta > 0.999) beta = 0.999;
      prod *= 1.0 - beta;
      ac[t - 1] = prod;
    }
    return SD_OK;
  }
  return SD_ERR_UNSUPPORTED;
}

sd_status sd_sampler_step(const sd_sampler_cfg* cfg, float* x, const void* eps_cond, const void* eps_uncond,
                          const float* noise, void* x_bf16, sd_stream_t stream) {
  if (!cfg) return SD_ERR_NULL_ARG;
  if (cfg->n <= 0 || cfg->out_ch <= 0 || cfg->n % cfg->out_ch) return SD_ERR_BAD_SHAPE;
  if (x_bf16 && cfg->ld < cfg->out_ch) return SD_ERR_BAD_SHAPE;
  if (!x || !eps_cond) return SD_ERR_NULL_ARG;
  if (!aligned16(x) || !aligned16(eps_cond) || (eps_uncond && !aligned16(eps_uncond)) || (noise && !aligned16(noise)) ||
      (x_bf16 && !aligned16(x_bf16)))
    return SD_ERR_MISALIGNED;
  return launch_step(cfg, x, eps_cond, eps_uncond, noise, x_bf16, nullptr, nullptr, nullptr,
                     static_cast<cudaStream_t>(stream));
}

size_t sd_denoise_workspace_size(const sd_unet_cfg* cfg) {
  const size_t u = sd_unet_workspace_size(cfg);
  if (u == 0 || cfg->in_channels < cfg->out_channels) return 0;
  return plan_denoise(cfg, u).total;
}

sd_status sd_denoise(const sd_unet_cfg* cfg, const void* pw, int32_t kind, const double* ac, int32_t T,
                     const int32_t* ts, int32_t n_steps, float guidance, float* x, const void* cond_latent,
                     const void* ctx_cond, const void* ctx_uncond, const void* text_c, const void* text_u,
                     const float* ids, const float* noise, void* ws, size_t ws_bytes, sd_stream_t stream) {
  if (!cfg) return SD_ERR_NULL_ARG;
  const size_t need = sd_denoise_workspace_size(cfg);
  if (need == 0) return SD_ERR_UNSUPPORTED;
  if (kind != SD_SAMPLER_DDPM && kind != SD_SAMPLER_DDIM) return SD_ERR_UNSUPPORTED;
  if (!pw || !ac || !ts || !x || !ctx_cond || !ws) return SD_ERR_NULL_ARG;
  if (n_steps < 1 || T < 1) return SD_ERR_BAD_SHAPE;
  const int in_ch = cfg->in_channels, out_ch = cfg->out_channels;
  if (in_ch > out_ch && !cond_latent) return SD_ERR_NULL_ARG;
  if (cfg->add_text_dim > 0 && (!text_c || (ctx_uncond && !text_u))) return SD_ERR_NULL_ARG;
  for (int i = 0; i < n_steps; ++i) {
    if (ts[i] < 1 || ts[i] > T) return SD_ERR_BAD_SHAPE;
    if (i > 0 && ts[i] >= ts[i - 1]) return SD_ERR_BAD_SHAPE;
  }
  if (!aligned16(x) || !aligned16(ws) || (cond_latent && in_ch > out_ch && !aligned16(cond_latent)) ||
      (noise && !aligned16(noise)))
    return SD_ERR_MISALIGNED;
  if (ws_bytes < need) return SD_ERR_WORKSPACE_TOO_SMALL;
  const DenoisePlan p = plan_denoise(cfg, sd_unet_workspace_size(cfg));
  uint8_t* base = static_cast<uint8_t*>(ws);
  void* ws_a = base + p.off_ws_a;
  void* ws_b = base + p.off_ws_b;
  bf16* ec = reinterpret_cast<bf16*>(base + p.off_ec);
  bf16* eu = reinterpret_cast<bf16*>(base + p.off_eu);
  bf16* in = reinterpret_cast<bf16*>(base + p.off_in);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int64_t hw = (int64_t)cfg->height * cfg->width;
  const int64_t n = hw * out_ch;
  if (cudaMemsetAsync(base, 0, kHeader, st) != cudaSuccess) return SD_ERR_LAUNCH;
  {
    sdp::Scope sc("assemble_input", sdp::F_OTHER, 0, hw * (4.0 * out_ch + 4.0 * in_ch - 2.0 * out_ch), st);
    if (sdk::launch_pdl(assemble_input_kernel, dim3(grid_for(hw * in_ch)), dim3(256), 0, st, (const float*)x,
                        static_cast<const bf16*>(cond_latent), hw, out_ch, in_ch, in) != cudaSuccess)
      return SD_ERR_LAUNCH;
  }
  for (int i = 0; i < n_steps; ++i) {
    const int t = ts[i];
    const float tf = (float)t;
    sd_status s = sd_unet_step_cond(cfg, pw, in, tf, ctx_cond, text_c, ids, ec, ws_a, p.unet_ws, stream);
    if (s != SD_OK) return s;
    if (ctx_uncond) {
      s = sd_unet_step_cond(cfg, pw, in, tf, ctx_uncond, text_u, ids, eu, ws_b, p.unet_ws, stream);
      if (s != SD_OK) return s;
    }
    sd_sampler_cfg sc;
    sc.kind = kind;
    sc.n = n;
    sc.out_ch = out_ch;
    sc.ld = in_ch;
    sc.guidance = guidance;
    sc.alpha_bar_t = ac[t - 1];
    sc.alpha_bar_prev = i + 1 < n_steps ? ac[ts[i + 1] - 1] : 1.0;
    s = launch_step(&sc, x, ec, ctx_uncond ? eu : nullptr, noise ? noise + (size_t)i * n : nullptr, in,
                    static_cast<const int*>(ws_a), ctx_uncond ? static_cast<const int*>(ws_b) : nullptr,
                    reinterpret_cast<int*>(base), st);
    if (s != SD_OK) return s;
  }
  return SD_OK;
}

}  // extern "C"
