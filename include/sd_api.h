/*
 * sd_api.h -- C ABI of the B200 (sm_100a) Stable-Diffusion U-Net denoiser library.
 *
 * One forward pass of a Stable-Diffusion-style U-Net denoiser timestep at batch 1
 * in BF16: ResnetBlock2D and Transformer2DModel blocks composed into the
 * Down / Mid / Up topology with skip concatenation, stride-2 downsampling and
 * nearest-2x upsampling.
 *
 * Sources (page title, section):
 *   [SD21]  "Stable Diffusion 2.1 Base 宏观架构": section 3 (full U-Net multi-scale
 *           topology: levels, skips, Conv_in 4->320, Conv_out 320->4), section 4
 *           (core operators: ResnetBlock2D and Transformer2DModel panels).
 *   [SDXLI] "Stable Diffusion XL Inpainting 宏观架构": sections 1-4 (9-channel
 *           input = noisy latent + masked latent + mask; context [1,77,2048]).
 *   [TUT]   SD/SDXL tutorial page (bfzx365.com, video 67462879): GSC bullet
 *           (GroupNorm + SiLU + Conv), FeedForward bullet (GEGLU), DownSample
 *           bullet (Conv k3 s2 p1), UpSample bullet (nearest + Conv k3 s1 p1),
 *           BasicTransformer Block bullet, Spatial Transformer bullets, the
 *           ResNetBlock paragraph and the sinusoidal time-embedding paragraph.
 *   [SD15]  SD1.5 anatomy page (hotelren.com), section 3.4: Softmax(QK^T/sqrt(d))V.
 *
 * Conventions shared by every entry point
 *   - Batch is 1. Activations are NHWC BF16, i.e. a token matrix [H*W, C] in
 *     row-major pixel order (y*W + x). Context is BF16 [ctx_len, ctx_dim].
 *   - Every device pointer is caller-owned device memory. The library never
 *     allocates, frees or synchronises inside a *_fwd / sd_unet_step call; all
 *     work is enqueued on the given stream, in order.
 *   - Device pointers must be 16-byte aligned (SD_ERR_MISALIGNED otherwise).
 *     Outputs must not alias inputs unless an entry point says otherwise.
 *   - Weights are a packed BF16 buffer in the library's layout: obtain the
 *     canonical tensor table with sd_*_weight_layout(), fill a canonical buffer
 *     (tensors in table order, row-major in the canonical shapes, no padding),
 *     convert it with sd_*_pack_weights() on the host and copy the result to the
 *     device.
 *   - All argument, shape, alignment and workspace checks run on the host before
 *     any launch; on error nothing is launched and a status is returned. No call
 *     aborts, prints or throws. Device-side waits are bounded; one that gives up
 *     sets a flag in the workspace header that sd_query_device_status() reports.
 *   - Thread safety: calls are re-entrant when they use distinct workspaces. The
 *     only shared state is a per-device attribute cache guarded by a mutex.
 */
#ifndef SD_API_H
#define SD_API_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef void* sd_stream_t; /* a cudaStream_t; NULL = the legacy default stream */

typedef enum {
  SD_OK = 0,
  SD_ERR_NULL_ARG = 1,             /* a required pointer is NULL */
  SD_ERR_BAD_SHAPE = 2,            /* inconsistent sizes, channel or context mismatch */
  SD_ERR_UNSUPPORTED = 3,          /* batch != 1, head_dim != 64, C % 64 != 0, groups ..., device index >= 64 */
  SD_ERR_MISALIGNED = 4,           /* a device pointer is not 16-byte aligned */
  SD_ERR_WORKSPACE_TOO_SMALL = 5,  /* ws_bytes below sd_*_workspace_size() */
  SD_ERR_NOT_SM100 = 6,            /* current device is not compute capability 10.0 */
  SD_ERR_LAUNCH = 7,               /* a kernel launch or CUDA runtime call failed */
  SD_ERR_DEVICE_TIMEOUT = 8,       /* a bounded device-side wait gave up */
  SD_ERR_CAPACITY = 9              /* caller-provided table too small */
} sd_status;

/* Tensor kinds in a weight table. */
enum { SD_KIND_WEIGHT = 0, SD_KIND_BIAS = 1, SD_KIND_NORM_GAMMA = 2, SD_KIND_NORM_BETA = 3 };

typedef struct {
  char name[80];          /* e.g. "down.0.res.1.conv1.weight" */
  int32_t ndim;
  int64_t shape[4];       /* canonical shape: conv [O, C, k, k], linear [out, in], vectors [n] */
  int32_t kind;           /* SD_KIND_* */
  int32_t fan_in;         /* C*k*k for conv, in_features for linear, 0 for norms */
  int64_t canon_offset;   /* element offset in the canonical buffer */
  int64_t packed_offset;  /* byte offset in the packed buffer */
} sd_tensor_desc;

/* ---------------------------------------------------------------- configurations */

/* Time embedding MLP [TUT, time-embedding paragraph]: phi(t) sinusoid of
 * proj_dim (cos half first, frequencies 10000^(-i/(proj_dim/2))), then
 * Linear proj_dim->temb_dim, SiLU, Linear temb_dim->temb_dim. */
typedef struct {
  int32_t proj_dim;  /* 320 */
  int32_t temb_dim;  /* 1280 */
} sd_time_cfg;

/* Plain convolutions: conv_in (3x3, c_in 4 or 9 -> c_out), downsample (3x3
 * stride 2 pad 1, c_in = c_out), upsample (nearest 2x then 3x3), and the output
 * head (GroupNorm + SiLU + 3x3 conv_out). height/width are the INPUT size. */
typedef struct {
  int32_t batch;   /* must be 1 */
  int32_t height;
  int32_t width;
  int32_t c_in;
  int32_t c_out;
  int32_t groups;  /* output head only (32) */
  float eps;       /* output head only (1e-5) */
} sd_conv_cfg;

/* ResnetBlock2D [SD21 section 4; TUT ResNetBlock paragraph]. Input is
 * concat_C(x, skip) when c_skip > 0 (x channels first). A 1x1 shortcut conv is
 * used when c_x + c_skip != c_out, else the identity. */
typedef struct {
  int32_t batch;     /* must be 1 */
  int32_t height;
  int32_t width;
  int32_t c_x;       /* channels of x */
  int32_t c_skip;    /* channels of the concatenated skip tensor, 0 = none */
  int32_t c_out;
  int32_t temb_dim;  /* 1280 */
  int32_t groups;    /* 32 */
  float eps;         /* 1e-5 */
} sd_resblock_cfg;

/* Transformer2DModel [SD21 section 4; TUT Spatial Transformer and
 * BasicTransformer Block bullets]: GN -> proj_in -> depth x (LN -> self-attn,
 * LN -> cross-attn on the context, LN -> GEGLU FF; each residual) -> proj_out,
 * plus the block input. */
typedef struct {
  int32_t batch;     /* must be 1 */
  int32_t height;
  int32_t width;
  int32_t channels;  /* C, a multiple of 64 */
  int32_t head_dim;  /* must be 64; heads = C / 64 */
  int32_t depth;     /* number of BasicTransformer blocks (1, 2, 10) */
  int32_t ctx_len;   /* 1 .. 256 (77) */
  int32_t ctx_dim;   /* 1024 or 2048 (multiple of 64) */
  int32_t groups;    /* 32 */
  float gn_eps;      /* 1e-5 */
  float ln_eps;      /* 1e-5 */
} sd_transformer_cfg;

/* Whole denoiser [SD21 section 3; SDXLI section 3]. The three add_* fields
 * describe SDXL's added conditioning [TUT, SDXL conditioning paragraphs]: a
 * pooled text vector of add_text_dim values and add_time_ids scalars (original
 * size, crop offset, target size), each Fourier-encoded like the timestep to
 * add_time_dim values and concatenated after the text (1280 + 6 x 256 = 2816 for
 * SDXL); that vector goes through Linear -> SiLU -> Linear (the time MLP's shape)
 * and is added to the time embedding. add_text_dim = 0 disables it (SD2.1). */
typedef struct {
  int32_t in_channels;        /* 4, or 9 for inpainting */
  int32_t out_channels;       /* 4 */
  int32_t height;             /* latent height, divisible by 2^(n_levels-1) */
  int32_t width;
  int32_t n_levels;           /* 1..4 */
  int32_t block_channels[4];  /* 320, 640, 1280, 1280 */
  int32_t attn_depth[4];      /* 1, 1, 1, 0 (0 = no transformer at that level) */
  int32_t layers_per_block;   /* 2 (the up path uses layers_per_block + 1) */
  int32_t mid_depth;          /* 1 */
  int32_t head_dim;           /* 64 */
  int32_t ctx_len;            /* 77 */
  int32_t ctx_dim;            /* 1024 */
  int32_t time_proj_dim;      /* 320 */
  int32_t temb_dim;           /* 1280 */
  int32_t groups;             /* 32 */
  float eps;                  /* 1e-5, for every GroupNorm and LayerNorm */
  int32_t add_text_dim;       /* 0 = no added conditioning; 1280 for SDXL */
  int32_t add_time_ids;       /* 0..8 scalars (6 for SDXL) */
  int32_t add_time_dim;       /* Fourier width per scalar (256 for SDXL), even */
} sd_unet_cfg;

/* VAE decoder [SD21 section 5; SDXLI section 5]: the denoised latent divided by
 * scaling_factor (0.18215, [TUT]), a 1x1 post-quantisation conv, conv_in 3x3 to
 * the widest channel count, a MidBlock (resblock, single-head self-attention
 * over the H*W tokens, resblock), n_levels UpDecoder blocks walking
 * block_channels backwards (512, 512, 256, 128) with layers_per_block + 1
 * resblocks each and a nearest-2x upsampling conv after all but the last, then
 * GroupNorm + SiLU + conv_out 3x3 to out_channels. The resblocks have no time
 * embedding. height/width are the LATENT size; the image is 2^(n_levels-1)
 * times larger. */
typedef struct {
  int32_t height;             /* latent height (96 for a 768x768 image) */
  int32_t width;
  int32_t latent_channels;    /* 4 */
  int32_t out_channels;       /* 3 */
  int32_t n_levels;           /* 4 */
  int32_t block_channels[4];  /* 128, 256, 512, 512 (encoder order) */
  int32_t layers_per_block;   /* 2 (each UpDecoder block has 3 resblocks) */
  int32_t groups;             /* 32 */
  float eps;                  /* 1e-5 */
  float scaling_factor;       /* 0.18215 */
} sd_vae_cfg;

/* ---------------------------------------------------------------- weights (host only) */

/* Enumerate the canonical tensor table. `out` may be NULL (sizes only); when
 * not NULL it must hold `capacity` entries (SD_ERR_CAPACITY otherwise, with
 * *n_tensors still set). canon_elems: BF16 elements of the canonical buffer;
 * packed_bytes: size of the packed buffer. Pure host code, no GPU needed. */
sd_status sd_time_weight_layout(const sd_time_cfg* cfg, sd_tensor_desc* out, int32_t capacity,
                                int32_t* n_tensors, int64_t* canon_elems, int64_t* packed_bytes);
sd_status sd_conv_weight_layout(const sd_conv_cfg* cfg, int32_t conv_kind, sd_tensor_desc* out,
                                int32_t capacity, int32_t* n_tensors, int64_t* canon_elems,
                                int64_t* packed_bytes);
sd_status sd_resblock_weight_layout(const sd_resblock_cfg* cfg, sd_tensor_desc* out, int32_t capacity,
                                    int32_t* n_tensors, int64_t* canon_elems, int64_t* packed_bytes);
sd_status sd_transformer_weight_layout(const sd_transformer_cfg* cfg, sd_tensor_desc* out,
                                       int32_t capacity, int32_t* n_tensors, int64_t* canon_elems,
                                       int64_t* packed_bytes);
sd_status sd_unet_weight_layout(const sd_unet_cfg* cfg, sd_tensor_desc* out, int32_t capacity,
                                int32_t* n_tensors, int64_t* canon_elems, int64_t* packed_bytes);
sd_status sd_vae_weight_layout(const sd_vae_cfg* cfg, sd_tensor_desc* out, int32_t capacity, int32_t* n_tensors,
                               int64_t* canon_elems, int64_t* packed_bytes);

/* conv_kind for sd_conv_weight_layout / sd_conv_pack_weights / sd_conv_fwd. */
enum { SD_CONV_IN = 0, SD_CONV_DOWNSAMPLE = 1, SD_CONV_UPSAMPLE = 2, SD_CONV_OUTPUT = 3 };

/* Convert a canonical BF16 buffer (host, uint16 bit patterns) into the packed
 * layout (host buffer of packed_bytes); host code only, no stream. Each tensor
 * starts on a 256-byte boundary, in table order:
 *   - 3x3 conv weights become [O][ky][kx][C]; conv_in weights become [O][Kp] in
 *     im2col order k = (ky*3 + kx)*C + c, zero-padded to a multiple of 64;
 *   - the three linear layers fed by a LayerNorm in each BasicTransformer block
 *     (attn1 q/k/v, attn2 q, ff.w1) are stored multiplied by that LayerNorm's
 *     gamma along K and rounded to BF16 (W' = W * gamma); ff.w1 rows and bias are
 *     also interleaved (value j, gate j);
 *   - after each block's tensors come two derived FP32 vectors per such layer:
 *     c1 = row sums of W' and c2 = W * beta + bias, which the GEMM epilogue uses
 *     to apply the LayerNorm from per-row statistics (no LayerNorm kernel runs);
 *   - in a whole U-Net (sd_unet_pack_weights) the cross-attention K and V weights
 *     of every BasicTransformer block are placed last, out of table order, as one
 *     [K of all blocks | V of all blocks] x ctx_dim matrix, so that one GEMM
 *     projects the context for every cross-attention of the step (the
 *     packed_offset of each tensor in sd_unet_weight_layout gives its place);
 *   - every other tensor is copied unchanged. */
sd_status sd_time_pack_weights(const sd_time_cfg* cfg, const uint16_t* canonical, void* packed);
sd_status sd_conv_pack_weights(const sd_conv_cfg* cfg, int32_t conv_kind, const uint16_t* canonical,
                               void* packed);
sd_status sd_resblock_pack_weights(const sd_resblock_cfg* cfg, const uint16_t* canonical, void* packed);
sd_status sd_transformer_pack_weights(const sd_transformer_cfg* cfg, const uint16_t* canonical,
                                      void* packed);
sd_status sd_unet_pack_weights(const sd_unet_cfg* cfg, const uint16_t* canonical, void* packed);
sd_status sd_vae_pack_weights(const sd_vae_cfg* cfg, const uint16_t* canonical, void* packed);

/* ---------------------------------------------------------------- workspace sizes */

size_t sd_time_workspace_size(const sd_time_cfg* cfg);
size_t sd_conv_workspace_size(const sd_conv_cfg* cfg, int32_t conv_kind);
size_t sd_resblock_workspace_size(const sd_resblock_cfg* cfg);
size_t sd_transformer_workspace_size(const sd_transformer_cfg* cfg);
size_t sd_unet_workspace_size(const sd_unet_cfg* cfg);
size_t sd_vae_workspace_size(const sd_vae_cfg* cfg);

/* ---------------------------------------------------------------- forward calls (device) */

/* temb_out: device FP32 [temb_dim], the MLP output before any SiLU. */
sd_status sd_time_embed(const sd_time_cfg* cfg, const void* packed_w, float timestep, float* temb_out,
                        void* workspace, size_t ws_bytes, sd_stream_t stream);

/* Allocation-free variant of sd_time_embed. The source pages have no
 * counterpart: it exists for callers that cannot give this library a workspace
 * because they may not allocate device memory themselves, e.g. the enqueue step
 * of a plugin inside another inference engine (the host engine owns every
 * allocation) or a latency-critical loop where cudaMalloc/cudaFree would
 * synchronise the device.
 * Same arguments and result as sd_time_embed without the workspace: the two
 * intermediate vectors live in a fixed device array of this library
 * (2 x 4096 FP32 = 32 KiB, resident on every GPU that loads the library until
 * the process exits). proj_dim and temb_dim above 4096 are rejected with
 * SD_ERR_UNSUPPORTED before anything is launched. No device or host memory is
 * allocated. Every call looks up that array's device address on the current
 * device (a host-side query, so the address stays right after a device reset);
 * the first lookup on a device may load the library's device code, so make the
 * first call on each device before any stream capture. All calls share the one
 * array: calls whose work overlaps on the GPU (different streams, or different
 * host threads, without ordering) race on it; serialise them. Each call
 * rewrites both vectors before reading them, so no state carries over between
 * calls. */
sd_status sd_time_embed_noalloc(const sd_time_cfg* cfg, const void* packed_w, float timestep, float* temb_out,
                                sd_stream_t stream);

/* SD_CONV_IN: x0 = latent [H, W, c_in] BF16, or for c_in = 9 the inpaint input
 *   assembled from x0 = noisy [H, W, 4], x1 = masked latent [H, W, 4],
 *   x2 = mask [H, W, 1] (channels in that order) without materialising it.
 *   y = [H, W, c_out].
 * SD_CONV_DOWNSAMPLE: x0 = [H, W, C] -> y = [H/2, W/2, C] (3x3, stride 2, pad 1).
 * SD_CONV_UPSAMPLE: x0 = [H, W, C] -> y = [2H, 2W, C] (nearest 2x, then 3x3).
 * SD_CONV_OUTPUT: x0 = [H, W, C] -> y = [H, W, c_out] = conv_out(SiLU(GN(x0))). */
sd_status sd_conv_fwd(const sd_conv_cfg* cfg, int32_t conv_kind, const void* packed_w, const void* x0,
                      const void* x1, const void* x2, void* y, void* workspace, size_t ws_bytes,
                      sd_stream_t stream);

/* x [H, W, c_x], skip [H, W, c_skip] or NULL, temb device FP32 [temb_dim]
 * (pre-SiLU MLP output), y [H, W, c_out]. */
sd_status sd_resblock_fwd(const sd_resblock_cfg* cfg, const void* packed_w, const void* x,
                          const void* skip, const float* temb, void* y, void* workspace, size_t ws_bytes,
                          sd_stream_t stream);

/* x [H, W, C], context [ctx_len, ctx_dim], y [H, W, C]; y may alias x (in-place
 * update of the residual stream). */
sd_status sd_transformer_fwd(const sd_transformer_cfg* cfg, const void* packed_w, const void* x,
                             const void* context, void* y, void* workspace, size_t ws_bytes,
                             sd_stream_t stream);

/* One denoiser timestep. latent: [H, W, in_channels] BF16 (for in_channels = 9
 * the caller passes the assembled 9-channel input), context [ctx_len, ctx_dim],
 * eps_out [H, W, out_channels]. The skip stack and every intermediate live in
 * the workspace. A config with added conditioning (add_text_dim > 0) needs
 * sd_unet_step_cond; here it returns SD_ERR_NULL_ARG. */
sd_status sd_unet_step(const sd_unet_cfg* cfg, const void* packed_w, const void* latent, float timestep,
                       const void* context, void* eps_out, void* workspace, size_t ws_bytes,
                       sd_stream_t stream);

/* sd_unet_step with SDXL's added conditioning [TUT, SDXL conditioning
 * paragraphs; SDXLI section 1]: add_text = device BF16 [add_text_dim] pooled
 * text vector; add_time_ids = HOST array of add_time_ids floats (SDXL: original
 * height, width, crop top, left, target height, width), read during this call
 * (a captured graph keeps the values it was captured with). Both may be NULL
 * when cfg->add_text_dim is 0. */
sd_status sd_unet_step_cond(const sd_unet_cfg* cfg, const void* packed_w, const void* latent, float timestep,
                            const void* context, const void* add_text, const float* add_time_ids, void* eps_out,
                            void* workspace, size_t ws_bytes, sd_stream_t stream);

/* ---------------------------------------------------------------- sampling
 * The steps either side of the denoiser [TUT, DDPM paragraphs]: the forward
 * process q(x_t | x_{t-1}) = N(sqrt(1 - beta_t) x_{t-1}, beta_t I), alpha_t =
 * 1 - beta_t, alpha_bar_t = prod_{s<=t} alpha_s, and the reverse step
 *   DDPM: x_{t-1} = (x_t - beta_t / sqrt(1 - alpha_bar_t) eps) / sqrt(alpha_t) + sqrt(beta_t) z
 * as printed there; the deterministic DDIM step (Song, Meng and Ermon 2021,
 * eta = 0; the page names the DDIM scheduler only):
 *   x0 = (x_t - sqrt(1 - alpha_bar_t) eps) / sqrt(alpha_bar_t),
 *   x_prev = sqrt(alpha_bar_prev) x0 + sqrt(1 - alpha_bar_prev) eps;
 * and classifier-free guidance (the "CFG scale" of the SD1.5 anatomy page):
 *   eps = eps_uncond + guidance * (eps_cond - eps_uncond).
 * Timesteps t run from 1 to T; alphas_cumprod[t - 1] is alpha_bar_t. */
enum { SD_SCHED_LINEAR = 0, SD_SCHED_COSINE = 1 };
enum { SD_SAMPLER_DDPM = 0, SD_SAMPLER_DDIM = 1 };

/* Host only. SD_SCHED_LINEAR: beta rises linearly from beta_start to beta_end
 * over T steps (the page: 0.0001 to 0.02, T = 1000; the DDIM scheduler's
 * beta_start 0.00085 is another choice). SD_SCHED_COSINE: the cosine schedule
 * of Nichol and Dhariwal (2021), named on the page, with s = 0.008 and beta
 * clipped at 0.999 (beta_start/end unused). Writes alphas_cumprod[T]. */
sd_status sd_schedule(int32_t kind, int32_t T, double beta_start, double beta_end, double* alphas_cumprod);

/* One reverse step on a latent of n elements, in place on the FP32 state x
 * (x_t in, x_prev out). alpha_bar_t / alpha_bar_prev: the schedule at the current
 * and the next timestep (alpha_bar_prev = 1 after the last step; for DDPM the
 * next timestep is t - 1, beta_t = 1 - alpha_bar_t / alpha_bar_prev).
 * eps_cond / eps_uncond: BF16 [n] U-Net outputs; eps_uncond = NULL means no
 * guidance. noise: FP32 [n] z of the DDPM step, NULL = none (always none for
 * DDIM). x_bf16: NULL, or a BF16 [n / out_ch][ld] buffer whose first out_ch
 * channels of each pixel receive the new x (the next U-Net input; the other
 * ld - out_ch channels are left as they are). Device pointers, 16-byte aligned. */
typedef struct {
  int32_t kind;          /* SD_SAMPLER_* */
  int64_t n;             /* latent elements (H * W * out_ch) */
  int32_t out_ch;        /* channels of the latent (4) */
  int32_t ld;            /* channels per pixel of x_bf16 (out_ch, or 9 for inpainting) */
  float guidance;        /* classifier-free guidance scale */
  double alpha_bar_t;
  double alpha_bar_prev;
} sd_sampler_cfg;

sd_status sd_sampler_step(const sd_sampler_cfg* cfg, float* x, const void* eps_cond, const void* eps_uncond,
                          const float* noise, void* x_bf16, sd_stream_t stream);

/* A whole sampling loop on the device, stream-ordered (no host synchronisation,
 * so it can be captured into one CUDA graph): for each of n_steps timesteps
 * (host array, descending, each in 1..T), run the denoiser on the current latent
 * with ctx_cond (and again with ctx_uncond when it is not NULL, then combine with
 * `guidance`), then sd_sampler_step to the next timestep (0 after the last).
 * x: device FP32 [H, W, out_channels], x_T in, x_0 out. For in_channels >
 * out_channels (inpainting) cond_latent = device BF16 [H, W, in - out] holds the
 * channels that follow the latent in the denoiser input (masked latent, mask);
 * else NULL. add_text_cond / add_text_uncond / add_time_ids: the SDXL added
 * conditioning of each pass (as in sd_unet_step_cond). noise: device FP32
 * [n_steps][H*W*out] (DDPM), or NULL. The U-Net is called with the timestep value
 * t. Workspace: sd_denoise_workspace_size(cfg) bytes. */
size_t sd_denoise_workspace_size(const sd_unet_cfg* cfg);
sd_status sd_denoise(const sd_unet_cfg* cfg, const void* packed_w, int32_t sampler_kind, const double* alphas_cumprod,
                     int32_t T, const int32_t* timesteps, int32_t n_steps, float guidance, float* x,
                     const void* cond_latent, const void* ctx_cond, const void* ctx_uncond, const void* add_text_cond,
                     const void* add_text_uncond, const float* add_time_ids, const float* noise, void* workspace,
                     size_t ws_bytes, sd_stream_t stream);

/* VAE decode: latent = device BF16 [height, width, latent_channels] (NHWC),
 * image = device BF16 [height * 2^(n_levels-1), width * 2^(n_levels-1),
 * out_channels]. The MidBlock attention forms the full [HW, HW] score matrix in
 * the workspace (FP32 scores, BF16 probabilities), so the workspace grows with
 * the square of the latent's pixel count. */
sd_status sd_vae_decode(const sd_vae_cfg* cfg, const void* packed_w, const void* latent, void* image,
                        void* workspace, size_t ws_bytes, sd_stream_t stream);

/* Synchronises `stream`, then reads the device error word of `workspace`:
 * SD_OK, or SD_ERR_DEVICE_TIMEOUT when a bounded wait gave up; the word is
 * cleared afterwards. */
sd_status sd_query_device_status(void* workspace, sd_stream_t stream);

/* ---------------------------------------------------------------- launch accounting
 * Optional per-thread recorder for measuring kernels in place: between
 * sd_profile_begin() and sd_profile_end() every kernel this library launches
 * from the calling thread is bracketed by two CUDA events on its stream and
 * tagged with its algorithmic FLOPs (2*M*N*K per contraction, 4*Nq*Nk*C per
 * attention) and bytes (each operand read once, each output written once).
 * Recording also works while the stream is being captured into a CUDA graph,
 * provided an earlier eager recording of the same call sequence created the
 * events; the graph then holds the event records and every replay overwrites
 * them. sd_profile_read() returns the records of the last recording with their
 * elapsed times (ms < 0 where the events have not completed). */
typedef struct {
  char kernel[24];  /* "gemm_tc", "attention", "groupnorm", "gemv", ... (SD_FAMILY_LAYERNORM is unused:
                       the LayerNorms are folded into the GEMMs) */
  int32_t family;   /* SD_FAMILY_* */
  int32_t kernels;  /* kernels enqueued by this launch (a split-K GEMM enqueues 2) */
  double flops;
  double bytes;
  float ms;         /* device time between the two events */
} sd_launch_record;

enum {
  SD_FAMILY_GEMM = 0, SD_FAMILY_ATTENTION = 1, SD_FAMILY_GN_STATS = 2, SD_FAMILY_GN_APPLY = 3,
  SD_FAMILY_LAYERNORM = 4, SD_FAMILY_GEMV = 5, SD_FAMILY_OTHER = 6
};

sd_status sd_profile_begin(void);
sd_status sd_profile_end(int32_t* n_kernels); /* kernels enqueued while recording */
sd_status sd_profile_read(sd_launch_record* out, int32_t capacity, int32_t* n);

/* Tuning and test hook for the tensor-core GEMM behind every convolution and
 * linear layer. bn (0 = automatic, else one of 32, 64, 96, 128, 160, 192, 224,
 * 256) fixes the output-feature width of a tile; splits (0 = automatic, 1 = no
 * split, up to 16) fixes the number of reduction splits. The setting is
 * process-wide and applies to calls issued after it. A split count above the
 * number of 64-wide reduction blocks of a GEMM is lowered to that number; one
 * that needs more FP32 workspace than the call has makes the call fail with
 * SD_ERR_UNSUPPORTED. Results are
 * the same for every setting up to FP32 summation order. Not thread-safe
 * against calls in flight on other host threads. The pages have no
 * counterpart: this only selects among equivalent schedules. */
sd_status sd_gemm_override(int32_t bn, int32_t splits);

/* ---------------------------------------------------------------- sublayer record (testing)
 * Per calling thread: between sd_record_begin() and sd_record_end(), every
 * ResnetBlock2D and Transformer2DModel this library runs also writes the
 * outputs of its sublayers BEFORE their residual add into `dev_buf` (caller-
 * owned device memory of `bytes` bytes), as BF16 token matrices:
 *   "h1"    conv1(SiLU(GN1(x))) + b1 + time projection of a resblock [HW, C_out];
 *   "attn1" the self-attention output after its out-projection and bias [HW, C];
 *   "attn2" the same for the cross-attention;
 *   "ff"    the GEGLU feed-forward output after its second linear and bias;
 * and the input each of them saw: "x_h1" (and "x_skip" for a concatenated
 * skip) = the resblock input; "x_attn1", "x_attn2", "x_ff" = the residual
 * stream entering that sublayer (before its LayerNorm).
 * These are the intermediate values of [SD21 section 4]'s block panels, for
 * comparing each sublayer with a reference. The extra outputs are computed by
 * extra launches enqueued on the call's stream (the normal outputs are
 * unchanged). `module` counts resblocks ("h1") or transformers (the others) in
 * the order they ran since sd_record_begin; `block` is the BasicTransformer block.
 * An entry that no longer fits is dropped and sd_record_end returns
 * SD_ERR_CAPACITY. */
typedef struct {
  char name[8];    /* "h1", "attn1", "attn2", "ff", or an input: "x_h1", "x_skip", "x_attn1", ... */
  int32_t module;
  int32_t block;
  int64_t offset;  /* byte offset in dev_buf */
  int64_t rows;    /* tokens (H*W) */
  int64_t cols;    /* channels */
} sd_record_entry;

sd_status sd_record_begin(void* dev_buf, size_t bytes);
sd_status sd_record_end(int32_t* n_entries);
sd_status sd_record_read(sd_record_entry* out, int32_t capacity, int32_t* n);

/* Test hook for the device-side timeout path (the pages have no counterpart).
 * The next n_launches tensor-core GEMM kernels enqueued by this process first
 * make one thread of every CTA wait on a barrier that nothing completes, for
 * at most spin_limit polls (1 .. 2^24); the wait gives up, raises the device
 * error flag in the workspace header and makes every role of the CTA skip its
 * work, so the kernel loads nothing, computes nothing, writes no output (the
 * output buffer keeps stale values) and releases its tensor memory before it
 * returns. sd_query_device_status then reports SD_ERR_DEVICE_TIMEOUT.
 * n_launches = 0 cancels. Process-wide. */
sd_status sd_debug_inject_timeout(int32_t n_launches, int32_t spin_limit);

/* Kernel launches issued by this library in this process so far. */
int64_t sd_launch_count(void);

const char* sd_status_string(sd_status s);

/* Library version string ("sd-b200 <major>.<minor>"). */
const char* sd_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SD_API_H */
