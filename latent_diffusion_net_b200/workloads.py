"""The synthetic workloads (shapes, seeds, value distributions).

Every input is N(0, 1) rounded to BF16; every convolution/linear weight and
bias is N(0, 1/fan_in) rounded to BF16; norm gains are 1 and shifts 0; the
timestep is 500. Activations are NHWC.

1. crossattn_block_320x32: time MLP + ResnetBlock2D 320->320 + Transformer2DModel
   depth 1 (5 heads x 64) at 32x32, context [77, 1024]; seed 0.
2. crossattn_block_320x96: the same block at the SD2.1-base level-0 size 96x96
   (9216 tokens); seed 1.
3. sdxl_level1_stage_640x64: time MLP + 2 x (ResnetBlock2D 640 + Transformer2DModel
   depth 2, 10 heads) at 64x64, context [77, 2048], then a stride-2 downsample;
   seed 2.
4. sdxl_level2_stage_1280x32: time MLP + ResnetBlock2D 1280 + Transformer2DModel
   depth 10 (20 heads) at 32x32, context [77, 2048]; plus the inpaint conv_in
   9->320 on a 128x128 input assembled from a noisy latent, a masked latent and a
   rectangle mask; seed 3.
5. sd21_base_unet_step_96: the whole SD2.1-base-shaped denoiser step on a 96x96
   latent with 4 channels, context [77, 1024]; seed 4.
6. sdxl_inpaint_unet_step_128: the whole SDXL-Inpainting-shaped denoiser step on
   a 128x128 latent: 9 input channels assembled from a noisy latent, a masked
   latent and a rectangle mask; 3 levels (320 without attention, 640 with depth-2
   and 1280 with depth-10 transformers), mid depth 10, context [77, 2048], and
   the added conditioning: a pooled text vector [1280] ~ N(0, 1) and the six
   size/crop values (1024, 1024, 0, 0, 1024, 1024); seed 5.
7. sd21_base_unet_step_64 and 8. sd21_base_unet_step_128: the SD2.1-base step of
   workload 5 (same weights, seed 4) on 64x64 and 128x128 latents: 4096 and 16384
   self-attention tokens at the first level.
9. sd21_base_guided_ddim_step_96: one iteration of a guided sampling loop on the
   workload-5 model and latent: the denoiser with the text context and again
   with an unconditional context [77, 1024] ~ N(0, 1) (seed 4, stream 7), the
   guidance combination (scale 7.5) and a DDIM update at t = 500 on the page's
   linear schedule (0.0001 -> 0.02, 1000 steps).
10. sd21_vae_decode_96: the VAE decoder on the 96x96 latent of workload 5's shape
   (N(0, 1), seed 4) to a 768x768 RGB image; weights N(0, 1/fan_in), seed 6.
"""

WORKLOADS = {
    1: dict(name="crossattn_block_320x32", seed=0, kind="block", H=32, W=32, C=320, depth=1, ctx_dim=1024),
    2: dict(name="crossattn_block_320x96", seed=1, kind="block", H=96, W=96, C=320, depth=1, ctx_dim=1024),
    3: dict(name="sdxl_level1_stage_640x64", seed=2, kind="stage3", H=64, W=64, C=640, depth=2, ctx_dim=2048),
    4: dict(name="sdxl_level2_stage_1280x32", seed=3, kind="stage4", H=32, W=32, C=1280, depth=10, ctx_dim=2048,
            inpaint_hw=128),
    5: dict(name="sd21_base_unet_step_96", seed=4, kind="unet", H=96, W=96, ctx_dim=1024, unet="sd21"),
    6: dict(name="sdxl_inpaint_unet_step_128", seed=5, kind="unet", H=128, W=128, ctx_dim=2048, unet="sdxl_inpaint"),
    7: dict(name="sd21_base_unet_step_64", seed=4, kind="unet", H=64, W=64, ctx_dim=1024, unet="sd21"),
    8: dict(name="sd21_base_unet_step_128", seed=4, kind="unet", H=128, W=128, ctx_dim=1024, unet="sd21"),
    9: dict(name="sd21_base_guided_ddim_step_96", seed=4, kind="denoise", H=96, W=96, ctx_dim=1024, unet="sd21",
            guidance=7.5, timestep=500),
    10: dict(name="sd21_vae_decode_96", seed=6, kind="vae", H=96, W=96),
}

# U-Net shapes (SD2.1 architecture page section 3; SDXL-Inpainting architecture
# page section 3; the SDXL added conditioning of the tutorial page).
UNETS = {
    "sd21": dict(in_channels=4, block_channels=(320, 640, 1280, 1280), attn_depth=(1, 1, 1, 0), mid_depth=1,
                 ctx_dim=1024, add_text_dim=0, add_time_ids=0),
    "sdxl_inpaint": dict(in_channels=9, block_channels=(320, 640, 1280), attn_depth=(0, 2, 10), mid_depth=10,
                         ctx_dim=2048, add_text_dim=1280, add_time_ids=6),
}
SDXL_TIME_IDS = (1024.0, 1024.0, 0.0, 0.0, 1024.0, 1024.0)  # original size, crop top-left, target size
TIMESTEP = 500.0
CTX_LEN = 77
