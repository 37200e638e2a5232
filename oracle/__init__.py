"""CPU oracle for the Stable-Diffusion U-Net denoiser step (test infrastructure).

This package is test infrastructure only. It is imported by ``tests/``, by
``__graft_entry__.smoke()`` and by the ``cpu_baseline`` / ``--impl reference``
legs of ``bench.py``; the product path never imports, links or runs it.

It is a plain, slow, float64 numpy restatement of what one denoiser timestep
computes, written from the source pages' definitions, with activations kept in
channel-major ``[C, H, W]`` layout (the CUDA path uses NHWC BF16) and sharing
no code with the CUDA path. Library primitives (``numpy.tensordot``, ``@``,
``scipy.special.erf``) serve as single steps; nothing is blocked, fused or
reordered beyond the definitions.

``sampler`` holds the noise schedules, the DDPM / DDIM reverse updates and
classifier-free guidance that sit on either side of the denoiser step; ``vae``
holds the VAE decoder that turns the denoised latent into pixels.

Parity pins: see ``tests/test_oracle_*.py``. Every function here is pinned by
at least one check that does not retype its own formula (brute-force loops,
closed forms, invariants, page-printed shapes and parameter totals). The
absolute output values of a whole block or step are not printed on any page, so
they are pinned only compositionally.
"""
from .ops import (bf16_round, group_norm, silu, conv2d, upsample_nearest2x, linear,
                  layer_norm, attention, gelu, geglu_ff, timestep_embedding)
from .model import (UNetConfig, SD21_BASE, SDXL_INPAINT, enumerate_unet_params,
                    enumerate_resblock_params, enumerate_transformer_params,
                    enumerate_time_mlp_params, time_mlp, resblock, transformer,
                    downsample, upsample, conv_in, unet_step, unet_stages, unet_shapes,
                    add_embedding, resblock_h1, self_attention_sublayer, cross_attention_sublayer,
                    ff_sublayer)
from . import sampler
from . import vae

__all__ = [n for n in dir() if not n.startswith("_")]
