"""The VAE decoder that turns a denoised latent into pixels, float64 (test
infrastructure only; see the package docstring).

Sources (page title, section):
* "Stable Diffusion 2.1 Base 宏观架构" section 5 and "Stable Diffusion XL
  Inpainting 宏观架构" section 5 (VAE boundary): the decoder is a MidBlock
  followed by four UpDecoder blocks, upsampling x8 in space ([1, 4, 96, 96] ->
  [1, 3, 768, 768]; [1, 4, 128, 128] -> [1, 3, 1024, 1024]), with the channel
  ladder 512 -> 512 -> 256 -> 128 and 4 latent channels.
* SD/SDXL tutorial page (bfzx365.com): the latent is divided by the scaling
  factor 0.18215 before the decoder (the "rescaling coefficient" paragraph), and
  the VAE weighs 167 MB in FP16 (the SDXL component-size paragraph).
* The decoder's blocks reuse the U-Net's operators (section 4 of the SD2.1
  page): GroupNorm + SiLU + 3x3 convolution, residual blocks with a 1x1 shortcut
  where the width changes, nearest-2x upsampling followed by a 3x3 convolution.

Readings where the pages are silent (listed with the design notes): a 1x1
post-quantisation convolution on the 4 latent channels first; every block has
layers_per_block + 1 = 3 residual blocks, as the U-Net's up path does; the
first three UpDecoder blocks end with the upsampling convolution; the MidBlock
is ResBlock -> single-head self-attention over the H*W tokens (GroupNorm, then
Q/K/V/out linear layers with biases, scale 1/sqrt(C), residual) -> ResBlock; the
residual blocks have no time embedding; GroupNorm uses 32 groups and eps 1e-5 as
everywhere else; the output head is GroupNorm + SiLU + 3x3 conv to 3 channels.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np

from .model import _w, enumerate_conv_params
from .ops import conv2d, group_norm, linear, silu, upsample_nearest2x


@dataclass(frozen=True)
class VAEConfig:
    latent_channels: int = 4
    out_channels: int = 3
    block_channels: tuple = (128, 256, 512, 512)  # encoder order; the decoder walks it backwards
    layers_per_block: int = 2
    groups: int = 32
    eps: float = 1e-5
    scaling_factor: float = 0.18215


SD_VAE = VAEConfig()


def enumerate_vae_resblock_params(prefix, c_in, c_out):
    p = [
        (f"{prefix}.norm1.gamma", (c_in,), "norm_gamma", 0),
        (f"{prefix}.norm1.beta", (c_in,), "norm_beta", 0),
        (f"{prefix}.conv1.weight", (c_out, c_in, 3, 3), "weight", c_in * 9),
        (f"{prefix}.conv1.bias", (c_out,), "bias", c_in * 9),
        (f"{prefix}.norm2.gamma", (c_out,), "norm_gamma", 0),
        (f"{prefix}.norm2.beta", (c_out,), "norm_beta", 0),
        (f"{prefix}.conv2.weight", (c_out, c_out, 3, 3), "weight", c_out * 9),
        (f"{prefix}.conv2.bias", (c_out,), "bias", c_out * 9),
    ]
    if c_in != c_out:
        p += [(f"{prefix}.skip.weight", (c_out, c_in, 1, 1), "weight", c_in),
              (f"{prefix}.skip.bias", (c_out,), "bias", c_in)]
    return p


def enumerate_vae_attention_params(prefix, c):
    return [
        (f"{prefix}.norm.gamma", (c,), "norm_gamma", 0),
        (f"{prefix}.norm.beta", (c,), "norm_beta", 0),
        (f"{prefix}.q.weight", (c, c), "weight", c),
        (f"{prefix}.k.weight", (c, c), "weight", c),
        (f"{prefix}.v.weight", (c, c), "weight", c),
        (f"{prefix}.q.bias", (c,), "bias", c),
        (f"{prefix}.k.bias", (c,), "bias", c),
        (f"{prefix}.v.bias", (c,), "bias", c),
        (f"{prefix}.out.weight", (c, c), "weight", c),
        (f"{prefix}.out.bias", (c,), "bias", c),
    ]


def enumerate_vae_decoder_params(cfg: VAEConfig = SD_VAE):
    ch = list(reversed(cfg.block_channels))  # 512, 512, 256, 128
    p = enumerate_conv_params("post_quant_conv", cfg.latent_channels, cfg.latent_channels, 1)
    p += enumerate_conv_params("conv_in", cfg.latent_channels, ch[0])
    p += enumerate_vae_resblock_params("mid.res.0", ch[0], ch[0])
    p += enumerate_vae_attention_params("mid.attn", ch[0])
    p += enumerate_vae_resblock_params("mid.res.1", ch[0], ch[0])
    c_prev = ch[0]
    for i, c in enumerate(ch):
        for j in range(cfg.layers_per_block + 1):
            p += enumerate_vae_resblock_params(f"up.{i}.res.{j}", c_prev, c)
            c_prev = c
        if i < len(ch) - 1:
            p += enumerate_conv_params(f"up.{i}.up", c, c)
    p += [("out.norm.gamma", (ch[-1],), "norm_gamma", 0), ("out.norm.beta", (ch[-1],), "norm_beta", 0)]
    p += enumerate_conv_params("conv_out", ch[-1], cfg.out_channels)
    return p


def enumerate_vae_encoder_params(cfg: VAEConfig = SD_VAE):
    """The encoder's table, shapes only (it is outside the decoder path; used to
    check the VAE's total size against the pages): conv_in 3 -> 128, four down
    blocks of layers_per_block residual blocks (stride-2 convolution after the
    first three), the same MidBlock, GroupNorm + conv to 2 x latent channels
    (mean and log-variance), and a 1x1 quantisation convolution."""
    ch = list(cfg.block_channels)
    p = enumerate_conv_params("enc.conv_in", 3, ch[0])
    c_prev = ch[0]
    for i, c in enumerate(ch):
        for j in range(cfg.layers_per_block):
            p += enumerate_vae_resblock_params(f"enc.down.{i}.res.{j}", c_prev, c)
            c_prev = c
        if i < len(ch) - 1:
            p += enumerate_conv_params(f"enc.down.{i}.down", c, c)
    p += enumerate_vae_resblock_params("enc.mid.res.0", ch[-1], ch[-1])
    p += enumerate_vae_attention_params("enc.mid.attn", ch[-1])
    p += enumerate_vae_resblock_params("enc.mid.res.1", ch[-1], ch[-1])
    p += [("enc.out.norm.gamma", (ch[-1],), "norm_gamma", 0), ("enc.out.norm.beta", (ch[-1],), "norm_beta", 0)]
    p += enumerate_conv_params("enc.conv_out", ch[-1], 2 * cfg.latent_channels)
    p += enumerate_conv_params("quant_conv", 2 * cfg.latent_channels, 2 * cfg.latent_channels, 1)
    return p


def vae_resblock(x, params, prefix, groups=32, eps=1e-5):
    """y = s(x) + Conv2(SiLU(GN2(Conv1(SiLU(GN1(x)))))), s = identity or a 1x1 conv."""
    x = np.asarray(x, dtype=np.float64)
    h = conv2d(silu(group_norm(x, _w(params, f"{prefix}.norm1.gamma"), _w(params, f"{prefix}.norm1.beta"),
                               groups, eps)),
               _w(params, f"{prefix}.conv1.weight"), _w(params, f"{prefix}.conv1.bias"), 1, 1)
    h = conv2d(silu(group_norm(h, _w(params, f"{prefix}.norm2.gamma"), _w(params, f"{prefix}.norm2.beta"),
                               groups, eps)),
               _w(params, f"{prefix}.conv2.weight"), _w(params, f"{prefix}.conv2.bias"), 1, 1)
    if f"{prefix}.skip.weight" in params:
        s = conv2d(x, _w(params, f"{prefix}.skip.weight"), _w(params, f"{prefix}.skip.bias"), 1, 0)
    else:
        s = x
    return s + h


def vae_attention(x, params, prefix, groups=32, eps=1e-5):
    """Single-head self-attention over the H*W tokens with a residual:
    t = GN(x) as tokens; y = x + (softmax(Q K^T / sqrt(C)) V) W_o^T + b_o."""
    x = np.asarray(x, dtype=np.float64)
    C, H, W = x.shape
    t = group_norm(x, _w(params, f"{prefix}.norm.gamma"), _w(params, f"{prefix}.norm.beta"), groups,
                   eps).reshape(C, H * W).T
    q = linear(t, _w(params, f"{prefix}.q.weight"), _w(params, f"{prefix}.q.bias"))
    k = linear(t, _w(params, f"{prefix}.k.weight"), _w(params, f"{prefix}.k.bias"))
    v = linear(t, _w(params, f"{prefix}.v.weight"), _w(params, f"{prefix}.v.bias"))
    s = (q @ k.T) / math.sqrt(C)
    s -= s.max(axis=1, keepdims=True)
    pr = np.exp(s)
    pr /= pr.sum(axis=1, keepdims=True)
    o = linear(pr @ v, _w(params, f"{prefix}.out.weight"), _w(params, f"{prefix}.out.bias"))
    return x + o.T.reshape(C, H, W)


def vae_stages(z, params, cfg: VAEConfig = SD_VAE):
    """The decode as a sequence of modules: yields (name, output) after the input
    convolutions, each resblock, the attention, each upsampling conv and the
    output head ("out", the image)."""
    z = np.asarray(z, dtype=np.float64) / cfg.scaling_factor
    G, eps = cfg.groups, cfg.eps
    h = conv2d(z, _w(params, "post_quant_conv.weight"), _w(params, "post_quant_conv.bias"), 1, 0)
    h = conv2d(h, _w(params, "conv_in.weight"), _w(params, "conv_in.bias"), 1, 1)
    yield "conv_in", h
    h = vae_resblock(h, params, "mid.res.0", G, eps)
    yield "mid.res.0", h
    h = vae_attention(h, params, "mid.attn", G, eps)
    yield "mid.attn", h
    h = vae_resblock(h, params, "mid.res.1", G, eps)
    yield "mid.res.1", h
    n = len(cfg.block_channels)
    for i in range(n):
        for j in range(cfg.layers_per_block + 1):
            h = vae_resblock(h, params, f"up.{i}.res.{j}", G, eps)
            yield f"up.{i}.res.{j}", h
        if i < n - 1:
            h = conv2d(upsample_nearest2x(h), _w(params, f"up.{i}.up.weight"), _w(params, f"up.{i}.up.bias"), 1, 1)
            yield f"up.{i}.up", h
    h = silu(group_norm(h, _w(params, "out.norm.gamma"), _w(params, "out.norm.beta"), G, eps))
    yield "out", conv2d(h, _w(params, "conv_out.weight"), _w(params, "conv_out.bias"), 1, 1)


def vae_decode(z, params, cfg: VAEConfig = SD_VAE):
    """Latent z [latent_channels, h, w] -> image [out_channels, 8h, 8w]: the
    modules of ``vae_stages`` in order."""
    out = None
    for _, out in vae_stages(z, params, cfg):
        pass
    return out
