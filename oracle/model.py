"""Blocks and the full U-Net denoiser step, float64 (test infrastructure only).

Topology sources (page title, section):
* "Stable Diffusion 2.1 Base 宏观架构", section 3 (完整 U-Net 多尺度拓扑): Down 0-2
  with ResNet x2 + CrossAttn at 320x96^2, 640x48^2, 1280x24^2; Down 3 ResNet x2
  at 1280x12^2; Mid ResNet + CrossAttn; Up 0 ResNet x3 (no attention) at
  1280x12^2; Up 1-3 ResNet x3 + CrossAttn at 1280x24^2, 640x48^2, 320x96^2;
  skips 320x96^2, 640x48^2, 1280x24^2, 1280x12^2; Conv_in 4->320,
  Conv_out 320->4, layers_per_block = 2.
* "Stable Diffusion XL Inpainting 宏观架构", section 3: the three-level variant
  (320x128^2 ResNet only, 640x64^2 and 1280x32^2 with CrossAttn), 9-channel
  input.
* Section 4 of both pages: ResnetBlock2D = GroupNorm + SiLU + Conv, add time
  embedding, GroupNorm + Dropout + Conv, residual / shortcut add;
  Transformer2DModel = Norm -> self-attention (Q = K = V = image tokens),
  Norm -> cross-attention (K = V = context), Norm -> GEGLU, residual after every
  sublayer; H x W flattened into a token sequence.
* Tutorial page (bfzx365.com): ResNetBlock paragraph (GSC, then add the
  SiLU + Linear time embedding, then GSC, then add the skip input); Spatial
  Transformer bullets (GroupNorm + Linear/Conv + BasicTransformer Blocks +
  Linear/Conv, with the block input added back); DownSample and UpSample bullets.

Readings where the pages are silent (each is listed with the design notes):
GroupNorm and LayerNorm eps 1e-5, 32 groups, biased variance; Q/K/V projections
without bias, out-projection / proj_in / proj_out / FF with bias; head_dim 64;
no attention mask; GEGLU value half first, exact-erf GELU; the 12-entry skip
stack popped last-in-first-out with concatenation order [h, skip]; symmetric
padding 1 for the stride-2 convolution.

Parity unpinned: the absolute output values of ``resblock``, ``transformer``
and ``unet_step``. No page prints a numeric output of a block or of the step,
so these compositions are pinned only through their parts (every op in
``ops`` is pinned), identities (zeroed sublayers reduce a block to a known
function), the pages' shapes and parameter totals.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

from .ops import (group_norm, silu, conv2d, upsample_nearest2x, linear, layer_norm,
                  attention, geglu_ff, timestep_embedding)


@dataclass(frozen=True)
class UNetConfig:
    in_channels: int = 4
    out_channels: int = 4
    block_channels: tuple = (320, 640, 1280, 1280)
    attn_depth: tuple = (1, 1, 1, 0)
    layers_per_block: int = 2
    mid_depth: int = 1
    head_dim: int = 64
    ctx_len: int = 77
    ctx_dim: int = 1024
    time_proj_dim: int = 320
    temb_dim: int = 1280
    groups: int = 32
    eps: float = 1e-5
    # SDXL added conditioning: a pooled text vector of add_text_dim values and
    # add_time_ids scalars (original size, crop offset, target size), each
    # Fourier-encoded to add_time_dim values like the timestep; 0 = none.
    add_text_dim: int = 0
    add_time_ids: int = 0
    add_time_dim: int = 256

    @property
    def add_embed_dim(self) -> int:
        return self.add_text_dim + self.add_time_ids * self.add_time_dim if self.add_text_dim else 0


SD21_BASE = UNetConfig()
SDXL_INPAINT = UNetConfig(in_channels=9, block_channels=(320, 640, 1280), attn_depth=(0, 2, 10),
                          mid_depth=10, ctx_dim=2048, add_text_dim=1280, add_time_ids=6)


# --------------------------------------------------------------------------- parameter tables
# Each entry: (name, shape, kind, fan_in); kind in weight | bias | norm_gamma | norm_beta.

def enumerate_time_mlp_params(prefix="time", proj_dim=320, temb_dim=1280):
    return [
        (f"{prefix}.lin1.weight", (temb_dim, proj_dim), "weight", proj_dim),
        (f"{prefix}.lin1.bias", (temb_dim,), "bias", proj_dim),
        (f"{prefix}.lin2.weight", (temb_dim, temb_dim), "weight", temb_dim),
        (f"{prefix}.lin2.bias", (temb_dim,), "bias", temb_dim),
    ]


def enumerate_resblock_params(prefix, c_in, c_out, temb_dim=1280):
    p = [
        (f"{prefix}.norm1.gamma", (c_in,), "norm_gamma", 0),
        (f"{prefix}.norm1.beta", (c_in,), "norm_beta", 0),
        (f"{prefix}.conv1.weight", (c_out, c_in, 3, 3), "weight", c_in * 9),
        (f"{prefix}.conv1.bias", (c_out,), "bias", c_in * 9),
        (f"{prefix}.temb.weight", (c_out, temb_dim), "weight", temb_dim),
        (f"{prefix}.temb.bias", (c_out,), "bias", temb_dim),
        (f"{prefix}.norm2.gamma", (c_out,), "norm_gamma", 0),
        (f"{prefix}.norm2.beta", (c_out,), "norm_beta", 0),
        (f"{prefix}.conv2.weight", (c_out, c_out, 3, 3), "weight", c_out * 9),
        (f"{prefix}.conv2.bias", (c_out,), "bias", c_out * 9),
    ]
    if c_in != c_out:
        p += [
            (f"{prefix}.skip.weight", (c_out, c_in, 1, 1), "weight", c_in),
            (f"{prefix}.skip.bias", (c_out,), "bias", c_in),
        ]
    return p


def enumerate_transformer_params(prefix, c, depth, ctx_dim):
    p = [
        (f"{prefix}.norm.gamma", (c,), "norm_gamma", 0),
        (f"{prefix}.norm.beta", (c,), "norm_beta", 0),
        (f"{prefix}.proj_in.weight", (c, c), "weight", c),
        (f"{prefix}.proj_in.bias", (c,), "bias", c),
    ]
    for d in range(depth):
        b = f"{prefix}.blocks.{d}"
        p += [
            (f"{b}.ln1.gamma", (c,), "norm_gamma", 0),
            (f"{b}.ln1.beta", (c,), "norm_beta", 0),
            (f"{b}.attn1.q.weight", (c, c), "weight", c),
            (f"{b}.attn1.k.weight", (c, c), "weight", c),
            (f"{b}.attn1.v.weight", (c, c), "weight", c),
            (f"{b}.attn1.out.weight", (c, c), "weight", c),
            (f"{b}.attn1.out.bias", (c,), "bias", c),
            (f"{b}.ln2.gamma", (c,), "norm_gamma", 0),
            (f"{b}.ln2.beta", (c,), "norm_beta", 0),
            (f"{b}.attn2.q.weight", (c, c), "weight", c),
            (f"{b}.attn2.k.weight", (c, ctx_dim), "weight", ctx_dim),
            (f"{b}.attn2.v.weight", (c, ctx_dim), "weight", ctx_dim),
            (f"{b}.attn2.out.weight", (c, c), "weight", c),
            (f"{b}.attn2.out.bias", (c,), "bias", c),
            (f"{b}.ln3.gamma", (c,), "norm_gamma", 0),
            (f"{b}.ln3.beta", (c,), "norm_beta", 0),
            (f"{b}.ff.w1.weight", (8 * c, c), "weight", c),
            (f"{b}.ff.w1.bias", (8 * c,), "bias", c),
            (f"{b}.ff.w2.weight", (c, 4 * c), "weight", 4 * c),
            (f"{b}.ff.w2.bias", (c,), "bias", 4 * c),
        ]
    p += [
        (f"{prefix}.proj_out.weight", (c, c), "weight", c),
        (f"{prefix}.proj_out.bias", (c,), "bias", c),
    ]
    return p


def enumerate_conv_params(prefix, c_in, c_out, k=3):
    return [
        (f"{prefix}.weight", (c_out, c_in, k, k), "weight", c_in * k * k),
        (f"{prefix}.bias", (c_out,), "bias", c_in * k * k),
    ]


def _skip_channels(cfg: UNetConfig):
    """Channel count of each skip-stack entry in push order."""
    ch = cfg.block_channels
    L = len(ch)
    s = [ch[0]]
    for lvl in range(L):
        s += [ch[lvl]] * cfg.layers_per_block
        if lvl < L - 1:
            s.append(ch[lvl])
    return s


def enumerate_unet_params(cfg: UNetConfig = SD21_BASE):
    ch = cfg.block_channels
    L = len(ch)
    p = enumerate_time_mlp_params("time", cfg.time_proj_dim, cfg.temb_dim)
    if cfg.add_embed_dim:
        p += enumerate_time_mlp_params("add", cfg.add_embed_dim, cfg.temb_dim)
    p += enumerate_conv_params("conv_in", cfg.in_channels, ch[0])
    c_prev = ch[0]
    for lvl in range(L):
        for i in range(cfg.layers_per_block):
            p += enumerate_resblock_params(f"down.{lvl}.res.{i}", c_prev, ch[lvl], cfg.temb_dim)
            c_prev = ch[lvl]
            if cfg.attn_depth[lvl] > 0:
                p += enumerate_transformer_params(f"down.{lvl}.attn.{i}", ch[lvl], cfg.attn_depth[lvl],
                                                  cfg.ctx_dim)
        if lvl < L - 1:
            p += enumerate_conv_params(f"down.{lvl}.down", ch[lvl], ch[lvl])
    p += enumerate_resblock_params("mid.res.0", ch[-1], ch[-1], cfg.temb_dim)
    p += enumerate_transformer_params("mid.attn.0", ch[-1], cfg.mid_depth, cfg.ctx_dim)
    p += enumerate_resblock_params("mid.res.1", ch[-1], ch[-1], cfg.temb_dim)
    skips = _skip_channels(cfg)
    c_prev = ch[-1]
    for up in range(L):
        lvl = L - 1 - up
        for i in range(cfg.layers_per_block + 1):
            c_skip = skips.pop()
            p += enumerate_resblock_params(f"up.{up}.res.{i}", c_prev + c_skip, ch[lvl], cfg.temb_dim)
            c_prev = ch[lvl]
            if cfg.attn_depth[lvl] > 0:
                p += enumerate_transformer_params(f"up.{up}.attn.{i}", ch[lvl], cfg.attn_depth[lvl],
                                                  cfg.ctx_dim)
        if up < L - 1:
            p += enumerate_conv_params(f"up.{up}.up", ch[lvl], ch[lvl])
    p += [
        ("out.norm.gamma", (ch[0],), "norm_gamma", 0),
        ("out.norm.beta", (ch[0],), "norm_beta", 0),
    ]
    p += enumerate_conv_params("conv_out", ch[0], cfg.out_channels)
    return p


# --------------------------------------------------------------------------- blocks

def _w(params, name):
    return np.asarray(params[name], dtype=np.float64)


def time_mlp(params, t: float, prefix="time", proj_dim=320):
    """temb = W2 SiLU(W1 phi(t) + b1) + b2 (sinusoid phi, then Linear -> SiLU ->
    Linear; tutorial page, time-embedding paragraphs)."""
    phi = timestep_embedding(t, proj_dim)[None, :]
    h = linear(phi, _w(params, f"{prefix}.lin1.weight"), _w(params, f"{prefix}.lin1.bias"))
    h = linear(silu(h), _w(params, f"{prefix}.lin2.weight"), _w(params, f"{prefix}.lin2.bias"))
    return h[0]


def add_embedding(params, text, time_ids, cfg: UNetConfig, prefix="add"):
    """SDXL added conditioning (tutorial page, SDXL conditioning paragraphs:
    the image-size, crop and target-size conditions are Fourier-encoded like the
    timestep and concatenated after the pooled text embedding, 2816 values for
    SDXL): a = [text | phi(v_0) | ... | phi(v_5)], then the same
    Linear -> SiLU -> Linear shape as the time MLP; the result is added to temb."""
    parts = [np.asarray(text, dtype=np.float64).reshape(-1)]
    for v in time_ids:
        parts.append(timestep_embedding(float(v), cfg.add_time_dim))
    a = np.concatenate(parts)[None, :]
    assert a.shape[1] == cfg.add_embed_dim
    h = linear(a, _w(params, f"{prefix}.lin1.weight"), _w(params, f"{prefix}.lin1.bias"))
    h = linear(silu(h), _w(params, f"{prefix}.lin2.weight"), _w(params, f"{prefix}.lin2.bias"))
    return h[0]


def resblock_h1(x, temb, params, prefix, groups=32, eps=1e-5):
    """The first half of a ResnetBlock2D: h1 = Conv1(SiLU(GN1(x))) + (W_t SiLU(temb) + b_t)
    broadcast over H, W."""
    x = np.asarray(x, dtype=np.float64)
    h = conv2d(silu(group_norm(x, _w(params, f"{prefix}.norm1.gamma"), _w(params, f"{prefix}.norm1.beta"),
                               groups, eps)),
               _w(params, f"{prefix}.conv1.weight"), _w(params, f"{prefix}.conv1.bias"), 1, 1)
    tp = linear(silu(np.asarray(temb, dtype=np.float64))[None, :], _w(params, f"{prefix}.temb.weight"),
                _w(params, f"{prefix}.temb.bias"))[0]
    return h + tp[:, None, None]


def resblock(x, temb, params, prefix, groups=32, eps=1e-5, record=None):
    """ResnetBlock2D on x [C_in, H, W] with temb [temb_dim].

    h = Conv1(SiLU(GN1(x))) + (W_t SiLU(temb) + b_t) broadcast over H, W;
    y = s(x) + Conv2(SiLU(GN2(h))), s = identity if C_in = C_out else a 1x1
    conv; Dropout is the identity. (Section 4 of the SD2.1 page; ResNetBlock
    paragraph of the tutorial page.)"""
    x = np.asarray(x, dtype=np.float64)
    h = resblock_h1(x, temb, params, prefix, groups, eps)
    if record is not None:
        record[f"{prefix}.h1"] = h
    h2 = conv2d(silu(group_norm(h, _w(params, f"{prefix}.norm2.gamma"), _w(params, f"{prefix}.norm2.beta"),
                                groups, eps)),
                _w(params, f"{prefix}.conv2.weight"), _w(params, f"{prefix}.conv2.bias"), 1, 1)
    if f"{prefix}.skip.weight" in params:
        s = conv2d(x, _w(params, f"{prefix}.skip.weight"), _w(params, f"{prefix}.skip.bias"), 1, 0)
    else:
        s = x
    return s + h2


def self_attention_sublayer(t, params, b, head_dim=64, ln_eps=1e-5):
    """Out-projection of SelfAttn(LN1(t)) of BasicTransformer block ``b`` (before the residual add)."""
    n1 = layer_norm(t, _w(params, f"{b}.ln1.gamma"), _w(params, f"{b}.ln1.beta"), ln_eps)
    a1 = attention(linear(n1, _w(params, f"{b}.attn1.q.weight"), None),
                   linear(n1, _w(params, f"{b}.attn1.k.weight"), None),
                   linear(n1, _w(params, f"{b}.attn1.v.weight"), None), head_dim)
    return linear(a1, _w(params, f"{b}.attn1.out.weight"), _w(params, f"{b}.attn1.out.bias"))


def cross_attention_sublayer(t, ctx, params, b, head_dim=64, ln_eps=1e-5):
    """Out-projection of CrossAttn(LN2(t), ctx) of block ``b`` (before the residual add)."""
    n2 = layer_norm(t, _w(params, f"{b}.ln2.gamma"), _w(params, f"{b}.ln2.beta"), ln_eps)
    a2 = attention(linear(n2, _w(params, f"{b}.attn2.q.weight"), None),
                   linear(ctx, _w(params, f"{b}.attn2.k.weight"), None),
                   linear(ctx, _w(params, f"{b}.attn2.v.weight"), None), head_dim)
    return linear(a2, _w(params, f"{b}.attn2.out.weight"), _w(params, f"{b}.attn2.out.bias"))


def ff_sublayer(t, params, b, ln_eps=1e-5):
    """GEGLU feed-forward of LN3(t) of block ``b`` (before the residual add)."""
    n3 = layer_norm(t, _w(params, f"{b}.ln3.gamma"), _w(params, f"{b}.ln3.beta"), ln_eps)
    return geglu_ff(n3, _w(params, f"{b}.ff.w1.weight"), _w(params, f"{b}.ff.w1.bias"),
                    _w(params, f"{b}.ff.w2.weight"), _w(params, f"{b}.ff.w2.bias"))


def transformer(x, ctx, params, prefix, depth, head_dim=64, groups=32, gn_eps=1e-5, ln_eps=1e-5,
                record=None):
    """Transformer2DModel on x [C, H, W] with context ctx [77, ctx_dim].

    t = proj_in(GN(x)) as tokens [H*W, C] (row-major pixel order); then, depth
    times: t += SelfAttn(LN1(t)); t += CrossAttn(LN2(t), ctx); t += FF(LN3(t));
    finally y = x + proj_out(t) reshaped back to [C, H, W]."""
    x = np.asarray(x, dtype=np.float64)
    ctx = np.asarray(ctx, dtype=np.float64)
    C, H, W = x.shape
    g = group_norm(x, _w(params, f"{prefix}.norm.gamma"), _w(params, f"{prefix}.norm.beta"), groups, gn_eps)
    t = linear(g.reshape(C, H * W).T, _w(params, f"{prefix}.proj_in.weight"), _w(params, f"{prefix}.proj_in.bias"))
    for d in range(depth):
        b = f"{prefix}.blocks.{d}"
        o1 = self_attention_sublayer(t, params, b, head_dim, ln_eps)
        t = t + o1
        o2 = cross_attention_sublayer(t, ctx, params, b, head_dim, ln_eps)
        t = t + o2
        f = ff_sublayer(t, params, b, ln_eps)
        t = t + f
        if record is not None:
            record[f"{b}.attn1"] = o1
            record[f"{b}.attn2"] = o2
            record[f"{b}.ff"] = f
    y = linear(t, _w(params, f"{prefix}.proj_out.weight"), _w(params, f"{prefix}.proj_out.bias"))
    return x + y.T.reshape(C, H, W)


def downsample(x, params, prefix):
    """Stride-2 3x3 convolution with padding 1 (DownSample bullet)."""
    return conv2d(np.asarray(x, dtype=np.float64), _w(params, f"{prefix}.weight"), _w(params, f"{prefix}.bias"), 2, 1)


def upsample(x, params, prefix):
    """Nearest 2x interpolation, then a 3x3 stride-1 convolution (UpSample bullet)."""
    return conv2d(upsample_nearest2x(np.asarray(x, dtype=np.float64)), _w(params, f"{prefix}.weight"),
                  _w(params, f"{prefix}.bias"), 1, 1)


def conv_in(x, params, prefix="conv_in"):
    """Input convolution, 3x3, stride 1, padding 1 (Conv_in 4->320 / 9->320)."""
    return conv2d(np.asarray(x, dtype=np.float64), _w(params, f"{prefix}.weight"), _w(params, f"{prefix}.bias"), 1, 1)


def unet_stages(latent, t, ctx, params, cfg: UNetConfig = SD21_BASE, add_text=None, add_time_ids=None,
                record=None):
    """The denoiser step as a sequence of modules: yields (name, output) after
    the time embedding, conv_in, every resblock, transformer, resampling conv and
    the output head, in forward order, and each up-path resblock's concatenated
    input as "up.<u>.res.<i>.in"; the last item is ("out", eps).

    h = conv_in(latent), pushed; per level: layers_per_block resblocks (each
    followed by a transformer where the level has attention), each output
    pushed, then a stride-2 downsample (except the last level), pushed; mid
    resblock -> transformer -> resblock; per up level: layers_per_block + 1 times
    pop a skip, concatenate [h, skip] on channels, resblock (+ transformer), then
    a nearest-2x upsample conv (except the last up level); output
    conv_out(SiLU(GN(h))). With SDXL added conditioning the add embedding is
    added to temb before any resblock uses it. ``record`` (a dict) receives
    each block's sublayer outputs under the module's name."""
    ch = cfg.block_channels
    L = len(ch)
    G, eps = cfg.groups, cfg.eps
    temb = time_mlp(params, t, "time", cfg.time_proj_dim)
    if cfg.add_embed_dim:
        temb = temb + add_embedding(params, add_text, add_time_ids, cfg)
    yield "temb", temb
    h = conv_in(latent, params, "conv_in")
    yield "conv_in", h
    skips = [h]
    for lvl in range(L):
        for i in range(cfg.layers_per_block):
            h = resblock(h, temb, params, f"down.{lvl}.res.{i}", G, eps, record)
            yield f"down.{lvl}.res.{i}", h
            if cfg.attn_depth[lvl] > 0:
                h = transformer(h, ctx, params, f"down.{lvl}.attn.{i}", cfg.attn_depth[lvl], cfg.head_dim, G, eps,
                                eps, record)
                yield f"down.{lvl}.attn.{i}", h
            skips.append(h)
        if lvl < L - 1:
            h = downsample(h, params, f"down.{lvl}.down")
            yield f"down.{lvl}.down", h
            skips.append(h)
    h = resblock(h, temb, params, "mid.res.0", G, eps, record)
    yield "mid.res.0", h
    h = transformer(h, ctx, params, "mid.attn.0", cfg.mid_depth, cfg.head_dim, G, eps, eps, record)
    yield "mid.attn.0", h
    h = resblock(h, temb, params, "mid.res.1", G, eps, record)
    yield "mid.res.1", h
    for up in range(L):
        lvl = L - 1 - up
        for i in range(cfg.layers_per_block + 1):
            s = skips.pop()
            h = np.concatenate([h, s], axis=0)
            yield f"up.{up}.res.{i}.in", h
            h = resblock(h, temb, params, f"up.{up}.res.{i}", G, eps, record)
            yield f"up.{up}.res.{i}", h
            if cfg.attn_depth[lvl] > 0:
                h = transformer(h, ctx, params, f"up.{up}.attn.{i}", cfg.attn_depth[lvl], cfg.head_dim, G, eps, eps,
                                record)
                yield f"up.{up}.attn.{i}", h
        if up < L - 1:
            h = upsample(h, params, f"up.{up}.up")
            yield f"up.{up}.up", h
    assert not skips
    h = silu(group_norm(h, _w(params, "out.norm.gamma"), _w(params, "out.norm.beta"), G, eps))
    out = conv2d(h, _w(params, "conv_out.weight"), _w(params, "conv_out.bias"), 1, 1)
    yield "out", out


def unet_step(latent, t, ctx, params, cfg: UNetConfig = SD21_BASE, record_shapes=None, add_text=None,
              add_time_ids=None, record=None):
    """One denoiser timestep: eps = UNet(latent [in_ch, H, W], t, ctx [77, D])
    (and the SDXL added conditioning when the config has it), the modules of
    ``unet_stages`` run in order. ``record_shapes`` (a list) receives the
    shape of every module output."""
    out = None
    for name, h in unet_stages(latent, t, ctx, params, cfg, add_text, add_time_ids, record):
        if record_shapes is not None and name != "temb":
            record_shapes.append((name, h.shape))
        out = h
    return out


def unet_shapes(cfg: UNetConfig = SD21_BASE, height=96, width=96):
    """Shape walk of the step without arithmetic: the skip-stack shapes in push
    order and the resblock input channel counts of the up path."""
    ch = cfg.block_channels
    L = len(ch)
    hw = (height, width)
    skips = [(ch[0],) + hw]
    for lvl in range(L):
        for i in range(cfg.layers_per_block):
            skips.append((ch[lvl],) + hw)
        if lvl < L - 1:
            hw = (hw[0] // 2, hw[1] // 2)
            skips.append((ch[lvl],) + hw)
    stack = list(skips)
    c = ch[-1]
    up_cin = []
    for up in range(L):
        lvl = L - 1 - up
        for i in range(cfg.layers_per_block + 1):
            s = stack.pop()
            up_cin.append(c + s[0])
            c = ch[lvl]
    return skips, up_cin
