"""Device-side driver of the synthetic workloads through the C ABI.

PyTorch supplies device memory and streams only; every step of the denoiser
runs in the library's kernels, called through ``binding``. Inputs and weights
come from ``synth`` (seeded, BF16-rounded), packed by the library and copied
to the device once.
"""
from __future__ import annotations

from contextlib import nullcontext as _nullcontext

import numpy as np
import torch

from . import binding as B
from . import synth
from .workloads import CTX_LEN, SDXL_TIME_IDS, TIMESTEP, UNETS, WORKLOADS


def to_dev_bf16(a: np.ndarray, device="cuda") -> torch.Tensor:
    """float32 array holding BF16 values -> BF16 device tensor (exact)."""
    bits = synth.f32_to_bf16_bits(np.ascontiguousarray(a, dtype=np.float32))
    t = torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16)
    return t.to(device)


def u16_to_dev(bits: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(device)


def bytes_to_dev(buf: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(buf)).to(device)


def workspace(nbytes: int, device="cuda") -> torch.Tensor:
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


class Module:
    """One packed weight set of a module kind (time / conv / res / attn / unet)."""

    def __init__(self, kind, cfg, conv_kind=None):
        self.kind = kind
        self.cfg = cfg
        self.conv_kind = conv_kind
        if kind == "time":
            self.rows, self.canon_n, self.packed_n = B.sd_time_weight_layout(cfg)
        elif kind == "conv":
            self.rows, self.canon_n, self.packed_n = B.sd_conv_weight_layout(cfg, conv_kind)
        elif kind == "res":
            self.rows, self.canon_n, self.packed_n = B.sd_resblock_weight_layout(cfg)
        elif kind == "attn":
            self.rows, self.canon_n, self.packed_n = B.sd_transformer_weight_layout(cfg)
        elif kind == "unet":
            self.rows, self.canon_n, self.packed_n = B.sd_unet_weight_layout(cfg)
        elif kind == "vae":
            self.rows, self.canon_n, self.packed_n = B.sd_vae_weight_layout(cfg)
        else:
            raise ValueError(kind)
        self.packed_dev = None
        self.ws = None
        self.ws_bytes = 0

    def gen_rows(self):
        return [(r["shape"], r["kind"], r["fan_in"]) for r in self.rows]

    def pack(self, canonical_u16):
        if self.kind == "time":
            return B.sd_time_pack_weights(self.cfg, canonical_u16, self.packed_n)
        if self.kind == "conv":
            return B.sd_conv_pack_weights(self.cfg, self.conv_kind, canonical_u16, self.packed_n)
        if self.kind == "res":
            return B.sd_resblock_pack_weights(self.cfg, canonical_u16, self.packed_n)
        if self.kind == "attn":
            return B.sd_transformer_pack_weights(self.cfg, canonical_u16, self.packed_n)
        if self.kind == "vae":
            return B.sd_vae_pack_weights(self.cfg, canonical_u16, self.packed_n)
        return B.sd_unet_pack_weights(self.cfg, canonical_u16, self.packed_n)

    def load(self, canonical_u16, device="cuda"):
        self.packed_dev = bytes_to_dev(self.pack(canonical_u16), device)
        if self.kind == "time":
            self.ws_bytes = B.sd_time_workspace_size(self.cfg)
        elif self.kind == "conv":
            self.ws_bytes = B.sd_conv_workspace_size(self.cfg, self.conv_kind)
        elif self.kind == "res":
            self.ws_bytes = B.sd_resblock_workspace_size(self.cfg)
        elif self.kind == "attn":
            self.ws_bytes = B.sd_transformer_workspace_size(self.cfg)
        elif self.kind == "vae":
            self.ws_bytes = B.sd_vae_workspace_size(self.cfg)
        else:
            self.ws_bytes = B.sd_unet_workspace_size(self.cfg)
        self.ws = workspace(self.ws_bytes, device)
        return self


def generate_canonical(modules, seed, affine_noise=False):
    """One canonical buffer per module; tensor indices run across the modules
    in order, as in the oracle's enumeration of the same workload."""
    out = []
    base = 0
    for m in modules:
        rows = m.gen_rows()
        out.append(synth.canonical_weights(rows, seed, affine_noise, index_base=base))
        base += len(rows)
    return out


class Workload:
    """Builds the modules, weights and inputs of workload ``wid`` on the device
    and runs one step through the ABI."""

    def __init__(self, wid, device="cuda", affine_noise=False, canonical=None):
        """``canonical``: already generated canonical buffers of this workload's
        modules (the same seed and tables), to skip drawing them again."""
        self.wid = wid
        self.spec = dict(WORKLOADS[wid])
        self.device = device
        s = self.spec
        seed = s["seed"]
        self.modules = []
        if s["kind"] in ("unet", "denoise"):
            self.cfg = B.unet_cfg(height=s["H"], width=s["W"], **UNETS[s["unet"]])
            self.modules = [Module("unet", self.cfg)]
        elif s["kind"] == "vae":
            self.cfg = B.vae_cfg(s["H"], s["W"])
            self.modules = [Module("vae", self.cfg)]
        else:
            self.modules.append(Module("time", B.time_cfg()))
            C, H, W = s["C"], s["H"], s["W"]
            nblocks = 2 if s["kind"] == "stage3" else 1
            for _ in range(nblocks):
                self.modules.append(Module("res", B.resblock_cfg(H, W, C, C)))
                self.modules.append(Module("attn", B.transformer_cfg(H, W, C, s["depth"], CTX_LEN, s["ctx_dim"])))
            if s["kind"] == "stage3":
                self.modules.append(Module("conv", B.conv_cfg(H, W, C, C), B.SD_CONV_DOWNSAMPLE))
            if s["kind"] == "stage4":
                hw = s["inpaint_hw"]
                self.modules.append(Module("conv", B.conv_cfg(hw, hw, 9, 320), B.SD_CONV_IN))
        self.canonical = canonical if canonical is not None else generate_canonical(self.modules, seed, affine_noise)
        for m, c in zip(self.modules, self.canonical):
            m.load(c, device)
        self.inputs = make_inputs(wid)
        self.dev_inputs = {k: to_dev_bf16(v, device) for k, v in self.inputs.items()}
        if s["kind"] == "denoise":
            # the sampler's FP32 latent state, updated in place by every step, and the
            # workload's latent it is reset to before each pass
            self.x_init = torch.from_numpy(self.inputs["x"].reshape(-1).astype(np.float32)).to(device)
            self.dev_inputs["x"] = self.x_init.clone()
            m = self.modules[0]
            m.ws_bytes = B.sd_denoise_workspace_size(self.cfg)
            m.ws = workspace(m.ws_bytes, device)
            self.alphas_cumprod = B.sd_schedule(B.SD_SCHED_LINEAR, 1000, 1e-4, 0.02)
        self._alloc_outputs()

    def _alloc_outputs(self):
        s = self.spec
        d = self.device
        if s["kind"] == "unet":
            self.out = torch.empty(s["H"] * s["W"] * 4, dtype=torch.bfloat16, device=d)
            return
        if s["kind"] == "denoise":
            self.out = self.dev_inputs["x"]
            return
        if s["kind"] == "vae":
            self.out = torch.empty(64 * s["H"] * s["W"] * 3, dtype=torch.bfloat16, device=d)
            return
        C, H, W = s["C"], s["H"], s["W"]
        self.temb = torch.empty(1280, dtype=torch.float32, device=d)
        self.bufs = [torch.empty(H * W * C, dtype=torch.bfloat16, device=d) for _ in range(2)]
        if s["kind"] == "stage3":
            self.out = torch.empty((H // 2) * (W // 2) * C, dtype=torch.bfloat16, device=d)
        else:
            self.out = self.bufs[1]
        if s["kind"] == "stage4":
            hw = s["inpaint_hw"]
            self.out2 = torch.empty(hw * hw * 320, dtype=torch.bfloat16, device=d)

    def step(self, stream=None, latent=None, context=None):
        """Enqueue one pass of the workload on ``stream``; returns the output tensor."""
        s = self.spec
        x = self.dev_inputs["x"] if latent is None else latent
        ctx = self.dev_inputs.get("ctx") if context is None else context
        if s["kind"] == "vae":
            m = self.modules[0]
            B.sd_vae_decode(self.cfg, m.packed_dev, x, self.out, m.ws, m.ws_bytes, stream)
            return self.out
        if s["kind"] == "denoise":
            m = self.modules[0]
            if latent is None:
                # Every pass is the same guided step from the workload's latent. Chained
                # passes would apply the step to its own output: with alpha_bar_prev = 1
                # the state grows by 1/sqrt(alpha_bar_t) (3.6 at t = 500) per pass and
                # within a few passes leaves the range of the fixed-point GroupNorm sums.
                with torch.cuda.stream(stream) if isinstance(stream, torch.cuda.Stream) else _nullcontext():
                    x.copy_(self.x_init)
            B.sd_denoise(self.cfg, m.packed_dev, B.SD_SAMPLER_DDIM, self.alphas_cumprod, [s["timestep"]],
                         s["guidance"], x, None, ctx, self.dev_inputs["ctx_uncond"], None, None, None, None, m.ws,
                         m.ws_bytes, stream)
            return x
        if s["kind"] == "unet":
            m = self.modules[0]
            if self.cfg.add_text_dim:
                B.sd_unet_step_cond(self.cfg, m.packed_dev, x, TIMESTEP, ctx, self.dev_inputs["text"], SDXL_TIME_IDS,
                                    self.out, m.ws, m.ws_bytes, stream)
            else:
                B.sd_unet_step(self.cfg, m.packed_dev, x, TIMESTEP, ctx, self.out, m.ws, m.ws_bytes, stream)
            return self.out
        tm = self.modules[0]
        B.sd_time_embed(tm.cfg, tm.packed_dev, TIMESTEP, self.temb, tm.ws, tm.ws_bytes, stream)
        cur = x
        nblocks = 2 if s["kind"] == "stage3" else 1
        for b in range(nblocks):
            rm, am = self.modules[1 + 2 * b], self.modules[2 + 2 * b]
            B.sd_resblock_fwd(rm.cfg, rm.packed_dev, cur, None, self.temb, self.bufs[0], rm.ws, rm.ws_bytes, stream)
            B.sd_transformer_fwd(am.cfg, am.packed_dev, self.bufs[0], ctx, self.bufs[1], am.ws, am.ws_bytes, stream)
            cur = self.bufs[1]
        if s["kind"] == "stage3":
            dm = self.modules[-1]
            B.sd_conv_fwd(dm.cfg, dm.conv_kind, dm.packed_dev, cur, None, None, self.out, dm.ws, dm.ws_bytes, stream)
        if s["kind"] == "stage4":
            cm = self.modules[-1]
            di = self.dev_inputs
            B.sd_conv_fwd(cm.cfg, cm.conv_kind, cm.packed_dev, di["noisy"], di["masked"], di["mask"], self.out2,
                          cm.ws, cm.ws_bytes, stream)
        return self.out


def make_inputs(wid):
    """Synthetic inputs of workload ``wid`` as float32 NHWC arrays (BF16 values)."""
    s = WORKLOADS[wid]
    seed = s["seed"]
    out = {}
    if s["kind"] == "unet" and UNETS[s["unet"]]["in_channels"] == 9:
        H, W = s["H"], s["W"]
        noisy = synth.normal_bf16(seed, synth.IDX_NOISY, (H, W, 4))
        masked = synth.normal_bf16(seed, synth.IDX_MASKED, (H, W, 4))
        mask = synth.mask_rectangle(seed, H, W)[0].reshape(H, W, 1)
        out["x"] = np.concatenate([noisy, masked, mask], axis=2)
        out["text"] = synth.normal_bf16(seed, synth.IDX_TEXT, (UNETS[s["unet"]]["add_text_dim"],))
    elif s["kind"] in ("unet", "denoise", "vae"):
        out["x"] = synth.normal_bf16(seed, synth.IDX_X, (s["H"], s["W"], 4))
        if s["kind"] == "vae":
            return out  # the decoder has no context
    else:
        out["x"] = synth.normal_bf16(seed, synth.IDX_X, (s["H"], s["W"], s["C"]))
    out["ctx"] = synth.normal_bf16(seed, synth.IDX_CTX, (CTX_LEN, s["ctx_dim"]))
    if s["kind"] == "denoise":
        out["ctx_uncond"] = synth.normal_bf16(seed, synth.IDX_CTX_UNCOND, (CTX_LEN, s["ctx_dim"]))
    if s["kind"] == "stage4":
        hw = s["inpaint_hw"]
        out["noisy"] = synth.normal_bf16(seed, synth.IDX_NOISY, (hw, hw, 4))
        out["masked"] = synth.normal_bf16(seed, synth.IDX_MASKED, (hw, hw, 4))
        out["mask"] = synth.mask_rectangle(seed, hw, hw)[0].reshape(hw, hw, 1)
    return out


def flops(wid):
    """Algorithmic FLOPs of one pass (2MNK per contraction, 4 Nq Nk C per attention)."""
    s = WORKLOADS[wid]

    def conv(hw, ci, co, k=3):
        return 2.0 * hw * co * ci * k * k

    def res(hw, ci, co):
        f = conv(hw, ci, co) + conv(hw, co, co)
        if ci != co:
            f += conv(hw, ci, co, 1)
        return f + 2.0 * 1280 * co

    def tx(hw, C, depth, D):
        f = 2 * (2.0 * hw * C * C)  # proj_in, proj_out
        per = 2.0 * hw * C * 3 * C + 4.0 * hw * hw * C + 2.0 * hw * C * C  # self
        per += 2.0 * hw * C * C + 2.0 * CTX_LEN * D * 2 * C + 4.0 * hw * CTX_LEN * C + 2.0 * hw * C * C  # cross
        per += 2.0 * hw * C * 8 * C + 2.0 * hw * 4 * C * C  # ff
        return f + depth * per

    tm = 2.0 * (320 * 1280 + 1280 * 1280)
    if s["kind"] == "block":
        hw = s["H"] * s["W"]
        return tm + res(hw, s["C"], s["C"]) + tx(hw, s["C"], s["depth"], s["ctx_dim"])
    if s["kind"] == "stage3":
        hw = s["H"] * s["W"]
        C = s["C"]
        return tm + 2 * (res(hw, C, C) + tx(hw, C, s["depth"], s["ctx_dim"])) + conv(hw // 4, C, C)
    if s["kind"] == "stage4":
        hw = s["H"] * s["W"]
        C = s["C"]
        return tm + res(hw, C, C) + tx(hw, C, s["depth"], s["ctx_dim"]) + conv(s["inpaint_hw"] ** 2, 9, 320)
    if s["kind"] == "denoise":
        return 2 * unet_flops(s["H"], s["W"], **UNETS[s["unet"]])
    if s["kind"] == "vae":
        return vae_flops(s["H"], s["W"])
    return unet_flops(s["H"], s["W"], **UNETS[s["unet"]])


def vae_flops(H, W, latent_channels=4, out_channels=3, block_channels=(128, 256, 512, 512), layers_per_block=2):
    """Algorithmic FLOPs of one VAE decode (2MNK per convolution and linear layer,
    4 N^2 C for the single-head attention)."""
    def conv(hw, ci, co, k=3):
        return 2.0 * hw * co * ci * k * k

    def res(hw, ci, co):
        return conv(hw, ci, co) + conv(hw, co, co) + (conv(hw, ci, co, 1) if ci != co else 0.0)

    ch = list(reversed(block_channels))
    hw = H * W
    f = conv(hw, latent_channels, latent_channels, 1) + conv(hw, latent_channels, ch[0])
    f += 2 * res(hw, ch[0], ch[0]) + 4 * 2.0 * hw * ch[0] * ch[0] + 4.0 * hw * hw * ch[0]
    c_prev = ch[0]
    for i, c in enumerate(ch):
        for _ in range(layers_per_block + 1):
            f += res(hw, c_prev, c)
            c_prev = c
        if i < len(ch) - 1:
            hw *= 4
            f += conv(hw, c, c)
    return f + conv(hw, ch[-1], out_channels)


def unet_flops(H, W, in_channels, block_channels, attn_depth, mid_depth, ctx_dim, add_text_dim=0, add_time_ids=0,
               add_time_dim=256, layers_per_block=2, temb_dim=1280, proj_dim=320):
    """Algorithmic FLOPs of one denoiser step of the given shape."""
    def conv(hw, ci, co, k=3):
        return 2.0 * hw * co * ci * k * k

    def res(hw, ci, co):
        f = conv(hw, ci, co) + conv(hw, co, co)
        if ci != co:
            f += conv(hw, ci, co, 1)
        return f + 2.0 * temb_dim * co

    def tx(hw, C, depth):
        f = 2 * (2.0 * hw * C * C)
        per = 2.0 * hw * C * 3 * C + 4.0 * hw * hw * C + 2.0 * hw * C * C
        per += 2.0 * hw * C * C + 2.0 * CTX_LEN * ctx_dim * 2 * C + 4.0 * hw * CTX_LEN * C + 2.0 * hw * C * C
        per += 2.0 * hw * C * 8 * C + 2.0 * hw * 4 * C * C
        return f + depth * per

    ch = block_channels
    L = len(ch)
    f = 2.0 * (proj_dim * temb_dim + temb_dim * temb_dim)
    if add_text_dim:
        f += 2.0 * ((add_text_dim + add_time_ids * add_time_dim) * temb_dim + temb_dim * temb_dim)
    hw = H * W
    f += conv(hw, in_channels, ch[0])
    c_prev = ch[0]
    skips = [ch[0]]
    for lvl in range(L):
        for _ in range(layers_per_block):
            f += res(hw, c_prev, ch[lvl])
            c_prev = ch[lvl]
            if attn_depth[lvl]:
                f += tx(hw, ch[lvl], attn_depth[lvl])
            skips.append(ch[lvl])
        if lvl < L - 1:
            f += conv(hw // 4, ch[lvl], ch[lvl])
            hw //= 4
            skips.append(ch[lvl])
    f += 2 * res(hw, ch[-1], ch[-1]) + tx(hw, ch[-1], mid_depth)
    for up in range(L):
        lvl = L - 1 - up
        for _ in range(layers_per_block + 1):
            cs = skips.pop()
            f += res(hw, c_prev + cs, ch[lvl])
            c_prev = ch[lvl]
            if attn_depth[lvl]:
                f += tx(hw, ch[lvl], attn_depth[lvl])
        if up < L - 1:
            hw *= 4
            f += conv(hw, ch[lvl], ch[lvl])
    f += conv(hw, ch[0], 4)
    return f
