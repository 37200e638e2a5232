"""Run one block of the denoiser a few times through the C ABI, for profilers.

Blocks: ``resblock``, ``transformer``, ``upsample`` and ``downsample`` (the
resampling convolutions), ``output`` (GroupNorm + SiLU + conv_out), ``conv_in``
(the 9-channel inpaint entry), ``time`` (the time-embedding MLP and one batch
of resblock time projections), ``vae`` (the VAE decoder on a [hw, hw, 4]
latent: 8x upsampling, GroupNorm in one or two passes depending on the size,
the single-head mid-block attention), ``sampler`` (the fused guidance + DDIM
update of a [hw, hw, 4] latent).

``python profile_case.py resblock --hw 96 --c 320``
runs a ResnetBlock2D (C -> C, time projection from a random embedding) on a
seeded [hw, hw, C] input; ``transformer`` runs a Transformer2DModel (depth 1,
77 context rows of width --ctx-dim). Each iteration is one eager call of the
block's entry point, so a kernel capture with ``-k`` and ``-c`` selects
launches by their order inside the block (the ResnetBlock2D issues GroupNorm,
conv1, GroupNorm, conv2; the Transformer2DModel issues its GroupNorm, the
proj_in GEMM, the QKV GEMM with LayerNorm folded in, self-attention, ...). Prints the mean
time per call measured with CUDA events after the warm-up calls.
"""
from __future__ import annotations

import argparse
import os
import sys

import numpy as np
import torch

sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))

from latent_diffusion_net_b200 import binding as B  # noqa: E402
from latent_diffusion_net_b200 import harness as Hn  # noqa: E402
from latent_diffusion_net_b200 import synth  # noqa: E402


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("block", choices=["resblock", "transformer", "upsample", "downsample", "output", "conv_in",
                                      "time", "vae", "sampler"])
    ap.add_argument("--hw", type=int, default=96, help="latent height = width")
    ap.add_argument("--c", type=int, default=320, help="channels")
    ap.add_argument("--ctx-dim", type=int, default=1024)
    ap.add_argument("--iters", type=int, default=3)
    ap.add_argument("--warmup", type=int, default=1)
    ap.add_argument("--seed", type=int, default=7)
    a = ap.parse_args(argv)
    if not torch.cuda.is_available():
        raise SystemExit("profile_case needs a CUDA device")
    hw, C = a.hw, a.c
    if a.block == "resblock":
        cfg = B.resblock_cfg(hw, hw, C, C)
        m = Hn.Module("res", cfg)
    elif a.block == "transformer":
        cfg = B.transformer_cfg(hw, hw, C, 1, 77, a.ctx_dim)
        m = Hn.Module("attn", cfg)
    elif a.block == "time":
        cfg = B.time_cfg()
        m = Hn.Module("time", cfg)
    elif a.block == "vae":
        cfg = B.vae_cfg(hw, hw)
        m = Hn.Module("vae", cfg)
    elif a.block == "sampler":
        m = None
    else:
        kind = {"upsample": B.SD_CONV_UPSAMPLE, "downsample": B.SD_CONV_DOWNSAMPLE, "output": B.SD_CONV_OUTPUT,
                "conv_in": B.SD_CONV_IN}[a.block]
        cin = 9 if a.block == "conv_in" else C
        cout = {"output": 4, "conv_in": 320}.get(a.block, C)
        cfg = B.conv_cfg(hw, hw, cin, cout)
        m = Hn.Module("conv", cfg, kind)
    if m is not None:
        m.load(Hn.generate_canonical([m], a.seed)[0])
    if a.block == "conv_in":
        x = Hn.to_dev_bf16(synth.normal_bf16(a.seed, synth.IDX_NOISY, (hw, hw, 4)))
        x1 = Hn.to_dev_bf16(synth.normal_bf16(a.seed, synth.IDX_MASKED, (hw, hw, 4)))
        x2 = Hn.to_dev_bf16(synth.mask_rectangle(a.seed, hw, hw)[0].reshape(hw, hw, 1))
    elif a.block in ("vae", "sampler"):
        x = Hn.to_dev_bf16(synth.normal_bf16(a.seed, synth.IDX_X, (hw, hw, 4)))
    else:
        x = Hn.to_dev_bf16(synth.normal_bf16(a.seed, synth.IDX_X, (hw, hw, C)))
    out_elems = {"upsample": 4 * hw * hw * C, "downsample": hw * hw * C // 4, "output": hw * hw * 4,
                 "conv_in": hw * hw * 320, "vae": 64 * hw * hw * 3, "sampler": hw * hw * 4}.get(a.block, hw * hw * C)
    y = torch.empty(out_elems, dtype=torch.bfloat16, device="cuda")
    if a.block == "resblock":
        temb = torch.from_numpy(synth.normal_bf16(a.seed, synth.IDX_CTX, (1280,)).astype(np.float32)).cuda()

        def call():
            B.sd_resblock_fwd(cfg, m.packed_dev, x, None, temb, y, m.ws, m.ws_bytes)
    elif a.block == "transformer":
        ctx = Hn.to_dev_bf16(synth.normal_bf16(a.seed, synth.IDX_CTX, (77, a.ctx_dim)))

        def call():
            B.sd_transformer_fwd(cfg, m.packed_dev, x, ctx, y, m.ws, m.ws_bytes)
    elif a.block == "time":
        temb = torch.empty(1280, dtype=torch.float32, device="cuda")

        def call():
            B.sd_time_embed(cfg, m.packed_dev, 500.0, temb, m.ws, m.ws_bytes)
    elif a.block == "conv_in":
        def call():
            B.sd_conv_fwd(cfg, B.SD_CONV_IN, m.packed_dev, x, x1, x2, y, m.ws, m.ws_bytes)
    elif a.block == "vae":
        def call():
            B.sd_vae_decode(cfg, m.packed_dev, x, y, m.ws, m.ws_bytes)
    elif a.block == "sampler":
        ac = B.sd_schedule(B.SD_SCHED_LINEAR, 1000, 1e-4, 0.02)
        scfg = B.sampler_cfg(B.SD_SAMPLER_DDIM, hw * hw * 4, ac[500], ac[480], guidance=7.5)
        xs = torch.from_numpy(synth.normal_bf16(a.seed, synth.IDX_CTX, (hw * hw * 4,)).astype(np.float32)).cuda()
        eu = Hn.to_dev_bf16(synth.normal_bf16(a.seed, synth.IDX_CTX_UNCOND, (hw * hw * 4,)))

        def call():
            B.sd_sampler_step(scfg, xs, x, eu, None, y)
    else:
        def call():
            B.sd_conv_fwd(cfg, kind, m.packed_dev, x, None, None, y, m.ws, m.ws_bytes)

    for _ in range(a.warmup):
        call()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record()
    for _ in range(a.iters):
        call()
    t1.record()
    torch.cuda.synchronize()
    status = B.sd_query_device_status(m.ws) if m is not None else 0
    print(f"{a.block} hw={hw} C={C}: {t0.elapsed_time(t1) / max(a.iters, 1) * 1e3:.1f} us per call, "
          f"device status {status}")
    return 0 if status == 0 else 1


if __name__ == "__main__":
    raise SystemExit(main())
