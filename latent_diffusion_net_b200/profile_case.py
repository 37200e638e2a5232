"""Run one block of the denoiser a few times through the C ABI, for profilers.

``python -m latent_diffusion_net_b200.profile_case resblock --hw 96 --c 320``
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

import numpy as np
import torch

from . import binding as B
from . import harness as Hn
from . import synth


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("block", choices=["resblock", "transformer"])
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
    else:
        cfg = B.transformer_cfg(hw, hw, C, 1, 77, a.ctx_dim)
        m = Hn.Module("attn", cfg)
    m.load(Hn.generate_canonical([m], a.seed)[0])
    x = Hn.to_dev_bf16(synth.normal_bf16(a.seed, synth.IDX_X, (hw, hw, C)))
    y = torch.empty(hw * hw * C, dtype=torch.bfloat16, device="cuda")
    if a.block == "resblock":
        temb = torch.from_numpy(synth.normal_bf16(a.seed, synth.IDX_CTX, (1280,)).astype(np.float32)).cuda()

        def call():
            B.sd_resblock_fwd(cfg, m.packed_dev, x, None, temb, y, m.ws, m.ws_bytes)
    else:
        ctx = Hn.to_dev_bf16(synth.normal_bf16(a.seed, synth.IDX_CTX, (77, a.ctx_dim)))

        def call():
            B.sd_transformer_fwd(cfg, m.packed_dev, x, ctx, y, m.ws, m.ws_bytes)

    for _ in range(a.warmup):
        call()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record()
    for _ in range(a.iters):
        call()
    t1.record()
    torch.cuda.synchronize()
    status = B.sd_query_device_status(m.ws)
    print(f"{a.block} hw={hw} C={C}: {t0.elapsed_time(t1) / max(a.iters, 1) * 1e3:.1f} us per call, "
          f"device status {status}")
    return 0 if status == 0 else 1


if __name__ == "__main__":
    raise SystemExit(main())
