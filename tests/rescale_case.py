"""A transformer case whose self-attention rows rescale their running output at
different key tiles (test infrastructure, oracle side only).

The attention kernel keeps each query row's output relative to a running
maximum and rescales it when a later 128-key tile raises that maximum by more
than 8 in the log2 domain. With the standard N(0, 1/fan_in) weights no row ever
gets there. Scaling the self-attention Q and K weights by a power of two (exact
in BF16) widens the scores until many rows do, at different tiles, so the 32 rows
of one warp disagree. ``divergent_events`` replays that rule on the oracle's
scores, so the tests can check that the case really drives the branch.
"""
import math

import numpy as np

from gpu_util import oracle_params
from latent_diffusion_net_b200 import synth
from oracle import model, ops

SEED = 17
QK_SCALE = 2.0
# (H, W, C, CTAs of the kernel's split schedule or None for one CTA per whole item)
CASES = [(48, 48, 320, None), (64, 64, 640, 296)]


def canonical(C, ctx_dim=1024, qk_scale=QK_SCALE):
    """(rows, canonical BF16 bits) of a depth-1 transformer, attn1 Q/K weights x qk_scale."""
    rows = model.enumerate_transformer_params("t", C, 1, ctx_dim)
    canon = synth.canonical_weights([(s, k, f) for _, s, k, f in rows], SEED, False)
    off = 0
    for name, shape, _, _ in rows:
        n = int(np.prod(shape))
        if name in ("t.blocks.0.attn1.q.weight", "t.blocks.0.attn1.k.weight"):
            v = synth.bf16_bits_to_f32(canon[off:off + n]) * np.float32(qk_scale)
            canon[off:off + n] = synth.f32_to_bf16_bits(v.astype(np.float32))
        off += n
    return rows, canon


def inputs(H, W, C, ctx_dim=1024, ctx_len=77):
    return synth.normal_bf16(SEED, 0, (H, W, C)), synth.normal_bf16(SEED, 1, (ctx_len, ctx_dim))


def divergent_events(H, W, C, ctas, qk_scale=QK_SCALE):
    """(warp-tile events where some row of a 32-row warp rescales, of those the ones
    where the warp's rows disagree), replaying the rescale rule on the oracle's
    self-attention scores. Steps run head-major, then query tile, then key tile;
    with ``ctas`` the steps are cut into equal contiguous ranges (CTA c takes
    [c*steps/ctas, (c+1)*steps/ctas)) and the maximum restarts at every range's
    first step, as it does at every item's first key tile."""
    rows, canon = canonical(C, qk_scale=qk_scale)
    p = oracle_params(rows, canon)
    x, _ = inputs(H, W, C)
    xc = np.asarray(x, np.float64).transpose(2, 0, 1)
    g = ops.group_norm(xc, p["t.norm.gamma"], p["t.norm.beta"], 32, 1e-5)
    t = ops.linear(g.reshape(C, H * W).T, p["t.proj_in.weight"], p["t.proj_in.bias"])
    n1 = ops.layer_norm(t, p["t.blocks.0.ln1.gamma"], p["t.blocks.0.ln1.beta"], 1e-5)
    q = ops.linear(n1, p["t.blocks.0.attn1.q.weight"], None)
    k = ops.linear(n1, p["t.blocks.0.attn1.k.weight"], None)
    N = H * W
    assert N % 128 == 0
    nt = N // 128
    heads = C // 64
    log2e = 1.0 / math.log(2.0)
    # per (head, query tile): the log2-domain maximum of every row over every key tile
    tmax = []
    for h in range(heads):
        s = (q[:, 64 * h:64 * h + 64] @ k[:, 64 * h:64 * h + 64].T) * (log2e / 8.0)
        tmax.append(s.reshape(nt, 128, nt, 128).max(axis=3))  # [q tile, row, k tile]
    steps = heads * nt * nt
    starts = {c * steps // ctas for c in range(ctas)} if ctas else set()
    events = divergent = 0
    m = None
    for st in range(steps):
        item, j = divmod(st, nt)
        h, qi = divmod(item, nt)
        tm = tmax[h][qi, :, j]
        if j == 0 or st in starts:
            m = tm.copy()
            continue
        r = tm > m + 8.0
        m = np.where(r, tm, m)
        w = r.reshape(-1, 32)
        some, every = w.any(axis=1), w.all(axis=1)
        events += int(some.sum())
        divergent += int((some & ~every).sum())
    return events, divergent
