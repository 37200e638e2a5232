"""Pins for the oracle's blocks and U-Net composition (CPU only).

Shapes and parameter totals come from the pages (tests/golden/*.json); block
identities are exact special cases of the definitions.
"""
import json
import os

import numpy as np
import pytest

import oracle
from oracle import model, ops
from latent_diffusion_net_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def count(table):
    return sum(int(np.prod(s)) for _, s, _, _ in table)


def make_params(table, seed=0, affine_noise=False):
    return {name: synth.param_value(seed, k, shape, kind, fan, affine_noise)
            for k, (name, shape, kind, fan) in enumerate(table)}


# ----------------------------------------------------------------------------- topology

def test_sd21_skip_shapes_match_page():
    g = load("sd21_base_topology.json")
    skips, up_cin = model.unet_shapes(model.SD21_BASE, 96, 96)
    # the page lists one skip shape per level; each must be among the pushed entries of that level
    for shp in g["skip_shapes"]:
        assert tuple(shp) in [tuple(s) for s in skips]
    # level outputs: the last skip pushed at each level's resolution has the level's channel count
    for c, h, w in g["levels"]:
        assert any(s == (c, h, w) for s in skips)
    assert len(skips) == 1 + 4 * g["layers_per_block"] + 3
    assert len(up_cin) == 4 * g["up_resnets_per_level"]
    assert up_cin == [2560, 2560, 2560, 2560, 2560, 1920, 1920, 1280, 960, 960, 640, 640]


def test_sdxl_skip_shapes_match_page():
    g = load("sdxl_inpaint_topology.json")
    skips, _ = model.unet_shapes(model.SDXL_INPAINT, 128, 128)
    for shp in g["skip_shapes"]:
        assert tuple(shp) in [tuple(s) for s in skips]
    assert model.SDXL_INPAINT.in_channels == g["input"][1]


def test_unet_shape_walk_small_model():
    """Run the real composition on a narrow model and check every recorded shape
    against the arithmetic-free shape walk."""
    cfg = model.UNetConfig(block_channels=(64, 64, 128, 128), attn_depth=(1, 1, 1, 0), ctx_dim=64,
                           time_proj_dim=32, temb_dim=64)
    table = model.enumerate_unet_params(cfg)
    p = make_params(table, seed=5)
    lat = synth.normal_bf16(5, synth.IDX_X, (4, 16, 16))
    ctx = synth.normal_bf16(5, synth.IDX_CTX, (77, 64))
    rec = []
    out = model.unet_step(lat, 500.0, ctx, p, cfg, record_shapes=rec)
    assert out.shape == (4, 16, 16)
    assert np.all(np.isfinite(out))
    skips, up_cin = model.unet_shapes(cfg, 16, 16)
    shapes = dict(rec)
    pushed = [shapes["conv_in"]]
    for lvl in range(4):
        for i in range(cfg.layers_per_block):
            pushed.append(shapes.get(f"down.{lvl}.attn.{i}", shapes[f"down.{lvl}.res.{i}"]))
        if lvl < 3:
            pushed.append(shapes[f"down.{lvl}.down"])
    assert [tuple(s) for s in pushed] == [tuple(s) for s in skips]
    ins = [s[0] for name, s in rec if name.endswith(".in")]
    assert ins == up_cin


# ----------------------------------------------------------------------------- parameter totals

def text_encoder_params(layers, hidden, vocab=49408, positions=77, mlp_ratio=4):
    per = 4 * (hidden * hidden + hidden) + 2 * (2 * hidden) \
        + (hidden * mlp_ratio * hidden + mlp_ratio * hidden) + (mlp_ratio * hidden * hidden + hidden)
    return layers * per + vocab * hidden + positions * hidden + 2 * hidden


def test_sd21_param_total_matches_page():
    """U-Net (this enumerator) + OpenCLIP text encoder (23 layers, hidden 1024,
    SD2.1 page section 2) + VAE (167 MB in FP16 on the tutorial page) must round
    to the 1.290B the SD2.1 page reports in its trace evidence."""
    g = load("sd21_base_topology.json")
    unet = count(model.enumerate_unet_params(model.SD21_BASE))
    assert unet == 865_910_724
    te = text_encoder_params(g["text_encoder"]["layers"], g["text_encoder"]["hidden"])
    vae = 167e6 / 2
    total = unet + te + vae
    assert abs(total / 1e9 - g["params_total_billion"]) < 0.0006


def test_sdxl_param_total_matches_page():
    """U-Net with its 2816-d added-conditioning MLP (this enumerator) + both text
    encoders + VAE round to the 3.469B of the SDXL-Inpainting page section 5."""
    g = load("sdxl_inpaint_topology.json")
    table = model.enumerate_unet_params(model.SDXL_INPAINT)
    unet = count(table)
    add = [(n, s) for n, s, _, _ in table if n.startswith("add.")]
    assert add[0][1] == (1280, 2816)  # pooled text 1280 + 6 Fourier-encoded size/crop values x 256
    assert model.SDXL_INPAINT.add_embed_dim == 2816
    total = unet + g["clip_l_params_million"] * 1e6 + g["openclip_bigg_params_million"] * 1e6 \
        + g["vae_fp16_file_mb"] * 1e6 / 2
    assert abs(total / 1e9 - g["params_total_billion"]) < 0.0006


def test_config_param_counts():
    c1 = model.enumerate_time_mlp_params() + model.enumerate_resblock_params("r", 320, 320) \
        + model.enumerate_transformer_params("t", 320, 1, 1024)
    assert count(c1) == 7_015_680
    t = model.enumerate_transformer_params("t", 320, 1, 1024)
    assert not any(n.endswith(("q.bias", "k.bias", "v.bias")) for n, *_ in t)


# ----------------------------------------------------------------------------- block identities

def small_block_params(c_in=64, c_out=64, c=64, depth=1, ctx_dim=96, seed=3, affine=True):
    table = model.enumerate_time_mlp_params("time", 32, 64) + model.enumerate_resblock_params("r", c_in, c_out, 64) \
        + model.enumerate_transformer_params("t", c, depth, ctx_dim)
    return make_params(table, seed, affine)


def test_resblock_zero_conv2_is_identity():
    p = small_block_params()
    p["r.conv2.weight"] = np.zeros_like(p["r.conv2.weight"])
    p["r.conv2.bias"] = np.zeros_like(p["r.conv2.bias"])
    x = synth.normal_bf16(3, 0, (64, 6, 5))
    temb = synth.normal_bf16(3, 1, (64,))
    np.testing.assert_array_equal(oracle.resblock(x, temb, p, "r"), x.astype(np.float64))


def test_resblock_zero_conv1_gives_gn_of_bias():
    """With conv1 = 0, h is the per-channel constant b1 + temb projection; GN2 of
    a per-channel constant within each group is (b - mean_g)/sqrt(var_g + eps)."""
    p = small_block_params()
    p["r.conv1.weight"] = np.zeros_like(p["r.conv1.weight"])
    x = synth.normal_bf16(3, 0, (64, 4, 4))
    temb = synth.normal_bf16(3, 1, (64,))
    rec = {}
    oracle.resblock(x, temb, p, "r", record=rec)
    tp = np.asarray(p["r.temb.weight"], np.float64) @ ops.silu(temb.astype(np.float64)) + p["r.temb.bias"]
    want = (p["r.conv1.bias"] + tp)[:, None, None] * np.ones((1, 4, 4))
    np.testing.assert_allclose(rec["r.h1"], want, atol=1e-12)


def test_resblock_shortcut_path():
    p = small_block_params(c_in=96, c_out=64)
    p["r.conv2.weight"] = np.zeros_like(p["r.conv2.weight"])
    p["r.conv2.bias"] = np.zeros_like(p["r.conv2.bias"])
    x = synth.normal_bf16(3, 0, (96, 5, 5))
    temb = synth.normal_bf16(3, 1, (64,))
    y = oracle.resblock(x, temb, p, "r")
    ws = p["r.skip.weight"][:, :, 0, 0].astype(np.float64)
    want = np.einsum("oc,chw->ohw", ws, x.astype(np.float64)) + p["r.skip.bias"][:, None, None]
    np.testing.assert_allclose(y, want, atol=1e-12)


def test_transformer_zero_proj_out_is_identity():
    p = small_block_params()
    p["t.proj_out.weight"] = np.zeros_like(p["t.proj_out.weight"])
    p["t.proj_out.bias"] = np.zeros_like(p["t.proj_out.bias"])
    x = synth.normal_bf16(4, 0, (64, 4, 6))
    ctx = synth.normal_bf16(4, 1, (77, 96))
    np.testing.assert_array_equal(oracle.transformer(x, ctx, p, "t", 1), x.astype(np.float64))


def test_transformer_zero_sublayers_reduce_to_projections():
    """With every sublayer's output projection zeroed, the block is
    x + proj_out(proj_in(GN(x))) with tokens in row-major pixel order."""
    p = small_block_params()
    for n in ("attn1.out", "attn2.out"):
        p[f"t.blocks.0.{n}.weight"] = np.zeros_like(p[f"t.blocks.0.{n}.weight"])
        p[f"t.blocks.0.{n}.bias"] = np.zeros_like(p[f"t.blocks.0.{n}.bias"])
    p["t.blocks.0.ff.w2.weight"] = np.zeros_like(p["t.blocks.0.ff.w2.weight"])
    p["t.blocks.0.ff.w2.bias"] = np.zeros_like(p["t.blocks.0.ff.w2.bias"])
    x = synth.normal_bf16(4, 0, (64, 3, 5))
    ctx = synth.normal_bf16(4, 1, (77, 96))
    y = oracle.transformer(x, ctx, p, "t", 1)
    g = ops.group_norm(x.astype(np.float64), p["t.norm.gamma"], p["t.norm.beta"], 32, 1e-5)
    want = x.astype(np.float64).copy()
    for i in range(3):
        for j in range(5):
            tok = np.asarray(p["t.proj_in.weight"], np.float64) @ g[:, i, j] + p["t.proj_in.bias"]
            want[:, i, j] += np.asarray(p["t.proj_out.weight"], np.float64) @ tok + p["t.proj_out.bias"]
    np.testing.assert_allclose(y, want, atol=1e-12)


def test_transformer_cross_attention_context_permutation_invariant():
    p = small_block_params()
    x = synth.normal_bf16(6, 0, (64, 4, 4))
    ctx = synth.normal_bf16(6, 1, (77, 96))
    perm = np.random.default_rng(0).permutation(77)
    a = oracle.transformer(x, ctx, p, "t", 1)
    b = oracle.transformer(x, ctx[perm], p, "t", 1)
    np.testing.assert_allclose(a, b, atol=1e-10)


def test_time_mlp_zero_weights():
    table = model.enumerate_time_mlp_params("time", 32, 64)
    p = make_params(table, 1)
    p["time.lin2.weight"] = np.zeros_like(p["time.lin2.weight"])
    np.testing.assert_array_equal(oracle.time_mlp(p, 500.0, "time", 32), p["time.lin2.bias"].astype(np.float64))


# ----------------------------------------------------------------------------- generator

def test_generator_is_counter_based_and_bf16():
    a = synth.normal_bf16_bits(7, 20, 5000)
    b = synth.normal_bf16_bits(7, 20, 3000)
    np.testing.assert_array_equal(a[:3000], b)
    v = synth.bf16_bits_to_f32(a)
    assert abs(v.mean()) < 0.05 and abs(v.std() - 1) < 0.05
    np.testing.assert_array_equal(ops.bf16_round(v), v.astype(np.float64))
    assert not np.array_equal(a, synth.normal_bf16_bits(8, 20, 5000))
    # SplitMix64 reference value: first output of a stream seeded with 0 is 0xE220A8397B1DCDAF
    assert int(synth.splitmix64(np.uint64(0), 0, 1)[0]) == 0xE220A8397B1DCDAF


def test_mask_rectangle_ranges():
    for s in range(20):
        m, (y0, x0, h, w) = synth.mask_rectangle(s)
        assert 0 <= y0 < 64 and 0 <= x0 < 64 and 32 <= h <= 64 and 32 <= w <= 64
        assert m.sum() == h * w and set(np.unique(m)) <= {0.0, 1.0}
