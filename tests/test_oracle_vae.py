"""Pins for the oracle's VAE decoder (CPU only): the page's VAE size and
shapes, and closed forms of its blocks."""
import math

import numpy as np
import pytest

from oracle import vae
from oracle.model import enumerate_unet_params, SD21_BASE
from latent_diffusion_net_b200 import synth


def count(table):
    return sum(int(np.prod(s)) for _, s, _, _ in table)


def params_of(table, seed, affine=False, zero=()):
    out = {}
    for k, (name, shape, kind, fan) in enumerate(table):
        v = synth.param_value(seed, k, shape, kind, fan, affine).astype(np.float64)
        if any(name.startswith(z) for z in zero):
            v = np.zeros(shape)
        out[name] = v
    return out


def test_vae_size_matches_page():
    """Encoder + decoder in FP16 = the 167 MB the tutorial page gives for the VAE;
    the decoder alone keeps the page's channel ladder 512 -> 512 -> 256 -> 128."""
    dec = vae.enumerate_vae_decoder_params()
    enc = vae.enumerate_vae_encoder_params()
    total = count(dec) + count(enc)
    assert abs(total * 2 / 1e6 - 167.0) < 0.5
    convs = [s[0] for n, s, _, _ in dec if n.endswith("conv2.weight")]
    assert [convs[i] for i in (0, 2, 5, 8, 11)] == [512, 512, 512, 256, 128]  # mid, then the four UpDecoder blocks
    # the same enumerator also closes the SD2.1 total: U-Net + text encoder + this VAE ~ 1.290B
    unet = count(enumerate_unet_params(SD21_BASE))
    hidden, layers = 1024, 23
    te = layers * (4 * (hidden * hidden + hidden) + 4 * hidden + (4 * hidden * hidden + 4 * hidden)
                   + (4 * hidden * hidden + hidden)) + 49408 * hidden + 77 * hidden + 2 * hidden
    assert abs((unet + te + total) / 1e9 - 1.290) < 0.0006


def narrow(channels=(32, 32, 64, 64)):
    return vae.VAEConfig(block_channels=channels)


def test_decode_upsamples_by_eight():
    cfg = narrow()
    p = params_of(vae.enumerate_vae_decoder_params(cfg), 3)
    z = synth.normal_bf16(3, 0, (4, 3, 2)).astype(np.float64)
    out = vae.vae_decode(z, p, cfg)
    assert out.shape == (3, 24, 16) and np.all(np.isfinite(out))


def test_resblock_identity_and_shortcut():
    r = np.random.default_rng(1)
    x = r.standard_normal((64, 5, 4))
    t = vae.enumerate_vae_resblock_params("r", 64, 64)
    p = params_of(t, 4, zero=("r.conv2",))
    np.testing.assert_allclose(vae.vae_resblock(x, p, "r"), x, atol=1e-14)
    t = vae.enumerate_vae_resblock_params("r", 64, 32)
    p = params_of(t, 5, zero=("r.conv2",))
    ref = np.einsum("oc,chw->ohw", p["r.skip.weight"][:, :, 0, 0], x) + p["r.skip.bias"][:, None, None]
    np.testing.assert_allclose(vae.vae_resblock(x, p, "r"), ref, atol=1e-12)


def test_attention_single_token_and_uniform_keys():
    """One token: the softmax has one key, so the block adds W_o v + b_o with
    v = W_v GN(x) + b_v. Keys all equal (W_k = 0, b_k = 0): every query
    averages V over the tokens."""
    C = 64
    t = vae.enumerate_vae_attention_params("a", C)
    p = params_of(t, 6, affine=True)
    x = np.random.default_rng(2).standard_normal((C, 1, 1))
    g = (x[:, 0, 0].reshape(32, 2) - x[:, 0, 0].reshape(32, 2).mean(1, keepdims=True))
    g = g / np.sqrt((g * g).mean(1, keepdims=True) + 1e-5)
    n = g.reshape(C) * p["a.norm.gamma"] + p["a.norm.beta"]
    v = p["a.v.weight"] @ n + p["a.v.bias"]
    ref = x[:, 0, 0] + p["a.out.weight"] @ v + p["a.out.bias"]
    np.testing.assert_allclose(vae.vae_attention(x, p, "a")[:, 0, 0], ref, atol=1e-12)
    p["a.k.weight"] = np.zeros((C, C))
    p["a.k.bias"] = np.zeros(C)
    x = np.random.default_rng(3).standard_normal((C, 3, 2))
    tok = x.reshape(C, 6).T
    mu = tok.reshape(6, 32, 2).mean(axis=(0, 2), keepdims=True)
    gn = tok.reshape(6, 32, 2) - mu
    gn = (gn / np.sqrt((gn * gn).mean(axis=(0, 2), keepdims=True) + 1e-5)).reshape(6, C)
    gn = gn * p["a.norm.gamma"] + p["a.norm.beta"]
    vmean = (gn @ p["a.v.weight"].T + p["a.v.bias"]).mean(axis=0)
    o = p["a.out.weight"] @ vmean + p["a.out.bias"]
    np.testing.assert_allclose(vae.vae_attention(x, p, "a"), x + o[:, None, None], atol=1e-12)


def test_decoder_output_head_only():
    """All convolution weights zero: the output is conv_out's bias everywhere."""
    cfg = narrow()
    table = vae.enumerate_vae_decoder_params(cfg)
    p = params_of(table, 7)
    for name, shape, kind, _ in table:
        if kind == "weight":
            p[name] = np.zeros(shape)
    out = vae.vae_decode(np.ones((4, 2, 2)), p, cfg)
    np.testing.assert_allclose(out, np.broadcast_to(p["conv_out.bias"][:, None, None], out.shape), atol=1e-14)
