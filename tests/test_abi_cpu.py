"""C-ABI checks that need no GPU: the library loads, exports every entry point
declared in include/sd_api.h, enumerates the same weight tables as the oracle,
packs weights as documented, and rejects bad arguments on the host before any
launch."""
import os
import re

import numpy as np
import pytest

from latent_diffusion_net_b200 import binding as B
from latent_diffusion_net_b200 import synth
from oracle import model

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def built():
    from latent_diffusion_net_b200 import build
    build.build()


def header_functions():
    txt = open(os.path.join(ROOT, "include", "sd_api.h")).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(sd_[a-z0-9_]+)\s*\(", txt)))


def test_library_exports_every_declared_function():
    import ctypes
    lib = ctypes.CDLL(B.LIB_PATH)
    declared = header_functions()
    assert len(declared) >= 20
    for name in declared:
        assert hasattr(lib, name), name
    assert set(declared) == set(B.exported_symbols())
    assert B.lib().sd_version().decode().startswith("sd-b200")


def strip(rows, prefix):
    return [(r["name"][len(prefix):] if r["name"].startswith(prefix) else r["name"], tuple(r["shape"]), r["kind"],
             r["fan_in"]) for r in rows]


def oracle_rows(table, prefix):
    return [(n[len(prefix):] if n.startswith(prefix) else n, tuple(s), k, f) for n, s, k, f in table]


@pytest.mark.parametrize("cfg", [model.SD21_BASE, model.SDXL_INPAINT])
def test_unet_table_matches_oracle(cfg):
    c = B.unet_cfg_from(cfg, 96, 96)
    rows, canon, packed = B.sd_unet_weight_layout(c)
    ora = model.enumerate_unet_params(cfg)
    assert strip(rows, "") == oracle_rows(ora, "")
    assert canon == sum(int(np.prod(s)) for _, s, _, _ in ora)
    if cfg is model.SD21_BASE:
        assert canon == 865_910_724
    offs = [r["packed_offset"] for r in rows]
    assert all(o % 256 == 0 for o in offs) and packed >= 2 * canon
    # packed tensors never overlap (the BF16 ones take 2 bytes per element; conv_in is padded wider)
    spans = sorted((r["packed_offset"], r["packed_offset"] + 2 * int(np.prod(r["shape"]))) for r in rows
                   if "conv_in" not in r["name"])
    assert all(a1 <= b0 for (_, a1), (b0, _) in zip(spans, spans[1:]))
    # every cross-attention's K then V weights form one [K of all blocks | V of all blocks] matrix at the end
    kv = [r for r in rows if ".attn2.k." in r["name"] or ".attn2.v." in r["name"]]
    ks = [r for r in kv if ".attn2.k." in r["name"]]
    vs = [r for r in kv if ".attn2.v." in r["name"]]
    order = ks + vs
    for a, b in zip(order, order[1:]):
        assert b["packed_offset"] == a["packed_offset"] + 2 * int(np.prod(a["shape"]))
    assert order[0]["packed_offset"] > max(r["packed_offset"] for r in rows if r not in kv)


@pytest.mark.parametrize("cin,cout,cs", [(320, 320, 0), (640, 320, 0), (1280, 1280, 1280), (640, 640, 320)])
def test_resblock_table_matches_oracle(cin, cout, cs):
    rows, canon, _ = B.sd_resblock_weight_layout(B.resblock_cfg(8, 8, cin, cout, c_skip=cs))
    assert strip(rows, "res") == oracle_rows(model.enumerate_resblock_params("", cin + cs, cout), "")


@pytest.mark.parametrize("C,depth,D", [(320, 1, 1024), (640, 2, 2048), (1280, 10, 2048)])
def test_transformer_table_matches_oracle(C, depth, D):
    rows, _, _ = B.sd_transformer_weight_layout(B.transformer_cfg(8, 8, C, depth, ctx_dim=D))
    assert strip(rows, "attn") == oracle_rows(model.enumerate_transformer_params("", C, depth, D), "")


def test_time_and_conv_tables():
    rows, _, _ = B.sd_time_weight_layout(B.time_cfg())
    assert strip(rows, "") == oracle_rows(model.enumerate_time_mlp_params(), "")
    rows, _, _ = B.sd_conv_weight_layout(B.conv_cfg(128, 128, 9, 320), B.SD_CONV_IN)
    assert strip(rows, "") == oracle_rows(model.enumerate_conv_params("conv_in", 9, 320), "")
    rows, _, _ = B.sd_conv_weight_layout(B.conv_cfg(64, 64, 640, 640), B.SD_CONV_DOWNSAMPLE)
    assert [r["shape"] for r in rows] == [(640, 640, 3, 3), (640,)]


def test_pack_conv_krsc_and_geglu_interleave():
    C = 64
    cfg = B.resblock_cfg(4, 4, 256, 256)
    rows, canon_n, packed_n = B.sd_resblock_weight_layout(cfg)
    canon = np.arange(canon_n, dtype=np.int64).astype(np.uint16)
    packed = B.sd_resblock_pack_weights(cfg, canon, packed_n).view(np.uint16)
    r = [x for x in rows if x["name"] == "res.conv1.weight"][0]
    O, Ci = r["shape"][0], r["shape"][1]
    src = canon[r["canon_offset"]:r["canon_offset"] + O * Ci * 9].reshape(O, Ci, 3, 3)
    dst = packed[r["packed_offset"] // 2:r["packed_offset"] // 2 + O * Ci * 9].reshape(O, 3, 3, Ci)
    np.testing.assert_array_equal(dst, src.transpose(0, 2, 3, 1))
    # FF1 rows: value/gate interleave of W * gamma(LN3), rounded to BF16 (the LayerNorm fold)
    tcfg = B.transformer_cfg(4, 4, 256, 1, ctx_dim=256)
    rows, canon_n, packed_n = B.sd_transformer_weight_layout(tcfg)
    canon = synth.normal_bf16_bits(99, 0, canon_n)
    packed = B.sd_transformer_pack_weights(tcfg, canon, packed_n).view(np.uint16)
    r = [x for x in rows if x["name"].endswith("ff.w1.weight")][0]
    g = [x for x in rows if x["name"].endswith("ln3.gamma")][0]
    R, K = r["shape"]
    src = synth.bf16_bits_to_f32(canon[r["canon_offset"]:r["canon_offset"] + R * K]).reshape(R, K)
    gamma = synth.bf16_bits_to_f32(canon[g["canon_offset"]:g["canon_offset"] + K])
    folded = synth.f32_to_bf16_bits((src * gamma[None, :]).astype(np.float32))
    dst = packed[r["packed_offset"] // 2:r["packed_offset"] // 2 + R * K].reshape(R, K)
    np.testing.assert_array_equal(dst[0::2], folded[:R // 2])
    np.testing.assert_array_equal(dst[1::2], folded[R // 2:])
    # q, k, v contiguous: [3C, C]
    q = [x for x in rows if x["name"].endswith("attn1.q.weight")][0]
    v = [x for x in rows if x["name"].endswith("attn1.v.weight")][0]
    assert v["packed_offset"] - q["packed_offset"] == 2 * 256 * 256 * 2
    del C


def test_pack_conv_in_im2col_order():
    cfg = B.conv_cfg(16, 16, 9, 320)
    rows, canon_n, packed_n = B.sd_conv_weight_layout(cfg, B.SD_CONV_IN)
    canon = (np.arange(canon_n, dtype=np.int64) % 60000 + 1).astype(np.uint16)
    packed = B.sd_conv_pack_weights(cfg, B.SD_CONV_IN, canon, packed_n).view(np.uint16)
    w = canon[:320 * 81].reshape(320, 9, 3, 3)
    p = packed[:320 * 128].reshape(320, 128)
    for o in (0, 7, 319):
        for c in range(9):
            for ky in range(3):
                for kx in range(3):
                    assert p[o, (ky * 3 + kx) * 9 + c] == w[o, c, ky, kx]
        assert np.all(p[o, 81:] == 0)


def test_host_validation_without_gpu():
    cfg = B.resblock_cfg(8, 8, 320, 320)
    ws = B.sd_resblock_workspace_size(cfg)
    assert ws > 0
    fake = 1 << 20
    # null pointer
    assert B.sd_resblock_fwd(cfg, None, fake, None, fake, fake, fake, ws, check=False) == 1
    # misaligned
    assert B.sd_resblock_fwd(cfg, fake, fake + 2, None, fake, fake, fake, ws, check=False) == 4
    # workspace too small
    assert B.sd_resblock_fwd(cfg, fake, fake, None, fake, fake, fake, ws - 1, check=False) == 5
    # unsupported: batch 2, channels not a multiple of 64, groups leaving < 8 channels
    bad = B.resblock_cfg(8, 8, 320, 320)
    bad.batch = 2
    assert B.sd_resblock_fwd(bad, fake, fake, None, fake, fake, fake, ws, check=False) == 3
    assert B.sd_resblock_fwd(B.resblock_cfg(8, 8, 100, 320), fake, fake, None, fake, fake, fake, ws,
                             check=False) == 3
    assert B.sd_resblock_fwd(B.resblock_cfg(8, 8, 128, 128), fake, fake, None, fake, fake, fake, ws,
                             check=False) == 3
    # skip channels declared but no skip pointer
    assert B.sd_resblock_fwd(B.resblock_cfg(8, 8, 320, 320, c_skip=320), fake, fake, None, fake, fake, fake,
                             10 ** 9, check=False) == 1
    t = B.transformer_cfg(8, 8, 320)
    t.head_dim = 80
    assert B.sd_transformer_fwd(t, fake, fake, fake, fake, fake, 10 ** 9, check=False) == 3
    t = B.transformer_cfg(8, 8, 320, ctx_len=0)
    assert B.sd_transformer_fwd(t, fake, fake, fake, fake, fake, 10 ** 9, check=False) == 2
    u = B.unet_cfg(height=90, width=96)
    assert B.sd_unet_step(u, fake, fake, 500.0, fake, fake, fake, 10 ** 10, check=False) == 2
    u = B.unet_cfg(in_channels=3)
    assert B.sd_unet_step(u, fake, fake, 500.0, fake, fake, fake, 10 ** 10, check=False) == 3
    d = B.conv_cfg(9, 8, 320, 320)
    assert B.sd_conv_fwd(d, B.SD_CONV_DOWNSAMPLE, fake, fake, None, None, fake, fake, 10 ** 9, check=False) == 2
    # empty images are rejected as bad shapes before anything is launched
    assert B.sd_resblock_fwd(B.resblock_cfg(0, 8, 320, 320), fake, fake, None, fake, fake, fake, 10 ** 9,
                             check=False) == 2
    assert B.sd_transformer_fwd(B.transformer_cfg(8, 0, 320), fake, fake, fake, fake, fake, 10 ** 9, check=False) == 2
    assert B.sd_conv_fwd(B.conv_cfg(0, 8, 320, 320), B.SD_CONV_UPSAMPLE, fake, fake, None, None, fake, fake, 10 ** 9,
                         check=False) == 2
    assert B.sd_unet_step(B.unet_cfg(height=0, width=96), fake, fake, 500.0, fake, fake, fake, 10 ** 10,
                          check=False) == 2
    # a well-formed call on a machine without a usable B200 fails cleanly, never crashes
    s = B.sd_resblock_fwd(cfg, fake, fake, None, fake, fake, fake, ws, check=False)
    assert s in (0, 6, 7) and (s != 0 or os.environ.get("CUDA_VISIBLE_DEVICES") != "")


def test_workspace_sizes():
    u = B.sd_unet_workspace_size(B.unet_cfg())
    assert 0 < u < 2 * 1024 ** 3
    assert B.sd_unet_workspace_size(B.unet_cfg(height=90)) == 0
    small = B.sd_transformer_workspace_size(B.transformer_cfg(32, 32, 320))
    large = B.sd_transformer_workspace_size(B.transformer_cfg(96, 96, 320))
    assert 0 < small < large
    assert B.status_string(5) == "workspace too small"


def test_gemm_override_validation():
    """The schedule hook accepts 0 or a multiple of 32 up to 256, and 0..16 splits."""
    for bn, sp in [(48, 0), (512, 0), (-32, 0), (0, 17), (0, -1), (16, 1)]:
        with pytest.raises(RuntimeError):
            B.sd_gemm_override(bn, sp)
    for bn, sp in [(32, 1), (256, 16), (160, 0), (0, 0)]:
        B.sd_gemm_override(bn, sp)


def test_conditioned_step_and_hooks_validate_on_host():
    """SDXL added conditioning is checked before any launch; the record and
    timeout-injection hooks reject bad arguments."""
    fake = 1 << 20
    sdxl = B.unet_cfg_from(model.SDXL_INPAINT, 128, 128)
    assert B.sd_unet_workspace_size(sdxl) > B.sd_unet_workspace_size(B.unet_cfg(height=128, width=128,
                                                                                   in_channels=9,
                                                                                   block_channels=(320, 640, 1280),
                                                                                   attn_depth=(0, 2, 10),
                                                                                   mid_depth=10, ctx_dim=2048))
    # the plain step cannot serve a config with added conditioning
    assert B.sd_unet_step(sdxl, fake, fake, 500.0, fake, fake, fake, 10 ** 11, check=False) == 1
    assert B.sd_unet_step_cond(sdxl, fake, fake, 500.0, fake, None, [1024.0] * 6, fake, fake, 10 ** 11,
                               check=False) == 1
    assert B.sd_unet_step_cond(sdxl, fake, fake, 500.0, fake, fake, None, fake, fake, 10 ** 11, check=False) == 1
    assert B.sd_unet_step_cond(sdxl, fake, fake, 500.0, fake, fake + 4, [0.0] * 6, fake, fake, 10 ** 11,
                               check=False) == 4
    bad = B.unet_cfg_from(model.SDXL_INPAINT, 128, 128)
    bad.add_time_ids = 9
    assert B.sd_unet_step_cond(bad, fake, fake, 500.0, fake, fake, [0.0] * 9, fake, fake, 10 ** 11,
                               check=False) == 3
    bad = B.unet_cfg_from(model.SDXL_INPAINT, 128, 128)
    bad.add_time_dim = 255
    assert B.sd_unet_step_cond(bad, fake, fake, 500.0, fake, fake, [0.0] * 6, fake, fake, 10 ** 11,
                               check=False) == 2
    for n, spins in [(-1, 10), (1, 0), (1, (1 << 24) + 1)]:
        with pytest.raises(RuntimeError):
            B.sd_debug_inject_timeout(n, spins)
    B.sd_debug_inject_timeout(0, 0)
    with pytest.raises(RuntimeError):
        B.sd_record_begin(fake + 8, 1024)
    B.sd_record_begin(fake, 0)
    assert B.sd_record_end() == (0, 0)
    assert B.sd_record_read() == []


def test_vae_table_matches_oracle_and_validates():
    from oracle import vae
    rows, canon, packed = B.sd_vae_weight_layout(B.vae_cfg(96, 96))
    assert strip(rows, "") == oracle_rows(vae.enumerate_vae_decoder_params(), "")
    assert canon == 49_490_199
    assert B.sd_vae_workspace_size(B.vae_cfg(96, 96)) > B.sd_vae_workspace_size(B.vae_cfg(32, 32)) > 0
    fake = 1 << 20
    assert B.sd_vae_decode(B.vae_cfg(10, 10), fake, fake, fake, fake, 10 ** 10, check=False) == 3  # 100 tokens
    assert B.sd_vae_decode(B.vae_cfg(16, 16, groups=64), fake, fake, fake, fake, 10 ** 10, check=False) == 3
    assert B.sd_vae_decode(B.vae_cfg(16, 16), fake, None, fake, fake, 10 ** 10, check=False) == 1


def test_sampler_schedules_and_validation_on_host():
    """The host-side schedules of the sampling entry points equal the oracle's
    (linear and cosine alpha_bar, float64), and the update and the loop reject
    bad arguments before any launch."""
    from oracle import sampler
    lin = np.array(B.sd_schedule(B.SD_SCHED_LINEAR, 1000, 1e-4, 0.02))
    np.testing.assert_allclose(lin, sampler.alphas_cumprod(sampler.linear_betas(1000, 1e-4, 0.02)), rtol=1e-12)
    cos = np.array(B.sd_schedule(B.SD_SCHED_COSINE, 1000, 1e-4, 0.02))
    np.testing.assert_allclose(cos, sampler.alphas_cumprod(sampler.cosine_betas(1000)), rtol=1e-12)
    for args in [(B.SD_SCHED_LINEAR, 0, 1e-4, 0.02), (B.SD_SCHED_LINEAR, 1000, 0.02, 1e-4), (7, 1000, 1e-4, 0.02)]:
        with pytest.raises(RuntimeError):
            B.sd_schedule(*args)
    fake = 1 << 20
    ac = lin
    ok = B.sampler_cfg(B.SD_SAMPLER_DDIM, 96 * 96 * 4, ac[499], ac[479], guidance=7.5)
    assert B.sd_sampler_step(ok, None, fake, check=False) == 1                        # no state
    assert B.sd_sampler_step(B.sampler_cfg(B.SD_SAMPLER_DDIM, 10, ac[499], ac[479]), fake, fake,
                             check=False) == 2                                           # n % out_ch
    assert B.sd_sampler_step(B.sampler_cfg(B.SD_SAMPLER_DDIM, 96 * 96 * 4, ac[499], ac[479], ld=2), fake, fake,
                             x_bf16=fake, check=False) == 2                              # ld < out_ch
    assert B.sd_sampler_step(ok, fake + 4, fake, check=False) == 4                    # misaligned
    assert B.sd_sampler_step(B.sampler_cfg(B.SD_SAMPLER_DDIM, 96 * 96 * 4, ac[479], ac[499]), fake, fake,
                             check=False) == 2                                           # alpha_bar_prev < alpha_bar_t
    cfg = B.unet_cfg_from(model.SD21_BASE, 96, 96)
    need = B.sd_denoise_workspace_size(cfg)
    assert need > 2 * B.sd_unet_workspace_size(cfg)

    def den(ts, kind=B.SD_SAMPLER_DDIM, ws_bytes=need, acs=ac, ctx=fake):
        return B.sd_denoise(cfg, fake, kind, acs, ts, 7.5, fake, None, ctx, fake, None, None, None, None, fake,
                            ws_bytes, check=False)

    assert den([500, 500]) == 2          # timesteps must fall
    assert den([1001]) == 2              # past T
    assert den([]) == 2                  # no step
    assert den([500], kind=5) == 3       # unknown sampler
    assert den([500], ws_bytes=need - 1) == 5
    assert den([500], ctx=None) == 1
