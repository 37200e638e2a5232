"""Every tensor-core GEMM schedule against the oracle: each N-tile width the
kernel is instantiated for, with and without a split reduction, through two
blocks that between them reach every epilogue (bias + time column vector +
fused 1x1 shortcut in a ResnetBlock2D; the folded LayerNorms, GEGLU and the
residual add in a Transformer2DModel). Sizes leave ragged M and N tails."""
import numpy as np
import pytest

from gpu_util import assert_close, chw, dev_np, hwc, oracle_params
from oracle import model
import oracle
from latent_diffusion_net_b200 import synth

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover - collected on CPU hosts too
    pytest.skip("no CUDA device", allow_module_level=True)

from latent_diffusion_net_b200 import binding as B  # noqa: E402
from latent_diffusion_net_b200 import harness as Hn  # noqa: E402

BLOCK_TOL = 2e-2
SCHEDULES = [(bn, sp) for bn in (32, 64, 96, 128, 160, 192, 224, 256) for sp in (1, 3)] + [(128, 12), (256, 7)]


@pytest.fixture(autouse=True)
def _reset_override():
    yield
    B.sd_gemm_override(0, 0)


def _module(kind, cfg, seed, rows):
    m = Hn.Module(kind, cfg)
    canon = synth.canonical_weights([(s, k, f) for _, s, k, f in rows], seed, True)
    m.load(canon)
    return m, oracle_params(rows, canon)


@pytest.fixture(scope="module")
def res_case():
    H, W, cx, co = 11, 13, 640, 320
    rows = model.enumerate_resblock_params("r", cx, co)
    cfg = B.resblock_cfg(H, W, cx, co)
    m, p = _module("res", cfg, 31, rows)
    x = synth.normal_bf16(31, 0, (H, W, cx))
    temb = synth.normal_bf16(31, 1, (1280,))
    ref = hwc(oracle.resblock(chw(x), temb, p, "r"))
    return H, W, co, cfg, m, x, temb, ref


@pytest.fixture(scope="module")
def tx_case():
    H, W, C, D, L = 9, 14, 320, 1024, 77
    rows = model.enumerate_transformer_params("t", C, 1, D)
    cfg = B.transformer_cfg(H, W, C, 1, L, D)
    m, p = _module("attn", cfg, 32, rows)
    x = synth.normal_bf16(32, 0, (H, W, C))
    ctx = synth.normal_bf16(32, 1, (L, D))
    ref = hwc(oracle.transformer(chw(x), ctx, p, "t", 1))
    return H, W, C, cfg, m, x, ctx, ref


@pytest.mark.parametrize("bn,splits", SCHEDULES)
def test_resblock_schedule(res_case, bn, splits):
    H, W, co, cfg, m, x, temb, ref = res_case
    B.sd_gemm_override(bn, splits)
    y = torch.empty(H * W * co, dtype=torch.bfloat16, device="cuda")
    temb_d = torch.from_numpy(temb.astype(np.float32)).cuda()
    B.sd_resblock_fwd(cfg, m.packed_dev, Hn.to_dev_bf16(x), None, temb_d, y, m.ws, m.ws_bytes)
    torch.cuda.synchronize()
    assert B.sd_query_device_status(m.ws) == 0
    assert_close(dev_np(y, (H, W, co)), ref, BLOCK_TOL)


@pytest.mark.parametrize("bn,splits", SCHEDULES)
def test_transformer_schedule(tx_case, bn, splits):
    H, W, C, cfg, m, x, ctx, ref = tx_case
    B.sd_gemm_override(bn, splits)
    y = torch.empty(H * W * C, dtype=torch.bfloat16, device="cuda")
    B.sd_transformer_fwd(cfg, m.packed_dev, Hn.to_dev_bf16(x), Hn.to_dev_bf16(ctx), y, m.ws, m.ws_bytes)
    torch.cuda.synchronize()
    assert B.sd_query_device_status(m.ws) == 0
    got = dev_np(y, (H, W, C))
    assert_close(got, ref, BLOCK_TOL)
    assert_close(got - x, ref - chw(x).transpose(1, 2, 0), 3 * BLOCK_TOL)

