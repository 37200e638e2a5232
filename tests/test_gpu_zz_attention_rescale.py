"""GPU parity of a transformer whose self-attention rows rescale their running
output at different key tiles, so the 32 rows of one softmax warp disagree on the
rescale (the Q/K weights are doubled; ``tests/test_attention_rescale_case.py``
counts those events on the oracle's scores). With the standard weights no row ever
rescales, so no other test reaches this branch of the attention kernel.

Whole items at 48x48x320; the split schedule and the merge kernel at 64x64x640.
Tolerance as for every transformer block: 2e-2 on the output, 6e-2 on the
block's own contribution. The file runs after the other GPU parity tests (before the
allocation-free entry point's file, which is collected last)."""
import pytest

import rescale_case
from gpu_util import assert_close, chw, dev_np, hwc, oracle_params
import oracle

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover - collected on CPU hosts too
    pytest.skip("no CUDA device", allow_module_level=True)

from latent_diffusion_net_b200 import binding as B  # noqa: E402
from latent_diffusion_net_b200 import harness as Hn  # noqa: E402

BLOCK_TOL = 2e-2


@pytest.mark.parametrize("H,W,C,ctas", rescale_case.CASES)
def test_transformer_rows_rescale_at_different_key_tiles(H, W, C, ctas):
    rows, canon = rescale_case.canonical(C)
    cfg = B.transformer_cfg(H, W, C, 1, 77, 1024)
    m = Hn.Module("attn", cfg)
    m.load(canon)
    p = oracle_params(rows, canon)
    x, ctx = rescale_case.inputs(H, W, C)
    y = torch.empty(H * W * C, dtype=torch.bfloat16, device="cuda")
    B.sd_transformer_fwd(cfg, m.packed_dev, Hn.to_dev_bf16(x), Hn.to_dev_bf16(ctx), y, m.ws, m.ws_bytes)
    torch.cuda.synchronize()
    assert B.sd_query_device_status(m.ws) == 0
    ref = hwc(oracle.transformer(chw(x), ctx, p, "t", 1))
    got = dev_np(y, (H, W, C))
    assert_close(got, ref, BLOCK_TOL, "output")
    assert_close(got - x, ref - chw(x).transpose(1, 2, 0), 3 * BLOCK_TOL, "block contribution")
