"""The device-side timeout path of the tensor-core GEMM, exercised without a
fault: sd_debug_inject_timeout makes one thread of every CTA of the next GEMM
wait on a barrier that nothing completes, with a short limit. The wait gives
up, raises the error flag, and every role of the kernel skips its work and
releases its tensor memory. The test checks that sd_query_device_status then
reports SD_ERR_DEVICE_TIMEOUT once, that the flag is cleared, and that the next
ordinary call on the same device and workspace is correct."""
import numpy as np
import pytest

from gpu_util import assert_close, chw, dev_np, hwc, oracle_params
from oracle import model
import oracle
from latent_diffusion_net_b200 import synth

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("no CUDA device", allow_module_level=True)

from latent_diffusion_net_b200 import binding as B  # noqa: E402
from latent_diffusion_net_b200 import harness as Hn  # noqa: E402

SD_ERR_DEVICE_TIMEOUT = 8


def test_gemm_wait_gives_up_and_the_next_call_is_correct():
    H = W = 16
    C = 320
    rows = model.enumerate_resblock_params("r", C, C)
    cfg = B.resblock_cfg(H, W, C, C)
    m = Hn.Module("res", cfg)
    canon = synth.canonical_weights([(s, k, f) for _, s, k, f in rows], 23)
    m.load(canon)
    p = oracle_params(rows, canon)
    x = synth.normal_bf16(23, 0, (H, W, C))
    temb = synth.normal_bf16(23, 1, (1280,))
    temb_d = torch.from_numpy(temb.astype(np.float32)).cuda()
    xd = Hn.to_dev_bf16(x)
    y = torch.empty(H * W * C, dtype=torch.bfloat16, device="cuda")
    ref = hwc(oracle.resblock(chw(x), temb, p, "r"))
    try:
        B.sd_debug_inject_timeout(1, 1000)  # the first of the block's two convolutions gives up
        B.sd_resblock_fwd(cfg, m.packed_dev, xd, None, temb_d, y, m.ws, m.ws_bytes)
        assert B.sd_query_device_status(m.ws) == SD_ERR_DEVICE_TIMEOUT
    finally:
        B.sd_debug_inject_timeout(0, 0)
    assert B.sd_query_device_status(m.ws) == 0  # reported once, then cleared
    for _ in range(2):
        B.sd_resblock_fwd(cfg, m.packed_dev, xd, None, temb_d, y, m.ws, m.ws_bytes)
        assert B.sd_query_device_status(m.ws) == 0
        assert_close(dev_np(y, (H, W, C)), ref, 2e-2, "resblock after a timeout")
