"""GPU parity of the VAE decoder (sd_vae_decode) against the oracle: the full SD
channel ladder (512 -> 512 -> 256 -> 128) on a 16x16 latent (a 128x128 image)
and on a 24x32 latent (192x256), bar 5e-2 as for a whole denoiser step. Source:
section 5 of the SD2.1 and SDXL-Inpainting architecture pages."""
import numpy as np
import pytest

from gpu_util import assert_close, chw, dev_np, hwc, oracle_params
from oracle import vae
from latent_diffusion_net_b200 import synth

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("no CUDA device", allow_module_level=True)

from latent_diffusion_net_b200 import binding as B  # noqa: E402
from latent_diffusion_net_b200 import harness as Hn  # noqa: E402

_W = {}


@pytest.mark.parametrize("h,w", [(16, 16), (24, 32)])
def test_vae_decode_matches_oracle(h, w):
    rows = vae.enumerate_vae_decoder_params()
    cfg = B.vae_cfg(h, w)
    m = Hn.Module("vae", cfg)
    if "canon" not in _W:
        _W["canon"] = synth.canonical_weights([(s, k, f) for _, s, k, f in rows], 51)
    m.load(_W["canon"])
    p = oracle_params(rows, _W["canon"])
    z = synth.normal_bf16(51, synth.IDX_X, (h, w, 4))
    img = torch.empty(64 * h * w * 3, dtype=torch.bfloat16, device="cuda")
    B.sd_vae_decode(cfg, m.packed_dev, Hn.to_dev_bf16(z), img, m.ws, m.ws_bytes)
    torch.cuda.synchronize()
    assert B.sd_query_device_status(m.ws) == 0
    ref = hwc(vae.vae_decode(chw(z), p))
    assert_close(dev_np(img, (8 * h, 8 * w, 3)), ref, 5e-2, f"vae decode {h}x{w}")
