"""GPU parity of the sampling steps around the denoiser: the fused guidance +
DDPM / DDIM update (sd_sampler_step) against the oracle's updates, and whole
guided sampling loops (sd_denoise: two denoiser passes per step, then the
update) against the oracle's loop on a narrow SD2.1-shaped U-Net, eagerly and
replayed from one CUDA graph.

Sources: the SD/SDXL tutorial page's DDPM paragraphs (reverse step, linear
schedule, sampling loop); the cosine schedule and the DDIM step from the papers
that page names; classifier-free guidance."""
import numpy as np
import pytest

from gpu_util import assert_close, chw, dev_np, hwc, oracle_params
from oracle import model, sampler
import oracle
from latent_diffusion_net_b200 import synth

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("no CUDA device", allow_module_level=True)

from latent_diffusion_net_b200 import binding as B  # noqa: E402
from latent_diffusion_net_b200 import harness as Hn  # noqa: E402

STEP_TOL = 5e-2


@pytest.mark.parametrize("kind,t,t_prev,guided,noisy", [
    (B.SD_SAMPLER_DDPM, 500, 499, True, True), (B.SD_SAMPLER_DDPM, 1, 0, False, False),
    (B.SD_SAMPLER_DDIM, 981, 961, True, False), (B.SD_SAMPLER_DDIM, 21, 0, False, False)])
def test_sampler_step_matches_oracle(kind, t, t_prev, guided, noisy):
    H, W = 20, 12
    n = H * W * 4
    betas = sampler.linear_betas()
    ac = B.sd_schedule(B.SD_SCHED_LINEAR)
    x = synth.normal_bf16(31, 0, (n,)).astype(np.float64) * 3.0
    ec = synth.normal_bf16(31, 1, (n,))
    eu = synth.normal_bf16(31, 2, (n,))
    z = synth.normal_bf16(31, 3, (n,))
    g = 7.5
    xd = torch.from_numpy(x.astype(np.float32)).cuda()
    xb = torch.zeros(n, dtype=torch.bfloat16, device="cuda")
    cfg = B.sampler_cfg(kind, n, ac[t - 1], ac[t_prev - 1] if t_prev > 0 else 1.0, guidance=g)
    B.sd_sampler_step(cfg, xd, Hn.to_dev_bf16(ec), Hn.to_dev_bf16(eu) if guided else None,
                      torch.from_numpy(z).cuda() if noisy else None, xb)
    torch.cuda.synchronize()
    eps = sampler.cfg_combine(ec, eu, g) if guided else ec.astype(np.float64)
    if kind == B.SD_SAMPLER_DDPM:
        ref = sampler.ddpm_step(x, eps, t, betas, z if noisy else None)
    else:
        ref = sampler.ddim_step(x, eps, t, t_prev, betas)
    got = xd.double().cpu().numpy()
    assert_close(got, ref, 1e-5, "sampler step")
    np.testing.assert_array_equal(xb.float().cpu().numpy(), torch.from_numpy(got.astype(np.float32)).bfloat16()
                                  .float().numpy())


def narrow_unet(seed=41):
    bc = (256, 256, 512, 512)
    ocfg = model.UNetConfig(block_channels=bc, ctx_dim=256)
    rows = model.enumerate_unet_params(ocfg)
    cfg = B.unet_cfg(height=16, width=16, block_channels=bc, ctx_dim=256)
    m = Hn.Module("unet", cfg)
    canon = synth.canonical_weights([(s, k, f) for _, s, k, f in rows], seed)
    m.load(canon)
    return ocfg, cfg, m, oracle_params(rows, canon)


@pytest.mark.parametrize("kind,sched,timesteps,guidance", [
    (B.SD_SAMPLER_DDPM, B.SD_SCHED_LINEAR, [3, 2, 1], 7.5),
    (B.SD_SAMPLER_DDIM, B.SD_SCHED_COSINE, [999, 666, 333], None)])
def test_denoise_loop_matches_oracle(kind, sched, timesteps, guidance):
    ocfg, cfg, m, p = narrow_unet()
    H = W = 16
    n = H * W * 4
    ac = B.sd_schedule(sched, 1000, 1e-4, 0.02)
    betas = sampler.linear_betas() if sched == B.SD_SCHED_LINEAR else sampler.cosine_betas()
    xT = synth.normal_bf16(41, synth.IDX_X, (H, W, 4))
    ctx_c = synth.normal_bf16(41, synth.IDX_CTX, (77, 256))
    ctx_u = synth.normal_bf16(42, synth.IDX_CTX, (77, 256))
    noise = synth.normal_bf16(41, synth.IDX_NOISE, (len(timesteps), H, W, 4)) if kind == B.SD_SAMPLER_DDPM else None
    ws_bytes = B.sd_denoise_workspace_size(cfg)
    ws = Hn.workspace(ws_bytes)
    x = torch.from_numpy(xT.reshape(-1).copy()).cuda()
    args = (cfg, m.packed_dev, kind, ac, timesteps, guidance or 1.0)
    tail = (None, Hn.to_dev_bf16(ctx_c), Hn.to_dev_bf16(ctx_u) if guidance else None, None, None, None,
            torch.from_numpy(noise.reshape(-1).copy()).cuda() if noise is not None else None, ws, ws_bytes)
    B.sd_denoise(*args, x, *tail)
    torch.cuda.synchronize()
    assert B.sd_query_device_status(ws) == 0

    def eps_fn(xc, t):
        lat = chw(xc)
        e_c = hwc(oracle.unet_step(lat, float(t), ctx_c, p, ocfg))
        e_u = hwc(oracle.unet_step(lat, float(t), ctx_u, p, ocfg)) if guidance else None
        return e_c, e_u

    ref = sampler.denoise(xT, timesteps, eps_fn, betas, "ddpm" if kind == B.SD_SAMPLER_DDPM else "ddim",
                          guidance, None if noise is None else list(noise))
    assert_close(dev_np(x, (H, W, 4)), ref, STEP_TOL, "denoise loop")

    # the same loop captured once in a CUDA graph and replayed gives the same bits
    x2 = torch.from_numpy(xT.reshape(-1).copy()).cuda()
    s = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        B.sd_denoise(*args, x2, *tail, stream=torch.cuda.current_stream())
    x2.copy_(torch.from_numpy(xT.reshape(-1).copy()).cuda())
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(x2, x)
    del g
