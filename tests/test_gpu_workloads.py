"""GPU parity of the workloads against the oracle at their full sizes, in the
launch configuration the benchmark times (same ABI calls, same shapes).

Bars: relative L2 <= 2e-2 per block workload (1-4) and <= 5e-2 for a whole
denoiser step: SD2.1-base at 96x96 (5), 64x64 (7) and 128x128 (8, 16384
self-attention tokens at the first level), and the SDXL-Inpainting step at
128x128 with its added conditioning (6)."""
import numpy as np
import pytest

from gpu_util import assert_close, chw, dev_np, hwc, oracle_params
from oracle import model
import oracle
from latent_diffusion_net_b200.workloads import SDXL_TIME_IDS, TIMESTEP, WORKLOADS

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("no CUDA device", allow_module_level=True)

from latent_diffusion_net_b200 import harness as Hn  # noqa: E402


UNET_CFGS = {"sd21": model.SD21_BASE, "sdxl_inpaint": model.SDXL_INPAINT}
_CANON = {}  # (unet, seed) -> canonical weights, shared by the workloads of one model


def oracle_rows_for(wid):
    s = WORKLOADS[wid]
    if s["kind"] == "unet":
        return [model.enumerate_unet_params(UNET_CFGS[s["unet"]])]
    C = s["C"]
    mods = [model.enumerate_time_mlp_params()]
    nb = 2 if s["kind"] == "stage3" else 1
    for b in range(nb):
        mods.append(model.enumerate_resblock_params(f"r{b}", C, C))
        mods.append(model.enumerate_transformer_params(f"t{b}", C, s["depth"], s["ctx_dim"]))
    if s["kind"] == "stage3":
        mods.append(model.enumerate_conv_params("down", C, C))
    if s["kind"] == "stage4":
        mods.append(model.enumerate_conv_params("conv_in", 9, 320))
    return mods


def make_workload(wid):
    s = WORKLOADS[wid]
    if s["kind"] != "unet":
        return Hn.Workload(wid)
    key = (s["unet"], s["seed"])
    wl = Hn.Workload(wid, canonical=_CANON.get(key))
    _CANON.clear()
    _CANON[key] = wl.canonical
    return wl


def workload_params(wid, wl):
    params = {}
    for r, canon in zip(oracle_rows_for(wid), wl.canonical):
        params.update(oracle_params(r, canon))
    return params


def oracle_forward(wid, wl, record=None):
    s = WORKLOADS[wid]
    params = workload_params(wid, wl)
    inp = wl.inputs
    if s["kind"] == "unet":
        cfg = UNET_CFGS[s["unet"]]
        kw = {"add_text": inp["text"], "add_time_ids": SDXL_TIME_IDS} if cfg.add_embed_dim else {}
        return {"out": hwc(oracle.unet_step(chw(inp["x"]), TIMESTEP, inp["ctx"], params, cfg, **kw))}
    temb = oracle.time_mlp(params, TIMESTEP)
    h = chw(inp["x"])
    nb = 2 if s["kind"] == "stage3" else 1
    for b in range(nb):
        h = oracle.resblock(h, temb, params, f"r{b}", record=record)
        h = oracle.transformer(h, inp["ctx"], params, f"t{b}", s["depth"], record=record)
    out = {}
    if s["kind"] == "stage3":
        h = oracle.downsample(h, params, "down")
    out["out"] = hwc(h)
    if s["kind"] == "stage4":
        x9 = np.concatenate([inp["noisy"], inp["masked"], inp["mask"]], axis=2)
        out["out2"] = hwc(oracle.conv_in(chw(x9), params, "conv_in"))
    return out


@pytest.mark.parametrize("wid", [1, 2, 3, 4, 5, 7, 8, 6])
def test_workload_parity(wid):
    s = WORKLOADS[wid]
    wl = make_workload(wid)
    wl.step()
    torch.cuda.synchronize()
    assert Hn.B.sd_query_device_status(wl.modules[0].ws) == 0
    ref = oracle_forward(wid, wl)
    if s["kind"] == "unet":
        got = dev_np(wl.out, (s["H"], s["W"], 4))
        assert_close(got, ref["out"], 5e-2, f"workload {wid} ({s['name']})")
        if wid == 6:
            _CANON.clear()  # 5 GB of SDXL weights
        return
    if s["kind"] == "stage3":
        shape = (s["H"] // 2, s["W"] // 2, s["C"])
    else:
        shape = (s["H"], s["W"], s["C"])
    assert_close(dev_np(wl.out, shape), ref["out"], 2e-2, f"workload {wid}")
    if s["kind"] == "stage4":
        hw = s["inpaint_hw"]
        assert_close(dev_np(wl.out2, (hw, hw, 320)), ref["out2"], 2e-2, f"workload {wid} conv_in")


def test_repeat_is_bitwise_deterministic():
    wl = Hn.Workload(1)
    a = wl.step().clone()
    b = wl.step().clone()
    torch.cuda.synchronize()
    assert torch.equal(a, b)
