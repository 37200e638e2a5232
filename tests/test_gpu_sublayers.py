"""Per-sublayer GPU parity: each ResnetBlock2D's h1 (conv1 output with its bias
and time projection) and each BasicTransformer block's self-attention,
cross-attention and feed-forward outputs BEFORE their residual add, recorded
from the library (sd_record_*) and compared with the oracle's record of the
same values at relative L2 <= 1e-2. The residual stream carries the block
input through, so a wrong sublayer could hide under a good block output; here
it cannot. Block panels: "Stable Diffusion 2.1 Base 宏观架构" section 4.

Cases: the 96x96x320 CrossAttn block (9216 tokens, one BasicTransformer block)
and the SDXL level-1 stage at 64x64x640 (two resblocks, two transformers of
depth 2)."""
import numpy as np
import pytest

from gpu_util import assert_close, hwc

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("no CUDA device", allow_module_level=True)

from latent_diffusion_net_b200 import binding as B  # noqa: E402
from test_gpu_workloads import make_workload, oracle_forward  # noqa: E402

SUBLAYER_TOL = 1e-2


@pytest.mark.parametrize("wid", [2, 3])
def test_sublayers_match_oracle(wid):
    wl = make_workload(wid)
    buf = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    B.sd_record_begin(buf, buf.numel())
    out_rec = wl.step().clone()
    status, n = B.sd_record_end()
    torch.cuda.synchronize()
    assert status == 0 and n > 0
    entries = B.sd_record_read()
    # recording leaves the block output unchanged
    plain = wl.step().clone()
    torch.cuda.synchronize()
    assert torch.equal(out_rec, plain)
    rec = {}
    oracle_forward(wid, wl, record=rec)
    raw = buf.cpu().numpy()
    names = []
    for e in entries:
        nbytes = e["rows"] * e["cols"] * 2
        bits = raw[e["offset"]:e["offset"] + nbytes].view(np.uint16)
        got = (bits.astype(np.uint32) << 16).view(np.float32).reshape(e["rows"], e["cols"]).astype(np.float64)
        if e["name"] == "h1":
            ref = hwc(rec[f"r{e['module']}.h1"]).reshape(e["rows"], e["cols"])
        else:
            ref = rec[f"t{e['module']}.blocks.{e['block']}.{e['name']}"]
        what = f"workload {wid} module {e['module']} block {e['block']} {e['name']}"
        assert_close(got, ref, SUBLAYER_TOL, what)
        names.append((e["name"], e["module"], e["block"]))
    depth = 1 if wid == 2 else 2
    nmod = 1 if wid == 2 else 2
    expect = {("h1", m, 0) for m in range(nmod)} | {(k, m, d) for m in range(nmod) for d in range(depth)
                                                     for k in ("attn1", "attn2", "ff")}
    assert set(names) == expect
