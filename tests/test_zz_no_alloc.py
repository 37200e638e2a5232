"""The allocation-free time embedding (sd_time_embed_noalloc) against the
workspace entry point sd_time_embed.

Callers that may not allocate device memory (for instance a plugin inside
another inference engine, which owns all allocations) use the no-allocation
entry point; it must give the same result as the regular one, call after call,
although all calls share one scratch array inside the library. This file is
named to be collected last."""
import numpy as np
import pytest

from latent_diffusion_net_b200 import synth

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("no CUDA device", allow_module_level=True)

from latent_diffusion_net_b200 import binding as B  # noqa: E402
from latent_diffusion_net_b200 import harness as Hn  # noqa: E402

TOL = 1e-4  # the time-embedding tolerance of the parity tests


def rel(a, b):
    a = a.double().cpu().numpy()
    b = b.double().cpu().numpy()
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


def test_noalloc_time_embed_matches_workspace_entry_point():
    cfg = B.time_cfg(320, 1280)
    m = Hn.Module("time", cfg)
    m.load(synth.canonical_weights(m.gen_rows(), seed=21))
    ref = torch.empty(1280, dtype=torch.float32, device="cuda")
    B.sd_time_embed(cfg, m.packed_dev, 500.0, ref, m.ws, m.ws_bytes)
    outs = []
    for t in (500.0, 500.0):  # two calls in a row share the scratch array
        o = torch.full((1280,), float("nan"), dtype=torch.float32, device="cuda")
        B.sd_time_embed_noalloc(cfg, m.packed_dev, t, o)
        outs.append(o)
    torch.cuda.synchronize()
    for o in outs:
        assert torch.isfinite(o).all()
        assert rel(o, ref) <= TOL
    # a different timestep in between must not leak into the next call
    other = torch.empty(1280, dtype=torch.float32, device="cuda")
    B.sd_time_embed_noalloc(cfg, m.packed_dev, 17.0, other)
    again = torch.empty(1280, dtype=torch.float32, device="cuda")
    B.sd_time_embed_noalloc(cfg, m.packed_dev, 500.0, again)
    torch.cuda.synchronize()
    assert rel(again, ref) <= TOL
    assert rel(other, ref) > 1e-2
    # sizes beyond the fixed scratch are rejected before any launch
    big = B.time_cfg(320, 8192)
    assert B.sd_time_embed_noalloc(big, m.packed_dev, 500.0, again, check=False) == 3
