"""Helpers shared by the GPU parity tests: oracle parameters from a canonical
buffer, layout conversions and the error metric."""
import numpy as np

import oracle
from latent_diffusion_net_b200 import synth


def oracle_params(rows, canonical_u16, prefix_map=None):
    """name -> float32 array (BF16 values), sliced from the canonical buffer by
    the oracle's own enumeration (rows = [(name, shape, kind, fan_in), ...])."""
    out = {}
    off = 0
    vals = synth.bf16_bits_to_f32(canonical_u16)
    for name, shape, _, _ in rows:
        n = int(np.prod(shape))
        out[name] = vals[off:off + n].reshape(shape)
        off += n
    assert off == canonical_u16.size
    return out


def chw(x_hwc):
    return np.ascontiguousarray(np.asarray(x_hwc, dtype=np.float64).transpose(2, 0, 1))


def hwc(x_chw):
    return np.ascontiguousarray(np.asarray(x_chw).transpose(1, 2, 0))


def dev_np(t, shape):
    return t.float().cpu().numpy().reshape(shape).astype(np.float64)


def rel_l2(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.all(np.isfinite(got)), "non-finite values in the GPU output"
    return float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-30))


__all__ = ["oracle_params", "chw", "hwc", "dev_np", "rel_l2", "oracle"]
