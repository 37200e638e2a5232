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


TILE_ROWS = 128  # one GEMM / attention tile of tokens (pixels)


def worst_tile(got, ref, rows=TILE_ROWS):
    """Worst 128-token tile of a [..., C] output: (index, error) where error is
    the tile's L2 error over the L2 norm the tile would have at the whole
    tensor's RMS (so a locally small reference does not inflate it), plus the
    largest element error over that RMS."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    cols = ref.shape[-1] if ref.ndim > 1 else 1
    g = got.reshape(-1, cols)
    r = ref.reshape(-1, cols)
    rms = max(float(np.sqrt(np.mean(r * r))), 1e-30)
    d = g - r
    n = g.shape[0]
    errs = []
    for t0 in range(0, n, rows):
        blk = d[t0:t0 + rows]
        errs.append(float(np.linalg.norm(blk)) / (rms * np.sqrt(blk.size)))
    i = int(np.argmax(errs))
    return i, errs[i], float(np.max(np.abs(d))) / rms


def assert_close(got, ref, tol, what="", tile_factor=3.0):
    """rel-L2 over the whole tensor below ``tol`` and no 128-token tile worse
    than ``tile_factor * tol`` (a wrong border strip or tail tile cannot hide
    under a good average); prints both."""
    err = rel_l2(got, ref)
    ti, terr, emax = worst_tile(got, ref)
    print(f"{what} rel_l2 {err:.3e} worst tile {ti} {terr:.3e} max |err|/rms {emax:.3e}")
    assert err < tol, (what, err)
    assert terr < tile_factor * tol, (what, ti, terr)
    return err


__all__ = ["oracle_params", "chw", "hwc", "dev_np", "rel_l2", "worst_tile", "assert_close", "oracle"]
