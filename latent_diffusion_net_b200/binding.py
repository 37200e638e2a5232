"""ctypes binding of the C ABI declared in include/sd_api.h.

Argument marshalling only: every function here has the name of the C entry
point it calls and passes plain pointers and sizes through. The CUDA library
must be built (``python -m latent_diffusion_net_b200.build``); loading fails
loudly when it is missing. There is no fallback implementation.
"""
from __future__ import annotations

import ctypes
import os
from ctypes import POINTER, c_char, c_char_p, c_float, c_int32, c_int64, c_size_t, c_uint16, c_void_p

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libsd_b200.so")

SD_OK = 0
STATUS_NAMES = {0: "SD_OK", 1: "SD_ERR_NULL_ARG", 2: "SD_ERR_BAD_SHAPE", 3: "SD_ERR_UNSUPPORTED",
                4: "SD_ERR_MISALIGNED", 5: "SD_ERR_WORKSPACE_TOO_SMALL", 6: "SD_ERR_NOT_SM100",
                7: "SD_ERR_LAUNCH", 8: "SD_ERR_DEVICE_TIMEOUT", 9: "SD_ERR_CAPACITY"}
SD_KIND_WEIGHT, SD_KIND_BIAS, SD_KIND_NORM_GAMMA, SD_KIND_NORM_BETA = 0, 1, 2, 3
KIND_NAMES = {0: "weight", 1: "bias", 2: "norm_gamma", 3: "norm_beta"}
SD_CONV_IN, SD_CONV_DOWNSAMPLE, SD_CONV_UPSAMPLE, SD_CONV_OUTPUT = 0, 1, 2, 3


class SdError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)} ({status_string(status)})")


class sd_tensor_desc(ctypes.Structure):
    _fields_ = [("name", c_char * 80), ("ndim", c_int32), ("shape", c_int64 * 4), ("kind", c_int32),
                ("fan_in", c_int32), ("canon_offset", c_int64), ("packed_offset", c_int64)]


class sd_time_cfg(ctypes.Structure):
    _fields_ = [("proj_dim", c_int32), ("temb_dim", c_int32)]


class sd_conv_cfg(ctypes.Structure):
    _fields_ = [("batch", c_int32), ("height", c_int32), ("width", c_int32), ("c_in", c_int32),
                ("c_out", c_int32), ("groups", c_int32), ("eps", c_float)]


class sd_resblock_cfg(ctypes.Structure):
    _fields_ = [("batch", c_int32), ("height", c_int32), ("width", c_int32), ("c_x", c_int32),
                ("c_skip", c_int32), ("c_out", c_int32), ("temb_dim", c_int32), ("groups", c_int32),
                ("eps", c_float)]


class sd_transformer_cfg(ctypes.Structure):
    _fields_ = [("batch", c_int32), ("height", c_int32), ("width", c_int32), ("channels", c_int32),
                ("head_dim", c_int32), ("depth", c_int32), ("ctx_len", c_int32), ("ctx_dim", c_int32),
                ("groups", c_int32), ("gn_eps", c_float), ("ln_eps", c_float)]


class sd_unet_cfg(ctypes.Structure):
    _fields_ = [("in_channels", c_int32), ("out_channels", c_int32), ("height", c_int32), ("width", c_int32),
                ("n_levels", c_int32), ("block_channels", c_int32 * 4), ("attn_depth", c_int32 * 4),
                ("layers_per_block", c_int32), ("mid_depth", c_int32), ("head_dim", c_int32),
                ("ctx_len", c_int32), ("ctx_dim", c_int32), ("time_proj_dim", c_int32), ("temb_dim", c_int32),
                ("groups", c_int32), ("eps", c_float), ("add_text_dim", c_int32), ("add_time_ids", c_int32),
                ("add_time_dim", c_int32)]


class sd_vae_cfg(ctypes.Structure):
    _fields_ = [("height", c_int32), ("width", c_int32), ("latent_channels", c_int32), ("out_channels", c_int32),
                ("n_levels", c_int32), ("block_channels", c_int32 * 4), ("layers_per_block", c_int32),
                ("groups", c_int32), ("eps", c_float), ("scaling_factor", c_float)]


class sd_sampler_cfg(ctypes.Structure):
    _fields_ = [("kind", c_int32), ("n", c_int64), ("out_ch", c_int32), ("ld", c_int32), ("guidance", c_float),
                ("alpha_bar_t", ctypes.c_double), ("alpha_bar_prev", ctypes.c_double)]


SD_SCHED_LINEAR, SD_SCHED_COSINE = 0, 1
SD_SAMPLER_DDPM, SD_SAMPLER_DDIM = 0, 1


class sd_record_entry(ctypes.Structure):
    _fields_ = [("name", c_char * 8), ("module", c_int32), ("block", c_int32), ("offset", c_int64),
                ("rows", c_int64), ("cols", c_int64)]


class sd_launch_record(ctypes.Structure):
    _fields_ = [("kernel", c_char * 24), ("family", c_int32), ("kernels", c_int32), ("flops", ctypes.c_double),
                ("bytes", ctypes.c_double), ("ms", c_float)]


FAMILY_NAMES = {0: "gemm_tc", 1: "attention", 2: "gn_stats", 3: "gn_apply", 4: "layernorm", 5: "gemv", 6: "other"}

# name -> (restype, argtypes)
_P = c_void_p
_SIGS = {
    "sd_version": (c_char_p, []),
    "sd_status_string": (c_char_p, [c_int32]),
    "sd_time_weight_layout": (c_int32, [POINTER(sd_time_cfg), POINTER(sd_tensor_desc), c_int32, POINTER(c_int32),
                                        POINTER(c_int64), POINTER(c_int64)]),
    "sd_conv_weight_layout": (c_int32, [POINTER(sd_conv_cfg), c_int32, POINTER(sd_tensor_desc), c_int32,
                                        POINTER(c_int32), POINTER(c_int64), POINTER(c_int64)]),
    "sd_resblock_weight_layout": (c_int32, [POINTER(sd_resblock_cfg), POINTER(sd_tensor_desc), c_int32,
                                            POINTER(c_int32), POINTER(c_int64), POINTER(c_int64)]),
    "sd_transformer_weight_layout": (c_int32, [POINTER(sd_transformer_cfg), POINTER(sd_tensor_desc), c_int32,
                                               POINTER(c_int32), POINTER(c_int64), POINTER(c_int64)]),
    "sd_unet_weight_layout": (c_int32, [POINTER(sd_unet_cfg), POINTER(sd_tensor_desc), c_int32, POINTER(c_int32),
                                        POINTER(c_int64), POINTER(c_int64)]),
    "sd_time_pack_weights": (c_int32, [POINTER(sd_time_cfg), POINTER(c_uint16), _P]),
    "sd_conv_pack_weights": (c_int32, [POINTER(sd_conv_cfg), c_int32, POINTER(c_uint16), _P]),
    "sd_resblock_pack_weights": (c_int32, [POINTER(sd_resblock_cfg), POINTER(c_uint16), _P]),
    "sd_transformer_pack_weights": (c_int32, [POINTER(sd_transformer_cfg), POINTER(c_uint16), _P]),
    "sd_unet_pack_weights": (c_int32, [POINTER(sd_unet_cfg), POINTER(c_uint16), _P]),
    "sd_time_workspace_size": (c_size_t, [POINTER(sd_time_cfg)]),
    "sd_conv_workspace_size": (c_size_t, [POINTER(sd_conv_cfg), c_int32]),
    "sd_resblock_workspace_size": (c_size_t, [POINTER(sd_resblock_cfg)]),
    "sd_transformer_workspace_size": (c_size_t, [POINTER(sd_transformer_cfg)]),
    "sd_unet_workspace_size": (c_size_t, [POINTER(sd_unet_cfg)]),
    "sd_time_embed": (c_int32, [POINTER(sd_time_cfg), _P, c_float, _P, _P, c_size_t, _P]),
    "sd_time_embed_noalloc": (c_int32, [POINTER(sd_time_cfg), _P, c_float, _P, _P]),
    "sd_conv_fwd": (c_int32, [POINTER(sd_conv_cfg), c_int32, _P, _P, _P, _P, _P, _P, c_size_t, _P]),
    "sd_resblock_fwd": (c_int32, [POINTER(sd_resblock_cfg), _P, _P, _P, _P, _P, _P, c_size_t, _P]),
    "sd_transformer_fwd": (c_int32, [POINTER(sd_transformer_cfg), _P, _P, _P, _P, _P, c_size_t, _P]),
    "sd_unet_step": (c_int32, [POINTER(sd_unet_cfg), _P, _P, c_float, _P, _P, _P, c_size_t, _P]),
    "sd_unet_step_cond": (c_int32, [POINTER(sd_unet_cfg), _P, _P, c_float, _P, _P, POINTER(c_float), _P, _P,
                                    c_size_t, _P]),
    "sd_vae_weight_layout": (c_int32, [POINTER(sd_vae_cfg), POINTER(sd_tensor_desc), c_int32, POINTER(c_int32),
                                       POINTER(c_int64), POINTER(c_int64)]),
    "sd_vae_pack_weights": (c_int32, [POINTER(sd_vae_cfg), POINTER(c_uint16), _P]),
    "sd_vae_workspace_size": (c_size_t, [POINTER(sd_vae_cfg)]),
    "sd_vae_decode": (c_int32, [POINTER(sd_vae_cfg), _P, _P, _P, _P, c_size_t, _P]),
    "sd_schedule": (c_int32, [c_int32, c_int32, ctypes.c_double, ctypes.c_double, POINTER(ctypes.c_double)]),
    "sd_sampler_step": (c_int32, [POINTER(sd_sampler_cfg), _P, _P, _P, _P, _P, _P]),
    "sd_denoise_workspace_size": (c_size_t, [POINTER(sd_unet_cfg)]),
    "sd_denoise": (c_int32, [POINTER(sd_unet_cfg), _P, c_int32, POINTER(ctypes.c_double), c_int32, POINTER(c_int32),
                             c_int32, c_float, _P, _P, _P, _P, _P, _P, POINTER(c_float), _P, _P, c_size_t, _P]),
    "sd_record_begin": (c_int32, [_P, c_size_t]),
    "sd_record_end": (c_int32, [POINTER(c_int32)]),
    "sd_record_read": (c_int32, [POINTER(sd_record_entry), c_int32, POINTER(c_int32)]),
    "sd_debug_inject_timeout": (c_int32, [c_int32, c_int32]),
    "sd_query_device_status": (c_int32, [_P, _P]),
    "sd_profile_begin": (c_int32, []),
    "sd_profile_end": (c_int32, [POINTER(c_int32)]),
    "sd_profile_read": (c_int32, [POINTER(sd_launch_record), c_int32, POINTER(c_int32)]),
    "sd_launch_count": (c_int64, []),
    "sd_gemm_override": (c_int32, [c_int32, c_int32]),
}

_lib = None


def lib():
    """Load the shared library (once). Raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"CUDA library not built: {LIB_PATH} is missing "
                               "(run python -m latent_diffusion_net_b200.build)")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def exported_symbols():
    return list(_SIGS)


def status_string(s: int) -> str:
    try:
        return lib().sd_status_string(int(s)).decode()
    except Exception:  # noqa: BLE001 - used while formatting another error
        return "?"


def _check(status: int, where: str):
    if status != SD_OK:
        raise SdError(status, where)
    return status


def _ptr(x):
    """Device or host address of a torch tensor, an int, or None."""
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(s):
    if s is None:
        return None
    if isinstance(s, int):
        return s
    return s.cuda_stream


# ---------------------------------------------------------------- tables and packing

def _table(fn, *args):
    n = c_int32(0)
    ce = c_int64(0)
    pb = c_int64(0)
    _check(fn(*args, None, 0, ctypes.byref(n), ctypes.byref(ce), ctypes.byref(pb)), fn.__name__)
    arr = (sd_tensor_desc * n.value)()
    _check(fn(*args, arr, n.value, ctypes.byref(n), ctypes.byref(ce), ctypes.byref(pb)), fn.__name__)
    rows = []
    for d in arr:
        rows.append({"name": d.name.decode(), "shape": tuple(d.shape[i] for i in range(d.ndim)),
                     "kind": KIND_NAMES[d.kind], "fan_in": d.fan_in, "canon_offset": d.canon_offset,
                     "packed_offset": d.packed_offset})
    return rows, ce.value, pb.value


def sd_time_weight_layout(cfg):
    return _table(lib().sd_time_weight_layout, ctypes.byref(cfg))


def sd_conv_weight_layout(cfg, kind):
    return _table(lib().sd_conv_weight_layout, ctypes.byref(cfg), int(kind))


def sd_resblock_weight_layout(cfg):
    return _table(lib().sd_resblock_weight_layout, ctypes.byref(cfg))


def sd_transformer_weight_layout(cfg):
    return _table(lib().sd_transformer_weight_layout, ctypes.byref(cfg))


def sd_unet_weight_layout(cfg):
    return _table(lib().sd_unet_weight_layout, ctypes.byref(cfg))


def sd_vae_weight_layout(cfg):
    return _table(lib().sd_vae_weight_layout, ctypes.byref(cfg))


def _pack(fn, args, canonical_u16, packed_bytes):
    import numpy as np
    canon = np.ascontiguousarray(canonical_u16, dtype=np.uint16)
    out = np.empty(packed_bytes, dtype=np.uint8)
    _check(fn(*args, canon.ctypes.data_as(POINTER(c_uint16)), out.ctypes.data_as(c_void_p)), fn.__name__)
    return out


def sd_time_pack_weights(cfg, canonical_u16, packed_bytes):
    return _pack(lib().sd_time_pack_weights, (ctypes.byref(cfg),), canonical_u16, packed_bytes)


def sd_conv_pack_weights(cfg, kind, canonical_u16, packed_bytes):
    return _pack(lib().sd_conv_pack_weights, (ctypes.byref(cfg), int(kind)), canonical_u16, packed_bytes)


def sd_resblock_pack_weights(cfg, canonical_u16, packed_bytes):
    return _pack(lib().sd_resblock_pack_weights, (ctypes.byref(cfg),), canonical_u16, packed_bytes)


def sd_transformer_pack_weights(cfg, canonical_u16, packed_bytes):
    return _pack(lib().sd_transformer_pack_weights, (ctypes.byref(cfg),), canonical_u16, packed_bytes)


def sd_unet_pack_weights(cfg, canonical_u16, packed_bytes):
    return _pack(lib().sd_unet_pack_weights, (ctypes.byref(cfg),), canonical_u16, packed_bytes)


def sd_vae_pack_weights(cfg, canonical_u16, packed_bytes):
    return _pack(lib().sd_vae_pack_weights, (ctypes.byref(cfg),), canonical_u16, packed_bytes)


# ---------------------------------------------------------------- workspace sizes

def sd_time_workspace_size(cfg):
    return lib().sd_time_workspace_size(ctypes.byref(cfg))


def sd_conv_workspace_size(cfg, kind):
    return lib().sd_conv_workspace_size(ctypes.byref(cfg), int(kind))


def sd_resblock_workspace_size(cfg):
    return lib().sd_resblock_workspace_size(ctypes.byref(cfg))


def sd_transformer_workspace_size(cfg):
    return lib().sd_transformer_workspace_size(ctypes.byref(cfg))


def sd_unet_workspace_size(cfg):
    return lib().sd_unet_workspace_size(ctypes.byref(cfg))


def sd_vae_workspace_size(cfg):
    return lib().sd_vae_workspace_size(ctypes.byref(cfg))


# ---------------------------------------------------------------- forward calls
# Each returns the status (SD_OK) or raises SdError; pass check=False to get
# the raw status instead.

def sd_time_embed(cfg, packed_w, timestep, temb_out, workspace, ws_bytes, stream=None, check=True):
    s = lib().sd_time_embed(ctypes.byref(cfg), _ptr(packed_w), float(timestep), _ptr(temb_out), _ptr(workspace),
                            int(ws_bytes), _stream(stream))
    return _check(s, "sd_time_embed") if check else s


def sd_time_embed_noalloc(cfg, packed_w, timestep, temb_out, stream=None, check=True):
    """Workspace-free time embedding (fixed device scratch inside the library)."""
    s = lib().sd_time_embed_noalloc(ctypes.byref(cfg), _ptr(packed_w), float(timestep), _ptr(temb_out),
                                    _stream(stream))
    return _check(s, "sd_time_embed_noalloc") if check else s


def sd_conv_fwd(cfg, kind, packed_w, x0, x1, x2, y, workspace, ws_bytes, stream=None, check=True):
    s = lib().sd_conv_fwd(ctypes.byref(cfg), int(kind), _ptr(packed_w), _ptr(x0), _ptr(x1), _ptr(x2), _ptr(y),
                          _ptr(workspace), int(ws_bytes), _stream(stream))
    return _check(s, "sd_conv_fwd") if check else s


def sd_resblock_fwd(cfg, packed_w, x, skip, temb, y, workspace, ws_bytes, stream=None, check=True):
    s = lib().sd_resblock_fwd(ctypes.byref(cfg), _ptr(packed_w), _ptr(x), _ptr(skip), _ptr(temb), _ptr(y),
                              _ptr(workspace), int(ws_bytes), _stream(stream))
    return _check(s, "sd_resblock_fwd") if check else s


def sd_transformer_fwd(cfg, packed_w, x, context, y, workspace, ws_bytes, stream=None, check=True):
    s = lib().sd_transformer_fwd(ctypes.byref(cfg), _ptr(packed_w), _ptr(x), _ptr(context), _ptr(y),
                                 _ptr(workspace), int(ws_bytes), _stream(stream))
    return _check(s, "sd_transformer_fwd") if check else s


def sd_unet_step(cfg, packed_w, latent, timestep, context, eps_out, workspace, ws_bytes, stream=None, check=True):
    s = lib().sd_unet_step(ctypes.byref(cfg), _ptr(packed_w), _ptr(latent), float(timestep), _ptr(context),
                           _ptr(eps_out), _ptr(workspace), int(ws_bytes), _stream(stream))
    return _check(s, "sd_unet_step") if check else s


def sd_unet_step_cond(cfg, packed_w, latent, timestep, context, add_text, add_time_ids, eps_out, workspace,
                      ws_bytes, stream=None, check=True):
    """add_time_ids: a sequence of host floats (or None)."""
    ids = None
    if add_time_ids is not None:
        vals = [float(v) for v in add_time_ids]
        ids = (c_float * max(len(vals), 1))(*vals)
    s = lib().sd_unet_step_cond(ctypes.byref(cfg), _ptr(packed_w), _ptr(latent), float(timestep), _ptr(context),
                                _ptr(add_text), ids, _ptr(eps_out), _ptr(workspace), int(ws_bytes), _stream(stream))
    return _check(s, "sd_unet_step_cond") if check else s


def sd_schedule(kind, T=1000, beta_start=1e-4, beta_end=0.02):
    """alpha_bar_t for t = 1..T as a list of floats (host only)."""
    out = (ctypes.c_double * int(T))()
    _check(lib().sd_schedule(int(kind), int(T), float(beta_start), float(beta_end), out), "sd_schedule")
    return list(out)


def sampler_cfg(kind, n, alpha_bar_t, alpha_bar_prev, guidance=1.0, out_ch=4, ld=None):
    return sd_sampler_cfg(int(kind), int(n), int(out_ch), int(out_ch if ld is None else ld), float(guidance),
                          float(alpha_bar_t), float(alpha_bar_prev))


def sd_sampler_step(cfg, x, eps_cond, eps_uncond=None, noise=None, x_bf16=None, stream=None, check=True):
    s = lib().sd_sampler_step(ctypes.byref(cfg), _ptr(x), _ptr(eps_cond), _ptr(eps_uncond), _ptr(noise),
                              _ptr(x_bf16), _stream(stream))
    return _check(s, "sd_sampler_step") if check else s


def sd_denoise_workspace_size(cfg):
    return lib().sd_denoise_workspace_size(ctypes.byref(cfg))


def sd_denoise(cfg, packed_w, kind, alphas_cumprod, timesteps, guidance, x, cond_latent, ctx_cond, ctx_uncond,
               add_text_cond, add_text_uncond, add_time_ids, noise, workspace, ws_bytes, stream=None, check=True):
    """alphas_cumprod, timesteps, add_time_ids: host sequences; the rest device tensors (or None)."""
    ac = (ctypes.c_double * len(alphas_cumprod))(*[float(v) for v in alphas_cumprod])
    ts = (c_int32 * len(timesteps))(*[int(t) for t in timesteps])
    ids = None
    if add_time_ids is not None:
        ids = (c_float * max(len(add_time_ids), 1))(*[float(v) for v in add_time_ids])
    s = lib().sd_denoise(ctypes.byref(cfg), _ptr(packed_w), int(kind), ac, len(alphas_cumprod), ts, len(timesteps),
                         float(guidance), _ptr(x), _ptr(cond_latent), _ptr(ctx_cond), _ptr(ctx_uncond),
                         _ptr(add_text_cond), _ptr(add_text_uncond), ids, _ptr(noise), _ptr(workspace),
                         int(ws_bytes), _stream(stream))
    return _check(s, "sd_denoise") if check else s


def sd_record_begin(dev_buf, nbytes):
    return _check(lib().sd_record_begin(_ptr(dev_buf), int(nbytes)), "sd_record_begin")


def sd_record_end(check=True):
    """Returns (status, number of entries)."""
    n = c_int32(0)
    s = lib().sd_record_end(ctypes.byref(n))
    if check:
        _check(s, "sd_record_end")
    return s, n.value


def sd_record_read():
    """Entries of the last recording: list of dicts (name, module, block, offset, rows, cols)."""
    n = c_int32(0)
    _check(lib().sd_record_read(None, 0, ctypes.byref(n)), "sd_record_read")
    arr = (sd_record_entry * max(n.value, 1))()
    _check(lib().sd_record_read(arr, n.value, ctypes.byref(n)), "sd_record_read")
    return [{"name": e.name.decode(), "module": e.module, "block": e.block, "offset": e.offset, "rows": e.rows,
             "cols": e.cols} for e in arr[:n.value]]


def sd_debug_inject_timeout(n_launches, spin_limit=1024):
    return _check(lib().sd_debug_inject_timeout(int(n_launches), int(spin_limit)), "sd_debug_inject_timeout")


def sd_vae_decode(cfg, packed_w, latent, image, workspace, ws_bytes, stream=None, check=True):
    s = lib().sd_vae_decode(ctypes.byref(cfg), _ptr(packed_w), _ptr(latent), _ptr(image), _ptr(workspace),
                            int(ws_bytes), _stream(stream))
    return _check(s, "sd_vae_decode") if check else s


def sd_query_device_status(workspace, stream=None):
    return lib().sd_query_device_status(_ptr(workspace), _stream(stream))


def sd_profile_begin():
    return _check(lib().sd_profile_begin(), "sd_profile_begin")


def sd_profile_end():
    n = c_int32(0)
    _check(lib().sd_profile_end(ctypes.byref(n)), "sd_profile_end")
    return n.value


def sd_profile_read():
    """Records of the last recording: list of dicts (kernel, family, flops, bytes, ms)."""
    n = c_int32(0)
    _check(lib().sd_profile_read(None, 0, ctypes.byref(n)), "sd_profile_read")
    arr = (sd_launch_record * max(n.value, 1))()
    _check(lib().sd_profile_read(arr, n.value, ctypes.byref(n)), "sd_profile_read")
    return [{"kernel": r.kernel.decode(), "family": FAMILY_NAMES.get(r.family, r.family), "kernels": r.kernels,
             "flops": r.flops, "bytes": r.bytes, "ms": r.ms} for r in arr[:n.value]]


def sd_launch_count():
    return int(lib().sd_launch_count())


def sd_gemm_override(bn=0, splits=0):
    """Fix the GEMM N tile and reduction split count (0 = automatic)."""
    _check(lib().sd_gemm_override(int(bn), int(splits)), "sd_gemm_override")


# ---------------------------------------------------------------- config helpers

def time_cfg(proj_dim=320, temb_dim=1280):
    return sd_time_cfg(proj_dim, temb_dim)


def conv_cfg(height, width, c_in, c_out, groups=32, eps=1e-5):
    return sd_conv_cfg(1, height, width, c_in, c_out, groups, eps)


def resblock_cfg(height, width, c_x, c_out, c_skip=0, temb_dim=1280, groups=32, eps=1e-5):
    return sd_resblock_cfg(1, height, width, c_x, c_skip, c_out, temb_dim, groups, eps)


def transformer_cfg(height, width, channels, depth=1, ctx_len=77, ctx_dim=1024, groups=32, eps=1e-5):
    return sd_transformer_cfg(1, height, width, channels, 64, depth, ctx_len, ctx_dim, groups, eps, eps)


def unet_cfg(in_channels=4, out_channels=4, height=96, width=96, block_channels=(320, 640, 1280, 1280),
             attn_depth=(1, 1, 1, 0), layers_per_block=2, mid_depth=1, ctx_len=77, ctx_dim=1024,
             time_proj_dim=320, temb_dim=1280, groups=32, eps=1e-5, add_text_dim=0, add_time_ids=0,
             add_time_dim=256):
    bc = list(block_channels) + [0] * (4 - len(block_channels))
    ad = list(attn_depth) + [0] * (4 - len(attn_depth))
    return sd_unet_cfg(in_channels, out_channels, height, width, len(block_channels), (c_int32 * 4)(*bc),
                       (c_int32 * 4)(*ad), layers_per_block, mid_depth, 64, ctx_len, ctx_dim, time_proj_dim,
                       temb_dim, groups, eps, add_text_dim, add_time_ids, add_time_dim)


def vae_cfg(height, width, latent_channels=4, out_channels=3, block_channels=(128, 256, 512, 512),
            layers_per_block=2, groups=32, eps=1e-5, scaling_factor=0.18215):
    bc = list(block_channels) + [0] * (4 - len(block_channels))
    return sd_vae_cfg(height, width, latent_channels, out_channels, len(block_channels), (c_int32 * 4)(*bc),
                      layers_per_block, groups, eps, scaling_factor)


def unet_cfg_from(ocfg, height, width):
    """C config of an oracle UNetConfig (same field names)."""
    return unet_cfg(in_channels=ocfg.in_channels, out_channels=ocfg.out_channels, height=height, width=width,
                    block_channels=ocfg.block_channels, attn_depth=ocfg.attn_depth,
                    layers_per_block=ocfg.layers_per_block, mid_depth=ocfg.mid_depth, ctx_len=ocfg.ctx_len,
                    ctx_dim=ocfg.ctx_dim, time_proj_dim=ocfg.time_proj_dim, temb_dim=ocfg.temb_dim,
                    groups=ocfg.groups, eps=ocfg.eps, add_text_dim=ocfg.add_text_dim,
                    add_time_ids=ocfg.add_time_ids, add_time_dim=ocfg.add_time_dim)
