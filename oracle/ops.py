"""Elementary operators of the U-Net denoiser, float64, plain definitions.

Test infrastructure only (see the package docstring). Activations are
``[C, H, W]`` arrays; token matrices are ``[N, C]``.

Sources (page title, then section or bullet):
* "Stable Diffusion 2.1 Base 宏观架构", section 4 (核心算子与任务差异): the
  ResnetBlock2D and Transformer2DModel panels list GroupNorm + SiLU + Conv,
  the time-embedding add, the residual/shortcut add, Norm -> self-attention,
  Norm -> cross-attention with K = V = context, Norm -> GEGLU.
* SD/SDXL tutorial page (bfzx365.com, video 67462879): the GSC bullet
  (GroupNorm + SiLU/Swish + Conv), the FeedForward bullet (GeGlU + Dropout +
  Linear), the DownSample bullet (Conv k3 s2 p1), the UpSample bullet (nearest
  interpolation + Conv k3 s1 p1), the BasicTransformer Block bullet (LayerNorm +
  self-attention + cross-attention + FeedForward, each residual), and the
  sinusoidal time embedding paragraph.
* SD1.5 anatomy page (hotelren.com, section 3.4, Conditioning Key): attention
  output Softmax(Q K^T / sqrt(d)) V.
"""
from __future__ import annotations

import math

import numpy as np
from scipy.special import erf as _erf


def bf16_round(x) -> np.ndarray:
    """Round to the nearest BF16 value (ties to even), returned as float64.

    The value is first rounded to float32, as the inputs of both sides are."""
    x32 = np.ascontiguousarray(np.asarray(x, dtype=np.float64).astype(np.float32))
    b = x32.view(np.uint32)
    with np.errstate(over="ignore"):
        r = (b + (np.uint32(0x7FFF) + ((b >> np.uint32(16)) & np.uint32(1)))) & np.uint32(0xFFFF0000)
    return r.view(np.float32).astype(np.float64)


def group_norm(x: np.ndarray, gamma: np.ndarray, beta: np.ndarray, groups: int = 32,
               eps: float = 1e-5) -> np.ndarray:
    """GroupNorm: channels split into ``groups`` runs of C/groups consecutive
    channels; each run is normalised by its mean and biased variance over
    (C/groups) x H x W, then scaled by gamma[c] and shifted by beta[c].
    (GSC bullet, tutorial page; ResnetBlock2D panel, SD2.1 page section 4.)"""
    C = x.shape[0]
    assert C % groups == 0
    xg = x.reshape(groups, -1)
    mean = xg.mean(axis=1, keepdims=True)
    var = ((xg - mean) ** 2).mean(axis=1, keepdims=True)
    y = ((xg - mean) / np.sqrt(var + eps)).reshape(x.shape)
    shape = (C,) + (1,) * (x.ndim - 1)
    return y * gamma.reshape(shape) + beta.reshape(shape)


def silu(x: np.ndarray) -> np.ndarray:
    """SiLU / Swish: x * sigmoid(x) = x / (1 + exp(-x)). (GSC bullet.)"""
    return x / (1.0 + np.exp(-x))


def conv2d(x: np.ndarray, w: np.ndarray, b: np.ndarray | None, stride: int = 1,
           pad: int = 1) -> np.ndarray:
    """2-D convolution of x [C_in, H, W] with w [C_out, C_in, k, k].

    y[o, i, j] = b[o] + sum_{c,u,v} w[o, c, u, v] * xp[c, s*i + u, s*j + v],
    where xp is x zero-padded by ``pad`` on every side. The zero padding applies
    to this function's own input (inside a GSC unit that is SiLU(GN(x))).
    Written as one tensor contraction over c per tap (u, v).
    (DownSample bullet: k3 s2 p1; UpSample bullet: k3 s1 p1.)"""
    C, H, W = x.shape
    O, C2, k, k2 = w.shape
    assert C == C2 and k == k2
    Ho = (H + 2 * pad - k) // stride + 1
    Wo = (W + 2 * pad - k) // stride + 1
    xp = np.zeros((C, H + 2 * pad, W + 2 * pad), dtype=np.float64)
    xp[:, pad:pad + H, pad:pad + W] = x
    y = np.zeros((O, Ho, Wo), dtype=np.float64)
    for u in range(k):
        for v in range(k):
            patch = xp[:, u:u + stride * (Ho - 1) + 1:stride, v:v + stride * (Wo - 1) + 1:stride]
            y += np.tensordot(w[:, :, u, v].astype(np.float64), patch, axes=([1], [0]))
    if b is not None:
        y += b.reshape(O, 1, 1)
    return y


def upsample_nearest2x(x: np.ndarray) -> np.ndarray:
    """Nearest-neighbour 2x: y[c, i, j] = x[c, floor(i/2), floor(j/2)].
    (UpSample bullet: nearest interpolation doubling the size.)"""
    return np.repeat(np.repeat(x, 2, axis=1), 2, axis=2)


def linear(t: np.ndarray, w: np.ndarray, b: np.ndarray | None) -> np.ndarray:
    """t [N, in] -> t w^T + b, w [out, in]."""
    y = t @ w.astype(np.float64).T
    if b is not None:
        y = y + b
    return y


def layer_norm(t: np.ndarray, gamma: np.ndarray, beta: np.ndarray, eps: float = 1e-5) -> np.ndarray:
    """LayerNorm over the channel axis of a token matrix t [N, C], biased
    variance, then gamma/beta. (BasicTransformer Block bullet.)"""
    mean = t.mean(axis=1, keepdims=True)
    var = ((t - mean) ** 2).mean(axis=1, keepdims=True)
    return (t - mean) / np.sqrt(var + eps) * gamma + beta


def attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, head_dim: int = 64) -> np.ndarray:
    """Multi-head scaled dot-product attention on projected tokens.

    q [Nq, C], k and v [Nk, C]; channel c belongs to head c // head_dim. Per
    head: S = Q_h K_h^T / sqrt(head_dim), P = row softmax of S (row maximum
    subtracted first), O_h = P V_h; the heads are concatenated back to [Nq, C].
    (SD1.5 anatomy page, section 3.4: Softmax(Q K^T / sqrt(d)) V.)"""
    Nq, C = q.shape
    assert C % head_dim == 0
    out = np.empty((Nq, C), dtype=np.float64)
    scale = 1.0 / math.sqrt(head_dim)
    for h in range(C // head_dim):
        sl = slice(h * head_dim, (h + 1) * head_dim)
        s = (q[:, sl] @ k[:, sl].T) * scale
        s -= s.max(axis=1, keepdims=True)
        p = np.exp(s)
        p /= p.sum(axis=1, keepdims=True)
        out[:, sl] = p @ v[:, sl]
    return out


def gelu(x: np.ndarray) -> np.ndarray:
    """Exact GELU: 0.5 x (1 + erf(x / sqrt(2)))."""
    return 0.5 * x * (1.0 + _erf(x / math.sqrt(2.0)))


def geglu_ff(t: np.ndarray, w1, b1, w2, b2) -> np.ndarray:
    """GEGLU feed-forward: u = t W1^T + b1 (8C wide), value a = u[:, :4C],
    gate g = u[:, 4C:], output (a * GELU(g)) W2^T + b2. Dropout is the
    identity at inference. (FeedForward bullet: GeGlU + Dropout + Linear.)"""
    u = linear(t, w1, b1)
    half = u.shape[1] // 2
    return linear(u[:, :half] * gelu(u[:, half:]), w2, b2)


def timestep_embedding(t: float, dim: int = 320) -> np.ndarray:
    """Sinusoidal embedding of a scalar timestep: [cos(t f_i) | sin(t f_i)],
    f_i = exp(-ln(10000) i / (dim/2)), i = 0 .. dim/2 - 1. The timestep is
    taken as a float32 value. (Tutorial page, sinusoidal embedding paragraph.)"""
    half = dim // 2
    i = np.arange(half, dtype=np.float64)
    f = np.exp(-math.log(10000.0) * i / half)
    a = float(np.float32(t)) * f
    return np.concatenate([np.cos(a), np.sin(a)])
