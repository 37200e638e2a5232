"""Noise schedules, the reverse-diffusion update and classifier-free guidance,
float64 (test infrastructure only; see the package docstring).

Sources (page title, then section or paragraph):
* SD/SDXL tutorial page (bfzx365.com, video 67462879), DDPM paragraphs: the
  forward step q(x_t | x_{t-1}) = N(sqrt(1 - beta_t) x_{t-1}, beta_t I); the
  linear schedule with beta_t rising linearly from 0.0001 to 0.02 over 1000
  steps (the schedule paragraph of the same page; beta_1 < ... < beta_T and
  alpha_bar_1 > ... > alpha_bar_T); the reverse-process mean
  mu = (x_t - (1 - alpha_t) / sqrt(1 - alpha_bar_t) * eps) / sqrt(alpha_t) with
  the untrained variance beta_t, i.e.
  x_{t-1} = (x_t - beta_t / sqrt(1 - alpha_bar_t) * eps) / sqrt(alpha_t) + sqrt(beta_t) z;
  the sampling loop that starts from Gaussian noise at step T and walks back to 0.
  The same page names the cosine schedule of "Improved Denoising Diffusion
  Probabilistic Models" (Nichol and Dhariwal, 2021) without printing it; it is
  written here from that paper: alpha_bar(t) = f(t) / f(0),
  f(t) = cos^2(((t / T + s) / (1 + s)) * pi / 2), s = 0.008, and
  beta_t = min(1 - alpha_bar_t / alpha_bar_{t-1}, 0.999).
* The same page names the DDIM scheduler (its beta_start default 0.00085)
  without printing its update; the deterministic DDIM step (eta = 0) is written
  from "Denoising Diffusion Implicit Models" (Song, Meng and Ermon, 2021):
  x0_hat = (x_t - sqrt(1 - alpha_bar_t) eps) / sqrt(alpha_bar_t),
  x_prev = sqrt(alpha_bar_prev) x0_hat + sqrt(1 - alpha_bar_prev) eps, with
  alpha_bar_prev = 1 past the first step.
* The SD1.5 anatomy page (section on the CFG scale) and the SD2.1 page
  (section 1, the "Timestep / Guidance" input) name classifier-free guidance
  without printing it; it is the standard combination
  eps = eps_uncond + s * (eps_cond - eps_uncond).

Timestep convention: arrays are indexed by t = 1 .. T stored at index t - 1.
"""
from __future__ import annotations

import math

import numpy as np


def linear_betas(T: int = 1000, beta_start: float = 1e-4, beta_end: float = 0.02) -> np.ndarray:
    """beta_t for t = 1 .. T, rising linearly from beta_start to beta_end."""
    if T == 1:
        return np.array([beta_start], dtype=np.float64)
    return np.array([beta_start + (beta_end - beta_start) * i / (T - 1) for i in range(T)], dtype=np.float64)


def cosine_betas(T: int = 1000, s: float = 0.008, max_beta: float = 0.999) -> np.ndarray:
    """beta_t of the cosine schedule (Nichol and Dhariwal, 2021)."""
    def f(t):
        return math.cos(((t / T + s) / (1.0 + s)) * math.pi / 2.0) ** 2
    out = []
    for t in range(1, T + 1):
        out.append(min(1.0 - f(t) / f(t - 1), max_beta))
    return np.array(out, dtype=np.float64)


def alphas_cumprod(betas: np.ndarray) -> np.ndarray:
    """alpha_bar_t = prod_{s <= t} (1 - beta_s), as a running product."""
    out = np.empty_like(betas)
    acc = 1.0
    for i, b in enumerate(betas):
        acc *= 1.0 - float(b)
        out[i] = acc
    return out


def cfg_combine(eps_cond, eps_uncond, scale: float):
    """Classifier-free guidance: eps_uncond + scale * (eps_cond - eps_uncond)."""
    eps_cond = np.asarray(eps_cond, dtype=np.float64)
    eps_uncond = np.asarray(eps_uncond, dtype=np.float64)
    return eps_uncond + scale * (eps_cond - eps_uncond)


def ddpm_step(x_t, eps, t: int, betas: np.ndarray, z=None):
    """One DDPM reverse step from t to t - 1 (t in 1 .. T): the page's update
    with alpha_t = 1 - beta_t and sigma_t = sqrt(beta_t); z = None adds no noise."""
    x_t = np.asarray(x_t, dtype=np.float64)
    eps = np.asarray(eps, dtype=np.float64)
    beta = float(betas[t - 1])
    alpha = 1.0 - beta
    abar = float(alphas_cumprod(betas)[t - 1])
    out = (x_t - beta / math.sqrt(1.0 - abar) * eps) / math.sqrt(alpha)
    if z is not None:
        out = out + math.sqrt(beta) * np.asarray(z, dtype=np.float64)
    return out


def ddim_step(x_t, eps, t: int, t_prev: int, betas: np.ndarray):
    """One deterministic DDIM step from t to t_prev (0 <= t_prev < t <= T)."""
    x_t = np.asarray(x_t, dtype=np.float64)
    eps = np.asarray(eps, dtype=np.float64)
    abar = alphas_cumprod(betas)
    a_t = float(abar[t - 1])
    a_prev = float(abar[t_prev - 1]) if t_prev > 0 else 1.0
    x0_hat = (x_t - math.sqrt(1.0 - a_t) * eps) / math.sqrt(a_t)
    return math.sqrt(a_prev) * x0_hat + math.sqrt(1.0 - a_prev) * eps


def denoise(x_T, timesteps, eps_fn, betas, kind="ddpm", guidance=None, noises=None):
    """The sampling loop: for each t of ``timesteps`` (descending), eps from
    ``eps_fn(x, t)`` -> (eps_cond, eps_uncond or None), guidance when given,
    then the DDPM or DDIM update to the next timestep (0 after the last).
    ``noises[i]`` is the z of step i (DDPM only; None = no noise)."""
    x = np.asarray(x_T, dtype=np.float64)
    ts = list(timesteps)
    for i, t in enumerate(ts):
        e_c, e_u = eps_fn(x, t)
        eps = cfg_combine(e_c, e_u, guidance) if (e_u is not None and guidance is not None) else \
            np.asarray(e_c, dtype=np.float64)
        if kind == "ddpm":
            z = None if noises is None else noises[i]
            x = ddpm_step(x, eps, t, betas, z)
        else:
            t_prev = ts[i + 1] if i + 1 < len(ts) else 0
            x = ddim_step(x, eps, t, t_prev, betas)
    return x
