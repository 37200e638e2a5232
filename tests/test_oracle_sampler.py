"""Pins for the oracle's noise schedules, reverse-diffusion updates, guidance
and SDXL added conditioning (CPU only).

Checks use values the pages print (the linear schedule's end points), textbook
identities of diffusion models (the DDPM posterior mean of Ho, Jain and Abbeel
2020, equation 7; the DDIM consistency property of Song, Meng and Ermon 2021),
closed forms and special cases, not the oracle's own formulas."""
import math

import numpy as np
import pytest

from oracle import model, sampler


def test_linear_schedule_matches_page():
    """Tutorial page, schedule paragraph: beta rises linearly from 0.0001 to
    0.02 over 1000 steps; beta increasing and alpha_bar decreasing."""
    b = sampler.linear_betas(1000, 1e-4, 0.02)
    assert b.shape == (1000,)
    assert b[0] == pytest.approx(1e-4, abs=1e-18) and b[-1] == pytest.approx(0.02, abs=1e-17)
    d = np.diff(b)
    np.testing.assert_allclose(d, (0.02 - 1e-4) / 999, rtol=1e-9)
    a = sampler.alphas_cumprod(b)
    assert a[0] == pytest.approx(1 - 1e-4, abs=1e-16)
    assert np.all(np.diff(a) < 0)
    # alpha_bar_T = prod (1 - beta): compare with the exponential of a sum of logs
    assert a[-1] == pytest.approx(math.exp(sum(math.log1p(-x) for x in b)), rel=1e-12)


def test_cosine_schedule_shape():
    """Cosine schedule: beta increasing and clipped at 0.999 at the end,
    alpha_bar near cos^2 (pi t / 2T), i.e. about 1/2 half way."""
    b = sampler.cosine_betas(1000)
    a = sampler.alphas_cumprod(b)
    assert np.all(np.diff(b) > 0)
    assert b[-1] == pytest.approx(0.999)
    assert abs(a[499] - 0.5) < 0.01
    assert a[0] > 0.9999 and a[-1] < 1e-6


def make_xt(seed, t, betas):
    r = np.random.default_rng(seed)
    x0 = r.standard_normal((4, 6, 5))
    eps = r.standard_normal((4, 6, 5))
    ab = sampler.alphas_cumprod(betas)[t - 1]
    return x0, eps, math.sqrt(ab) * x0 + math.sqrt(1 - ab) * eps


@pytest.mark.parametrize("t", [2, 17, 500, 1000])
def test_ddpm_mean_is_the_posterior_mean(t):
    """With the true noise, the reverse mean equals the posterior mean
    mu~(x_t, x_0) = sqrt(ab_{t-1}) beta_t / (1 - ab_t) x_0
    + sqrt(alpha_t) (1 - ab_{t-1}) / (1 - ab_t) x_t."""
    betas = sampler.linear_betas()
    x0, eps, xt = make_xt(t, t, betas)
    ab = sampler.alphas_cumprod(betas)
    abt, abp, beta = ab[t - 1], ab[t - 2], betas[t - 1]
    mu = math.sqrt(abp) * beta / (1 - abt) * x0 + math.sqrt(1 - beta) * (1 - abp) / (1 - abt) * xt
    np.testing.assert_allclose(sampler.ddpm_step(xt, eps, t, betas), mu, rtol=1e-10, atol=1e-12)


def test_ddpm_zero_eps_and_noise():
    betas = sampler.linear_betas()
    r = np.random.default_rng(3)
    x = r.standard_normal(10)
    z = r.standard_normal(10)
    t = 321
    beta = betas[t - 1]
    np.testing.assert_allclose(sampler.ddpm_step(x, np.zeros(10), t, betas, z),
                               x / math.sqrt(1 - beta) + math.sqrt(beta) * z, rtol=1e-14)


@pytest.mark.parametrize("t,t_prev", [(981, 961), (500, 480), (21, 1), (21, 0)])
def test_ddim_consistency(t, t_prev):
    """Deterministic DDIM with the true noise lands on the same trajectory:
    sqrt(ab_prev) x_0 + sqrt(1 - ab_prev) eps (x_0 itself at t_prev = 0)."""
    betas = sampler.linear_betas(1000, 0.00085, 0.012)
    x0, eps, xt = make_xt(t + t_prev, t, betas)
    ab = sampler.alphas_cumprod(betas)
    ap = ab[t_prev - 1] if t_prev > 0 else 1.0
    np.testing.assert_allclose(sampler.ddim_step(xt, eps, t, t_prev, betas),
                               math.sqrt(ap) * x0 + math.sqrt(1 - ap) * eps, rtol=1e-9, atol=1e-11)


def test_ddim_loop_recovers_x0():
    betas = sampler.cosine_betas(1000)
    ab = sampler.alphas_cumprod(betas)
    r = np.random.default_rng(9)
    x0 = r.standard_normal(32)
    e0 = r.standard_normal(32)
    ts = list(range(999, 0, -111))
    xT = math.sqrt(ab[ts[0] - 1]) * x0 + math.sqrt(1 - ab[ts[0] - 1]) * e0

    def eps_fn(x, t):
        return (x - math.sqrt(ab[t - 1]) * x0) / math.sqrt(1 - ab[t - 1]), None

    np.testing.assert_allclose(sampler.denoise(xT, ts, eps_fn, betas, kind="ddim"), x0, rtol=1e-8, atol=1e-9)


def test_cfg_combine_special_cases():
    r = np.random.default_rng(4)
    c, u = r.standard_normal(7), r.standard_normal(7)
    np.testing.assert_array_equal(sampler.cfg_combine(c, u, 0.0), u)
    np.testing.assert_allclose(sampler.cfg_combine(c, u, 1.0), c, rtol=0, atol=1e-15)
    np.testing.assert_allclose(sampler.cfg_combine(c, u, 7.5) - sampler.cfg_combine(c, u, 6.5), c - u, atol=1e-13)


def test_add_embedding_order_and_fourier_blocks():
    """SDXL added conditioning: the pooled text comes first, then six 256-wide
    Fourier blocks; phi(0) is 128 ones then 128 zeros, so an all-ones first
    layer sees sum(text) + 6 * 128."""
    cfg = model.SDXL_INPAINT
    D, T = cfg.add_embed_dim, cfg.temb_dim
    r = np.random.default_rng(5)
    text = r.standard_normal(1280)
    p = {"add.lin1.weight": np.ones((T, D)), "add.lin1.bias": np.zeros(T),
         "add.lin2.weight": np.eye(T), "add.lin2.bias": np.zeros(T)}
    out = model.add_embedding(p, text, [0.0] * 6, cfg)
    h = text.sum() + 6 * 128
    np.testing.assert_allclose(out, np.full(T, h / (1 + math.exp(-h))), rtol=1e-12)
    # selecting the text columns returns SiLU(text)
    w1 = np.zeros((T, D))
    w1[:, :1280] = np.eye(1280)
    p["add.lin1.weight"] = w1
    out = model.add_embedding(p, text, [1024.0, 1024.0, 0.0, 0.0, 1024.0, 1024.0], cfg)
    np.testing.assert_allclose(out, text / (1 + np.exp(-text)), rtol=1e-12)
