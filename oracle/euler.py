"""Flow-matching Euler update, fp64 (oracle side).

Source: blog "Learning Video Generation from the Wan2.2 Source Code",
chapter 1 ("From DDPM to Flow Matching": x_s = (1-s) x0 + s x1, velocity
v = x1 - x0, x0 = x_s - s v) and chapter 5 ("UniPC": the Euler step
x <- x - delta_sigma * v, first order).  Written with the signed step
sigma_next - sigma, which is negative while denoising.
"""
from __future__ import annotations

import numpy as np

#: The four-step schedule used here: sigma 1, .75, .5, .25 then 0.  The model
#: card fixes four steps per chunk and a sigma = 0 sink pass but prints no
#: sigmas; equal spacing is the plain reading.
SIGMAS_4 = (1.0, 0.75, 0.5, 0.25, 0.0)


def euler_step(x, v, sigma: float, sigma_next: float) -> np.ndarray:
    """x' = x + (sigma_next - sigma) * v, in fp64."""
    return np.asarray(x, np.float64) + (float(sigma_next) - float(sigma)) * np.asarray(v, np.float64)


def x0_prediction(x, v, sigma: float) -> np.ndarray:
    """Clean-data estimate x - sigma * v (blog chapter 1, flow_prediction)."""
    return np.asarray(x, np.float64) - float(sigma) * np.asarray(v, np.float64)


# ------------------------------------------------------------------ sampler variants
#: num_train_timesteps: t = 1000 * sigma (blog chapter 1, "Two Scales on One Ruler").
TRAIN_TIMESTEPS = 1000


def shift_sigma(sigma, shift: float):
    """The shift transform of the schedule (blog chapter 5, "shift: Where the 40
    Stops Land"): sigma' = shift * sigma / (1 + (shift - 1) * sigma)."""
    s = np.asarray(sigma, np.float64)
    return shift * s / (1.0 + (shift - 1.0) * s)


def shifted_schedule(n_steps: int, shift: float,
                     sigma_max: float = 1.0 - 1.0 / TRAIN_TIMESTEPS) -> np.ndarray:
    """n_steps + 1 sigmas: a uniform grid sigma_max * (1 - i / n_steps), shifted,
    then 0.  Reading: the blog says the points are first laid out uniformly and
    then shifted; a grid that starts one tick (1/1000) below the top of the ruler
    reproduces the timesteps it prints."""
    i = np.arange(n_steps, dtype=np.float64)
    s = shift_sigma(sigma_max * (1.0 - i / n_steps), shift)
    return np.concatenate([s, [0.0]])


def timesteps(sigmas) -> np.ndarray:
    """Integer timesteps of sigmas: 1000 * sigma, truncated (the blog prints the
    shifted schedule "rounded to integers"; truncation matches its values)."""
    return np.floor(TRAIN_TIMESTEPS * np.asarray(sigmas, np.float64)).astype(np.int64)


def cfg_combine(v_uncond, v_cond, guide_scale: float) -> np.ndarray:
    """Classifier-free guidance (blog chapter 5, "CFG"): uncond + w * (cond - uncond)."""
    u = np.asarray(v_uncond, np.float64)
    return u + float(guide_scale) * (np.asarray(v_cond, np.float64) - u)


def euler_cfg_step(x, v_cond, v_uncond, guide_scale: float, sigma: float,
                   sigma_next: float) -> np.ndarray:
    """The Euler step on the guided velocity."""
    return euler_step(x, cfg_combine(v_uncond, v_cond, guide_scale), sigma, sigma_next)
