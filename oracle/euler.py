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
