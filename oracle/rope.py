"""3D rotary position embedding, fp64 (oracle side).

Source: blog "Learning Video Generation from the Wan2.2 Source Code",
chapter 4, section "3D RoPE: Letting Tokens Know Where They Are".  Each
head's d dimensions split into a time block of d - 4*(d//6) dimensions and
two spatial blocks of 2*(d//6) each; a token at (f, h, w) rotates each
(even, odd) pair of its q and k by an angle taken from its own coordinate on
that pair's axis, as one complex multiplication.  The blog states Wan runs
the rotation in float64.

Readings (the blog prints the split but not the frequency table): the pair
(x[2i], x[2i+1]) is the complex number x[2i] + i*x[2i+1]; within an axis
block of width d_a the local pair k turns at frequency theta^(-2k/d_a) with
theta = 10000, the usual RoPE base.
"""
from __future__ import annotations

import numpy as np


def axis_dims(head_dim: int) -> tuple[int, int, int]:
    """Widths (time, height, width) of the three axis blocks, in dimensions."""
    s = head_dim // 6
    return head_dim - 4 * s, 2 * s, 2 * s


def axis_pairs(head_dim: int) -> tuple[int, int, int]:
    t, h, w = axis_dims(head_dim)
    return t // 2, h // 2, w // 2


def pair_angles(f, h, w, head_dim: int, theta: float = 10000.0,
                pairs: tuple[int, int, int] | None = None) -> np.ndarray:
    """Rotation angle of every pair for tokens at coordinates (f, h, w).

    f, h, w are integer arrays of equal length n; returns [n, head_dim/2] fp64.
    """
    f = np.asarray(f, dtype=np.float64)
    h = np.asarray(h, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    pt, ph, pw = pairs if pairs is not None else axis_pairs(head_dim)
    if pt + ph + pw != head_dim // 2:
        raise ValueError("axis pairs must cover head_dim/2")
    cols = []
    for pos, npairs in ((f, pt), (h, ph), (w, pw)):
        width = 2 * npairs
        k = np.arange(npairs, dtype=np.float64)
        freq = theta ** (-2.0 * k / width)
        cols.append(pos[:, None] * freq[None, :])
    return np.concatenate(cols, axis=1)


def rotate(x: np.ndarray, f, h, w, theta: float = 10000.0,
           pairs: tuple[int, int, int] | None = None) -> np.ndarray:
    """Rotate x [n, heads, head_dim] (any float) by the 3D RoPE of each token; fp64 out."""
    x = np.asarray(x, dtype=np.float64)
    n, heads, d = x.shape
    ang = pair_angles(f, h, w, d, theta, pairs)            # [n, d/2]
    z = x[..., 0::2] + 1j * x[..., 1::2]                   # [n, heads, d/2]
    z = z * np.exp(1j * ang)[:, None, :]
    out = np.empty_like(x)
    out[..., 0::2] = z.real
    out[..., 1::2] = z.imag
    return out


def token_coords(n_tokens: int, width: int, height: int, frame0: int):
    """(f, h, w) of the tokens of consecutive frames starting at frame0.

    Tokens of a frame are row-major: t = h*width + w (reading adopted; the
    pages do not print the flattening order).
    """
    t = np.arange(n_tokens)
    per = width * height
    return frame0 + t // per, (t % per) // width, t % width
