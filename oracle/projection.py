"""q, k, v projection with QK-Norm, fp64 (oracle side).  Test infrastructure:
only tests, the smoke check and the benchmark's CPU baseline use it.

Source: blog "Learning Video Generation from the Wan2.2 Source Code",
chapter 4, "3D RoPE: Letting Tokens Know Where They Are" (last paragraph):
inside the self-attention, q and k each pass through their linear layer and
then an RMSNorm (QK-Norm) that bounds the scale of the inner products; v
passes through its linear layer alone.  RoPE follows (oracle/rope.py).

Readings (the blog names the norm but prints none of its details): the linear
layers carry a bias (y = x W^T + b, W stored [out][in]); the RMSNorm runs over
the whole projected vector of a token (all heads, dim = heads x head_dim),
y / sqrt(mean(y^2) + eps) times a learned per-feature gain g, with eps = 1e-6;
the normalised vector is then split into heads, feature f to head f // D,
dimension f % D.
"""
from __future__ import annotations

import numpy as np

EPS = 1e-6


def linear(x, w, b=None) -> np.ndarray:
    """x [T][Din], w [Dout][Din], b [Dout] -> x w^T + b, fp64."""
    y = np.asarray(x, np.float64) @ np.asarray(w, np.float64).T
    if b is not None:
        y = y + np.asarray(b, np.float64)
    return y


def rms_norm(y, g, eps: float = EPS) -> np.ndarray:
    """Each row divided by its root mean square (plus eps under the root), then
    times the per-feature gain g."""
    y = np.asarray(y, np.float64)
    ms = np.mean(y * y, axis=-1, keepdims=True)
    return y / np.sqrt(ms + eps) * np.asarray(g, np.float64)


def split_heads(y, heads: int) -> np.ndarray:
    """[T][heads*D] -> [T][heads][D]: feature f to head f // D, dimension f % D."""
    y = np.asarray(y, np.float64)
    return y.reshape(y.shape[0], heads, y.shape[1] // heads)


def qkv(x, w, b, g_q, g_k, heads: int, eps: float = EPS):
    """q, k, v of the tokens x [T][dim]: w [3*dim][dim] holds W_q, W_k, W_v
    (rows 0..dim-1, dim..2*dim-1, 2*dim..3*dim-1), b [3*dim] their biases.
    Returns three [T][heads][D] fp64 arrays: q and k normalised, v not."""
    x = np.asarray(x, np.float64)
    w = np.asarray(w, np.float64)
    b = np.asarray(b, np.float64)
    dim = x.shape[1]
    q = rms_norm(linear(x, w[:dim], b[:dim]), g_q, eps)
    k = rms_norm(linear(x, w[dim:2 * dim], b[dim:2 * dim]), g_k, eps)
    v = linear(x, w[2 * dim:], b[2 * dim:])
    return split_heads(q, heads), split_heads(k, heads), split_heads(v, heads)
