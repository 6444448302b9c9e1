"""Softmax attention by its definition, fp64 (oracle side).

Source: the attention a chunk computes over its same-step key set (PhysisServe
Wan2.2-5B model card, "Inference profile" and the paragraph below it): every
query of the chunk attends to every key of the set, with no causal mask
(blog "Learning Video Generation from the Wan2.2 Source Code", chapter 4:
full 3D joint attention).  Scale 1/sqrt(d) (standard scaled dot product).
"""
from __future__ import annotations

import numpy as np


def attend(q: np.ndarray, k: np.ndarray, v: np.ndarray):
    """One head: q [Lq, d], k [Lk, d], v [Lk, dv] -> (o [Lq, dv], lse [Lq]).

    z = q k^T / sqrt(d);  o = sum_k e^(z - m) v_k / sum_k e^(z - m);
    lse = m + ln sum_k e^(z - m), with m the row maximum.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    z = (q @ k.T) / np.sqrt(q.shape[1])
    m = z.max(axis=1, keepdims=True)
    e = np.exp(z - m)
    s = e.sum(axis=1, keepdims=True)
    return (e @ v) / s, (m + np.log(s))[:, 0]


def attend_heads(q: np.ndarray, k: np.ndarray, v: np.ndarray):
    """Token-major multi-head: q [Lq, H, d], k/v [Lk, H, d] -> (o [Lq, H, d], lse [Lq, H])."""
    Lq, H, d = q.shape
    o = np.empty((Lq, H, v.shape[2]))
    lse = np.empty((Lq, H))
    for hh in range(H):
        o[:, hh], lse[:, hh] = attend(q[:, hh], k[:, hh], v[:, hh])
    return o, lse


def softmax_weights(q: np.ndarray, k: np.ndarray) -> np.ndarray:
    """The attention matrix itself (one head), for invariant checks."""
    z = (np.asarray(q, np.float64) @ np.asarray(k, np.float64).T) / np.sqrt(q.shape[1])
    e = np.exp(z - z.max(axis=1, keepdims=True))
    return e / e.sum(axis=1, keepdims=True)


def masked_dense(q: np.ndarray, k: np.ndarray, v: np.ndarray, mask: np.ndarray):
    """Brute force: dense attention of q [Lq, d] over ALL keys k [N, d] with an explicit
    boolean mask [Lq, N]; masked logits are -inf.  Written element by element with a
    separate log-sum-exp so that it shares no vectorised path with `attend`."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    Lq, d = q.shape
    N = k.shape[0]
    out = np.zeros((Lq, v.shape[1]))
    lse = np.zeros(Lq)
    scale = 1.0 / np.sqrt(d)
    for i in range(Lq):
        logits = np.full(N, -np.inf)
        for j in range(N):
            if mask[i, j]:
                logits[j] = float(np.dot(q[i], k[j])) * scale
        top = np.max(logits)
        total = 0.0
        acc = np.zeros(v.shape[1])
        for j in range(N):
            if mask[i, j]:
                wgt = np.exp(logits[j] - top)
                total += wgt
                acc += wgt * v[j]
        out[i] = acc / total
        lse[i] = top + np.log(total)
    return out, lse
