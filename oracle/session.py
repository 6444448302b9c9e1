"""One stream's same-step KV history, driven through a chunk schedule (oracle side).

Source: PhysisServe Wan2.2-5B model card, "Inference profile" and the
paragraph below it.  Per (layer, step) the stream keeps the K/V that each
chunk recorded at that step; the first chunk's clean K/V from the sigma = 0
bootstrap pass form the sink that every later chunk reads at every step.

Order of use for one chunk and one (layer, step): rotate q and k, record the
chunk's k and v, then attend (append before attend).  Keys are rotated once,
at the frame where they were recorded (absolute latent-frame positions;
reading adopted, the card does not say).
"""
from __future__ import annotations

import numpy as np

from . import attention, rope
from .schedule import BOOT, FIRST, STEADY, Geometry, RingModel

SINK_STEP = "sink"


class StreamSession:
    def __init__(self, geom: Geometry, pairs: tuple[int, int, int] | None = None):
        self.geom = geom
        self.pairs = pairs
        self.ring = RingModel(geom)
        self.sink: dict = {}      # layer -> (K, V)   fp64 [n, H, d]
        self.first: dict = {}     # (layer, step) -> (K, V) while the first chunk denoises
        self.slot_kv: dict = {}   # (layer, step, slot) -> (K, V)

    # --- schedule -------------------------------------------------------
    def begin_chunk(self, nframes: int) -> None:
        self.ring.begin_chunk(nframes)

    def coords(self):
        frames = self.ring.current_frames()
        n = len(frames) * self.geom.tokens_per_frame
        return rope.token_coords(n, self.geom.width, self.geom.height, frames[0])

    # --- the hot path ----------------------------------------------------
    def rope_append(self, layer: int, step, q, k, v) -> np.ndarray:
        """Rotate q, k [n, H, d]; record (k_rot, v); return q_rot (fp64)."""
        f, h, w = self.coords()
        q_rot = rope.rotate(q, f, h, w, self.geom.theta, self.pairs)
        k_rot = rope.rotate(k, f, h, w, self.geom.theta, self.pairs)
        v = np.asarray(v, np.float64)
        if step == SINK_STEP:
            self.ring.bootstrap()
            self.sink[layer] = (k_rot, v)
        elif self.ring.phase == FIRST:
            self.first[(layer, step)] = (k_rot, v)
        elif self.ring.phase == STEADY:
            self.slot_kv[(layer, step, self.ring.current_slot())] = (k_rot, v)
        else:
            raise ValueError("only the sink pass may run between the first chunk and chunk 1")
        return q_rot

    def key_set(self, layer: int, step):
        """(K, V) [Lk, H, d] that the current chunk reads at (layer, step)."""
        if step == SINK_STEP:
            if self.ring.phase != BOOT:
                raise ValueError("sink attention belongs to the bootstrap pass")
            return self.sink[layer]
        if self.ring.phase == FIRST:
            return self.first[(layer, step)]
        if self.ring.phase != STEADY:
            raise ValueError("no denoising step between the bootstrap and chunk 1")
        ks, vs = [self.sink[layer][0]], [self.sink[layer][1]]
        for slot, c in enumerate(self.ring.slots):
            if c is not None:
                kk, vv = self.slot_kv[(layer, step, slot)]
                ks.append(kk)
                vs.append(vv)
        return np.concatenate(ks, axis=0), np.concatenate(vs, axis=0)

    def chunk_attn(self, layer: int, step, q_rot):
        """(o [Lq, H, d], lse [Lq, H]) of the current chunk at (layer, step)."""
        K, V = self.key_set(layer, step)
        return attention.attend_heads(q_rot, K, V)
