"""Chunk / ring bookkeeping of same-step KV inference (oracle side).

Source: PhysisServe Wan2.2-5B model card, "Inference profile" table (first
chunk 3 latent frames, later chunks 1 frame, 29 chunks, attention sink from a
clean bootstrap at sigma = 0, history of up to 18 recent chunks plus the sink
without duplication) and the paragraph below it (at step s a chunk reads KV
recorded at the same step s; the first chunk gets one extra pass that builds
the sink).

Reading adopted where the card is silent: the ring of R slots includes the
current chunk (append, then attend), so a chunk j >= 1 sees chunks
max(1, j-R+1)..j; the first chunk lives only in the sink.

This model keeps an explicit list of slots and evicts the oldest chunk when
all slots are taken; it does not use the closed forms that the tests check
it against.
"""
from __future__ import annotations

from dataclasses import dataclass, field

NEW, FIRST, BOOT, STEADY = "NEW", "FIRST", "BOOT", "STEADY"


@dataclass
class Geometry:
    """Token geometry of one latent frame and the KV history.

    width x height tokens per latent frame (1280x704 at 32x32 compression gives
    40 x 22, Wan2.2 TI2V-5B page, "High Compression"); heads x head_dim.
    """
    width: int
    height: int
    heads: int
    head_dim: int
    first_frames: int = 3
    ring_slots: int = 18
    steps: int = 4
    theta: float = 10000.0

    @property
    def tokens_per_frame(self) -> int:
        return self.width * self.height

    @property
    def sink_tokens(self) -> int:
        return self.first_frames * self.tokens_per_frame


@dataclass
class RingModel:
    """Phase machine and slot table of one stream."""
    geom: Geometry
    phase: str = NEW
    chunk: int = -1
    slots: list = field(default_factory=list)   # slot -> chunk id or None

    def __post_init__(self):
        self.slots = [None] * self.geom.ring_slots

    def begin_chunk(self, nframes: int) -> None:
        if self.phase == NEW:
            if nframes != self.geom.first_frames:
                raise ValueError("the first chunk has first_frames frames")
            self.phase, self.chunk = FIRST, 0
            return
        if self.phase == FIRST:
            raise ValueError("the sink bootstrap pass must run before chunk 1")
        if nframes != 1:
            raise ValueError("chunks after the first hold one latent frame")
        self.chunk += 1
        self.phase = STEADY
        free = [i for i, c in enumerate(self.slots) if c is None]
        if free:
            slot = free[0]
        else:
            oldest = min(self.slots)
            slot = self.slots.index(oldest)
        self.slots[slot] = self.chunk

    def bootstrap(self) -> None:
        """The extra sigma = 0 pass over the clean first chunk."""
        if self.phase not in (FIRST, BOOT):
            raise ValueError("bootstrap belongs to the first chunk")
        self.phase = BOOT

    # --- queries -------------------------------------------------------
    def frame_of_chunk(self, j: int) -> int:
        """Latent-frame index of chunk j >= 1 (chunk 0 holds frames 0..first_frames-1)."""
        return self.geom.first_frames - 1 + j

    def current_frames(self) -> list[int]:
        if self.chunk == 0:
            return list(range(self.geom.first_frames))
        return [self.frame_of_chunk(self.chunk)]

    def current_slot(self) -> int:
        """Slot that the current chunk (>= 1) occupies; -1 during the first chunk."""
        if self.chunk < 1:
            return -1
        return self.slots.index(self.chunk)

    def fill(self) -> int:
        return sum(c is not None for c in self.slots)

    def slot_frames(self) -> list[int]:
        return [-1 if c is None else self.frame_of_chunk(c) for c in self.slots]

    def chunks_in_history(self) -> list[int]:
        """Chunk ids (>= 1) whose same-step KV the current chunk reads, by slot order."""
        return [c for c in self.slots if c is not None]

    def n_keys(self) -> int:
        """Keys the current chunk attends to at one step."""
        if self.phase in (FIRST, BOOT):
            return self.geom.sink_tokens
        return self.geom.sink_tokens + self.fill() * self.geom.tokens_per_frame


def attention_flops(n_queries: int, n_keys: int, heads: int, head_dim: int) -> int:
    """Algorithmic FLOPs of one softmax attention: two matrix products of
    2*Lq*Lk*d each (blog, chapter 8: 2 x 2 x L^2 x dim for self-attention)."""
    return 4 * n_queries * n_keys * heads * head_dim


def latent_frames_of_schedule(n_chunks: int, first_frames: int = 3) -> int:
    """Latent frames produced by a schedule of n_chunks (first chunk first_frames)."""
    return first_frames + (n_chunks - 1)


def video_frames_of_latent(latent_frames: int, time_stride: int = 4) -> int:
    """Decoded frames of a causal VAE: the first frame alone, then time_stride per latent
    frame (blog, chapter 2, "Where 4n+1 Comes From")."""
    return (latent_frames - 1) * time_stride + 1
