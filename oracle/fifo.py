"""Oracle FIFO queue of latent chunks (float64), test infrastructure only.

DualParal write-up ("双重并行：让AI视频生成突破时长限制…", techwalker.com), §二:
the queue holds chunks of frames, each chunk sharing one noise level; levels
fall from T at the tail to 1 at the head.  After every diffusion step every
chunk moves one place toward the head, a new noisy chunk joins at the tail and
the clean chunk leaves at the head for the decoder.  The same section notes
that the frames per chunk are fixed, so chunks can be pushed without end.

reading: the queue starts empty.  "A new chunk joins after step s" is taken
as "step s+1 begins by pushing it"; both orders put the same chunks at the same
levels in every denoising pass.  Each pass denoises every queued chunk once
(x <- x + (sigma_{j-1} - sigma_j) v, the Euler step of a flow model), then the
level of every chunk drops by one and a chunk that reaches level 0 leaves.  A
stream of N chunks therefore takes N + T - 1 steps.  Fresh chunks are plain
N(0,1) noise (the write-up's coordinated noise initialisation is not used).
"""
from __future__ import annotations

import dataclasses
from typing import Callable, List, Optional

import numpy as np

from .dit import sigma

PRED_NONE = 0
PRED_IN_BATCH = 1
PRED_CACHE = 2


@dataclasses.dataclass
class Entry:
    chunk_id: int
    level: int
    latent: np.ndarray  # float64 [C][F][H][W]


@dataclasses.dataclass
class QueueState:
    T: int
    n_chunks: int               # -1 = unbounded
    step: int = 0
    next_id: int = 0
    entries: List[Entry] = dataclasses.field(default_factory=list)  # head first
    pred_id: int = -1           # chunk whose K/V are persisted, -1 = none
    pred_kv: Optional[list] = None
    ready: List[tuple] = dataclasses.field(default_factory=list)     # (id, latent)
    closed: bool = False

    def pushing(self) -> bool:
        if self.closed:
            return False
        return self.n_chunks < 0 or self.next_id < self.n_chunks

    def drained(self) -> bool:
        return not self.entries and not self.pushing()


@dataclasses.dataclass
class StepTrace:
    step: int
    chunk_ids: List[int]
    levels: List[int]
    positions: List[int]
    head_pred: int              # PRED_* of the head chunk
    popped: List[int]


def queue_step(st: QueueState, velocity_fn: Callable, noise: Optional[np.ndarray],
               use_pred: bool = True) -> StepTrace:
    """One queue step: push (tail), denoise every queued chunk, pop (head).

    velocity_fn(latents, levels, chunk_ids, pred_kv, keep_kv_of) -> (v list,
    kept kv) is the batched model of ``dit.make_velocity_fn`` or a stub.
    """
    if st.pushing():
        if noise is None:
            raise ValueError("a chunk is due for push but no noise was given")
        st.entries.append(Entry(st.next_id, st.T, np.asarray(noise, np.float64).copy()))
        st.next_id += 1
    if not st.entries:
        raise RuntimeError("queue drained")
    ids = [e.chunk_id for e in st.entries]
    levels = [e.level for e in st.entries]
    head = st.entries[0]
    if not use_pred or head.chunk_id == 0:
        head_pred, pred_kv = PRED_NONE, None
    else:
        # the head's predecessor left the queue in the previous step
        assert st.pred_id == head.chunk_id - 1, (st.pred_id, head.chunk_id)
        head_pred, pred_kv = PRED_CACHE, st.pred_kv
    # the chunk at level 1 leaves after this step: keep its K/V for the next head
    keep = 0 if head.level == 1 else None
    vs, kept = velocity_fn([e.latent for e in st.entries], levels, ids, pred_kv, keep)
    for e, v in zip(st.entries, vs):
        e.latent = e.latent + (sigma(e.level - 1, st.T) - sigma(e.level, st.T)) * v
        e.level -= 1
    popped = []
    while st.entries and st.entries[0].level == 0:
        e = st.entries.pop(0)
        st.ready.append((e.chunk_id, e.latent))
        popped.append(e.chunk_id)
        st.pred_id, st.pred_kv = e.chunk_id, kept
    tr = StepTrace(st.step, ids, levels, [j - 1 for j in levels], head_pred, popped)
    st.step += 1
    return tr


def run_stream(velocity_fn: Callable, noise_fn: Callable[[int], np.ndarray], T: int,
               n_chunks: int, use_pred: bool = True, max_steps: Optional[int] = None):
    """Runs a finite stream to the end.  Returns (popped [(id, latent)], traces)."""
    st = QueueState(T=T, n_chunks=n_chunks)
    traces = []
    while not st.drained():
        if max_steps is not None and st.step >= max_steps:
            break
        noise = noise_fn(st.next_id) if st.pushing() else None
        traces.append(queue_step(st, velocity_fn, noise, use_pred))
    return st.ready, traces


def euler_chunk(velocity_fn: Callable, noise: np.ndarray, T: int, chunk_id: int = 0):
    """A single chunk denoised alone from level T to 0 (no queue, no neighbour).

    Used to check that the queue, with the neighbour link off, reduces to the
    ordinary per-chunk Euler loop.
    """
    x = np.asarray(noise, np.float64).copy()
    for j in range(T, 0, -1):
        (v,), _ = velocity_fn([x], [j], [chunk_id], None, None)
        x = x + (sigma(j - 1, T) - sigma(j, T)) * v
    return x
