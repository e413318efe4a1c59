"""Oracle of the coordinated noise initialisation (test infrastructure only).

DualParal write-up ("双重并行：让AI视频生成突破时长限制…", techwalker.com), §三
(coordinated noise initialisation): the full noise space keeps the video
globally consistent, repeated noise inside one denoising neighbourhood
hurts; so a new chunk takes its noise from a pool, avoiding what the last
NumC/2 latents of the tail chunk B_T use, and shuffles it.

reading (NumC is not defined on the pages): NumC = 2F, the latent frames of a
concatenated neighbourhood [B_{i-1}, B_i] of F-frame chunks.  The pool holds
2F noise frames drawn once.  Chunk k takes the F pool frames that chunk k-1
(the tail when k is pushed) does not use: frames 0..F-1 for even k, F..2F-1
for odd k; their order is a Fisher-Yates shuffle driven by the SplitMix64
stream (seed, 1002, k): for i = F-1 down to 1, swap position i with
position (draw_{F-1-i} mod (i+1)).
"""
from __future__ import annotations

import numpy as np

import synth


def chunk_frames(k: int, F: int, seed: int) -> list:
    """Pool frame indices of chunk k, in the order they fill frames 0..F-1."""
    base = 0 if k % 2 == 0 else F
    order = list(range(base, base + F))
    draws = synth.uniform_bits(synth.stream_key(seed, synth.TID_SHUFFLE, k), 0, max(F - 1, 0))
    for t, i in enumerate(range(F - 1, 0, -1)):
        j = int(draws[t] % np.uint64(i + 1))
        order[i], order[j] = order[j], order[i]
    return order


def coordinated_noise(pool: np.ndarray, k: int, seed: int) -> np.ndarray:
    """Chunk k's initial latent [C][F][H][W] gathered from the pool [2F][C][H][W]."""
    F = pool.shape[0] // 2
    fr = chunk_frames(k, F, seed)
    return np.stack([pool[b] for b in fr], axis=1)
