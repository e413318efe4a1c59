"""Seeded synthetic inputs shared by the oracle, the tests and the benchmark.

This module holds the workload shapes and the random-number generator that
produces every input (weights, biases, modulation tables, text tokens and the
per-chunk latent noise).  It holds none of the denoising arithmetic: nothing
here knows what a layer, an attention or an Euler step computes.

Generator (a published counter-based construction, restated):

* SplitMix64 (Steele, Lea and Flood, "Fast splittable pseudorandom number
  generators", OOPSLA 2014): the state advances by the odd constant
  GAMMA = 0x9E3779B97F4A7C15 and each output is the 64-bit finaliser
  ``mix64`` of the state.  The i-th draw of a stream with key ``k`` is
  ``mix64(k + (i + 1) * GAMMA)`` (mod 2**64), so any draw can be computed
  without the ones before it.
* A stream key is derived from ``(seed, a, b)`` by three chained mixes:
  ``k = mix64((seed + 1) * GAMMA); k = mix64(k + (a + 1) * GAMMA);
  k = mix64(k + (b + 1) * GAMMA)``.  ``a`` names the tensor, ``b`` a layer or
  a chunk id.
* Normal deviates come from the Box-Muller transform (Box and Muller, 1958)
  evaluated in float64: draws ``2i`` and ``2i+1`` give
  ``u1 = ((d0 >> 11) + 1) * 2**-53`` in (0, 1] and ``u2 = (d1 >> 11) * 2**-53``
  in [0, 1); ``r = sqrt(-2 ln u1)``; outputs ``r cos(2 pi u2)`` then
  ``r sin(2 pi u2)``.  The result is scaled by ``std`` in float64 and rounded
  once to float32.

Seeds follow the workload recipe: weights use seed 1, text seed 2 and the
noise of chunk ``k`` uses seed 3 with ``b = k``.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)
_MASK = (1 << 64) - 1

SEED_WEIGHTS = 1
SEED_TEXT = 2
SEED_NOISE = 3

# Tensor ids used as ``a`` in the stream key.
TID_TEXT = 1000
TID_NOISE = 1001
TID_SHUFFLE = 1002      # draws of the coordinated-noise permutation of chunk b
TID_NOISE_POOL = 1003   # noise pool frame b (coordinated noise)


def _mix64_int(z: int) -> int:
    z &= _MASK
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _MASK
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _MASK
    return z ^ (z >> 31)


def stream_key(seed: int, a: int, b: int) -> int:
    g = 0x9E3779B97F4A7C15
    k = _mix64_int(((seed + 1) * g) & _MASK)
    k = _mix64_int((k + (a + 1) * g) & _MASK)
    k = _mix64_int((k + (b + 1) * g) & _MASK)
    return k


def _mix64_vec(z: np.ndarray) -> np.ndarray:
    z = (z ^ (z >> np.uint64(30))) * _M1
    z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def uniform_bits(key: int, start: int, count: int) -> np.ndarray:
    """Draws ``start .. start+count-1`` of the SplitMix64 stream with ``key``."""
    with np.errstate(over="ignore"):
        i = np.arange(start + 1, start + count + 1, dtype=np.uint64)
        z = np.uint64(key) + i * GAMMA
        return _mix64_vec(z)


def normal(seed: int, a: int, b: int, n: int, std: float = 1.0) -> np.ndarray:
    """``n`` float32 N(0, std^2) deviates of stream (seed, a, b), Box-Muller."""
    key = stream_key(seed, a, b)
    out = np.empty(n, dtype=np.float32)
    chunk = 1 << 22  # pairs per block; bounds the temporaries
    npairs = (n + 1) // 2
    for p0 in range(0, npairs, chunk):
        p1 = min(npairs, p0 + chunk)
        d = uniform_bits(key, 2 * p0, 2 * (p1 - p0))
        d0 = d[0::2] >> np.uint64(11)
        d1 = d[1::2] >> np.uint64(11)
        u1 = (d0.astype(np.float64) + 1.0) * 2.0 ** -53
        u2 = d1.astype(np.float64) * 2.0 ** -53
        r = np.sqrt(-2.0 * np.log(u1))
        th = 2.0 * math.pi * u2
        z = np.empty(2 * (p1 - p0), dtype=np.float64)
        z[0::2] = r * np.cos(th)
        z[1::2] = r * np.sin(th)
        lo = 2 * p0
        hi = min(n, 2 * p1)
        out[lo:hi] = (z[: hi - lo] * std).astype(np.float32)
    return out


# --------------------------------------------------------------------------
# Workload shapes
# --------------------------------------------------------------------------


@dataclasses.dataclass(frozen=True)
class ModelShape:
    n_layers: int
    dim: int
    n_heads: int
    ffn_dim: int
    freq_dim: int
    text_len: int
    text_in_dim: int
    latent_ch: int = 16
    patch_t: int = 1
    patch_h: int = 2
    patch_w: int = 2
    qk_norm_rope: bool = False   # per-head RMSNorm of q, k and 3-D rotary positions

    @property
    def head_dim(self) -> int:
        return self.dim // self.n_heads

    @property
    def patch_dim(self) -> int:
        return self.latent_ch * self.patch_t * self.patch_h * self.patch_w


@dataclasses.dataclass(frozen=True)
class QueueShape:
    T: int
    frames_per_chunk: int
    lat_h: int
    lat_w: int
    n_chunks: int

    def chunk_shape(self, m: ModelShape):
        return (m.latent_ch, self.frames_per_chunk, self.lat_h, self.lat_w)

    def chunk_numel(self, m: ModelShape) -> int:
        return m.latent_ch * self.frames_per_chunk * self.lat_h * self.lat_w

    def tokens_per_chunk(self, m: ModelShape) -> int:
        return ((self.frames_per_chunk // m.patch_t) * (self.lat_h // m.patch_h)
                * (self.lat_w // m.patch_w))


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    model: ModelShape
    queue: QueueShape
    precision: str  # "fp32" (validation mode) or "bf16"


WORKLOADS = {
    # 2 layers, dim 64, 4 heads, FFN 256; 8x8 latent, 2 frames per chunk
    "tiny_fp32": Workload(
        "tiny_fp32",
        ModelShape(n_layers=2, dim=64, n_heads=4, ffn_dim=256, freq_dim=64,
                   text_len=8, text_in_dim=64),
        QueueShape(T=4, frames_per_chunk=2, lat_h=8, lat_w=8, n_chunks=6),
        "fp32"),
    # 8 layers, dim 512, 8 heads, FFN 2048; 32x32 latent, 4 frames per chunk
    "small_bf16": Workload(
        "small_bf16",
        ModelShape(n_layers=8, dim=512, n_heads=8, ffn_dim=2048, freq_dim=256,
                   text_len=64, text_in_dim=512),
        QueueShape(T=10, frames_per_chunk=4, lat_h=32, lat_w=32, n_chunks=32),
        "bf16"),
    # Wan2.1-1.3B-shaped: 30 layers, dim 1536, 12 heads, FFN 8960; 480x832 video
    "wan1.3b_480p": Workload(
        "wan1.3b_480p",
        ModelShape(n_layers=30, dim=1536, n_heads=12, ffn_dim=8960, freq_dim=256,
                   text_len=512, text_in_dim=4096),
        QueueShape(T=50, frames_per_chunk=2, lat_h=60, lat_w=104, n_chunks=64),
        "bf16"),
    # the same model streaming 128 chunks (256 latent frames)
    "wan1.3b_480p_long": Workload(
        "wan1.3b_480p_long",
        ModelShape(n_layers=30, dim=1536, n_heads=12, ffn_dim=8960, freq_dim=256,
                   text_len=512, text_in_dim=4096),
        QueueShape(T=50, frames_per_chunk=2, lat_h=60, lat_w=104, n_chunks=128),
        "bf16"),
    # Wan2.1-14B-shaped: 40 layers, dim 5120, 40 heads, FFN 13824; 720x1280 video
    "wan14b_720p": Workload(
        "wan14b_720p",
        ModelShape(n_layers=40, dim=5120, n_heads=40, ffn_dim=13824, freq_dim=256,
                   text_len=512, text_in_dim=4096),
        QueueShape(T=50, frames_per_chunk=2, lat_h=90, lat_w=160, n_chunks=16),
        "bf16"),
}


def truncated(w: Workload, n_layers: int) -> Workload:
    """The same workload with fewer layers (per-chunk shapes unchanged)."""
    return dataclasses.replace(w, model=dataclasses.replace(w.model, n_layers=n_layers))


def with_qk_norm_rope(w: Workload) -> Workload:
    """The same workload with per-head QK RMSNorm and 3-D rotary positions."""
    return dataclasses.replace(w, model=dataclasses.replace(w.model, qk_norm_rope=True))


# --------------------------------------------------------------------------
# Parameter inventory: (name, shape, per_layer).  Linear weights are stored
# [out][in] row-major.  Tensor id ``a`` of a parameter is its index here.
# --------------------------------------------------------------------------


def param_specs(m: ModelShape):
    d, F, D, P = m.dim, m.ffn_dim, m.freq_dim, m.patch_dim
    specs = [
        ("patch.w", (d, P), False),
        ("patch.b", (d,), False),
    ]
    if m.text_in_dim != d:
        specs += [("text.w", (d, m.text_in_dim), False), ("text.b", (d,), False)]
    specs += [
        ("time1.w", (d, D), False),
        ("time1.b", (d,), False),
        ("time2.w", (d, d), False),
        ("time2.b", (d,), False),
        ("mod.w", (6 * d, d), False),
        ("mod.b", (6 * d,), False),
        ("headmod.w", (2 * d, d), False),
        ("headmod.b", (2 * d,), False),
        ("out.w", (P, d), False),
        ("out.b", (P,), False),
        ("layer.mod", (6 * d,), True),
        ("layer.qkv.w", (3 * d, d), True),
        ("layer.qkv.b", (3 * d,), True),
        ("layer.o.w", (d, d), True),
        ("layer.o.b", (d,), True),
        ("layer.cq.w", (d, d), True),
        ("layer.cq.b", (d,), True),
        ("layer.ck.w", (d, d), True),
        ("layer.ck.b", (d,), True),
        ("layer.cv.w", (d, d), True),
        ("layer.cv.b", (d,), True),
        ("layer.co.w", (d, d), True),
        ("layer.co.b", (d,), True),
        ("layer.ffn1.w", (F, d), True),
        ("layer.ffn1.b", (F,), True),
        ("layer.ffn2.w", (d, F), True),
        ("layer.ffn2.b", (d,), True),
    ]
    if m.qk_norm_rope:
        specs += [("layer.qnorm.w", (d,), True), ("layer.knorm.w", (d,), True)]
    return specs


ALL_PARAM_NAMES = [s[0] for s in param_specs(ModelShape(1, 8, 1, 8, 8, 1, 16, qk_norm_rope=True))]


def param_tensor_id(name: str) -> int:
    return ALL_PARAM_NAMES.index(name)


WEIGHT_STD = 0.02


def make_params(m: ModelShape, seed: int = SEED_WEIGHTS, std: float = WEIGHT_STD):
    """Every parameter ~ N(0, std^2), float32, except the RMSNorm weights
    (names ending in "norm.w"), which are 1 + N(0, std^2).  Per-layer ones are
    lists."""
    out = {}
    for name, shape, per_layer in param_specs(m):
        a = param_tensor_id(name)
        n = int(np.prod(shape))
        mean = np.float32(1.0) if name.endswith("norm.w") else np.float32(0.0)
        if per_layer:
            out[name] = [normal(seed, a, l, n, std).reshape(shape) + mean for l in range(m.n_layers)]
        else:
            out[name] = normal(seed, a, 0, n, std).reshape(shape) + mean
    return out


def make_text(m: ModelShape, seed: int = SEED_TEXT) -> np.ndarray:
    return normal(seed, TID_TEXT, 0, m.text_len * m.text_in_dim).reshape(
        m.text_len, m.text_in_dim)


def make_noise_pool(m: ModelShape, q: QueueShape, seed: int = SEED_NOISE) -> np.ndarray:
    """2F latent frames of N(0,1) noise, [2F][C][H][W]; frame b from stream b."""
    n = m.latent_ch * q.lat_h * q.lat_w
    return np.stack([normal(seed, TID_NOISE_POOL, b, n).reshape(m.latent_ch, q.lat_h, q.lat_w)
                     for b in range(2 * q.frames_per_chunk)])


def make_noise(m: ModelShape, q: QueueShape, chunk_id: int, seed: int = SEED_NOISE) -> np.ndarray:
    shape = q.chunk_shape(m)
    return normal(seed, TID_NOISE, chunk_id, int(np.prod(shape))).reshape(shape)
