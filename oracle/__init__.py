"""Oracle: a plain, slow, float64 CPU statement of one block-wise FIFO denoising
queue, used ONLY as test infrastructure.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and
its Python binding) never imports, links or executes anything here, and this
package never imports the product.  The two share only the seeded input
generator in ``synth`` (which holds none of the method's arithmetic).

Source of the method: the DualParal write-up
"双重并行：让AI视频生成突破时长限制，新加坡国立大学团队实现分钟级长视频创作"
(techwalker.com, 2025-05-30), on "Minute-Long Videos with Dual Parallelisms":

* §一 (dual-parallel architecture): the video is cut into non-overlapping
  temporal chunks, each at its own noise level, later chunks noisier; one
  inference step denoises all chunks at once.
* §二 (FIFO queue and block-wise denoising): queue elements are chunks that
  share one noise level, decreasing from T at the tail to 1 at the head; after
  every diffusion step each chunk moves one place forward, a fresh noisy chunk
  enters at the tail and the clean one leaves at the head for decoding.
* §三 (feature cache and coordinated noise init): a chunk needs its neighbour's
  information only in self-attention; the neighbour's self-attention K/V are
  reused from a cache instead of concatenating the neighbour's input;
  cross-attention and the FFN are strictly per chunk.

The pages give no formula for the DiT block, the timestep embedding or the
flow parameterisation.  Every step they leave open is written here in its
plainest form and marked ``reading:`` at the point of use.

Parity status: every function here is pinned by tests that do not reuse this
code (tests/test_oracle_pins.py, tests/test_oracle_composition_pins.py):
closed forms, brute-force loops, textbook values, invariants, a hand-derived
queue trace, and hand-derived values (fixtures under tests/golden/) for the
per-level timestep embedding and modulation, the prompt's per-layer K/V and
the composed DiT velocity of a one-layer d = 4 model on two chunks.  Planted
mistakes (a swapped shift and scale, a misordered modulation split, swapped
gates, a missing SiLU, an unscaled timestep, the tanh GELU, a dropped LN eps)
each break one of them.
"""

from . import dit, fifo  # noqa: F401
