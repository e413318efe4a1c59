"""Block-wise FIFO video denoising (DualParal-style queue) on one B200.

The compute lives in the CUDA library ``libdp_b200.so`` (C ABI in
``include/dp.h`` and ``include/dp_ops.h``); this package only loads it and
marshals arguments.  Build it with ``python -m chunked_fifo_denoising_b200.build``.
"""
from . import _binding  # noqa: F401
from ._binding import DPError, lib  # noqa: F401
from .queue import Model, Queue  # noqa: F401
