"""Object wrappers over the C ABI (argument marshalling only).

``Model`` and ``Queue`` hold the C handles and turn numpy arrays (host) and
torch tensors (host or device) into pointers plus a dp_loc.  All work runs in
the CUDA library; nothing here computes.
"""
from __future__ import annotations

import ctypes as C

import numpy as np

from . import _binding as B


def _ptr(x, want_f32=True):
    """(pointer, location) of a numpy array or torch tensor (None -> NULL)."""
    if x is None:
        return None, B.DP_LOC_DEVICE
    if isinstance(x, np.ndarray):
        if want_f32 and x.dtype != np.float32:
            raise TypeError("expected float32")
        if not x.flags.c_contiguous:
            raise ValueError("expected a C-contiguous array")
        return x.ctypes.data, B.DP_LOC_HOST
    try:
        import torch
    except ImportError:  # pragma: no cover
        torch = None
    if torch is not None and isinstance(x, torch.Tensor):
        if want_f32 and x.dtype != torch.float32:
            raise TypeError("expected float32")
        if not x.is_contiguous():
            raise ValueError("expected a contiguous tensor")
        return x.data_ptr(), (B.DP_LOC_DEVICE if x.is_cuda else B.DP_LOC_HOST)
    raise TypeError(f"unsupported buffer type {type(x)}")


def _stream_handle(stream):
    if stream is None:
        return None
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream  # torch.cuda.Stream


class Model:
    """A DiT of the given shape on the current CUDA device.

    ``shape`` needs the attributes n_layers, dim, n_heads, ffn_dim, freq_dim,
    text_len, text_in_dim, latent_ch, patch_t, patch_h, patch_w.
    """

    def __init__(self, shape, precision="bf16", stream=None, neighbours="pred"):
        self.shape = shape
        self.cfg = B.dp_model_config(
            shape.n_layers, shape.dim, shape.n_heads, shape.ffn_dim, shape.freq_dim,
            shape.latent_ch, shape.patch_t, shape.patch_h, shape.patch_w, shape.text_len,
            shape.text_in_dim,
            B.DP_PREC_BF16 if precision == "bf16" else B.DP_PREC_FP32_VALIDATE,
            B.DP_NEIGHBOURS_BOTH if neighbours == "both" else B.DP_NEIGHBOURS_PRED,
            1 if getattr(shape, "qk_norm_rope", False) else 0)
        self.handle = C.c_void_p()
        B.check(B.dp_model_create(self.cfg, _stream_handle(stream), self.handle), "dp_model_create")
        self.queues = []

    def numel(self, name):
        n = C.c_longlong()
        B.check(B.dp_param_numel(self.cfg, B.PARAM_IDS[name], n), "dp_param_numel")
        return n.value

    def set_param(self, name, value, layer=0):
        p, loc = _ptr(value)
        n = value.size if isinstance(value, np.ndarray) else value.numel()
        B.check(B.dp_model_set_param(self.handle, B.PARAM_IDS[name], layer, p, n, loc),
                f"dp_model_set_param({name}, layer {layer})")

    def set_params(self, params):
        """params: name -> array, or name -> list of per-layer arrays."""
        for name, v in params.items():
            if isinstance(v, (list, tuple)):
                for l, a in enumerate(v):
                    self.set_param(name, a, l)
            else:
                self.set_param(name, v)

    def close(self):
        if self.handle:
            B.dp_destroy(self.handle)
            self.handle = C.c_void_p()
            for q in self.queues:
                q.handle = C.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


class Queue:
    """A FIFO denoising queue of ``T`` levels on a model."""

    def __init__(self, model, text, T, frames_per_chunk, lat_h, lat_w, n_chunks=-1,
                 ready_capacity=2, seed=3, noise="fresh"):
        self.model = model
        self.qc = B.dp_queue_config(T, frames_per_chunk, lat_h, lat_w, n_chunks, ready_capacity, seed,
                                    1 if noise == "coordinated" else 0)
        s = model.shape
        self.chunk_shape = (s.latent_ch, frames_per_chunk, lat_h, lat_w)
        self.chunk_numel = int(np.prod(self.chunk_shape))
        self.tokens = (frames_per_chunk // s.patch_t) * (lat_h // s.patch_h) * (lat_w // s.patch_w)
        p, loc = _ptr(text)
        self.handle = C.c_void_p()
        B.check(B.dp_queue_init(model.handle, self.qc, p, loc, self.handle), "dp_queue_init")
        model.queues.append(self)

    def step(self, noise=None):
        """One queue step; returns the dp status (raises on anything but OK)."""
        p, loc = _ptr(noise)
        return B.check(B.dp_queue_step(self.handle, p, loc), "dp_queue_step")

    def try_step(self, noise=None):
        p, loc = _ptr(noise)
        return B.dp_queue_step(self.handle, p, loc)

    def pop(self, out):
        p, loc = _ptr(out)
        cid = C.c_longlong(-1)
        B.check(B.dp_queue_pop(self.handle, p, loc, cid), "dp_queue_pop")
        return cid.value

    def try_pop(self, out):
        p, loc = _ptr(out)
        cid = C.c_longlong(-1)
        st = B.dp_queue_pop(self.handle, p, loc, cid)
        return st, cid.value

    def set_noise_pool(self, pool):
        p, loc = _ptr(pool)
        B.check(B.dp_queue_set_noise_pool(self.handle, p, loc), "dp_queue_set_noise_pool")

    def close_stream(self):
        B.check(B.dp_queue_close(self.handle), "dp_queue_close")

    def sync(self):
        return B.check(B.dp_queue_sync(self.handle), "dp_queue_sync")

    def selftest_timeout(self):
        """Enqueues the bounded-wait self test on the queue's stream."""
        B.check(B.dp_queue_selftest_timeout(self.handle), "dp_queue_selftest_timeout")

    def inspect(self):
        info = B.dp_queue_info()
        cap = self.qc.T
        ids = (C.c_longlong * cap)()
        lv = (C.c_int * cap)()
        sl = (C.c_int * cap)()
        pos = (C.c_int * cap)()
        B.check(B.dp_queue_inspect(self.handle, info, ids, lv, sl, pos, cap), "dp_queue_inspect")
        n = info.n
        return {"step": info.step, "next_push_id": info.next_push_id, "n": n,
                "head_pred": info.head_pred, "writes_cache": info.writes_cache,
                "n_ready": info.n_ready, "next_pop_id": info.next_pop_id,
                "drained": info.drained, "ids": list(ids[:n]), "levels": list(lv[:n]),
                "slots": list(sl[:n]), "positions": list(pos[:n])}

    def read_latents(self, n):
        out = np.empty((n,) + self.chunk_shape, np.float32)
        B.check(B.dp_queue_read_latents(self.handle, out.ctypes.data, n, B.DP_LOC_HOST),
                "dp_queue_read_latents")
        return out

    def load_state(self, step, n_pushed, latents, pred_kv=None):
        """latents [n][C][F][H][W] and pred_kv [layers][2][tokens][dim], float32:
        numpy arrays (host) or torch tensors, both at the same location."""
        if isinstance(latents, np.ndarray) or not hasattr(latents, "data_ptr"):
            latents = np.ascontiguousarray(latents, np.float32)
            if pred_kv is not None:
                pred_kv = np.ascontiguousarray(pred_kv, np.float32)
        lat, loc = _ptr(latents)
        kv, kv_loc = _ptr(pred_kv)
        if pred_kv is not None and kv_loc != loc:
            raise ValueError("latents and pred_kv must be at the same location")
        B.check(B.dp_queue_load_state(self.handle, step, n_pushed, latents.shape[0], lat, kv, loc),
                "dp_queue_load_state")

    def read_pred_kv(self):
        s = self.model.shape
        out = np.empty((s.n_layers, 2, self.tokens, s.dim), np.float32)
        cid = C.c_longlong(-1)
        B.check(B.dp_queue_read_pred_kv(self.handle, out.ctypes.data, B.DP_LOC_HOST, cid),
                "dp_queue_read_pred_kv")
        return out, cid.value

    def set_timing(self, on=True):
        B.check(B.dp_queue_set_timing(self.handle, 1 if on else 0), "dp_queue_set_timing")

    def timing(self):
        res = {}
        for k, name in enumerate(B.KCLASS_NAMES):
            ms, n, fl, by = C.c_double(), C.c_longlong(), C.c_double(), C.c_double()
            B.check(B.dp_queue_timing(self.handle, k, ms, n, fl, by), "dp_queue_timing")
            res[name] = {"ms": ms.value, "launches": n.value, "flops": fl.value, "bytes": by.value}
        return res

    def close(self):
        if self.handle:
            B.dp_queue_destroy(self.handle)
            self.handle = C.c_void_p()
            if self in self.model.queues:
                self.model.queues.remove(self)
