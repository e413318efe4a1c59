"""ctypes binding of libdp_b200.so (include/dp.h and include/dp_ops.h).

Argument marshalling only: every function here forwards to the C entry point
of the same name.  The library must have been built (``build.py``); importing
this module without it raises, so there is no silent fallback.
"""
from __future__ import annotations

import ctypes as C
import os

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libdp_b200.so")

# --- enums (mirror dp.h / dp_ops.h) -----------------------------------------
DP_OK, DP_ERR_INVALID_ARG, DP_ERR_OOM, DP_ERR_CUDA, DP_ERR_EMPTY, DP_ERR_FULL, \
    DP_ERR_DRAINED, DP_ERR_STATE, DP_ERR_KERNEL = range(9)
STATUS_NAMES = ["DP_OK", "DP_ERR_INVALID_ARG", "DP_ERR_OOM", "DP_ERR_CUDA", "DP_ERR_EMPTY",
                "DP_ERR_FULL", "DP_ERR_DRAINED", "DP_ERR_STATE", "DP_ERR_KERNEL"]
DP_PREC_BF16, DP_PREC_FP32_VALIDATE = 0, 1
DP_LOC_DEVICE, DP_LOC_HOST = 0, 1
DP_NEIGHBOURS_PRED, DP_NEIGHBOURS_BOTH = 0, 1
DP_DT_F32, DP_DT_BF16 = 0, 1
DP_EPI_STORE, DP_EPI_GELU, DP_EPI_RESID, DP_EPI_RESID_GATED = 0, 1, 2, 3
DP_KCLASS_COUNT = 7
KCLASS_NAMES = ["gemm", "self_attention", "cross_attention", "layernorm_mod", "patch_embed",
                "head_euler", "other"]

PARAM_IDS = {
    "patch.w": 0, "patch.b": 1, "text.w": 2, "text.b": 3,
    "time1.w": 4, "time1.b": 5, "time2.w": 6, "time2.b": 7,
    "mod.w": 8, "mod.b": 9, "headmod.w": 10, "headmod.b": 11, "out.w": 12, "out.b": 13,
    "layer.mod": 14, "layer.qkv.w": 15, "layer.qkv.b": 16, "layer.o.w": 17, "layer.o.b": 18,
    "layer.cq.w": 19, "layer.cq.b": 20, "layer.ck.w": 21, "layer.ck.b": 22,
    "layer.cv.w": 23, "layer.cv.b": 24, "layer.co.w": 25, "layer.co.b": 26,
    "layer.ffn1.w": 27, "layer.ffn1.b": 28, "layer.ffn2.w": 29, "layer.ffn2.b": 30,
    "layer.qnorm.w": 31, "layer.knorm.w": 32,
}
DP_PARAM_COUNT = 33


class dp_model_config(C.Structure):
    _fields_ = [("n_layers", C.c_int), ("dim", C.c_int), ("n_heads", C.c_int),
                ("ffn_dim", C.c_int), ("freq_dim", C.c_int), ("latent_ch", C.c_int),
                ("patch_t", C.c_int), ("patch_h", C.c_int), ("patch_w", C.c_int),
                ("text_len", C.c_int), ("text_in_dim", C.c_int), ("prec", C.c_int),
                ("neighbours", C.c_int), ("qk_norm_rope", C.c_int)]


class dp_queue_config(C.Structure):
    _fields_ = [("T", C.c_int), ("frames_per_chunk", C.c_int), ("lat_h", C.c_int),
                ("lat_w", C.c_int), ("n_chunks", C.c_longlong), ("ready_capacity", C.c_int),
                ("seed", C.c_ulonglong), ("noise_mode", C.c_int)]


class dp_queue_info(C.Structure):
    _fields_ = [("step", C.c_longlong), ("next_push_id", C.c_longlong), ("n", C.c_int),
                ("head_pred", C.c_int), ("writes_cache", C.c_int), ("n_ready", C.c_int),
                ("next_pop_id", C.c_longlong), ("drained", C.c_int)]


class dp_gemm_args(C.Structure):
    _fields_ = [("dtype", C.c_int), ("A", C.c_void_p), ("lda", C.c_longlong), ("W", C.c_void_p),
                ("bias", C.c_void_p), ("M", C.c_int), ("N", C.c_int), ("K", C.c_int),
                ("epi", C.c_int), ("out", C.c_void_p), ("ldo", C.c_longlong),
                ("resid", C.c_void_p), ("ldr", C.c_longlong), ("gate", C.c_void_p),
                ("gate_stride", C.c_longlong), ("chunk_sel", C.c_void_p),
                ("rows_per_chunk", C.c_int), ("cache", C.c_void_p), ("cache_row0", C.c_longlong),
                ("cache_rows", C.c_int), ("cache_col0", C.c_int), ("ldc", C.c_longlong)]


class dp_attn_args(C.Structure):
    _fields_ = [("dtype", C.c_int), ("n_chunks", C.c_int), ("Lq", C.c_int), ("n_heads", C.c_int),
                ("head_dim", C.c_int), ("q", C.c_void_p), ("ldq", C.c_longlong),
                ("k", C.c_void_p), ("v", C.c_void_p), ("ldkv", C.c_longlong),
                ("kv_chunk_rows", C.c_longlong), ("Lk", C.c_int), ("pred_in_batch", C.c_int),
                ("k0_pred", C.c_void_p), ("v0_pred", C.c_void_p), ("ld_pred", C.c_longlong),
                ("Lk_pred", C.c_int), ("out", C.c_void_p), ("ldo", C.c_longlong),
                ("succ_in_batch", C.c_int)]


class dp_ln_args(C.Structure):
    _fields_ = [("out_dtype", C.c_int), ("x", C.c_void_p), ("ldx", C.c_longlong), ("M", C.c_int),
                ("d", C.c_int), ("shift", C.c_void_p), ("scale", C.c_void_p),
                ("mod_stride", C.c_longlong), ("chunk_sel", C.c_void_p),
                ("rows_per_chunk", C.c_int), ("out", C.c_void_p), ("ldo", C.c_longlong)]


# name: (restype, argtypes)
_SIGS = {
    "dp_set_allocator": (C.c_int, [C.c_void_p, C.c_void_p, C.c_void_p]),
    "dp_param_numel": (C.c_int, [C.POINTER(dp_model_config), C.c_int, C.POINTER(C.c_longlong)]),
    "dp_model_create": (C.c_int, [C.POINTER(dp_model_config), C.c_void_p, C.POINTER(C.c_void_p)]),
    "dp_model_set_param": (C.c_int, [C.c_void_p, C.c_int, C.c_int, C.c_void_p, C.c_longlong, C.c_int]),
    "dp_queue_init": (C.c_int, [C.c_void_p, C.POINTER(dp_queue_config), C.c_void_p, C.c_int,
                                C.POINTER(C.c_void_p)]),
    "dp_queue_step": (C.c_int, [C.c_void_p, C.c_void_p, C.c_int]),
    "dp_queue_pop": (C.c_int, [C.c_void_p, C.c_void_p, C.c_int, C.POINTER(C.c_longlong)]),
    "dp_queue_close": (C.c_int, [C.c_void_p]),
    "dp_queue_set_noise_pool": (C.c_int, [C.c_void_p, C.c_void_p, C.c_int]),
    "dp_queue_sync": (C.c_int, [C.c_void_p]),
    "dp_queue_selftest_timeout": (C.c_int, [C.c_void_p]),
    "dp_queue_inspect": (C.c_int, [C.c_void_p, C.POINTER(dp_queue_info), C.c_void_p, C.c_void_p,
                                   C.c_void_p, C.c_void_p, C.c_int]),
    "dp_queue_read_latents": (C.c_int, [C.c_void_p, C.c_void_p, C.c_int, C.c_int]),
    "dp_queue_load_state": (C.c_int, [C.c_void_p, C.c_longlong, C.c_longlong, C.c_int, C.c_void_p,
                                      C.c_void_p, C.c_int]),
    "dp_queue_read_pred_kv": (C.c_int, [C.c_void_p, C.c_void_p, C.c_int, C.POINTER(C.c_longlong)]),
    "dp_queue_set_timing": (C.c_int, [C.c_void_p, C.c_int]),
    "dp_queue_timing": (C.c_int, [C.c_void_p, C.c_int, C.POINTER(C.c_double),
                                  C.POINTER(C.c_longlong), C.POINTER(C.c_double),
                                  C.POINTER(C.c_double)]),
    "dp_queue_destroy": (None, [C.c_void_p]),
    "dp_destroy": (None, [C.c_void_p]),
    "dp_last_error": (C.c_char_p, []),
    "dp_op_gemm": (C.c_int, [C.POINTER(dp_gemm_args), C.c_void_p]),
    "dp_op_attention": (C.c_int, [C.POINTER(dp_attn_args), C.c_void_p]),
    "dp_op_layernorm_mod": (C.c_int, [C.POINTER(dp_ln_args), C.c_void_p]),
    "dp_op_ln_gemm_noalloc": (C.c_int, [C.POINTER(dp_ln_args), C.POINTER(dp_gemm_args), C.c_void_p]),
    "dp_op_check": (C.c_int, [C.c_void_p]),
    "dp_op_selftest_timeout": (C.c_int, [C.c_void_p]),
}

EXPORTED = sorted(_SIGS)

_lib = None


def lib():
    """The loaded library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise ImportError(f"{_LIB_PATH} is missing: build it with __graft_entry__.build() "
                              "or python -m chunked_fifo_denoising_b200.build")
        L = C.CDLL(_LIB_PATH)
        for name, (res, args) in _SIGS.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


class DPError(RuntimeError):
    def __init__(self, status, where):
        self.status = status
        msg = lib().dp_last_error().decode(errors="replace")
        name = STATUS_NAMES[status] if 0 <= status < len(STATUS_NAMES) else str(status)
        super().__init__(f"{where}: {name}: {msg}")


def check(status, where):
    if status != DP_OK:
        raise DPError(status, where)
    return status


def _call(name, *args):
    return getattr(lib(), name)(*args)


# Same-name wrappers (status returned, not raised).
def dp_set_allocator(alloc, free_fn, ctx): return _call("dp_set_allocator", alloc, free_fn, ctx)
def dp_param_numel(cfg, pid, out): return _call("dp_param_numel", C.byref(cfg), pid, C.byref(out))
def dp_model_create(cfg, stream, out): return _call("dp_model_create", C.byref(cfg), stream, C.byref(out))
def dp_model_set_param(m, pid, layer, src, numel, loc): return _call("dp_model_set_param", m, pid, layer, src, numel, loc)
def dp_queue_init(m, qc, text, loc, out): return _call("dp_queue_init", m, C.byref(qc), text, loc, C.byref(out))
def dp_queue_step(q, noise, loc): return _call("dp_queue_step", q, noise, loc)
def dp_queue_pop(q, out, loc, cid): return _call("dp_queue_pop", q, out, loc, C.byref(cid))
def dp_queue_close(q): return _call("dp_queue_close", q)
def dp_queue_set_noise_pool(q, pool, loc): return _call("dp_queue_set_noise_pool", q, pool, loc)
def dp_queue_sync(q): return _call("dp_queue_sync", q)
def dp_queue_selftest_timeout(q): return _call("dp_queue_selftest_timeout", q)
def dp_queue_inspect(q, info, ids, levels, slots, positions, cap): return _call("dp_queue_inspect", q, C.byref(info), ids, levels, slots, positions, cap)
def dp_queue_read_latents(q, out, n, loc): return _call("dp_queue_read_latents", q, out, n, loc)
def dp_queue_load_state(q, step, n_pushed, n, lat, kv, loc): return _call("dp_queue_load_state", q, step, n_pushed, n, lat, kv, loc)
def dp_queue_read_pred_kv(q, out, loc, cid): return _call("dp_queue_read_pred_kv", q, out, loc, C.byref(cid))
def dp_queue_set_timing(q, on): return _call("dp_queue_set_timing", q, on)
def dp_queue_timing(q, k, ms, n, fl, by): return _call("dp_queue_timing", q, k, C.byref(ms), C.byref(n), C.byref(fl), C.byref(by))
def dp_queue_destroy(q): return _call("dp_queue_destroy", q)
def dp_destroy(m): return _call("dp_destroy", m)
def dp_last_error(): return lib().dp_last_error().decode(errors="replace")
def dp_op_gemm(args, stream): return _call("dp_op_gemm", C.byref(args), stream)
def dp_op_attention(args, stream): return _call("dp_op_attention", C.byref(args), stream)
def dp_op_layernorm_mod(args, stream): return _call("dp_op_layernorm_mod", C.byref(args), stream)
def dp_op_ln_gemm_noalloc(ln, gemm, stream): return _call("dp_op_ln_gemm_noalloc", C.byref(ln), C.byref(gemm), stream)
def dp_op_check(stream): return _call("dp_op_check", stream)
def dp_op_selftest_timeout(stream): return _call("dp_op_selftest_timeout", stream)
