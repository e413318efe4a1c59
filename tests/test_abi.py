"""The C library loads and exports every entry point its headers declare (no GPU)."""
import os
import re

import pytest

from tests.conftest import ROOT


def declared_symbols():
    names = set()
    for h in ("dp.h", "dp_ops.h"):
        src = open(os.path.join(ROOT, "include", h)).read()
        names |= set(re.findall(r"^DP_API [^;(]*?\b(dp_\w+)\s*\(", src, flags=re.M))
    return names


def test_headers_declare_the_queue_abi():
    names = declared_symbols()
    for n in ("dp_model_create", "dp_queue_init", "dp_queue_step", "dp_queue_pop", "dp_destroy"):
        assert n in names


def test_library_exports_every_declared_symbol():
    from chunked_fifo_denoising_b200 import _binding as B
    lib = B.lib()
    names = declared_symbols()
    for n in names:
        assert hasattr(lib, n), n
    assert names == set(B.EXPORTED), "binding and headers disagree"


def test_param_numel_and_config_errors():
    import ctypes as C
    from chunked_fifo_denoising_b200 import _binding as B
    import synth
    m = synth.WORKLOADS["wan1.3b_480p"].model
    cfg = B.dp_model_config(m.n_layers, m.dim, m.n_heads, m.ffn_dim, m.freq_dim, m.latent_ch,
                            m.patch_t, m.patch_h, m.patch_w, m.text_len, m.text_in_dim, 0)
    n = C.c_longlong()
    for name, shape, per_layer in synth.param_specs(m):
        assert B.dp_param_numel(cfg, B.PARAM_IDS[name], n) == 0
        assert n.value == int(__import__("numpy").prod(shape)), name
    bad = B.dp_model_config(*[getattr(cfg, f) for f, _ in cfg._fields_])
    bad.n_heads = 7
    assert B.dp_param_numel(bad, 0, n) == B.DP_ERR_INVALID_ARG
    assert "n_heads" in B.dp_last_error() or "head" in B.dp_last_error()


def test_binding_marshals_buffers_by_location_and_rejects_bad_ones():
    """The binding only marshals: numpy arrays and CPU tensors are host buffers,
    CUDA tensors device buffers; wrong dtypes or layouts are refused before any
    call into the library."""
    import numpy as np
    import torch
    from chunked_fifo_denoising_b200 import _binding as B
    from chunked_fifo_denoising_b200.queue import _ptr
    a = np.zeros((3, 4), np.float32)
    assert _ptr(a) == (a.ctypes.data, B.DP_LOC_HOST)
    t = torch.zeros(3, 4)
    assert _ptr(t) == (t.data_ptr(), B.DP_LOC_HOST)
    assert _ptr(None) == (None, B.DP_LOC_DEVICE)
    with pytest.raises(TypeError):
        _ptr(np.zeros(4, np.float64))
    with pytest.raises(ValueError):
        _ptr(np.zeros((4, 4), np.float32)[:, ::2])
    with pytest.raises(TypeError):
        _ptr(torch.zeros(4, dtype=torch.float16))
    with pytest.raises(ValueError):
        _ptr(torch.zeros(4, 4).t())
    with pytest.raises(TypeError):
        _ptr([1.0, 2.0])


def test_attention_rejects_keys_running_into_the_next_chunk():
    """With per-chunk keys, Lk > kv_chunk_rows would read the next chunk's rows
    (and the f32 and bf16 paths would disagree past the last chunk): refused
    by the argument checks, before anything reaches the device."""
    from chunked_fifo_denoising_b200 import _binding as B
    a = B.dp_attn_args()
    a.dtype, a.n_chunks, a.Lq, a.n_heads, a.head_dim = B.DP_DT_F32, 2, 8, 1, 16
    a.q = a.k = a.v = a.out = 4096          # never dereferenced: the call fails first
    a.ldq = a.ldkv = a.ldo = 16
    a.kv_chunk_rows, a.Lk, a.pred_in_batch = 8, 9, 1
    assert B.dp_op_attention(a, None) == B.DP_ERR_INVALID_ARG
    assert "kv_chunk_rows" in B.dp_last_error()


def test_noalloc_projection_refuses_oversized_rows_before_any_device_work():
    from chunked_fifo_denoising_b200 import _binding as B
    ln, g = B.dp_ln_args(), B.dp_gemm_args()
    ln.out_dtype = g.dtype = B.DP_DT_BF16
    ln.x, ln.ldx = 4096, 6144
    ln.M = g.M = 4096
    ln.d = g.K = 6144                       # 4096 x 6144 bf16 = 48 MiB > 32 MiB
    g.W, g.N, g.out, g.ldo = 4096, 64, 8192, 64
    assert B.dp_op_ln_gemm_noalloc(ln, g, None) == B.DP_ERR_INVALID_ARG
    assert "static scratch" in B.dp_last_error()
