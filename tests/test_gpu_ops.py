"""Kernel-level parity on the GPU: each kernel of the queue step, run alone
through the C ABI (include/dp_ops.h), against the float64 oracle on the same
inputs.  Small cases span several tiles plus ragged tails; full-size cases use
the Wan-1.3B / Wan-14B shapes in the launch configuration of a queue step and
compare sampled rows that the oracle computes one by one."""
import ctypes as C
import math

import numpy as np
import pytest

torch = pytest.importorskip("torch")

from oracle import dit  # noqa: E402

pytestmark = pytest.mark.gpu

B = None


@pytest.fixture(scope="module", autouse=True)
def _lib():
    global B
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from chunked_fifo_denoising_b200 import _binding
    B = _binding
    B.lib()


def rel_l2(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30))


def f64(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def gen(shape, std=1.0, dtype=torch.bfloat16, seed=0):
    g = torch.Generator(device="cuda").manual_seed(seed)
    return (torch.randn(shape, generator=g, device="cuda", dtype=torch.float32) * std).to(dtype)


def run_gemm(A, W, bias, epi, out=None, resid=None, gate=None, sel=None, rpc=1, cache=None,
             cache_row0=0, cache_rows=0, cache_col0=0, dtype=None):
    M, K = A.shape
    N = W.shape[0]
    a = B.dp_gemm_args()
    a.dtype = B.DP_DT_BF16 if A.dtype == torch.bfloat16 else B.DP_DT_F32
    a.A, a.lda, a.W = A.data_ptr(), A.stride(0), W.data_ptr()
    a.bias = bias.data_ptr() if bias is not None else None
    a.M, a.N, a.K, a.epi = M, N, K, epi
    if out is not None:
        a.out, a.ldo = out.data_ptr(), out.stride(0)
    if resid is not None:
        a.resid, a.ldr = resid.data_ptr(), resid.stride(0)
    if gate is not None:
        a.gate, a.gate_stride = gate.data_ptr(), gate.stride(0)
        a.chunk_sel = sel.data_ptr() if sel is not None else None
        a.rows_per_chunk = rpc
    if cache is not None:
        a.cache, a.cache_row0, a.cache_rows, a.cache_col0, a.ldc = (
            cache.data_ptr(), cache_row0, cache_rows, cache_col0, cache.stride(0))
    st = B.dp_op_gemm(a, torch.cuda.current_stream().cuda_stream)
    assert st == 0, B.dp_last_error()
    assert B.dp_op_check(torch.cuda.current_stream().cuda_stream) == 0, B.dp_last_error()


@pytest.mark.parametrize("M,N,K", [(300, 256, 128), (129, 64, 64), (1000, 384, 192),
                                   (300, 192, 128), (200, 96, 64), (100, 256, 64),
                                   (2048, 1536, 512), (257, 4608, 1536)])
def test_gemm_store_bf16(M, N, K):
    """N a multiple of 256 runs in CTA pairs (256-row tiles): M = 100 leaves the
    second CTA of the only pair without rows, M = 257 and 300 leave the second
    CTA of the last pair without rows; N = 64, 96, 192, 384 take single CTAs."""
    A, W = gen((M, K), seed=1), gen((N, K), 0.02, seed=2)
    bias = gen((N,), 0.02, torch.float32, seed=3)
    out = torch.empty((M, N), device="cuda", dtype=torch.bfloat16)
    run_gemm(A, W, bias, B.DP_EPI_STORE, out=out)
    ref = dit.linear(f64(A), f64(W), f64(bias))
    assert rel_l2(f64(out), ref) < 5e-3


def test_gemm_store_f32_out_patch_shape():
    """The patch embedding (K = 64) writes the fp32 residual stream: the
    tensor-core GEMM with an fp32 store through the queue step (checked there);
    here the same kernel stores bf16, and rows beyond a ragged M stay intact."""
    M, N, K = 3120 * 3 + 17, 1536, 64
    A, W = gen((M, K), seed=4), gen((N, K), 0.02, seed=5)
    bias = gen((N,), 0.02, torch.float32, seed=6)
    out = torch.full((M + 5, N), 7.0, device="cuda", dtype=torch.bfloat16)
    run_gemm(A, W, bias, B.DP_EPI_STORE, out=out[:M])
    ref = dit.linear(f64(A), f64(W), f64(bias))
    assert rel_l2(f64(out[:M]), ref) < 5e-3
    assert torch.all(out[M:] == 7.0)


def test_gemm_gelu():
    M, N, K = 700, 2048, 512
    A, W = gen((M, K), seed=7), gen((N, K), 0.05, seed=8)
    bias = gen((N,), 0.02, torch.float32, seed=9)
    out = torch.empty((M, N), device="cuda", dtype=torch.bfloat16)
    run_gemm(A, W, bias, B.DP_EPI_GELU, out=out)
    ref = dit.gelu(dit.linear(f64(A), f64(W), f64(bias)))
    assert rel_l2(f64(out), ref) < 5e-3


def test_gemm_residual_and_gated_residual():
    M, N, K, rpc = 1000, 512, 2048, 300
    A, W = gen((M, K), seed=10), gen((N, K), 0.02, seed=11)
    bias = gen((N,), 0.02, torch.float32, seed=12)
    x0 = gen((M, N), 1.0, torch.float32, seed=13)
    x = x0.clone()
    run_gemm(A, W, bias, B.DP_EPI_RESID, resid=x)
    y = dit.linear(f64(A), f64(W), f64(bias))
    assert rel_l2(f64(x) - f64(x0), y) < 1e-4
    # gated: chunk c of 300 rows uses gate row sel[c] of a level table
    table = gen((7, N), 0.5, torch.float32, seed=14)
    sel = torch.tensor([5, 0, 3, 6], device="cuda", dtype=torch.int32)
    x = x0.clone()
    run_gemm(A, W, bias, B.DP_EPI_RESID_GATED, resid=x, gate=table, sel=sel, rpc=rpc)
    g = f64(table)[f64(sel).astype(int)[np.arange(M) // rpc]]
    assert rel_l2(f64(x) - f64(x0), g * y) < 1e-4


def test_gemm_qkv_cache_copy():
    """QKV epilogue: rows of the head chunk also land, K and V columns only, in
    the persisted neighbour cache [Lc][2d]."""
    d, Lc, n = 256, 200, 3
    M = n * Lc
    A, W = gen((M, d), seed=15), gen((3 * d, d), 0.02, seed=16)
    bias = gen((3 * d,), 0.02, torch.float32, seed=17)
    out = torch.empty((M, 3 * d), device="cuda", dtype=torch.bfloat16)
    cache = torch.zeros((Lc, 2 * d), device="cuda", dtype=torch.bfloat16)
    run_gemm(A, W, bias, B.DP_EPI_STORE, out=out, cache=cache, cache_row0=0, cache_rows=Lc,
             cache_col0=d)
    assert torch.equal(cache, out[:Lc, d:])
    assert rel_l2(f64(out), dit.linear(f64(A), f64(W), f64(bias))) < 5e-3


@pytest.mark.parametrize("name,M,N,K", [
    ("wan1.3b ffn1", 156000, 8960, 1536),
    ("wan1.3b ffn2", 156000, 1536, 8960),
    ("wan1.3b qkv", 156000, 4608, 1536),
    ("wan14b ffn1", 115200, 13824, 5120),
])
def test_gemm_full_size_sampled_rows(name, M, N, K):
    A, W = gen((M, K), seed=20), gen((N, K), 0.02, seed=21)
    bias = gen((N,), 0.02, torch.float32, seed=22)
    out = torch.empty((M, N), device="cuda", dtype=torch.bfloat16)
    run_gemm(A, W, bias, B.DP_EPI_GELU if "ffn1" in name else B.DP_EPI_STORE, out=out)
    rows = np.unique(np.concatenate([np.random.default_rng(0).integers(0, M, 48), [0, 127, 128, M - 1]]))
    ref = dit.linear(f64(A[rows]), f64(W), f64(bias))
    if "ffn1" in name:
        ref = dit.gelu(ref)
    assert rel_l2(f64(out[rows]), ref) < 5e-3
    del A, W, out
    torch.cuda.empty_cache()


# ---------------------------------------------------------------------------
# attention
# ---------------------------------------------------------------------------

def run_attn(q, k, v, n_chunks, Lq, H, hd, Lk, kv_chunk_rows, pred_in_batch, kp=None, vp=None,
             dtype=None, succ=0):
    out = torch.empty((n_chunks * Lq, H * hd), device="cuda", dtype=q.dtype)
    a = B.dp_attn_args()
    a.dtype = B.DP_DT_BF16 if q.dtype == torch.bfloat16 else B.DP_DT_F32
    a.n_chunks, a.Lq, a.n_heads, a.head_dim = n_chunks, Lq, H, hd
    a.q, a.ldq = q.data_ptr(), q.stride(0)
    a.k, a.v, a.ldkv = k.data_ptr(), v.data_ptr(), k.stride(0)
    a.kv_chunk_rows, a.Lk, a.pred_in_batch = kv_chunk_rows, Lk, pred_in_batch
    if kp is not None:
        a.k0_pred, a.v0_pred, a.ld_pred, a.Lk_pred = kp.data_ptr(), vp.data_ptr(), kp.stride(0), kp.shape[0]
    a.out, a.ldo = out.data_ptr(), out.stride(0)
    a.succ_in_batch = succ
    st = B.dp_op_attention(a, torch.cuda.current_stream().cuda_stream)
    assert st == 0, B.dp_last_error()
    assert B.dp_op_check(torch.cuda.current_stream().cuda_stream) == 0, B.dp_last_error()
    return out


def oracle_self_attention(q, k, v, n, Lc, H, kp, vp, rows=None, succ=False):
    """Per chunk: own keys plus the predecessor's (in batch, or kp/vp for chunk 0)
    and, with succ, the successor's (in batch)."""
    outs = []
    for c in range(n):
        sl = slice(c * Lc, (c + 1) * Lc)
        qq = q[sl] if rows is None else q[sl][rows]
        if c > 0:
            pk, pv = k[(c - 1) * Lc:c * Lc], v[(c - 1) * Lc:c * Lc]
        else:
            pk, pv = kp, vp
        sk = sv = None
        if succ and c + 1 < n:
            sk, sv = k[(c + 1) * Lc:(c + 2) * Lc], v[(c + 1) * Lc:(c + 2) * Lc]
        outs.append(dit.self_attention_with_neighbours(qq, k[sl], v[sl], pk, pv, sk, sv, H))
    return np.concatenate(outs)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("hd,Lc,n,cached,succ,H", [(64, 200, 3, True, False, 2), (128, 333, 2, False, False, 2),
                                                   (128, 130, 4, True, False, 2), (128, 200, 3, True, True, 2),
                                                   (64, 333, 2, False, True, 2), (128, 100, 3, True, False, 2),
                                                   (64, 300, 2, True, True, 3)])
def test_self_attention_neighbour_buffers(dtype, hd, Lc, n, cached, succ, H):
    """Ragged chunks: the last 256-query block of a chunk holds Lc mod 256
    rows; with one tile's worth (333, 100, 300 rows) and an even head count the
    tensor-core path pairs two heads' last blocks in one CTA (H = 3 keeps them
    apart)."""
    d = H * hd
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    qkv = gen((n * Lc, 3 * d), 1.0, tdt, seed=30)
    q, k, v = qkv[:, :d], qkv[:, d:2 * d], qkv[:, 2 * d:]
    cache = gen((Lc, 2 * d), 1.0, tdt, seed=31) if cached else None
    kp = cache[:, :d] if cached else None
    vp = cache[:, d:] if cached else None
    out = run_attn(q, k, v, n, Lc, H, hd, Lc, Lc, 1, kp, vp, succ=int(succ))
    ref = oracle_self_attention(f64(q), f64(k), f64(v), n, Lc, H,
                                None if kp is None else f64(kp), None if vp is None else f64(vp),
                                succ=succ)
    assert rel_l2(f64(out), ref) < (1e-2 if dtype == "bf16" else 1e-5)


@pytest.mark.parametrize("hd", [64, 128])
@pytest.mark.parametrize("Lc", [5, 20])
def test_attention_chunks_shorter_than_an_output_box(hd, Lc):
    """Chunks of fewer query rows than the 32-row output box of the
    tensor-core path: self-attention with a cached predecessor, and
    cross-attention to a short prompt."""
    H, n = 2, 3
    d = H * hd
    qkv = gen((n * Lc, 3 * d), 1.0, torch.bfloat16, seed=34)
    q, k, v = qkv[:, :d], qkv[:, d:2 * d], qkv[:, 2 * d:]
    cache = gen((Lc, 2 * d), 1.0, torch.bfloat16, seed=35)
    out = run_attn(q, k, v, n, Lc, H, hd, Lc, Lc, 1, cache[:, :d], cache[:, d:])
    ref = oracle_self_attention(f64(q), f64(k), f64(v), n, Lc, H, f64(cache[:, :d]), f64(cache[:, d:]))
    assert rel_l2(f64(out), ref) < 1e-2
    kv = gen((9, 2 * d), 1.0, torch.bfloat16, seed=36)
    out = run_attn(q, kv[:, :d], kv[:, d:], n, Lc, H, hd, 9, 0, 0)
    assert rel_l2(f64(out), dit.attention(f64(q), f64(kv[:, :d]), f64(kv[:, d:]), H)) < 1e-2


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("Lq", [257, 700])
@pytest.mark.parametrize("hd,Lt", [(64, 64), (128, 77)])
def test_cross_attention_shared_keys(dtype, Lq, hd, Lt):
    """Several 256-query blocks per CTA (short key set); Lq = 257 ends in a
    one-tile block of 1 row, Lq = 700 in a block of two tiles (188 rows).
    77 prompt keys leave most of the one key tile masked; the output rows of a
    chunk's last block that fall past Lq must not land in the next chunk."""
    H, n = 4, 3
    d = H * hd
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    q = gen((n * Lq, d), 1.0, tdt, seed=32)
    kv = gen((Lt, 2 * d), 1.0, tdt, seed=33)
    out = run_attn(q, kv[:, :d], kv[:, d:], n, Lq, H, hd, Lt, 0, 0)
    ref = dit.attention(f64(q), f64(kv[:, :d]), f64(kv[:, d:]), H)
    assert rel_l2(f64(out), ref) < (1e-2 if dtype == "bf16" else 1e-5)


@pytest.mark.parametrize("succ", [False, True])
def test_self_attention_full_size_sampled_rows(succ):
    """Wan-1.3B steady state: 50 chunks of 3120 tokens, 12 heads of 128, every
    chunk with its predecessor (chunk 0 from the persisted cache), and with the
    bidirectional neighbourhood also its successor."""
    n, Lc, H, hd = 50, 3120, 12, 128
    d = H * hd
    qkv = gen((n * Lc, 3 * d), 1.0, torch.bfloat16, seed=40)
    q, k, v = qkv[:, :d], qkv[:, d:2 * d], qkv[:, 2 * d:]
    cache = gen((Lc, 2 * d), 1.0, torch.bfloat16, seed=41)
    out = run_attn(q, k, v, n, Lc, H, hd, Lc, Lc, 1, cache[:, :d], cache[:, d:], succ=int(succ))
    rows = np.array([0, 1, 127, 128, 1000, 3071, 3072, 3100, 3119])   # 3072..: the paired last block
    qf, kf, vf = f64(q), f64(k), f64(v)
    for c in (0, 1, 17, 49):
        sl = slice(c * Lc, (c + 1) * Lc)
        if c > 0:
            pk, pv = kf[(c - 1) * Lc:c * Lc], vf[(c - 1) * Lc:c * Lc]
        else:
            pk, pv = f64(cache[:, :d]), f64(cache[:, d:])
        sk = sv = None
        if succ and c + 1 < n:
            sk, sv = kf[(c + 1) * Lc:(c + 2) * Lc], vf[(c + 1) * Lc:(c + 2) * Lc]
        ref = dit.self_attention_with_neighbours(qf[sl][rows], kf[sl], vf[sl], pk, pv, sk, sv, H)
        assert rel_l2(f64(out[sl][rows]), ref) < 1e-2, c


def test_cross_attention_full_size_sampled_rows():
    """Wan-1.3B: 156 000 queries against the 512 prompt keys of one layer."""
    n, Lc, H, hd, Lt = 50, 3120, 12, 128, 512
    d = H * hd
    q = gen((n * Lc, d), 1.0, torch.bfloat16, seed=60)
    kv = gen((Lt, 2 * d), 1.0, torch.bfloat16, seed=61)
    out = run_attn(q, kv[:, :d], kv[:, d:], n, Lc, H, hd, Lt, 0, 0)
    rows = np.unique(np.concatenate([np.random.default_rng(1).integers(0, n * Lc, 40), [0, n * Lc - 1]]))
    ref = dit.attention(f64(q[rows]), f64(kv[:, :d]), f64(kv[:, d:]), H)
    assert rel_l2(f64(out[rows]), ref) < 1e-2


# ---------------------------------------------------------------------------
# layer norm + modulation
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("out_dtype", ["bf16", "f32"])
@pytest.mark.parametrize("M,d", [(1000, 1536), (33, 64), (257, 5120), (333, 512), (156000, 1536)])
def test_layernorm_mod(out_dtype, M, d):
    x = gen((M, d), 2.0, torch.float32, seed=50) + 0.5
    table = gen((5, 2 * d), 0.3, torch.float32, seed=51)
    rpc = max(1, M // 3)
    sel = torch.tensor([4, 1, 0, 2], device="cuda", dtype=torch.int32)
    tdt = torch.bfloat16 if out_dtype == "bf16" else torch.float32
    out = torch.empty((M, d), device="cuda", dtype=tdt)
    a = B.dp_ln_args()
    a.out_dtype = B.DP_DT_BF16 if out_dtype == "bf16" else B.DP_DT_F32
    a.x, a.ldx, a.M, a.d = x.data_ptr(), d, M, d
    a.shift, a.scale, a.mod_stride = table.data_ptr(), table[:, d:].data_ptr(), 2 * d
    a.chunk_sel, a.rows_per_chunk = sel.data_ptr(), rpc
    a.out, a.ldo = out.data_ptr(), d
    assert B.dp_op_layernorm_mod(a, torch.cuda.current_stream().cuda_stream) == 0, B.dp_last_error()
    torch.cuda.synchronize()
    t = f64(table)[f64(sel).astype(int)[np.minimum(np.arange(M) // rpc, 3)]]
    ref = dit.modulate(dit.layer_norm(f64(x)), t[:, :d], t[:, d:])
    assert rel_l2(f64(out), ref) < (5e-3 if out_dtype == "bf16" else 1e-6)


def test_bounded_wait_gives_up_and_reports():
    """A kernel whose mbarrier is never completed gives up after the wait limit,
    sets the status word (reported once as DP_ERR_KERNEL) and leaves the
    context usable: the next GEMM runs and checks clean."""
    s = torch.cuda.current_stream().cuda_stream
    assert B.dp_op_check(s) == 0
    assert B.dp_op_selftest_timeout(s) == 0
    assert B.dp_op_check(s) == B.DP_ERR_KERNEL
    assert "bounded wait" in B.dp_last_error()
    assert B.dp_op_check(s) == 0          # the word was cleared
    test_gemm_store_bf16(300, 256, 128)   # and kernels still run
