"""dp_op_ln_gemm_noalloc: the modulated projection (LN + adaLN, then a GEMM)
for callers that may not allocate device memory.  Its normalised rows live
in a static device array instead of a caller buffer; its results must equal
those of the two allocating-caller entry points it stands in for,
dp_op_layernorm_mod into a caller buffer followed by dp_op_gemm reading it.

Runs last (file name) so that a stop at the first failure has already run
every other test; it also passes alone in a fresh process.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

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
    a = a.detach().double().cpu().numpy()
    b = b.detach().double().cpu().numpy()
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30))


def gen(shape, std, dtype, seed):
    g = torch.Generator(device="cuda").manual_seed(seed)
    return (torch.randn(shape, generator=g, device="cuda", dtype=torch.float32) * std).to(dtype)


class Case:
    """Inputs of one modulated projection: x [M][d] fp32, a per-chunk
    shift/scale table, W [N][d], bias [N], and (gated residual) a gate table
    plus the fp32 residual it adds into."""

    def __init__(self, M, d, N, epi, dtype, rpc, seed):
        self.M, self.d, self.N, self.epi, self.dtype, self.rpc = M, d, N, epi, dtype, rpc
        self.x = gen((M, d), 2.0, torch.float32, seed) + 0.25
        self.table = gen((6, 2 * d), 0.3, torch.float32, seed + 1)
        n_chunks = (M + rpc - 1) // rpc
        self.sel = torch.arange(n_chunks, device="cuda", dtype=torch.int32) % 6
        self.W = gen((N, d), 0.03, dtype, seed + 2)
        self.bias = gen((N,), 0.02, torch.float32, seed + 3)
        self.gate = gen((6, N), 0.5, torch.float32, seed + 4)
        self.resid0 = gen((M, N), 1.0, torch.float32, seed + 5)

    def ln_args(self, out=None):
        a = B.dp_ln_args()
        a.out_dtype = B.DP_DT_BF16 if self.dtype == torch.bfloat16 else B.DP_DT_F32
        a.x, a.ldx, a.M, a.d = self.x.data_ptr(), self.d, self.M, self.d
        a.shift, a.scale, a.mod_stride = (self.table.data_ptr(), self.table[:, self.d:].data_ptr(),
                                          2 * self.d)
        a.chunk_sel, a.rows_per_chunk = self.sel.data_ptr(), self.rpc
        if out is not None:
            a.out, a.ldo = out.data_ptr(), self.d
        return a

    def gemm_args(self, out, resid, A=None):
        g = B.dp_gemm_args()
        g.dtype = B.DP_DT_BF16 if self.dtype == torch.bfloat16 else B.DP_DT_F32
        if A is not None:
            g.A, g.lda = A.data_ptr(), self.d
        g.W, g.bias = self.W.data_ptr(), self.bias.data_ptr()
        g.M, g.N, g.K, g.epi = self.M, self.N, self.d, self.epi
        if self.epi in (B.DP_EPI_STORE, B.DP_EPI_GELU):
            g.out, g.ldo = out.data_ptr(), self.N
        else:
            g.resid, g.ldr = resid.data_ptr(), self.N
            g.gate, g.gate_stride = self.gate.data_ptr(), self.N
            g.chunk_sel, g.rows_per_chunk = self.sel.data_ptr(), self.rpc
        return g

    def result(self, out, resid):
        return out if self.epi in (B.DP_EPI_STORE, B.DP_EPI_GELU) else resid

    def buffers(self):
        return (torch.full((self.M, self.N), 9.0, device="cuda", dtype=self.dtype),
                self.resid0.clone())


def run_existing(c, stream):
    """dp_op_layernorm_mod into a caller buffer, then dp_op_gemm reading it."""
    h = torch.empty((c.M, c.d), device="cuda", dtype=c.dtype)
    out, resid = c.buffers()
    assert B.dp_op_layernorm_mod(c.ln_args(h), stream) == 0, B.dp_last_error()
    assert B.dp_op_gemm(c.gemm_args(out, resid, A=h), stream) == 0, B.dp_last_error()
    assert B.dp_op_check(stream) == 0, B.dp_last_error()
    return c.result(out, resid)


def run_noalloc(c, stream):
    out, resid = c.buffers()
    assert B.dp_op_ln_gemm_noalloc(c.ln_args(), c.gemm_args(out, resid), stream) == 0, B.dp_last_error()
    return c.result(out, resid)


@pytest.mark.parametrize("dtype,tol", [(torch.bfloat16, 5e-3), (torch.float32, 1e-6)])
def test_noalloc_matches_the_allocating_entry_points_on_two_calls(dtype, tol):
    """Two calls in a row, the second with other inputs, fewer rows and
    another epilogue, so a stale scratch row from the first call would show.
    Tolerances are those of the single-kernel GEMM tests (bf16 5e-3, f32 1e-6)."""
    s = torch.cuda.current_stream().cuda_stream
    first = Case(M=1000, d=1536, N=2048, epi=B.DP_EPI_GELU, dtype=dtype, rpc=300, seed=10)
    second = Case(M=700, d=512, N=768, epi=B.DP_EPI_RESID_GATED, dtype=dtype, rpc=200, seed=20)
    ref1 = run_existing(first, s)
    ref2 = run_existing(second, s)
    got1 = run_noalloc(first, s)
    got2 = run_noalloc(second, s)
    assert B.dp_op_check(s) == 0, B.dp_last_error()
    torch.cuda.synchronize()
    assert rel_l2(got1, ref1) <= tol
    assert rel_l2(got2 - second.resid0, ref2 - second.resid0) <= tol
    # and once more with the first inputs: the result does not depend on what
    # the previous call left in the scratch
    again = run_noalloc(first, s)
    torch.cuda.synchronize()
    assert rel_l2(again, ref1) <= tol


def test_noalloc_rejects_sizes_beyond_the_static_scratch():
    s = torch.cuda.current_stream().cuda_stream
    c = Case(M=64, d=512, N=256, epi=B.DP_EPI_STORE, dtype=torch.bfloat16, rpc=64, seed=30)
    out, resid = c.buffers()
    ln, g = c.ln_args(), c.gemm_args(out, resid)
    ln.M = g.M = 32769                  # 32769 x 512 bf16 rows: 32 MiB + 1 KiB
    assert B.dp_op_ln_gemm_noalloc(ln, g, s) == B.DP_ERR_INVALID_ARG
    assert "static scratch" in B.dp_last_error()
    ln.M = g.M = 64
    h = torch.empty((64, 512), device="cuda", dtype=torch.bfloat16)
    ln.out, ln.ldo = h.data_ptr(), 512  # a caller buffer is refused, not used
    assert B.dp_op_ln_gemm_noalloc(ln, g, s) == B.DP_ERR_INVALID_ARG
