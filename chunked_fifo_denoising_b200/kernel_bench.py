"""Times one kernel of the queue step alone through include/dp_ops.h.

    python -m chunked_fifo_denoising_b200.kernel_bench --case NAME [--iters N] [--chunks C]

Cases use the Wan-1.3B / Wan-14B shapes of a steady-state step (random
inputs on the device).  Prints one JSON line per case with the mean time of
`iters` launches (CUDA events, after two untimed launches) and the achieved
TFLOP/s or GB/s of the kernel's algorithmic work.  --chunks scales the token
count (chunks x 3120 tokens for the 1.3B shapes) for small profiling runs.
"""
from __future__ import annotations

import argparse
import json

import torch

from . import _binding as B

CASES = {
    # name: (kind, dict)
    "qkv": ("gemm", dict(N=4608, K=1536, epi=B.DP_EPI_STORE)),
    "oproj": ("gemm", dict(N=1536, K=1536, epi=B.DP_EPI_RESID_GATED)),
    "crossq": ("gemm", dict(N=1536, K=1536, epi=B.DP_EPI_STORE)),
    "crosso": ("gemm", dict(N=1536, K=1536, epi=B.DP_EPI_RESID)),
    "ffn1": ("gemm", dict(N=8960, K=1536, epi=B.DP_EPI_GELU)),
    "ffn2": ("gemm", dict(N=1536, K=8960, epi=B.DP_EPI_RESID_GATED)),
    "ffn1_14b": ("gemm", dict(N=13824, K=5120, epi=B.DP_EPI_GELU, Lc=7200)),
    "self_attn": ("attn", dict(H=12, hd=128, Lk=3120, shared=False)),
    "cross_attn": ("attn", dict(H=12, hd=128, Lk=512, shared=True)),
    "self_attn_14b": ("attn", dict(H=40, hd=128, Lk=7200, shared=False, Lc=7200)),
    "ln": ("ln", dict(d=1536)),
}


class _ClockSampler:
    """Median SM clock (MHz) over a timed loop, read through NVML in a thread."""

    def __init__(self):
        import threading
        self.samples = []
        self.stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.h = pynvml.nvmlDeviceGetHandleByIndex(torch.cuda.current_device())
            self.nv = pynvml
        except Exception:
            self.nv = None
        self.t = threading.Thread(target=self._run, daemon=True)

    def _run(self):
        while not self.stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
            except Exception:
                return
            self.stop.wait(0.005)

    def __enter__(self):
        if self.nv is not None:
            self.t.start()
        return self

    def __exit__(self, *a):
        self.stop.set()
        if self.nv is not None:
            self.t.join()

    def median(self):
        s = sorted(self.samples)
        return float(s[len(s) // 2]) if s else None


def _time(fn, iters, stream):
    """Mean ms per launch and the median SM clock (MHz) while timing."""
    for _ in range(2):
        fn()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with _ClockSampler() as ck:
        e0.record(stream)
        for _ in range(iters):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
    return e0.elapsed_time(e1) / iters, ck.median()


def _res(d, ms, mhz, tflops=None, gbs=None):
    d["ms"] = ms
    d["sm_mhz"] = mhz
    if tflops is not None:
        d["tflops"] = tflops
        if mhz:  # the same work at the 1965 MHz maximum clock, for comparing runs
            d["tflops_at_max_clock"] = tflops * 1965.0 / mhz
    if gbs is not None:
        d["gbs"] = gbs
    return d


def run_case(name, iters, chunks):
    kind, c = CASES[name]
    Lc = c.get("Lc", 3120)
    M = chunks * Lc
    stream = torch.cuda.current_stream()
    sh = stream.cuda_stream
    g = torch.Generator(device="cuda").manual_seed(0)
    if kind == "gemm":
        N, K, epi = c["N"], c["K"], c["epi"]
        A = torch.randn(M, K, device="cuda", generator=g).to(torch.bfloat16)
        W = (torch.randn(N, K, device="cuda", generator=g) * 0.02).to(torch.bfloat16)
        bias = torch.zeros(N, device="cuda")
        a = B.dp_gemm_args()
        a.dtype, a.A, a.lda, a.W, a.bias = B.DP_DT_BF16, A.data_ptr(), K, W.data_ptr(), bias.data_ptr()
        a.M, a.N, a.K, a.epi = M, N, K, epi
        keep = [A, W, bias]
        if epi in (B.DP_EPI_RESID, B.DP_EPI_RESID_GATED):
            x = torch.zeros(M, N, device="cuda")
            gate = torch.ones(chunks, N, device="cuda")
            a.resid, a.ldr, a.gate, a.gate_stride, a.rows_per_chunk = x.data_ptr(), N, gate.data_ptr(), N, Lc
            keep += [x, gate]
        else:
            out = torch.empty(M, N, device="cuda", dtype=torch.bfloat16)
            a.out, a.ldo = out.data_ptr(), N
            keep.append(out)

        def fn():
            B.check(B.dp_op_gemm(a, sh), "dp_op_gemm")
        ms, mhz = _time(fn, iters, stream)
        B.check(B.dp_op_check(sh), "dp_op_check")
        return _res({"case": name, "M": M, "N": N, "K": K}, ms, mhz, tflops=2.0 * M * N * K / ms / 1e9)
    if kind == "attn":
        H, hd, Lk, shared = c["H"], c["hd"], c["Lk"], c["shared"]
        d = H * hd
        a = B.dp_attn_args()
        a.dtype, a.n_chunks, a.Lq, a.n_heads, a.head_dim = B.DP_DT_BF16, chunks, Lc, H, hd
        if shared:
            q = torch.randn(M, d, device="cuda", generator=g).to(torch.bfloat16)
            kv = torch.randn(Lk, 2 * d, device="cuda", generator=g).to(torch.bfloat16)
            a.q, a.ldq, a.k, a.v, a.ldkv, a.kv_chunk_rows, a.Lk = q.data_ptr(), d, kv.data_ptr(), kv[:, d:].data_ptr(), 2 * d, 0, Lk
            keys = Lk * chunks
            keep = [q, kv]
        else:
            qkv = torch.randn(M, 3 * d, device="cuda", generator=g).to(torch.bfloat16)
            cache = torch.randn(Lc, 2 * d, device="cuda", generator=g).to(torch.bfloat16)
            a.q, a.ldq = qkv.data_ptr(), 3 * d
            a.k, a.v, a.ldkv, a.kv_chunk_rows, a.Lk = qkv[:, d:].data_ptr(), qkv[:, 2 * d:].data_ptr(), 3 * d, Lc, Lk
            a.pred_in_batch = 1
            a.k0_pred, a.v0_pred, a.ld_pred, a.Lk_pred = cache.data_ptr(), cache[:, d:].data_ptr(), 2 * d, Lc
            keys = 2 * Lk * chunks
            keep = [qkv, cache]
        out = torch.empty(M, d, device="cuda", dtype=torch.bfloat16)
        a.out, a.ldo = out.data_ptr(), d
        keep.append(out)

        def fn():
            B.check(B.dp_op_attention(a, sh), "dp_op_attention")
        ms, mhz = _time(fn, iters, stream)
        B.check(B.dp_op_check(sh), "dp_op_check")
        flops = 4.0 * Lc * keys * d
        return _res({"case": name, "chunks": chunks, "Lq": Lc, "heads": H}, ms, mhz, tflops=flops / ms / 1e9)
    if kind == "ln":
        d = c["d"]
        x = torch.randn(M, d, device="cuda", generator=g)
        mod = torch.zeros(chunks, 2 * d, device="cuda")
        out = torch.empty(M, d, device="cuda", dtype=torch.bfloat16)
        a = B.dp_ln_args()
        a.out_dtype, a.x, a.ldx, a.M, a.d = B.DP_DT_BF16, x.data_ptr(), d, M, d
        a.shift, a.scale, a.mod_stride, a.rows_per_chunk = mod.data_ptr(), mod[:, d:].data_ptr(), 2 * d, Lc
        a.out, a.ldo = out.data_ptr(), d

        def fn():
            B.check(B.dp_op_layernorm_mod(a, sh), "dp_op_layernorm_mod")
        ms, mhz = _time(fn, iters, stream)
        return _res({"case": name, "M": M, "d": d}, ms, mhz, gbs=M * d * 6.0 / ms / 1e6)
    raise ValueError(name)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--case", action="append", required=True, choices=sorted(CASES))
    ap.add_argument("--iters", type=int, default=10)
    ap.add_argument("--chunks", type=int, default=50)
    args = ap.parse_args()
    B.lib()
    for name in args.case:
        print(json.dumps(run_case(name, args.iters, args.chunks)), flush=True)


if __name__ == "__main__":
    main()
