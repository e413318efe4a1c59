"""Host logic of bench.py (no GPU): the algorithmic FLOP count of a step, the
whole-job rate, the roofline traffic guard and the JSON contract keys."""
import hashlib
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import synth  # noqa: E402


def per_token_layer(m, q):
    """12 d^2 (QKV, O-proj, cross Q and O) + 4 d F (FFN) + 4 (2 Lc) d
    (self-attention over own and predecessor keys) + 4 Lt d (cross-attention)."""
    Lc = q.tokens_per_chunk(m)
    return 12 * m.dim ** 2 + 4 * m.dim * m.ffn_dim + 4 * 2 * Lc * m.dim + 4 * m.text_len * m.dim


@pytest.mark.parametrize("name,tflop", [("wan1.3b_480p", 584.3), ("wan14b_720p", 13005.0)])
def test_step_flops_full_queue(name, tflop):
    """Per full-queue step: Wan-1.3B 584.3 TFLOP, Wan-14B 13.0 PFLOP (every
    chunk with a predecessor, plus the patch and head projections)."""
    w = synth.WORKLOADS[name]
    got = bench.step_flops(w.model, w.queue, w.queue.T) / 1e12
    assert abs(got - tflop) / tflop < 1e-3, got


def test_step_flops_terms():
    w = synth.WORKLOADS["wan1.3b_480p"]
    m, q = w.model, w.queue
    Lc = q.tokens_per_chunk(m)
    assert per_token_layer(m, q) == 124_846_080  # the 124.8 M of the Wan-1.3B row
    body = 50 * Lc * m.n_layers * per_token_layer(m, q)
    proj = 50 * Lc * 2 * 2 * 64 * m.dim
    assert bench.step_flops(m, q, 50) == body + proj
    # the successor link adds Lc keys for every chunk but the last
    both = bench.step_flops(m, q, 50, "both") - bench.step_flops(m, q, 50)
    assert both == m.n_layers * 4 * Lc * (49 * Lc) * m.dim


def test_plateau_flops_of_a_short_stream():
    """Wan-14B, 16 chunks: 16/50 of the full step (4.16 PFLOP) less the
    predecessor keys chunk 0 does not have."""
    w = synth.WORKLOADS["wan14b_720p"]
    m, q = w.model, w.queue
    Lc = q.tokens_per_chunk(m)
    plateau = bench.step_flops(m, q, 16) - m.n_layers * 4.0 * Lc * Lc * m.dim
    assert abs(bench.step_flops(m, q, 16) / 1e15 - 4.16) < 0.01
    assert abs(plateau / 1e15 - 4.119) < 0.001


def test_whole_job_rate_is_units_of_all_ranks_over_slowest_time():
    # 4 ranks, 5 steps of 2 frames each in 2.5 s (max over ranks) -> 16 frames/s
    assert bench.whole_job_rate(4, 5, 2, 2500.0) == pytest.approx(16.0)
    assert bench.whole_job_rate(1, 5, 2, 2500.0) == pytest.approx(4.0)


def test_gemm_traffic_follows_the_kernel_source():
    """The committed ncu traffic line is used only while its hash matches the
    GEMM source; it is then the per-launch DRAM bytes."""
    src = os.path.join(ROOT, "chunked_fifo_denoising_b200", "csrc")
    h = hashlib.sha256()
    for f in ("k_gemm_tc.cu", "tc_common.cuh"):
        with open(os.path.join(src, f), "rb") as fh:
            h.update(fh.read())
    with open(os.path.join(ROOT, "profiles", "gemm_traffic_wan1.3b.md")) as fh:
        text = fh.read()
    line = [l for l in text.splitlines() if l.startswith("traffic gemm_tc_kernel")]
    assert len(line) == 1
    want = int(line[0].split("bytes_per_launch=")[1].split()[0])
    if f"source_sha256_16={h.hexdigest()[:16]}" in line[0]:
        assert bench.gemm_traffic() == want
    else:
        assert bench.gemm_traffic() is None


def test_peaks_come_from_the_measured_file():
    pk = bench.peaks()
    assert pk["_source"] in ("measured", "fallback")
    assert pk["bf16_tflops_sustained"] > 0 and pk["hbm_gbs"] > 0


def test_stream_summary_rates():
    """Whole stream: N chunks x F frames over the wall time; steady state: the
    median step with all T levels occupied (one chunk leaves per step)."""
    T, F = 3, 2
    occ = [1, 2, 3, 3, 3, 2, 1]          # N = 5 chunks, N + T - 1 = 7 steps
    ms = [100.0, 200.0, 300.0, 310.0, 290.0, 200.0, 100.0]
    r = bench.stream_summary(ms, occ, T, F, wall_s=1.6, n_chunks=5)
    assert r["steps"] == 7 and r["steady_steps"] == 3
    assert r["steady_ms_per_step"] == 300.0
    assert r["steady_frames_per_s"] == pytest.approx(F / 0.3)
    assert r["whole_stream_frames_per_s"] == pytest.approx(10 / 1.6)


def test_long_stream_schedule_is_177_steps():
    """128 chunks through a T = 50 queue: 128 + 50 - 1 = 177 steps, 79 of them
    with all 50 levels occupied."""
    w = synth.WORKLOADS["wan1.3b_480p_long"]
    N, T = w.queue.n_chunks, w.queue.T
    occ = [min(s, N - 1) - max(0, s - T + 1) + 1 for s in range(N + T - 1)]
    assert len(occ) == 177 and occ.count(T) == N - T + 1 == 79
