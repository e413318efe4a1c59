"""bench.py's whole-stream mode on the small bf16 workload (a B200 run of the
real entry point, in a child process): every chunk pops in push order, the
stream takes N + T - 1 steps, and the peak device memory in use does not depend
on the stream length (the write-up's claim that memory does not grow with the
length of the video: DualParal write-up, techwalker.com, section 二)."""
import json
import os
import subprocess
import sys

import pytest

torch = pytest.importorskip("torch")

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_stream_mode_small_workload():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--stream", "--workload", "small_bf16",
           "--stream-lengths", "12"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["mode"] == "stream" and line["config"]["workload"] == "small_bf16"
    runs = {s["chunks"]: s for s in line["streams"]}
    assert sorted(runs) == [12, 32]
    T = line["config"]["T"]
    for n, s in runs.items():
        assert s["steps"] == n + T - 1
        assert s["steady_steps"] == n - T + 1
        assert s["whole_stream_frames_per_s"] > 0
    assert line["memory_flat_in_stream_length"] is True
    assert runs[12]["peak_device_bytes_used"] == runs[32]["peak_device_bytes_used"]
    assert line["value"] > 0
