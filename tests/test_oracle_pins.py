"""Pins of the oracle against facts that do not come from the oracle itself:
textbook values, closed forms, brute-force loops, invariants and a queue trace
derived by hand from the FIFO rules of the DualParal write-up
("双重并行：让AI视频生成突破时长限制…", techwalker.com, §二 and §三).
"""
import math

import numpy as np
import pytest

import synth
from oracle import dit, fifo
from tests.conftest import read_golden


# ---------------------------------------------------------------------------
# generator
# ---------------------------------------------------------------------------

def test_splitmix64_published_outputs():
    want = [int(s, 16) for s in read_golden("splitmix64_seed0.txt")]
    got = [int(x) for x in synth.uniform_bits(0, 0, 3)]
    assert got == want


def test_generator_deterministic_and_normal():
    a = synth.normal(5, 7, 9, 200001)
    b = synth.normal(5, 7, 9, 200001)
    assert np.array_equal(a, b)
    assert abs(a.mean()) < 0.01 and abs(a.std() - 1.0) < 0.01
    c = synth.normal(5, 7, 10, 1000)
    assert not np.array_equal(a[:1000], c)
    # any draw is addressable without the ones before it
    key = synth.stream_key(5, 7, 9)
    assert np.array_equal(synth.uniform_bits(key, 10, 4), synth.uniform_bits(key, 0, 14)[10:])


# ---------------------------------------------------------------------------
# elementwise pieces
# ---------------------------------------------------------------------------

def test_gelu_is_exact_erf_form():
    for ln in read_golden("normal_cdf.txt"):
        x, phi = (float(t) for t in ln.split())
        assert dit.gelu(np.array([x]))[0] == pytest.approx(x * phi, abs=2e-10)
    # the tanh approximation differs at x = 1 by 1.5e-4: make sure it is not used
    tanh_form = 0.5 * (1 + math.tanh(math.sqrt(2 / math.pi) * (1 + 0.044715)))
    assert abs(dit.gelu(np.array([1.0]))[0] - tanh_form) > 1e-4
    x = np.linspace(-5, 5, 101)
    assert np.allclose(dit.gelu(x) - dit.gelu(-x), x, atol=1e-14)


def test_silu():
    assert dit.silu(np.array([0.0]))[0] == 0.0
    assert dit.silu(np.array([1.0]))[0] == pytest.approx(1.0 / (1.0 + math.exp(-1.0)), rel=1e-15)
    x = np.linspace(-6, 6, 49)
    assert np.allclose(dit.silu(x) - dit.silu(-x), x, atol=1e-14)


def test_layer_norm_closed_form():
    rng = np.random.default_rng(0)
    x = rng.normal(3.0, 2.0, size=(7, 64))
    y = dit.layer_norm(x)
    var = x.var(axis=1)
    assert np.allclose(y.mean(axis=1), 0, atol=1e-13)
    assert np.allclose((y ** 2).mean(axis=1), var / (var + dit.LN_EPS), rtol=1e-12)
    # invariant to a positive affine map of the row when eps vanishes
    assert np.allclose(dit.layer_norm(5 * x - 1, eps=0.0), dit.layer_norm(x, eps=0.0), atol=1e-12)
    assert np.all(dit.layer_norm(np.full((2, 8), 4.0)) == 0)


def test_modulate():
    h = np.arange(6.0).reshape(2, 3)
    z = np.zeros(3)
    assert np.array_equal(dit.modulate(h, z, z), h)
    s = np.array([1.0, -2.0, 0.5])
    assert np.array_equal(dit.modulate(h, s, -np.ones(3)), np.broadcast_to(s, h.shape))


def test_linear_hand_example_and_brute_force():
    w = np.array([[1.0, 2.0], [3.0, 4.0], [-1.0, 0.5]])
    b = np.array([1.0, 1.0, 0.0])
    assert np.array_equal(dit.linear(np.array([[5.0, 6.0]]), w, b), [[18.0, 40.0, -2.0]])
    rng = np.random.default_rng(1)
    x, w, b = rng.normal(size=(4, 5)), rng.normal(size=(3, 5)), rng.normal(size=3)
    ref = np.zeros((4, 3))
    for i in range(4):
        for o in range(3):
            ref[i, o] = b[o] + sum(x[i, k] * w[o, k] for k in range(5))
    assert np.allclose(dit.linear(x, w, b), ref, atol=1e-13)


def test_sinusoid():
    assert np.array_equal(dit.sinusoid(0.0, 8), [1, 1, 1, 1, 0, 0, 0, 0])
    # D = 4: frequencies 1 and 10000^(-1/2) = 0.01
    t = 100.0
    want = [math.cos(100.0), math.cos(1.0), math.sin(100.0), math.sin(1.0)]
    assert np.allclose(dit.sinusoid(t, 4), want, atol=1e-12)
    e = dit.sinusoid(123.4, 64)
    assert np.allclose(e[:32] ** 2 + e[32:] ** 2, 1.0)


def test_sigma_schedule():
    assert dit.sigma(0, 50) == 0.0 and dit.sigma(50, 50) == 1.0
    assert dit.sigma(2, 4) == 0.5


def test_patchify_index_order_and_round_trip():
    C, F, H, W = 3, 2, 4, 6
    lat = np.zeros((C, F, H, W))
    for c in range(C):
        for f in range(F):
            for y in range(H):
                for x in range(W):
                    lat[c, f, y, x] = 1000 * c + 100 * f + 10 * y + x
    tok = dit.patchify(lat, 1, 2, 2)
    assert tok.shape == (F * (H // 2) * (W // 2), C * 4)
    # token (f=1, row=1, col=2), feature (c=2, dy=1, dx=0)
    t = (1 * (H // 2) + 1) * (W // 2) + 2
    assert tok[t, 2 * 4 + 1 * 2 + 0] == 1000 * 2 + 100 * 1 + 10 * (2 * 1 + 1) + (2 * 2 + 0)
    assert np.array_equal(dit.unpatchify(tok, C, F, H, W, 1, 2, 2), lat)


# ---------------------------------------------------------------------------
# attention
# ---------------------------------------------------------------------------

def brute_attention(q, k, v, n_heads):
    Lq, d = q.shape
    hd = d // n_heads
    out = np.zeros((Lq, d))
    for h in range(n_heads):
        for i in range(Lq):
            s = [sum(q[i, h * hd + c] * k[j, h * hd + c] for c in range(hd)) / math.sqrt(hd)
                 for j in range(k.shape[0])]
            mx = max(s)
            e = [math.exp(x - mx) for x in s]
            z = sum(e)
            for c in range(hd):
                out[i, h * hd + c] = sum(e[j] * v[j, h * hd + c] for j in range(len(e))) / z
    return out


def streaming_two_buffer(q, bufs, n_heads):
    """Online softmax over a sequence of key buffers, one key at a time."""
    Lq, d = q.shape
    hd = d // n_heads
    out = np.zeros((Lq, d))
    for h in range(n_heads):
        c = slice(h * hd, (h + 1) * hd)
        for i in range(Lq):
            m, l, acc = -math.inf, 0.0, np.zeros(hd)
            for k, v in bufs:
                for j in range(k.shape[0]):
                    s = float(q[i, c] @ k[j, c]) / math.sqrt(hd)
                    mn = max(m, s)
                    a = math.exp(m - mn) if m > -math.inf else 0.0
                    p = math.exp(s - mn)
                    acc = acc * a + p * v[j, c]
                    l = l * a + p
                    m = mn
            out[i, c] = acc / l
    return out


def test_attention_matches_brute_force():
    rng = np.random.default_rng(2)
    q, k, v = rng.normal(size=(5, 8)), rng.normal(size=(7, 8)), rng.normal(size=(7, 8))
    assert np.allclose(dit.attention(q, k, v, 2), brute_attention(q, k, v, 2), atol=1e-12)


def test_softmax_rows_sum_to_one():
    rng = np.random.default_rng(3)
    p = dit.softmax_rows(rng.normal(scale=30, size=(9, 33)))
    assert np.allclose(p.sum(axis=1), 1.0, atol=1e-12)
    assert np.all(p >= 0)


def test_attention_closed_forms():
    rng = np.random.default_rng(4)
    k, v = rng.normal(size=(11, 8)), rng.normal(size=(11, 8))
    # zero queries: uniform weights, the mean of V over all keys
    assert np.allclose(dit.attention(np.zeros((3, 8)), k, v, 2), np.broadcast_to(v.mean(0), (3, 8)))
    # one key: the output is that key's value row
    assert np.allclose(dit.attention(rng.normal(size=(4, 8)), k[:1], v[:1], 4), np.broadcast_to(v[0], (4, 8)))
    # a dominant score selects its value row
    q = np.zeros((1, 4)); q[0, 0] = 1.0
    kk = np.zeros((3, 4)); kk[1, 0] = 200.0
    vv = np.arange(12.0).reshape(3, 4)
    assert np.allclose(dit.attention(q, kk, vv, 1), vv[1:2])


def test_attention_heads_are_independent():
    rng = np.random.default_rng(5)
    q, k, v = rng.normal(size=(4, 8)), rng.normal(size=(6, 8)), rng.normal(size=(6, 8))
    a = dit.attention(q, k, v, 2)
    k2 = k.copy(); k2[:, 4:] = rng.normal(size=(6, 4))
    b = dit.attention(q, k2, v, 2)
    assert np.array_equal(a[:, :4], b[:, :4]) and not np.allclose(a[:, 4:], b[:, 4:])


def test_two_buffer_attention_equals_streaming_and_concat():
    """Pin (a): attention over [pred; own] from two buffers equals one softmax
    over their explicit concatenation, streamed buffer after buffer."""
    rng = np.random.default_rng(6)
    q, k, v = rng.normal(size=(5, 8)), rng.normal(size=(6, 8)), rng.normal(size=(6, 8))
    kp, vp = rng.normal(size=(6, 8)), rng.normal(size=(6, 8))
    got = dit.self_attention_with_predecessor(q, k, v, kp, vp, 2)
    assert np.allclose(got, streaming_two_buffer(q, [(kp, vp), (k, v)], 2), rtol=1e-6, atol=1e-12)
    assert np.allclose(got, brute_attention(q, np.vstack([kp, k]), np.vstack([vp, v]), 2), atol=1e-12)
    # the predecessor's token order is irrelevant
    perm = rng.permutation(6)
    assert np.allclose(got, dit.self_attention_with_predecessor(q, k, v, kp[perm], vp[perm], 2), atol=1e-13)
    # permuting own tokens (keys and queries together) permutes the outputs (no position code)
    pr = rng.permutation(5)
    assert np.allclose(got[pr], dit.self_attention_with_predecessor(q[pr], k, v, kp, vp, 2), atol=1e-13)
    # no predecessor: own keys only
    assert np.allclose(dit.self_attention_with_predecessor(q, k, v, None, None, 2),
                       brute_attention(q, k, v, 2), atol=1e-12)


# ---------------------------------------------------------------------------
# queue
# ---------------------------------------------------------------------------

def stub_velocity(c):
    def fn(latents, levels, ids, pred_kv, keep):
        return [np.full_like(x, c) for x in latents], None
    return fn


def test_fifo_trace_matches_hand_derivation():
    rows = [ln.split("|") for ln in read_golden("fifo_T4_N6.txt")]
    zero = np.zeros((1, 1, 1, 1))
    _, traces = fifo.run_stream(stub_velocity(0.0), lambda k: zero, T=4, n_chunks=6)
    assert len(traces) == len(rows) == 6 + 4 - 1
    names = {fifo.PRED_NONE: "none", fifo.PRED_CACHE: "cache"}
    for tr, r in zip(traces, rows):
        assert tr.step == int(r[0])
        assert tr.chunk_ids == [int(t) for t in r[1].split()]
        assert tr.levels == [int(t) for t in r[2].split()]
        assert tr.popped == ([] if r[3].strip() == "-" else [int(t) for t in r[3].split()])
        assert names[tr.head_pred] == r[4].strip()
        assert tr.positions == [j - 1 for j in tr.levels]


@pytest.mark.parametrize("T,N", [(1, 3), (4, 6), (10, 32), (50, 64), (50, 128), (50, 16)])
def test_fifo_closed_form_schedule(T, N):
    """Step s holds chunks max(0, s-T+1) .. min(s, N-1); chunk k sits at level
    T - (s - k); pops are in increasing id order; N + T - 1 steps; every chunk
    exits after exactly T steps (pin (d))."""
    zero = np.zeros((1, 1, 1, 1))
    ready, traces = fifo.run_stream(stub_velocity(0.0), lambda k: zero, T=T, n_chunks=N)
    assert len(traces) == N + T - 1
    assert [k for k, _ in ready] == list(range(N))
    entered, left = {}, {}
    for s, tr in enumerate(traces):
        lo, hi = max(0, s - T + 1), min(s, N - 1)
        assert tr.chunk_ids == list(range(lo, hi + 1))
        assert tr.levels == [T - (s - k) for k in tr.chunk_ids]
        for k in tr.chunk_ids:
            entered.setdefault(k, s)
        for k in tr.popped:
            left[k] = s
    assert all(left[k] - entered[k] + 1 == T for k in range(N))


def test_euler_constant_velocity():
    """A stub model with constant v = c moves x by exactly -c over T steps."""
    for T in (4, 8):
        noise = np.full((1, 1, 2, 2), 3.0)
        ready, _ = fifo.run_stream(stub_velocity(0.5), lambda k: noise, T=T, n_chunks=3)
        for _, x in ready:
            assert np.array_equal(x, noise - 0.5)
    noise = np.full((1, 1, 2, 2), 3.0)
    ready, _ = fifo.run_stream(stub_velocity(0.5), lambda k: noise, T=50, n_chunks=2)
    for _, x in ready:
        assert np.allclose(x, 2.5, atol=1e-13)


def test_level_seen_by_model():
    """Each chunk is denoised at levels T, T-1, ..., 1 in that order."""
    seen = {}

    def fn(latents, levels, ids, pred_kv, keep):
        for k, j in zip(ids, levels):
            seen.setdefault(k, []).append(j)
        return [np.zeros_like(x) for x in latents], None
    fifo.run_stream(fn, lambda k: np.zeros((1, 1, 1, 1)), T=5, n_chunks=7)
    assert all(seen[k] == [5, 4, 3, 2, 1] for k in range(7))


# ---------------------------------------------------------------------------
# the DiT velocity on the tiny workload
# ---------------------------------------------------------------------------

W = synth.WORKLOADS["tiny_fp32"]


@pytest.fixture(scope="module")
def tiny():
    p = synth.make_params(W.model)
    text = synth.make_text(W.model)
    noise = [synth.make_noise(W.model, W.queue, k) for k in range(W.queue.n_chunks)]
    return p, text, noise


def test_T1_no_cache_is_single_chunk_euler(tiny):
    """Pin (c): with T = 1 and no neighbour, one queue step is x - v(x, sigma=1)."""
    p, text, noise = tiny
    fn = dit.make_velocity_fn(p, text, W.model, T=1, use_pred=False)
    ready, traces = fifo.run_stream(fn, lambda k: noise[k], T=1, n_chunks=3, use_pred=False)
    assert len(traces) == 3
    for k, x in ready:
        (v,), _ = fn([np.asarray(noise[k], np.float64)], [1], [k], None, None)
        assert np.allclose(x, noise[k] - v, atol=1e-14)


def test_no_cache_queue_equals_standalone_euler(tiny):
    """With the neighbour link off, every popped chunk equals a T-step Euler
    loop of that chunk alone: batching never mixes chunks or levels."""
    p, text, noise = tiny
    T = W.queue.T
    fn = dit.make_velocity_fn(p, text, W.model, T, use_pred=False)
    ready, _ = fifo.run_stream(fn, lambda k: noise[k], T=T, n_chunks=W.queue.n_chunks,
                               use_pred=False)
    for k, x in ready:
        assert np.allclose(x, fifo.euler_chunk(fn, noise[k], T, k), atol=1e-13)


def test_predecessor_link_is_causal(tiny):
    """A chunk only sees the chunk before it, one hop per layer: changing
    chunk 1 leaves chunk 0 unchanged, changes chunks 1..1+L, and leaves any
    chunk further away unchanged."""
    p, text, noise = tiny
    L = W.model.n_layers
    fn = dit.make_velocity_fn(p, text, W.model, T=8)
    lat = [np.asarray(noise[k % 6], np.float64) for k in range(6)]
    lv = [1, 2, 3, 4, 5, 6]
    ids = list(range(6))
    v0, _ = fn(lat, lv, ids, None, None)
    lat2 = list(lat)
    lat2[1] = lat[1] + 0.5
    v1, _ = fn(lat2, lv, ids, None, None)
    assert np.array_equal(v0[0], v1[0])
    for k in range(1, 2 + L):
        assert not np.allclose(v0[k], v1[k])
    for k in range(2 + L, 6):
        assert np.array_equal(v0[k], v1[k])


def test_persisted_kv_equals_in_batch_kv(tiny):
    """Running chunks 2..4 with chunk 1's persisted K/V equals running 1..4
    together (for chunks 2..4)."""
    p, text, noise = tiny
    fn = dit.make_velocity_fn(p, text, W.model, T=6)
    lat = [np.asarray(noise[k], np.float64) for k in range(5)]
    vs, _ = fn(lat[1:5], [2, 3, 4, 5], [1, 2, 3, 4], None, None)
    _, kv1 = fn(lat[1:2], [2], [1], None, 0)
    vs2, _ = fn(lat[2:5], [3, 4, 5], [2, 3, 4], kv1, None)
    for a, b in zip(vs[1:], vs2):
        assert np.allclose(a, b, atol=1e-14)


def test_zero_gates_bypass_the_blocks(tiny):
    """Gates and the cross-attention output projection at zero: the residual
    stream carries the patch embedding unchanged, so the attention and FFN
    weights cannot influence v."""
    p, text, noise = tiny
    d = W.model.dim
    q = {k: (list(v) if isinstance(v, list) else v) for k, v in p.items()}
    gates = np.ones(6 * d, bool)
    gates[2 * d:3 * d] = gates[5 * d:6 * d] = False
    q["mod.w"] = np.where(gates[:, None], p["mod.w"], 0).astype(np.float32)
    q["mod.b"] = np.where(gates, p["mod.b"], 0).astype(np.float32)
    q["layer.mod"] = [np.where(gates, t, 0).astype(np.float32) for t in p["layer.mod"]]
    q["layer.co.w"] = [np.zeros_like(t) for t in p["layer.co.w"]]
    q["layer.co.b"] = [np.zeros_like(t) for t in p["layer.co.b"]]
    a = dit.make_velocity_fn(q, text, W.model, T=4)
    r = dict(q)
    rng = np.random.default_rng(7)
    for name in ("layer.qkv.w", "layer.o.w", "layer.ffn1.w", "layer.ffn2.w", "layer.cq.w"):
        r[name] = [rng.normal(size=t.shape).astype(np.float32) for t in q[name]]
    b = dit.make_velocity_fn(r, text, W.model, T=4)
    lat = [np.asarray(noise[k], np.float64) for k in range(3)]
    va, _ = a(lat, [2, 3, 4], [0, 1, 2], None, None)
    vb, _ = b(lat, [2, 3, 4], [0, 1, 2], None, None)
    for x, y in zip(va, vb):
        assert np.allclose(x, y, atol=1e-15)
    # while with the gates on, the same change does move v
    c = dict(p)
    c["layer.ffn2.w"] = r["layer.ffn2.w"]
    v1, _ = dit.make_velocity_fn(p, text, W.model, T=4)(lat, [2, 3, 4], [0, 1, 2], None, None)
    v2, _ = dit.make_velocity_fn(c, text, W.model, T=4)(lat, [2, 3, 4], [0, 1, 2], None, None)
    assert not np.allclose(v1[0], v2[0])


def test_single_text_token_cross_attention_closed_form():
    """One text token: every query's cross-attention output is that token's value."""
    rng = np.random.default_rng(8)
    q = rng.normal(size=(7, 16))
    kt, vt = rng.normal(size=(1, 16)), rng.normal(size=(1, 16))
    assert np.allclose(dit.attention(q, kt, vt, 4), np.broadcast_to(vt, (7, 16)))


def test_level_changes_velocity(tiny):
    p, text, noise = tiny
    fn = dit.make_velocity_fn(p, text, W.model, T=4)
    x = np.asarray(noise[0], np.float64)
    (va,), _ = fn([x], [1], [0], None, None)
    (vb,), _ = fn([x], [4], [0], None, None)
    assert not np.allclose(va, vb)


def test_three_buffer_attention_equals_streaming_and_concat():
    """Bidirectional neighbourhood: [pred; own; succ] from three buffers equals
    one streamed softmax over them and brute force over the concatenation; the
    order of the buffers is irrelevant."""
    rng = np.random.default_rng(9)
    q, k, v = rng.normal(size=(4, 8)), rng.normal(size=(5, 8)), rng.normal(size=(5, 8))
    kp, vp = rng.normal(size=(5, 8)), rng.normal(size=(5, 8))
    ks, vs = rng.normal(size=(5, 8)), rng.normal(size=(5, 8))
    got = dit.self_attention_with_neighbours(q, k, v, kp, vp, ks, vs, 2)
    assert np.allclose(got, streaming_two_buffer(q, [(ks, vs), (kp, vp), (k, v)], 2), rtol=1e-6, atol=1e-12)
    assert np.allclose(got, brute_attention(q, np.vstack([kp, k, ks]), np.vstack([vp, v, vs]), 2), atol=1e-12)
    # no successor: the predecessor-only form
    assert np.allclose(dit.self_attention_with_neighbours(q, k, v, kp, vp, None, None, 2),
                       dit.self_attention_with_predecessor(q, k, v, kp, vp, 2), atol=1e-15)


def test_bidirectional_link_reaches_both_ways(tiny):
    """With both neighbours, changing chunk 2 changes chunks 0..4 (one hop per
    layer each way, 2 layers) and leaves chunk 5 unchanged."""
    p, text, noise = tiny
    L = W.model.n_layers
    fn = dit.make_velocity_fn(p, text, W.model, T=8, neighbours="both")
    lat = [np.asarray(noise[k % 6], np.float64) for k in range(6)]
    lv, ids = [1, 2, 3, 4, 5, 6], list(range(6))
    v0, _ = fn(lat, lv, ids, None, None)
    lat2 = list(lat)
    lat2[2] = lat[2] + 0.5
    v1, _ = fn(lat2, lv, ids, None, None)
    for k in range(2 - L, 2 + L + 1):
        assert not np.allclose(v0[k], v1[k]), k
    assert np.array_equal(v0[5], v1[5])
    # the predecessor-only model never looks forward
    fp = dit.make_velocity_fn(p, text, W.model, T=8)
    w0, _ = fp(lat, lv, ids, None, None)
    w1, _ = fp(lat2, lv, ids, None, None)
    assert np.array_equal(w0[0], w1[0]) and np.array_equal(w0[1], w1[1])


# ---------------------------------------------------------------------------
# per-head QK RMSNorm and 3-D rotary positions
# ---------------------------------------------------------------------------

def test_rms_norm_heads_closed_form():
    rng = np.random.default_rng(10)
    x = rng.normal(2.0, 3.0, size=(5, 16))
    y = dit.rms_norm_heads(x, np.ones(16), 4, eps=0.0)
    assert np.allclose((y.reshape(5, 4, 4) ** 2).mean(-1), 1.0)
    # per head: scaling one head's slice leaves the other heads unchanged
    x2 = x.copy(); x2[:, 4:8] *= 7.0
    y2 = dit.rms_norm_heads(x2, np.ones(16), 4, eps=0.0)
    assert np.allclose(y, y2)
    w = rng.normal(size=16)
    assert np.allclose(dit.rms_norm_heads(x, w, 4), dit.rms_norm_heads(x, np.ones(16), 4) * w)


def test_rope_bands_and_rotation():
    assert dit.rope_bands(128) == (22, 21, 21)
    assert dit.rope_bands(64) == (12, 10, 10)
    assert dit.rope_bands(16) == (4, 2, 2)
    rng = np.random.default_rng(11)
    x = rng.normal(size=(6, 32))
    t, y, xx = rng.integers(0, 50, 6), rng.integers(0, 30, 6), rng.integers(0, 52, 6)
    ang = dit.rope_angles(t, y, xx, 16)
    r = dit.apply_rope(x, ang, 2)
    # rotation: every pair keeps its length
    assert np.allclose(np.hypot(r[:, 0::2], r[:, 1::2]), np.hypot(x[:, 0::2], x[:, 1::2]))
    # position zero is the identity; a hand example: pair 0 of the temporal band
    # turns by t radians (base^0 = 1)
    assert np.allclose(dit.apply_rope(x, dit.rope_angles(np.zeros(6), np.zeros(6), np.zeros(6), 16), 2), x)
    one = np.zeros((1, 16)); one[0, 0] = 1.0
    got = dit.apply_rope(one, dit.rope_angles([2.0], [0.0], [0.0], 16), 1)
    assert np.allclose(got[0, :2], [math.cos(2.0), math.sin(2.0)])
    # the last temporal pair of hd = 16 (band of 4) turns by t * 10000^(-3/4)
    one = np.zeros((1, 16)); one[0, 6] = 1.0
    got = dit.apply_rope(one, dit.rope_angles([3.0], [0.0], [0.0], 16), 1)
    a = 3.0 * 10000.0 ** (-3 / 4)
    assert np.allclose(got[0, 6:8], [math.cos(a), math.sin(a)])


def test_rope_scores_depend_on_relative_position_only():
    """q(p1) . k(p2) after rotation is a function of p1 - p2: shifting every
    position by the same offset leaves attention unchanged."""
    rng = np.random.default_rng(12)
    q, k, v = rng.normal(size=(5, 32)), rng.normal(size=(7, 32)), rng.normal(size=(7, 32))
    pq = [rng.integers(0, 40, 5) for _ in range(3)]
    pk = [rng.integers(0, 40, 7) for _ in range(3)]
    o1 = dit.attention(dit.apply_rope(q, dit.rope_angles(*pq, 16), 2),
                       dit.apply_rope(k, dit.rope_angles(*pk, 16), 2), v, 2)
    shift = (1000, 17, 5)
    o2 = dit.attention(dit.apply_rope(q, dit.rope_angles(*[a + s for a, s in zip(pq, shift)], 16), 2),
                       dit.apply_rope(k, dit.rope_angles(*[a + s for a, s in zip(pk, shift)], 16), 2), v, 2)
    assert np.allclose(o1, o2, atol=1e-10)


def test_token_positions_follow_patch_order():
    t, y, x = dit.token_positions(3, 2, 4, 6, 1, 2, 2)
    assert len(t) == 2 * 2 * 3
    # token index (f=1, row=1, col=2) = (1 * 2 + 1) * 3 + 2
    i = (1 * 2 + 1) * 3 + 2
    assert (t[i], y[i], x[i]) == (3 * 2 + 1, 1, 2)


def test_rope_model_shift_invariance_over_chunk_ids(tiny):
    """With rotary positions the velocity of a batch does not depend on the
    absolute chunk ids, only on their offsets (relative positions)."""
    p, text, noise = tiny
    m = dataclasses_replace_rope(W.model)
    q = synth.make_params(m)
    fn = dit.make_velocity_fn(q, text, m, T=6)
    lat = [np.asarray(noise[k], np.float64) for k in range(3)]
    va, _ = fn(lat, [2, 3, 4], [0, 1, 2], None, None)
    vb, _ = fn(lat, [2, 3, 4], [40, 41, 42], None, None)
    for a, b in zip(va, vb):
        assert np.allclose(a, b, atol=1e-10)
    # and it does depend on the positions: swapping in a non-contiguous layout
    # of frames is visible (rotary positions are active)
    fn0 = dit.make_velocity_fn(p, text, W.model, T=6)
    v0, _ = fn0(lat, [2, 3, 4], [0, 1, 2], None, None)
    assert not np.allclose(v0[1], va[1])


def dataclasses_replace_rope(m):
    import dataclasses
    return dataclasses.replace(m, qk_norm_rope=True)


# ---------------------------------------------------------------------------
# coordinated noise initialisation
# ---------------------------------------------------------------------------

def test_coordinated_noise_sets_alternate_and_cover_the_pool():
    from oracle import noise
    F = 4
    for k in range(20):
        a, b = noise.chunk_frames(k, F, 3), noise.chunk_frames(k + 1, F, 3)
        assert sorted(a) == list(range(0, F) if k % 2 == 0 else range(F, 2 * F))
        assert not set(a) & set(b)                     # no repeat between neighbours
        assert sorted(a + b) == list(range(2 * F))     # together the whole pool


def test_coordinated_noise_shuffle_is_a_uniform_permutation():
    from oracle import noise
    F = 3
    counts = np.zeros((F, F))
    perms = set()
    for k in range(0, 6000, 2):
        fr = noise.chunk_frames(k, F, 7)
        perms.add(tuple(fr))
        for pos, b in enumerate(fr):
            counts[pos, b] += 1
    assert len(perms) == 6                             # every order of 3 frames occurs
    assert np.allclose(counts / counts.sum(axis=1, keepdims=True), 1 / F, atol=0.04)


def test_coordinated_noise_gathers_pool_frames():
    from oracle import noise
    rng = np.random.default_rng(13)
    pool = rng.normal(size=(4, 3, 2, 5))               # 2F = 4 frames, C=3, H=2, W=5
    lat = noise.coordinated_noise(pool, 1, 3)
    fr = noise.chunk_frames(1, 2, 3)
    assert lat.shape == (3, 2, 2, 5)
    for f in range(2):
        assert np.array_equal(lat[:, f], pool[fr[f]])
