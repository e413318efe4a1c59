"""Queue-level parity on the GPU through the C ABI (dp_queue_*), against the
float64 oracle on identical seeded inputs:

* fp32 validation mode, tiny workload: every popped chunk of the whole stream
  within relative L2 1e-4;
* bookkeeping (chunk ids, levels, positions, neighbour source, pop order)
  exactly equal to the oracle queue on the (T, N) schedule of every workload;
* bf16 production mode: one queue step from the same state within relative L2
  2e-2 on the velocity of every chunk, on the persisted K/V and on the latents
  (small workload; Wan-1.3B shapes with two layers; Wan-14B shapes with one
  layer; the bidirectional neighbourhood; QK RMSNorm with rotary positions);
* resuming from latents and persisted K/V read mid-stream is bit-exact, and
  matches the oracle (whole fp32 stream; one bf16 step from the checkpoint);
* load_state accepts only states a FIFO stream reaches; a host pop reports a
  kernel that gave up a bounded wait;
* error codes, the internal noise generator, flat device memory.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import synth  # noqa: E402
from oracle import dit, fifo  # noqa: E402

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def rel_l2(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30))


def bf16_round(x):
    return torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(torch.bfloat16).float().numpy()


def make(w, precision, params=None, text=None, n_chunks=None, T=None, ready=2, neighbours="pred"):
    from chunked_fifo_denoising_b200 import Model, Queue
    m, q = w.model, w.queue
    params = synth.make_params(m) if params is None else params
    text = synth.make_text(m) if text is None else text
    model = Model(m, precision, neighbours=neighbours)
    model.set_params(params)
    queue = Queue(model, text, q.T if T is None else T, q.frames_per_chunk, q.lat_h, q.lat_w,
                  q.n_chunks if n_chunks is None else n_chunks, ready_capacity=ready)
    return model, queue, params, text


@pytest.mark.parametrize("neighbours,rope", [("pred", False), ("both", False), ("pred", True)])
def test_tiny_fp32_stream_matches_oracle(neighbours, rope):
    w = synth.WORKLOADS["tiny_fp32"]
    if rope:
        w = synth.with_qk_norm_rope(w)
    m, q = w.model, w.queue
    model, queue, p, text = make(w, "fp32", neighbours=neighbours)
    noise = [synth.make_noise(m, q, k) for k in range(q.n_chunks)]
    fn = dit.make_velocity_fn(p, text, m, q.T, neighbours=neighbours)
    ready, traces = fifo.run_stream(fn, lambda k: noise[k], q.T, q.n_chunks)
    out = np.empty(q.chunk_shape(m), np.float32)
    got = {}
    for tr in traces:
        info = queue.inspect()
        assert info["step"] == tr.step
        assert info["ids"] == tr.chunk_ids and info["levels"] == tr.levels
        assert info["positions"] == tr.positions
        assert info["head_pred"] == tr.head_pred
        queue.step(noise[tr.step] if tr.step < q.n_chunks else None)
        queue.sync()
        popped = []
        while True:
            st, cid = queue.try_pop(out)
            if st != 0:
                break
            popped.append(cid)
            got[cid] = out.copy()
        assert popped == tr.popped
    assert queue.inspect()["drained"] == 1
    assert list(got) == list(range(q.n_chunks))
    for k, ref in ready:
        assert rel_l2(got[k], ref) <= 1e-4, k
    model.close()


@pytest.mark.parametrize("precision,T,N", [("fp32", 1, 3), ("fp32", 4, 1), ("fp32", 6, 3),
                                             ("bf16", 1, 3)])
def test_degenerate_queues_match_oracle(precision, T, N):
    """T = 1 (every step persists the head's K/V and each chunk's neighbour comes
    from the cache), a single chunk, and a stream shorter than the queue, on
    the tiny model (fp32: 1e-4 on every popped chunk; bf16: 2e-2)."""
    w = synth.WORKLOADS["tiny_fp32"]
    if precision == "bf16":  # bf16 path needs head_dim 64: 64 wide, one head
        import dataclasses
        w = dataclasses.replace(w, model=dataclasses.replace(w.model, n_heads=1))
    m, q = w.model, w.queue
    model, queue, p, text = make(w, precision, n_chunks=N, T=T)
    noise = [synth.make_noise(m, q, k) for k in range(N)]
    fn = dit.make_velocity_fn(p, text, m, T)
    ready, traces = fifo.run_stream(fn, lambda k: noise[k], T, N)
    assert len(traces) == N + T - 1
    out = np.empty(q.chunk_shape(m), np.float32)
    got = {}
    for tr in traces:
        queue.step(noise[tr.step] if tr.step < N else None)
        while True:
            st, cid = queue.try_pop(out)
            if st != 0:
                break
            got[cid] = out.copy()
    queue.sync()
    assert sorted(got) == list(range(N))
    tol = 1e-4 if precision == "fp32" else 2e-2
    for k, ref in ready:
        assert rel_l2(got[k], ref) <= tol, (k, rel_l2(got[k], ref))
    model.close()


def test_host_noise_buffer_is_free_when_step_returns():
    """One page-locked host buffer carries every pushed chunk: it is refilled
    with the next chunk's noise (and poisoned in between) as soon as each step
    returns, while the queue's stream may still be busy; the popped chunks
    must still match the oracle stream (fp32, 1e-4)."""
    w = synth.WORKLOADS["tiny_fp32"]
    m, q = w.model, w.queue
    model, queue, p, text = make(w, "fp32")
    noise = [synth.make_noise(m, q, k) for k in range(q.n_chunks)]
    fn = dit.make_velocity_fn(p, text, m, q.T)
    ready, traces = fifo.run_stream(fn, lambda k: noise[k], q.T, q.n_chunks)
    buf = torch.empty(q.chunk_shape(m), dtype=torch.float32).pin_memory()
    out = np.empty(q.chunk_shape(m), np.float32)
    got = {}
    for tr in traces:
        if tr.step < q.n_chunks:
            buf.copy_(torch.from_numpy(noise[tr.step]))
            queue.step(buf)
            buf.fill_(float("nan"))
        else:
            queue.step(None)
        while True:
            st, cid = queue.try_pop(out)
            if st != 0:
                break
            got[cid] = out.copy()
    queue.sync()
    assert sorted(got) == list(range(q.n_chunks))
    for k, ref in ready:
        assert rel_l2(got[k], ref) <= 1e-4, (k, rel_l2(got[k], ref))
    model.close()


def test_invalid_configurations_are_rejected():
    import ctypes as C
    from chunked_fifo_denoising_b200 import Model, Queue, DPError
    from chunked_fifo_denoising_b200 import _binding as B
    w = synth.WORKLOADS["tiny_fp32"]
    m, q = w.model, w.queue
    import dataclasses
    with pytest.raises(DPError) as e:   # bf16 needs head_dim 64 or 128 (here 16)
        Model(m, "bf16")
    assert e.value.status == B.DP_ERR_INVALID_ARG
    with pytest.raises(DPError):
        Model(dataclasses.replace(m, n_heads=3), "fp32")
    model = Model(m, "fp32")
    text = synth.make_text(m)
    with pytest.raises(DPError) as e:   # parameters not set yet
        Queue(model, text, q.T, q.frames_per_chunk, q.lat_h, q.lat_w, 4)
    assert e.value.status == B.DP_ERR_STATE
    model.set_params(synth.make_params(m))
    for kw in (dict(T=0), dict(n=0), dict(lat_h=7)):
        with pytest.raises(DPError) as e:
            Queue(model, text, kw.get("T", q.T), q.frames_per_chunk, kw.get("lat_h", q.lat_h), q.lat_w,
                  kw.get("n", 4))
        assert e.value.status == B.DP_ERR_INVALID_ARG
    with pytest.raises(DPError):        # wrong element count
        model.set_param("patch.w", np.zeros(5, np.float32))
    queue = Queue(model, text, q.T, q.frames_per_chunk, q.lat_h, q.lat_w, 4)
    with pytest.raises(DPError):        # read_latents with a wrong count
        queue.read_latents(3)
    assert B.dp_queue_step(None, None, 0) == B.DP_ERR_INVALID_ARG
    # a location that is neither host nor device is rejected before any copy
    buf = np.empty(q.chunk_numel(m) * 4, np.float32)
    assert B.dp_queue_read_latents(queue.handle, buf.ctypes.data, 0, 7) == B.DP_ERR_INVALID_ARG
    cid = C.c_longlong()
    assert B.dp_queue_read_pred_kv(queue.handle, buf.ctypes.data, 7, cid) == B.DP_ERR_INVALID_ARG
    assert B.dp_queue_step(queue.handle, buf.ctypes.data, 7) == B.DP_ERR_INVALID_ARG
    assert B.dp_queue_pop(queue.handle, buf.ctypes.data, 7, cid) == B.DP_ERR_INVALID_ARG
    model.close()


@pytest.mark.parametrize("name", list(synth.WORKLOADS))
def test_bookkeeping_exact_on_every_schedule(name):
    """The (T, N) schedule of each workload, run at full N on the tiny model."""
    w = synth.WORKLOADS[name]
    T, N = w.queue.T, w.queue.n_chunks
    tiny = synth.WORKLOADS["tiny_fp32"]
    model, queue, _, _ = make(tiny, "fp32", n_chunks=N, T=T)
    _, traces = fifo.run_stream(lambda lat, lv, ids, kv, keep: ([np.zeros_like(x) for x in lat], None),
                                lambda k: np.zeros((1, 1, 1, 1)), T, N)
    assert len(traces) == N + T - 1
    out = torch.empty(tiny.queue.chunk_shape(tiny.model), device="cuda")
    order = []
    for tr in traces:
        info = queue.inspect()
        assert (info["step"], info["ids"], info["levels"], info["positions"], info["head_pred"]) == \
            (tr.step, tr.chunk_ids, tr.levels, tr.positions, tr.head_pred)
        assert info["writes_cache"] == int(tr.levels[0] == 1)
        assert info["slots"] == [k % (T + 2) for k in tr.chunk_ids]
        queue.step(None)
        while True:
            st, cid = queue.try_pop(out)
            if st != 0:
                break
            order.append(cid)
    assert order == list(range(N))
    assert queue.try_step(None) == 6  # DP_ERR_DRAINED
    queue.sync()
    model.close()


def _one_step_parity(w, n_layers=None, n_occ=3, seed_state=7, neighbours="pred"):
    """Queue state just before a step: chunks at levels 1 .. n_occ (no push),
    the head's predecessor K/V persisted; compare one GPU step with the oracle."""
    if n_layers is not None:
        w = synth.truncated(w, n_layers)
    m, q = w.model, w.queue
    T = q.T
    n_chunks = 20
    head = n_chunks - n_occ
    step = head + T - 1              # the head chunk is at level 1
    model, queue, p, text = make(w, "bf16", n_chunks=n_chunks, neighbours=neighbours)
    rng = np.random.default_rng(seed_state)
    lat = rng.standard_normal((n_occ,) + q.chunk_shape(m)).astype(np.float32)
    Lc = q.tokens_per_chunk(m)
    kv = bf16_round(rng.standard_normal((m.n_layers, 2, Lc, m.dim)).astype(np.float32) * 0.5)
    queue.load_state(step, n_chunks, lat, kv)
    info = queue.inspect()
    assert info["ids"] == list(range(head, n_chunks)) and info["levels"] == list(range(1, n_occ + 1))
    assert info["head_pred"] == 2 and info["writes_cache"] == 1
    queue.step(None)
    queue.sync()
    popped = np.empty(q.chunk_shape(m), np.float32)
    assert queue.pop(popped) == head
    rest = queue.read_latents(n_occ - 1)
    new_kv, kv_id = queue.read_pred_kv()
    assert kv_id == head
    # oracle
    fn = dit.make_velocity_fn(p, text, m, T, neighbours=neighbours)
    st = fifo.QueueState(T=T, n_chunks=n_chunks, step=step, next_id=n_chunks,
                         entries=[fifo.Entry(head + i, 1 + i, lat[i].astype(np.float64)) for i in range(n_occ)],
                         pred_id=head - 1, pred_kv=[(kv[l, 0], kv[l, 1]) for l in range(m.n_layers)])
    tr = fifo.queue_step(st, fn, None)
    assert tr.popped == [head]
    ref_pop = st.ready[0][1]
    ref_rest = [e.latent for e in st.entries]
    dsig = -1.0 / T
    v_gpu = [(popped - lat[0]) / dsig] + [(rest[i] - lat[i + 1]) / dsig for i in range(n_occ - 1)]
    v_ref = [(ref_pop - lat[0]) / dsig] + [(ref_rest[i] - lat[i + 1]) / dsig for i in range(n_occ - 1)]
    errs = [rel_l2(a, b) for a, b in zip(v_gpu, v_ref)]
    assert max(errs) <= 2e-2, errs
    assert rel_l2(popped, ref_pop) <= 2e-2
    for l in range(m.n_layers):
        assert rel_l2(new_kv[l, 0], st.pred_kv[l][0]) <= 2e-2, l
        assert rel_l2(new_kv[l, 1], st.pred_kv[l][1]) <= 2e-2, l
    model.close()
    return errs


def test_bf16_step_small():
    _one_step_parity(synth.WORKLOADS["small_bf16"])


def test_bf16_step_small_bidirectional():
    """The bidirectional neighbourhood: chunk k also reads chunk k+1's K/V."""
    _one_step_parity(synth.WORKLOADS["small_bf16"], neighbours="both")


def test_bf16_step_small_qk_norm_rope():
    """Per-head QK RMSNorm and 3-D rotary positions; the persisted K of the
    head chunk is the rotated one."""
    _one_step_parity(synth.with_qk_norm_rope(synth.WORKLOADS["small_bf16"]))


def test_bf16_step_wan13b_shapes_two_layers():
    _one_step_parity(synth.WORKLOADS["wan1.3b_480p"], n_layers=2)


def test_bf16_step_wan14b_shapes_one_layer():
    """Wan-14B shapes (d 5120, 40 heads, 7200 tokens per chunk), one layer,
    three chunks: the head with its persisted predecessor and two chunks whose
    predecessors are rows of the same batch (the oracle needs about 40 s per
    chunk and layer at these shapes; two layers are composed at Wan-1.3B shapes)."""
    _one_step_parity(synth.WORKLOADS["wan14b_720p"], n_layers=1, n_occ=3)


def test_checkpoint_resume_is_bit_exact():
    """Latents and persisted K/V read mid-stream and loaded into a new queue
    continue the stream with bit-identical outputs."""
    from chunked_fifo_denoising_b200 import Queue
    w = synth.truncated(synth.WORKLOADS["small_bf16"], 2)
    m, q = w.model, w.queue
    N, s_ck = 14, 12
    model, qa, p, text = make(w, "bf16", n_chunks=N)
    out = np.empty(q.chunk_shape(m), np.float32)
    got_a, got_b = {}, {}
    for _ in range(s_ck):
        qa.step(None)
        while qa.try_pop(out)[0] == 0:
            pass
    info = qa.inspect()
    n_q = info["n"] - (1 if info["next_push_id"] >= 0 else 0)
    lat = qa.read_latents(n_q)
    kv, kv_id = qa.read_pred_kv()
    n_pushed = info["next_push_id"] if info["next_push_id"] >= 0 else N
    qb = Queue(model, text, q.T, q.frames_per_chunk, q.lat_h, q.lat_w, N)
    qb.load_state(info["step"], n_pushed, lat, kv if kv_id >= 0 else None)
    for qq, got in ((qa, got_a), (qb, got_b)):
        while qq.try_step(None) == 0:
            while True:
                st, cid = qq.try_pop(out)
                if st != 0:
                    break
                got[cid] = out.copy()
        while True:
            st, cid = qq.try_pop(out)
            if st != 0:
                break
            got[cid] = out.copy()
    assert sorted(got_a) == sorted(got_b) and len(got_a) > 0
    for k in got_a:
        assert np.array_equal(got_a[k], got_b[k]), k
    model.close()


def test_resume_matches_the_oracle_stream():
    """fp32 validation mode, tiny workload: a checkpoint read mid-stream (head
    chunk with a persisted predecessor, pushes still due) and loaded into a new
    queue finishes the stream; every chunk popped before and after the
    checkpoint matches the oracle's unbroken stream (relative L2 1e-4)."""
    from chunked_fifo_denoising_b200 import Queue
    w = synth.WORKLOADS["tiny_fp32"]
    m, q = w.model, w.queue
    N, T, s_ck = q.n_chunks, q.T, 5
    model, qa, p, text = make(w, "fp32")
    noise = [synth.make_noise(m, q, k) for k in range(N)]
    out = np.empty(q.chunk_shape(m), np.float32)
    got = {}

    def drain(qq):
        while True:
            st, cid = qq.try_pop(out)
            if st != 0:
                return
            got[cid] = out.copy()
    for s in range(s_ck):
        qa.step(noise[s])
        drain(qa)
    info = qa.inspect()
    n_pushed = info["next_push_id"]
    assert info["step"] == s_ck and n_pushed == s_ck          # pushes still due
    n_q = info["n"] - 1
    lat = qa.read_latents(n_q)
    kv, kv_id = qa.read_pred_kv()
    assert kv_id == n_pushed - n_q - 1 >= 0                  # the head has a persisted predecessor
    qa.close()
    qb = Queue(model, text, T, q.frames_per_chunk, q.lat_h, q.lat_w, N)
    qb.load_state(s_ck, n_pushed, lat, kv)
    assert qb.inspect()["ids"] == info["ids"] and qb.inspect()["levels"] == info["levels"]
    s = s_ck
    while qb.try_step(noise[s] if s < N else None) == 0:
        s += 1
        drain(qb)
    drain(qb)
    assert s == N + T - 1
    fn = dit.make_velocity_fn(p, text, m, T)
    ready, _ = fifo.run_stream(fn, lambda k: noise[k], T, N)
    assert sorted(got) == list(range(N))
    for k, ref in ready:
        assert rel_l2(got[k], ref) <= 1e-4, k
    model.close()


def test_resumed_bf16_step_matches_the_oracle_step():
    """bf16, small workload with two layers: the checkpoint of a GPU stream,
    loaded into a new queue, takes one step (with a push) that matches the
    oracle's step from the same checkpoint within relative L2 2e-2 on every
    chunk's latent and on the newly persisted K/V."""
    from chunked_fifo_denoising_b200 import Queue
    w = synth.truncated(synth.WORKLOADS["small_bf16"], 2)
    m, q = w.model, w.queue
    N, T, s_ck = 14, q.T, 12
    model, qa, p, text = make(w, "bf16", n_chunks=N)
    noise = [synth.make_noise(m, q, k) for k in range(N)]
    out = np.empty(q.chunk_shape(m), np.float32)
    for s in range(s_ck):
        qa.step(noise[s])
        while qa.try_pop(out)[0] == 0:
            pass
    info = qa.inspect()
    n_pushed, n_q = info["next_push_id"], info["n"] - 1
    lat = qa.read_latents(n_q)
    kv, kv_id = qa.read_pred_kv()
    head = n_pushed - n_q
    assert kv_id == head - 1 >= 0 and info["levels"][0] == 1
    qa.close()
    qb = Queue(model, text, T, q.frames_per_chunk, q.lat_h, q.lat_w, N)
    qb.load_state(s_ck, n_pushed, lat, kv)
    qb.step(noise[n_pushed])
    qb.sync()
    popped = np.empty(q.chunk_shape(m), np.float32)
    assert qb.pop(popped) == head
    rest = qb.read_latents(n_q)              # the chunks after the head, plus the one pushed
    new_kv, new_id = qb.read_pred_kv()
    assert new_id == head
    fn = dit.make_velocity_fn(p, text, m, T)
    st = fifo.QueueState(T=T, n_chunks=N, step=s_ck, next_id=n_pushed,
                         entries=[fifo.Entry(head + i, info["levels"][i], lat[i].astype(np.float64))
                                  for i in range(n_q)],
                         pred_id=head - 1, pred_kv=[(kv[l, 0], kv[l, 1]) for l in range(m.n_layers)])
    tr = fifo.queue_step(st, fn, noise[n_pushed])
    assert tr.popped == [head] and tr.chunk_ids == info["ids"]
    assert rel_l2(popped, st.ready[0][1]) <= 2e-2
    for i, e in enumerate(st.entries):
        assert rel_l2(rest[i], e.latent) <= 2e-2, i
    for l in range(m.n_layers):
        assert rel_l2(new_kv[l, 0], st.pred_kv[l][0]) <= 2e-2, l
        assert rel_l2(new_kv[l, 1], st.pred_kv[l][1]) <= 2e-2, l
    model.close()


def test_load_state_rejects_states_no_stream_reaches():
    """A state is accepted only if a FIFO stream reaches it; a rejected one
    leaves the queue unchanged.  A state past its last push is restored closed."""
    w = synth.WORKLOADS["tiny_fp32"]
    m, q = w.model, w.queue
    model, queue, _, _ = make(w, "fp32", n_chunks=-1, T=4)
    shape = q.chunk_shape(m)
    Lc = q.tokens_per_chunk(m)
    kv = np.zeros((m.n_layers, 2, Lc, m.dim), np.float32)
    queue.step(None)
    before = queue.inspect()
    lat2 = np.zeros((2,) + shape, np.float32)
    from chunked_fifo_denoising_b200 import DPError
    # head chunk 3 at level 2 while chunk 2 (level 1) has not left
    with pytest.raises(DPError, match="INVALID_ARG"):
        queue.load_state(5, 5, lat2, kv)
    # empty queue at step 3 with 3 chunks pushed: chunks 0..2 are still queued
    with pytest.raises(DPError, match="INVALID_ARG"):
        queue.load_state(3, 3, np.zeros((0,) + shape, np.float32))
    # chunk 2 would be at level 0: it has already left
    with pytest.raises(DPError, match="INVALID_ARG"):
        queue.load_state(6, 6, np.zeros((4,) + shape, np.float32), kv)
    assert queue.inspect() == before
    # reachable: step 5, chunks 2..4 at levels 1..3, chunk 5 due (open)
    queue.load_state(5, 5, np.zeros((3,) + shape, np.float32), kv)
    info = queue.inspect()
    assert info["ids"] == [2, 3, 4, 5] and info["levels"] == [1, 2, 3, 4] and info["next_push_id"] == 5
    # past the last push: chunk 4 alone at level 1 at step 7 -> closed, drains in one step
    queue.load_state(7, 5, np.zeros((1,) + shape, np.float32), kv)
    info = queue.inspect()
    assert info["ids"] == [4] and info["levels"] == [1] and info["next_push_id"] == -1
    queue.step(None)
    assert queue.try_step(None) == 6          # DP_ERR_DRAINED
    queue.sync()
    model.close()


def test_host_pop_reports_a_kernel_that_gave_up_a_wait():
    """After a kernel on the queue's stream gives up a bounded wait (the self
    test: an mbarrier nothing completes, 2 s), the next host pop returns
    DP_ERR_KERNEL (the chunk is consumed); the status word is then clear and the
    next pop returns DP_OK with a chunk that matches the oracle."""
    w = synth.WORKLOADS["tiny_fp32"]
    m, q = w.model, w.queue
    T, N = 1, 3
    model, queue, p, text = make(w, "fp32", n_chunks=N, T=T, ready=2)
    noise = [synth.make_noise(m, q, k) for k in range(N)]
    queue.step(noise[0])
    queue.step(noise[1])                      # chunks 0 and 1 ready
    queue.selftest_timeout()
    out = np.empty(q.chunk_shape(m), np.float32)
    st, cid = queue.try_pop(out)
    assert st == 8 and cid == 0               # DP_ERR_KERNEL
    st, cid = queue.try_pop(out)
    assert st == 0 and cid == 1
    fn = dit.make_velocity_fn(p, text, m, T)
    ready, _ = fifo.run_stream(fn, lambda k: noise[k], T, N)
    assert rel_l2(out, dict(ready)[1]) <= 1e-4
    queue.sync()
    model.close()


def test_errors_full_empty_drained():
    w = synth.WORKLOADS["tiny_fp32"]
    model, queue, _, _ = make(w, "fp32", n_chunks=-1, T=2, ready=1)
    out = np.empty(w.queue.chunk_shape(w.model), np.float32)
    st, _ = queue.try_pop(out)
    assert st == 4  # DP_ERR_EMPTY
    queue.step(None)                      # chunk 0 at level 2
    queue.step(None)                      # chunk 0 level 1 -> ready
    assert queue.inspect()["n_ready"] == 1
    queue.step(None)                      # uses the last free slot (T + 1 = 3 slots)
    assert queue.try_step(None) == 5      # DP_ERR_FULL: chunk 0 and 1 wait for pop
    assert queue.pop(out) == 0
    queue.step(None)
    queue.close_stream()
    while queue.try_step(None) == 0:
        pass
    ids = []
    while True:
        st, cid = queue.try_pop(out)
        if st != 0:
            break
        ids.append(cid)
    assert ids == sorted(ids) and ids[0] == 1
    assert queue.try_step(None) == 6
    model.close()


def test_internal_generator_matches_seeded_noise():
    """NULL noise draws chunk k from the same SplitMix64/Box-Muller stream as
    the host generator.  With the output layer at zero the step leaves it as is."""
    w = synth.WORKLOADS["tiny_fp32"]
    m, q = w.model, w.queue
    p = synth.make_params(m)
    p["out.w"] = np.zeros_like(p["out.w"])
    p["out.b"] = np.zeros_like(p["out.b"])
    model, queue, _, _ = make(w, "fp32", params=p)
    queue.step(None)
    queue.step(None)
    lat = queue.read_latents(2)
    for k in range(2):
        ref = synth.make_noise(m, q, k)
        assert np.allclose(lat[k], ref, rtol=1e-6, atol=1e-6)
    model.close()


def test_coordinated_noise_pushes_the_oracle_frames():
    """noise_mode 1: each pushed chunk is the oracle's selection and order of
    the pool frames (bit-exact with the pool uploaded); the default pool is the
    seeded N(0,1) frames of the device generator."""
    from chunked_fifo_denoising_b200 import Model, Queue
    from oracle import noise
    w = synth.WORKLOADS["tiny_fp32"]
    m, q = w.model, w.queue
    p = synth.make_params(m)
    p["out.w"] = np.zeros_like(p["out.w"])   # zero velocity: the latents stay as pushed
    p["out.b"] = np.zeros_like(p["out.b"])
    model = Model(m, "fp32")
    model.set_params(p)
    text = synth.make_text(m)
    pool = synth.make_noise_pool(m, q).astype(np.float32)
    qa = Queue(model, text, 6, q.frames_per_chunk, q.lat_h, q.lat_w, 6, seed=5, noise="coordinated")
    qa.set_noise_pool(pool)
    for k in range(5):
        qa.step(None)
        lat = qa.read_latents(k + 1)
        assert np.array_equal(lat[-1], noise.coordinated_noise(pool, k, 5).astype(np.float32)), k
    qb = Queue(model, text, 6, q.frames_per_chunk, q.lat_h, q.lat_w, 6, seed=3, noise="coordinated")
    qb.step(None)
    got = qb.read_latents(1)[0]
    ref = noise.coordinated_noise(synth.make_noise_pool(m, q, seed=3), 0, 3)
    assert np.allclose(got, ref, rtol=1e-6, atol=1e-6)
    model.close()


def test_device_memory_flat_in_stream_length():
    """Long-stream workload (Wan-1.3B shapes, all 30 layers, zero weights):
    device memory after init is the same for 32, 64 and 128 chunks and the
    steps allocate nothing."""
    from chunked_fifo_denoising_b200 import Model, Queue
    w = synth.WORKLOADS["wan1.3b_480p_long"]
    m, q = w.model, w.queue
    model = Model(m, "bf16")
    for name, shape, per_layer in synth.param_specs(m):
        t = torch.zeros(shape, device="cuda")
        model.set_params({name: [t] * m.n_layers if per_layer else t})
    text = torch.zeros((m.text_len, m.text_in_dim), device="cuda")
    # the driver loads each kernel's module at its first launch: load them all
    # with a throwaway queue before measuring
    warm = Queue(model, text, q.T, q.frames_per_chunk, q.lat_h, q.lat_w, 4)
    for _ in range(3):
        warm.step(None)
    warm.sync()
    warm.close()
    torch.cuda.synchronize()
    used = []
    for n in (32, 64, 128):
        free0 = torch.cuda.mem_get_info()[0]
        queue = Queue(model, text, q.T, q.frames_per_chunk, q.lat_h, q.lat_w, n)
        free1 = torch.cuda.mem_get_info()[0]
        for _ in range(3):
            queue.step(None)
        queue.sync()
        free2 = torch.cuda.mem_get_info()[0]
        print(f"N = {n}: queue device bytes {free0 - free1}, allocated by 3 steps {free1 - free2}")
        assert free2 == free1
        used.append(free0 - free1)
        queue.close()
    print(f"queue device bytes at N = 32, 64, 128: {used}")
    assert used[0] == used[1] == used[2]
    model.close()
