"""Pins of the oracle's composition functions against hand-derived values:
the per-level timestep embedding and modulation, the prompt's per-layer K/V,
and the whole DiT velocity on a case small enough to follow by calculator.

Every expected value comes from a derivation written out in the fixture under
tests/golden/ (selector weights, closed forms, a textbook normal probability),
never from a call to the oracle.  The last test plants plausible mistakes in
the oracle (on the CPU) and checks that these pins then fail.

Method: the DualParal write-up ("双重并行：让AI视频生成突破时长限制…",
techwalker.com), section 一 (each chunk at its own noise level) and section 三
(only self-attention reads the neighbour; cross-attention and FFN are per chunk).
"""
import numpy as np
import pytest

import synth
from oracle import dit
from tests.conftest import read_golden

# ---------------------------------------------------------------------------
# per-level timestep embedding and modulation
# ---------------------------------------------------------------------------


def level_params():
    """Selector weights of tests/golden/level_modulation_d2.txt (d = 2, D = 2)."""
    mod_w = np.zeros((12, 2))
    for i in range(12):
        mod_w[i, i % 2] = 0.1 * (i + 1)
    return {
        "time1.w": np.array([[2.0, 0.0], [0.0, 1.0]]), "time1.b": np.array([0.0, 0.5]),
        "time2.w": np.array([[0.0, 1.0], [1.0, 0.0]]), "time2.b": np.array([0.25, 0.0]),
        "mod.w": mod_w, "mod.b": np.arange(12.0),
        "headmod.w": np.array([[1.0, 0.0], [0.0, 1.0], [1.0, 1.0], [0.0, 0.0]]),
        "headmod.b": np.array([0.0, 0.0, 0.0, 7.0]),
    }


def level_golden():
    out = {}
    for ln in read_golden("level_modulation_d2.txt"):
        kind, j, T, *vals = ln.split()
        out[(kind, int(j), int(T))] = np.array([float(v) for v in vals])
    return out


def test_level_embedding_hand_values():
    """t_j = 1000 j / T, sinusoid [cos, sin], SiLU between the two layers of
    the time MLP, both biases."""
    g, p = level_golden(), level_params()
    for j, T in ((4, 4), (2, 4)):
        assert np.allclose(dit.level_embedding(j, T, p, 2), g[("embed", j, T)], rtol=1e-13, atol=1e-15)


def test_level_modulation_hand_values():
    """SiLU of the embedding before the 6d and 2d projections, biases added."""
    g, p = level_golden(), level_params()
    for j, T in ((4, 4), (2, 4)):
        m, hm = dit.level_modulation(j, T, p, 2)
        assert m.shape == (12,) and hm.shape == (4,)
        assert np.allclose(m, g[("mod", j, T)], rtol=1e-13, atol=1e-15)
        assert np.allclose(hm, g[("headmod", j, T)], rtol=1e-13, atol=1e-15)


def test_split_mod_order():
    """The 6d vector splits in the order shift_a, scale_a, gate_a, shift_f,
    scale_f, gate_f, each d wide."""
    parts = dit.split_mod(np.arange(18.0), 3)
    assert [list(x) for x in parts] == [[0, 1, 2], [3, 4, 5], [6, 7, 8], [9, 10, 11],
                                        [12, 13, 14], [15, 16, 17]]


# ---------------------------------------------------------------------------
# the prompt's per-layer K/V
# ---------------------------------------------------------------------------

def text_params():
    rev = np.eye(4)[::-1].copy()
    return {
        "text.w": np.array([[1.0, 0, 0], [0, 1, 0], [0, 0, 1], [1, 1, 1]]),
        "text.b": np.array([0.5, 0.0, 0.0, -1.0]),
        "layer.ck.w": [np.eye(4), rev], "layer.ck.b": [np.zeros(4), np.array([10.0, 20, 30, 40])],
        "layer.cv.w": [2 * np.eye(4), np.zeros((4, 4))],
        "layer.cv.b": [np.ones(4), np.array([-1.0, -2, -3, -4])],
    }


def test_text_kv_hand_values():
    """The projection to the model width comes first, then each layer's own K
    and V projections (K first, V second)."""
    want = {}
    for ln in read_golden("text_kv_d4.txt"):
        l, kind, tok, *vals = ln.split()
        want[(int(l), kind, int(tok))] = [float(v) for v in vals]
    kv = dit.text_kv(np.array([[1.0, 2, 3], [4, 5, 6]]), text_params(), 2)
    assert len(kv) == 2
    for l in range(2):
        for i, kind in enumerate("KV"):
            for tok in range(2):
                assert np.array_equal(kv[l][i][tok], want[(l, kind, tok)]), (l, kind, tok)


def test_text_kv_without_projection_uses_the_prompt_directly():
    p = text_params()
    del p["text.w"], p["text.b"]
    t = np.array([[1.0, 2, 3, 4]])
    kv = dit.text_kv(t, p, 2)
    assert np.array_equal(kv[0][0], t) and np.array_equal(kv[0][1], 2 * t + 1)


# ---------------------------------------------------------------------------
# the composed velocity
# ---------------------------------------------------------------------------

SHAPE = synth.ModelShape(n_layers=1, dim=4, n_heads=1, ffn_dim=4, freq_dim=2, text_len=1,
                         text_in_dim=4, latent_ch=4, patch_t=1, patch_h=1, patch_w=1)


def velocity_params():
    """Weights of tests/golden/velocity_d4_two_chunks.txt."""
    d = 4
    z = lambda *s: np.zeros(s)  # noqa: E731
    target = np.concatenate([
        [0, 0, 0.5, 0], [1, 0, 0, 0], [0, 0, 0.5, 0.5],       # shift_a, scale_a, gate_a
        [0, 0, 1, -1], [0, 0, -1, -1], [2, 2, 0.5, 0.5]])     # shift_f, scale_f, gate_f
    table = np.full(6 * d, 0.25)
    qkv_w = z(3 * d, d)
    qkv_w[d:2 * d] = 1.0                                      # W_k: all ones
    qkv_w[2 * d + 2] = [1, 0, 1, 0]                           # v2 = h0 + h2
    qkv_w[2 * d + 3] = [-1, 0, -1, 0]                         # v3 = -(h0 + h2)
    qkv_b = z(3 * d)
    qkv_b[d:2 * d] = 5.0
    ck_w = z(d, d)
    ck_w[:, 0] = 3.0
    cv_w = z(d, d)
    cv_w[:, 0] = [0.5, -0.5, 0, 0]
    ffn2_w = np.array([[1.0, -1, 0, 0], [-1, 1, 0, 0], [0, 0, 1, 1], [0, 0, -1, -1]])
    return {
        "patch.w": np.eye(d), "patch.b": z(d),
        "time1.w": z(d, 2), "time1.b": z(d), "time2.w": z(d, d), "time2.b": z(d),
        "mod.w": z(6 * d, d), "mod.b": target - table,
        "headmod.w": z(2 * d, d), "headmod.b": np.array([0, 0, 0, 0.1, 1, 0, 0, 0]),
        "out.w": np.eye(d), "out.b": np.array([0, 0, 0.01, 0]),
        "layer.mod": [table],
        "layer.qkv.w": [qkv_w], "layer.qkv.b": [qkv_b],
        "layer.o.w": [np.eye(d)], "layer.o.b": [z(d)],
        "layer.cq.w": [np.ones((d, d))], "layer.cq.b": [z(d)],
        "layer.ck.w": [ck_w], "layer.ck.b": [z(d)],
        "layer.cv.w": [cv_w], "layer.cv.b": [z(d)],
        "layer.co.w": [np.eye(d)], "layer.co.b": [np.array([0.25, -0.25, 0, 0])],
        "layer.ffn1.w": [np.eye(d)], "layer.ffn1.b": [z(d)],
        "layer.ffn2.w": [ffn2_w], "layer.ffn2.b": [z(d)],
    }


def velocity_case(p=None, use_pred=True):
    p = velocity_params() if p is None else p
    fn = dit.make_velocity_fn(p, np.array([[1.0, 0, 0, 0]]), SHAPE, T=4, use_pred=use_pred)
    lat = [np.array([1.0, -1, 0, 0]).reshape(4, 1, 1, 1), np.array([0.0, 0, 1, -1]).reshape(4, 1, 1, 1)]
    vs, _ = fn(lat, [1, 2], [0, 1], None, None)
    return [v.reshape(4) for v in vs]


def velocity_golden():
    rows = [ln.split() for ln in read_golden("velocity_d4_two_chunks.txt")]
    return [np.array([float(v) for v in r[1:]]) for r in sorted(rows, key=lambda r: int(r[0]))]


def velocity_matches(vs):
    return all(np.allclose(v, w, rtol=1e-12, atol=1e-13) for v, w in zip(vs, velocity_golden()))


def test_velocity_hand_values():
    """The whole block on two chunks: adaLN split and modulate, gated and
    ungated residuals, block order, the prompt's V, the predecessor link and
    the head modulation, against the derivation in the fixture."""
    assert velocity_matches(velocity_case())




# ---------------------------------------------------------------------------
# planted mistakes: each one must break at least one pin above
# ---------------------------------------------------------------------------

def _pins_hold():
    g, lp = level_golden(), level_params()
    ok = True
    for j, T in ((4, 4), (2, 4)):
        ok &= bool(np.allclose(dit.level_embedding(j, T, lp, 2), g[("embed", j, T)], rtol=1e-13))
        m, hm = dit.level_modulation(j, T, lp, 2)
        ok &= bool(np.allclose(m, g[("mod", j, T)], rtol=1e-13))
        ok &= bool(np.allclose(hm, g[("headmod", j, T)], rtol=1e-13))
    return ok and velocity_matches(velocity_case())


def _swap(order):
    def split(m, d):
        parts = [m[i * d:(i + 1) * d] for i in range(6)]
        return [parts[i] for i in order]
    return split


PLANTS = {
    "shift and scale swapped in modulate": ("modulate", lambda h, shift, scale: h * (1.0 + shift) + scale),
    "shift_a and scale_a swapped": ("split_mod", _swap([1, 0, 2, 3, 4, 5])),
    "gate_a and gate_f swapped": ("split_mod", _swap([0, 1, 5, 3, 4, 2])),
    "attention and FFN modulation swapped": ("split_mod", _swap([3, 4, 2, 0, 1, 5])),
    "no SiLU": ("silu", lambda x: x),
    "timestep not scaled by 1000": ("sinusoid", None),
    "tanh GELU": ("gelu", lambda x: 0.5 * x * (1 + np.tanh(np.sqrt(2 / np.pi) * (x + 0.044715 * x ** 3)))),
    "LayerNorm eps inside the square root dropped": ("LN_EPS", 0.0),
}


@pytest.mark.parametrize("name", sorted(PLANTS))
def test_pins_catch_planted_mistakes(name, monkeypatch):
    assert _pins_hold()
    attr, repl = PLANTS[name]
    if attr == "sinusoid":
        orig = dit.sinusoid
        repl = lambda t, D: orig(t / 1000.0, D)  # noqa: E731
    if attr == "LN_EPS":
        orig_ln = dit.layer_norm
        monkeypatch.setattr(dit, "layer_norm", lambda x, eps=dit.LN_EPS: orig_ln(x, eps=repl))
    else:
        monkeypatch.setattr(dit, attr, repl)
    assert not _pins_hold(), name


def test_velocity_pin_sees_the_predecessor_link():
    """With the neighbour link off, chunk 1 no longer averages chunk 0's value
    into its attention output, and the pin fails for chunk 1 only."""
    vs = velocity_case(use_pred=False)
    want = velocity_golden()
    assert np.allclose(vs[0], want[0], rtol=1e-12)
    assert not np.allclose(vs[1], want[1], rtol=1e-6)
