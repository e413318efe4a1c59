"""Oracle DiT velocity for a batch of queued chunks (float64, numpy).

Test infrastructure only (see the package docstring).  Every function takes
and returns float64 arrays; parameters arrive as the float32 arrays made by
``synth.make_params`` and are widened once.

Page cited throughout: "双重并行：让AI视频生成突破时长限制，新加坡国立大学团队实现
分钟级长视频创作" (techwalker.com), abbreviated "DualParal write-up".
"""
from __future__ import annotations

import math

import numpy as np
from scipy.special import erf

LN_EPS = 1e-6


# ---------------------------------------------------------------------------
# Elementwise pieces
# ---------------------------------------------------------------------------

def silu(x):
    """x * sigmoid(x)."""
    return x / (1.0 + np.exp(-x))


def gelu(x):
    """GELU, exact erf form: x * Phi(x), Phi the standard normal CDF.

    reading: the write-up names an FFN but not its activation; the exact erf
    form (Hendrycks and Gimpel, 2016) is taken, the tanh approximation being
    the alternative.
    """
    return 0.5 * x * (1.0 + erf(x / math.sqrt(2.0)))


def layer_norm(x, eps=LN_EPS):
    """Normalise each row over its last axis: (x - mean) / sqrt(var + eps).

    reading: no affine weight (adaLN supplies scale and shift), biased
    variance, eps = 1e-6.
    """
    mu = x.mean(axis=-1, keepdims=True)
    var = ((x - mu) ** 2).mean(axis=-1, keepdims=True)
    return (x - mu) / np.sqrt(var + eps)


def modulate(h, shift, scale):
    """adaLN: h * (1 + scale) + shift, per-chunk vectors broadcast over rows."""
    return h * (1.0 + scale) + shift


def linear(x, w, b):
    """x @ w^T + b with w stored [out][in]."""
    return x @ np.asarray(w, np.float64).T + np.asarray(b, np.float64)


# ---------------------------------------------------------------------------
# Timestep embedding and per-level modulation
# ---------------------------------------------------------------------------

def sigma(j, T):
    """Noise level of queue level j: sigma_j = j / T (linear schedule).

    DualParal write-up §二: levels run from T at the tail down to 1 at the
    head; a chunk at level 0 is clean.  The linear sigma_j = j/T is the
    schedule of the workload definition.
    """
    return j / T


def sinusoid(t, D):
    """[cos(t w_i), sin(t w_i)], w_i = 10000^(-i/(D/2)), i = 0 .. D/2-1.

    reading: the pages give no timestep embedding; the standard sinusoidal
    embedding of the DiT family is taken.
    """
    half = D // 2
    i = np.arange(half, dtype=np.float64)
    w = np.power(10000.0, -i / half)
    return np.concatenate([np.cos(t * w), np.sin(t * w)])


def level_embedding(j, T, p, D):
    """e_j = W_t2 SiLU(W_t1 sinusoid(t_j) + b_t1) + b_t2 with t_j = 1000 sigma_j.

    reading: timesteps scaled by 1000 so that the sinusoid separates levels.
    """
    e0 = sinusoid(1000.0 * sigma(j, T), D)
    h = silu(linear(e0, p["time1.w"], p["time1.b"]))
    return linear(h, p["time2.w"], p["time2.b"])


def level_modulation(j, T, p, D):
    """Per-level modulation m_j = W_mod SiLU(e_j) + b_mod (6d) and the head's
    (shift_o, scale_o) = W_hm SiLU(e_j) + b_hm (2d).

    DualParal write-up §一: every chunk carries its own noise level, so the
    modulation is a per-chunk quantity.  reading: one 6d projection shared by
    the layers, plus a per-layer 6d table added to it.
    """
    s = silu(level_embedding(j, T, p, D))
    m = linear(s, p["mod.w"], p["mod.b"])
    hm = linear(s, p["headmod.w"], p["headmod.b"])
    return m, hm


def split_mod(m, d):
    """(shift_a, scale_a, gate_a, shift_f, scale_f, gate_f), each of length d."""
    return [m[i * d:(i + 1) * d] for i in range(6)]


# ---------------------------------------------------------------------------
# Patches
# ---------------------------------------------------------------------------

def patchify(lat, pt, ph, pw):
    """Latent chunk [C][F][H][W] -> tokens [(F/pt)(H/ph)(W/pw)][C pt ph pw].

    Token order is (frame, row, column) row-major; inside a patch the feature
    index is ((c pt + dt) ph + dy) pw + dx.  reading: the 1x2x2 patch size is
    the workload's; the index order is this library's convention.
    """
    C, F, H, W = lat.shape
    x = lat.reshape(C, F // pt, pt, H // ph, ph, W // pw, pw)
    # -> (F', H', W', C, pt, ph, pw)
    x = x.transpose(1, 3, 5, 0, 2, 4, 6)
    return x.reshape((F // pt) * (H // ph) * (W // pw), C * pt * ph * pw)


def unpatchify(tok, C, F, H, W, pt, ph, pw):
    """Inverse of ``patchify``."""
    x = tok.reshape(F // pt, H // ph, W // pw, C, pt, ph, pw)
    x = x.transpose(3, 0, 4, 1, 5, 2, 6)
    return x.reshape(C, F, H, W)


# ---------------------------------------------------------------------------
# Attention
# ---------------------------------------------------------------------------

def softmax_rows(s):
    """Row softmax; subtracts the row maximum first."""
    s = s - s.max(axis=-1, keepdims=True)
    e = np.exp(s)
    return e / e.sum(axis=-1, keepdims=True)


def attention(q, k, v, n_heads):
    """Multi-head scaled dot-product attention, softmax(q k^T / sqrt(hd)) v.

    q [Lq][d], k and v [Lk][d]; head h uses columns h*hd .. (h+1)*hd-1.
    """
    Lq, d = q.shape
    hd = d // n_heads
    out = np.empty((Lq, d), dtype=np.float64)
    scale = 1.0 / math.sqrt(hd)
    for h in range(n_heads):
        c = slice(h * hd, (h + 1) * hd)
        p = softmax_rows((q[:, c] @ k[:, c].T) * scale)
        out[:, c] = p @ v[:, c]
    return out


def self_attention_with_neighbours(q, k, v, k_pred, v_pred, k_succ, v_succ, n_heads):
    """Self-attention of a chunk over its predecessor's, its own and its
    successor's K/V in one joint softmax (the key set written out as the
    concatenation).  Either neighbour may be None.

    DualParal write-up §三: processing chunk B_i with both neighbours,
    [B_{i-1}, B_i, B_{i+1}], is the starting point; the neighbours enter only
    through self-attention.  This is the bidirectional reading of the
    neighbourhood (the predecessor-only reading is the default).
    """
    ks, vs = [], []
    if k_pred is not None:
        ks.append(k_pred)
        vs.append(v_pred)
    ks.append(k)
    vs.append(v)
    if k_succ is not None:
        ks.append(k_succ)
        vs.append(v_succ)
    return attention(q, np.concatenate(ks), np.concatenate(vs), n_heads)


def self_attention_with_predecessor(q, k, v, k_pred, v_pred, n_heads):
    """A chunk's self-attention: its queries see its own keys plus the K/V of
    the chunk before it, in one joint softmax.

    DualParal write-up §三 (feature cache): the neighbour's self-attention K/V
    are reused instead of concatenating the neighbour's input; only
    self-attention needs the neighbour.  The key set is the union of the two
    buffers, written out here as their concatenation (the plain definition).
    ``k_pred``/``v_pred`` are None for the first chunk of the video.
    """
    if k_pred is None:
        return attention(q, k, v, n_heads)
    return attention(q, np.concatenate([k_pred, k]), np.concatenate([v_pred, v]), n_heads)


# ---------------------------------------------------------------------------
# Per-head QK RMSNorm and 3-D rotary positions (optional block variant)
# ---------------------------------------------------------------------------

RMS_EPS = 1e-6


def rms_norm_heads(x, w, n_heads, eps=RMS_EPS):
    """Each head's slice of every row divided by its root mean square, then
    scaled per channel by w (length d).

    reading: the write-up names Wan2.1's DiT without its block; this variant
    normalises q and k per head (over head_dim) with a learned weight.
    """
    L, d = x.shape
    hd = d // n_heads
    xh = x.reshape(L, n_heads, hd)
    r = np.sqrt((xh ** 2).mean(axis=-1, keepdims=True) + eps)
    return (xh / r).reshape(L, d) * np.asarray(w, np.float64)


def rope_bands(hd):
    """Pairs per axis (temporal, height, width) of a head of hd channels:
    h = w = floor(hd / 6), t = hd / 2 - 2 h."""
    nh = (hd // 2) // 3
    return hd // 2 - 2 * nh, nh, nh


def rope_angles(pos_t, pos_y, pos_x, hd, base=10000.0):
    """Rotation angle of every pair of a head for each token.

    reading: rotary embedding (Su et al., 2021) on interleaved pairs
    (x_{2i}, x_{2i+1}); the hd/2 pairs are split into a temporal, a height and
    a width band; pair l of a band of n pairs turns by pos * base^(-l / n).
    Positions are absolute: the temporal one is chunk id * frames per chunk +
    frame, so a chunk and its persisted neighbour keep their offset.
    """
    nt, nh, nw = rope_bands(hd)
    cols = []
    for pos, n in ((pos_t, nt), (pos_y, nh), (pos_x, nw)):
        theta = np.power(base, -np.arange(n, dtype=np.float64) / n)
        cols.append(np.outer(np.asarray(pos, np.float64), theta))
    return np.concatenate(cols, axis=1)   # [tokens][hd/2]


def apply_rope(x, angles, n_heads):
    """Rotates every pair (x_{2i}, x_{2i+1}) of every head by angles[:, i]."""
    L, d = x.shape
    hd = d // n_heads
    xh = x.reshape(L, n_heads, hd // 2, 2)
    c = np.cos(angles)[:, None, :]
    s = np.sin(angles)[:, None, :]
    a, b = xh[..., 0], xh[..., 1]
    out = np.stack([a * c - b * s, a * s + b * c], axis=-1)
    return out.reshape(L, d)


def token_positions(chunk_id, F, H, W, pt, ph, pw):
    """(t, y, x) of every token of a chunk, in patchify order."""
    Fq, Hq, Wq = F // pt, H // ph, W // pw
    f, y, x = np.meshgrid(np.arange(Fq), np.arange(Hq), np.arange(Wq), indexing="ij")
    return (chunk_id * Fq + f).ravel(), y.ravel(), x.ravel()


# ---------------------------------------------------------------------------
# Text
# ---------------------------------------------------------------------------

def text_kv(text, p, n_layers):
    """Per-layer cross-attention K/V of the prompt, computed once.

    reading: a single Linear projects the text features to the model width
    when their width differs; each layer then has its own K and V projection.
    """
    t = np.asarray(text, np.float64)
    if "text.w" in p:
        t = linear(t, p["text.w"], p["text.b"])
    kv = []
    for l in range(n_layers):
        kv.append((linear(t, p["layer.ck.w"][l], p["layer.ck.b"][l]),
                   linear(t, p["layer.cv.w"][l], p["layer.cv.b"][l])))
    return kv


# ---------------------------------------------------------------------------
# The batched velocity of one queue step
# ---------------------------------------------------------------------------

def velocity(latents, levels, chunk_ids, pred_kv, p, tkv, shape, T, use_pred=True,
             keep_kv_of=None, neighbours="pred"):
    """Model output v for every queued chunk of one step.

    latents   list of [C][F][H][W] arrays, one per queued chunk, ordered by
              chunk id (consecutive ids).
    levels    queue level j of each chunk (1..T).
    pred_kv   None, or a list over layers of (K, V) [L_c][d]: the persisted
              self-attention K/V of the chunk just before the first queued one.
    tkv       ``text_kv`` output.
    shape     synth.ModelShape.
    use_pred  False disables the neighbour links entirely.
    keep_kv_of  index into the batch whose per-layer (K, V) are returned.
    neighbours  "pred" (the predecessor only) or "both" (also the successor
              k+1, read from this pass when it is queued; the chunk pushed last
              has none).

    Returns (v list, kept kv list-or-None).

    DualParal write-up §一/§二: all queued chunks are denoised in the same
    step, each with its own noise level.  §三: only self-attention looks at
    the neighbour; cross-attention and the FFN are per chunk.

    reading (the main ambiguity): the neighbour is the temporally preceding
    chunk k-1 (one place nearer the head, one level cleaner).  Its K/V at
    layer l are the ones computed in this same step from its own layer-l
    input; when k-1 already left the queue, they are the values it produced at
    level 1 in the previous step; chunk 0 has no neighbour.  No RoPE and no
    QK-norm (neither is on the pages).  Cross-attention has no gate and no
    modulation.
    """
    m = shape
    d, H = m.dim, m.n_heads
    n = len(latents)
    for i in range(1, n):
        assert chunk_ids[i] == chunk_ids[i - 1] + 1
    C, F, Hh, W = latents[0].shape
    x = [linear(patchify(np.asarray(l, np.float64), m.patch_t, m.patch_h, m.patch_w),
                p["patch.w"], p["patch.b"]) for l in latents]
    rope = getattr(m, "qk_norm_rope", False)
    if rope:
        ang = [rope_angles(*token_positions(k, F, Hh, W, m.patch_t, m.patch_h, m.patch_w), d // H)
               for k in chunk_ids]
    mods = [level_modulation(j, T, p, m.freq_dim) for j in levels]
    kept = [] if keep_kv_of is not None else None
    for l in range(m.n_layers):
        tab = np.asarray(p["layer.mod"][l], np.float64)
        q, k, v = [], [], []
        for i in range(n):
            sh_a, sc_a, g_a, sh_f, sc_f, g_f = split_mod(mods[i][0] + tab, d)
            h = modulate(layer_norm(x[i]), sh_a, sc_a)
            qkv = linear(h, p["layer.qkv.w"][l], p["layer.qkv.b"][l])
            qi, ki = qkv[:, :d], qkv[:, d:2 * d]
            if rope:
                qi = apply_rope(rms_norm_heads(qi, p["layer.qnorm.w"][l], H), ang[i], H)
                ki = apply_rope(rms_norm_heads(ki, p["layer.knorm.w"][l], H), ang[i], H)
            q.append(qi)
            k.append(ki)
            v.append(qkv[:, 2 * d:])
        if kept is not None:
            kept.append((k[keep_kv_of].copy(), v[keep_kv_of].copy()))
        for i in range(n):
            sh_a, sc_a, g_a, sh_f, sc_f, g_f = split_mod(mods[i][0] + tab, d)
            if not use_pred:
                kp = vp = None
            elif i > 0:
                kp, vp = k[i - 1], v[i - 1]
            elif pred_kv is not None:
                kp, vp = (np.asarray(a, np.float64) for a in pred_kv[l])
            else:
                kp = vp = None
            ksu = vsu = None
            if use_pred and neighbours == "both" and i + 1 < n:
                ksu, vsu = k[i + 1], v[i + 1]
            o = self_attention_with_neighbours(q[i], k[i], v[i], kp, vp, ksu, vsu, H)
            x[i] = x[i] + g_a * linear(o, p["layer.o.w"][l], p["layer.o.b"][l])
            # cross-attention to the prompt (no modulation, no gate)
            h = layer_norm(x[i])
            qc = linear(h, p["layer.cq.w"][l], p["layer.cq.b"][l])
            oc = attention(qc, tkv[l][0], tkv[l][1], H)
            x[i] = x[i] + linear(oc, p["layer.co.w"][l], p["layer.co.b"][l])
            # FFN
            h = modulate(layer_norm(x[i]), sh_f, sc_f)
            u = gelu(linear(h, p["layer.ffn1.w"][l], p["layer.ffn1.b"][l]))
            x[i] = x[i] + g_f * linear(u, p["layer.ffn2.w"][l], p["layer.ffn2.b"][l])
    vs = []
    for i in range(n):
        sh_o, sc_o = mods[i][1][:d], mods[i][1][d:]
        h = modulate(layer_norm(x[i]), sh_o, sc_o)
        tok = linear(h, p["out.w"], p["out.b"])
        vs.append(unpatchify(tok, C, F, Hh, W, m.patch_t, m.patch_h, m.patch_w))
    return vs, kept


def make_velocity_fn(p, text, shape, T, use_pred=True, neighbours="pred"):
    """Binds parameters and the prompt into the callable the queue expects."""
    tkv = text_kv(text, p, shape.n_layers)

    def fn(latents, levels, chunk_ids, pred_kv, keep_kv_of):
        return velocity(latents, levels, chunk_ids, pred_kv, p, tkv, shape, T,
                        use_pred=use_pred, keep_kv_of=keep_kv_of, neighbours=neighbours)
    return fn
