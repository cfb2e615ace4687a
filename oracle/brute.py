"""float64 per-token brute force of one FlashHead DiT block (small sizes only).

TEST INFRASTRUCTURE ONLY. Written apart from ``oracle.model`` to pin it: every
token is handled on its own with scalar loops and ``math`` functions; the rotary
embedding is a complex multiplication by exp(i * angle) with the angle derived
per pair from the axis split; softmax is an explicit max/exp/sum. Only
matrix-vector products use numpy (``W @ v``), as a library primitive.

Same readings (R1-R16) as ``oracle.model``; see that module's docstring.
"""
from __future__ import annotations

import cmath
import math

import numpy as np


def _layer_norm(v, eps):
    n = len(v)
    mu = math.fsum(v) / n
    var = math.fsum((a - mu) * (a - mu) for a in v) / n
    inv = 1.0 / math.sqrt(var + eps)
    return np.array([(a - mu) * inv for a in v])


def _rms(v, eps):
    n = len(v)
    ms = math.fsum(a * a for a in v) / n
    return np.array(v) / math.sqrt(ms + eps)


def _silu(a):
    return a / (1.0 + math.exp(-a))


def _gelu_tanh(a):
    return 0.5 * a * (1.0 + math.tanh(math.sqrt(2.0 / math.pi) * (a + 0.044715 * a * a * a)))


def _matvec(w, b, v):
    return np.asarray(w, dtype=np.float64) @ np.asarray(v, dtype=np.float64) + np.asarray(b, dtype=np.float64)


def _conditioning(W, t):
    cfg = W.cfg
    g = W.glob
    half = cfg.time_freq_dim // 2
    tau = 1000.0 * t
    sinus = [math.cos(tau * 10000.0 ** (-k / half)) for k in range(half)]
    sinus += [math.sin(tau * 10000.0 ** (-k / half)) for k in range(half)]
    hid = [_silu(a) for a in _matvec(g["t_w1"], g["t_b1"], sinus)]
    e = _matvec(g["t_w2"], g["t_b2"], hid)
    e0 = _matvec(g["t_wp"], g["t_bp"], [_silu(a) for a in e])
    return e, e0.reshape(6, cfg.dim)


def _pair_angle(cfg, n, d):
    """Angle of rotary pair d for token n, from the frame/row/column split."""
    hw = cfg.lat_h * cfg.lat_w
    f, r, c = n // hw, (n % hw) // cfg.lat_w, n % cfg.lat_w
    nf, nh, nw = cfg.rope_split
    if d < nf // 2:
        pos, j, ndim = f, d, nf
    elif d < nf // 2 + nh // 2:
        pos, j, ndim = r, d - nf // 2, nh
    else:
        pos, j, ndim = c, d - nf // 2 - nh // 2, nw
    return pos * cfg.rope_theta ** (-2.0 * j / ndim)


def _rotate(cfg, v, n):
    out = np.empty_like(v)
    hd = cfg.head_dim
    for h in range(cfg.heads):
        for d in range(hd // 2):
            i0 = h * hd + 2 * d
            z = complex(v[i0], v[i0 + 1]) * cmath.exp(1j * _pair_angle(cfg, n, d))
            out[i0], out[i0 + 1] = z.real, z.imag
    return out


def _attend(q, keys, values, hd):
    """softmax(q.k/sqrt(hd)) weighted sum of values, one head, explicit loops."""
    s = [float(np.dot(q, kj)) / math.sqrt(hd) for kj in keys]
    m = max(s)
    p = [math.exp(a - m) for a in s]
    z = math.fsum(p)
    out = np.zeros(hd)
    for pj, vj in zip(p, values):
        out += (pj / z) * np.asarray(vj)
    return out


def block_tokens(W, k, x, audio, t, tokens):
    """Block output rows ``tokens`` for a single stream. x [L, D], audio [F, A, D], t scalar."""
    cfg = W.cfg
    p = W.blocks[k]
    L, D = x.shape
    NH, hd = cfg.heads, cfg.head_dim
    eps = cfg.eps
    _, e0 = _conditioning(W, t)
    mods = np.asarray(p["mod"], dtype=np.float64) + e0
    sh1, sc1, g1, sh2, sc2, g2 = mods
    x = np.asarray(x, dtype=np.float64)

    # keys and values of every token, query of every token
    Q, K, V = [], [], []
    for n in range(L):
        h = _layer_norm(list(x[n]), eps) * (1.0 + sc1) + sh1
        q = _rms(list(_matvec(p["wq"], p["bq"], h)), eps) * p["gq"]
        kk = _rms(list(_matvec(p["wk"], p["bk"], h)), eps) * p["gk"]
        Q.append(_rotate(cfg, q, n))
        K.append(_rotate(cfg, kk, n))
        V.append(_matvec(p["wv"], p["bv"], h))

    # audio keys/values per frame
    F, A, _ = audio.shape
    AK, AV = [], []
    for f in range(F):
        ks, vs = [], []
        for a in range(A):
            ks.append(_rms(list(_matvec(p["wck"], p["bck"], audio[f, a])), eps) * p["gck"])
            vs.append(_matvec(p["wcv"], p["bcv"], audio[f, a]))
        AK.append(ks)
        AV.append(vs)

    out = []
    hw = cfg.lat_h * cfg.lat_w
    for i in tokens:
        o = np.zeros(D)
        for h in range(NH):
            sl = slice(h * hd, (h + 1) * hd)
            o[sl] = _attend(Q[i][sl], [kj[sl] for kj in K], [vj[sl] for vj in V], hd)
        xi = x[i] + g1 * _matvec(p["wo"], p["bo"], o)
        hc = _layer_norm(list(xi), eps) * p["ln3_w"] + p["ln3_b"]
        qc = _rms(list(_matvec(p["wcq"], p["bcq"], hc)), eps) * p["gcq"]
        f = i // hw
        oc = np.zeros(D)
        for h in range(NH):
            sl = slice(h * hd, (h + 1) * hd)
            oc[sl] = _attend(qc[sl], [kj[sl] for kj in AK[f]], [vj[sl] for vj in AV[f]], hd)
        xi = xi + _matvec(p["wco"], p["bco"], oc)
        h2 = _layer_norm(list(xi), eps) * (1.0 + sc2) + sh2
        u = [_gelu_tanh(a) for a in _matvec(p["w1"], p["b1"], h2)]
        xi = xi + g2 * _matvec(p["w2"], p["b2"], u)
        out.append(xi)
    return np.array(out)


def predict_flow(W, x_noisy, ref, audio, sigma):
    """Velocity [C, F, H, W] of one stream for one sigma, token by token in float64.

    x_noisy, ref [C, F, H, W]; audio [F, A, D]. The steps of a flow prediction as the
    gizai:flashhead page (opening paragraph; Types > FlashHead: ``patch``, ``head``,
    ``headMods``) and readings R9, R10, R16 give them, written without ``oracle.model``:
    each token's input is its noisy channels followed by its reference channels, mapped by
    the patch Linear; the blocks are ``block_tokens`` chained over every token; the output
    norm is an RMSNorm without gain followed by (1 + scale) and shift, where (shift, scale)
    are the head's table rows plus the conditioning vector e of this sigma; the head Linear
    gives the token's C velocity channels, written back to (channel, frame, row, column).
    """
    cfg = W.cfg
    g = W.glob
    C, F, H, Wd = x_noisy.shape
    eps = cfg.eps
    e, _ = _conditioning(W, sigma)
    shift = np.asarray(g["head_mod"][0], dtype=np.float64) + e
    scale = np.asarray(g["head_mod"][1], dtype=np.float64) + e
    coords = [(f, r, c) for f in range(F) for r in range(H) for c in range(Wd)]   # token n = f*H*W + r*W + c
    rows = []
    for (f, r, c) in coords:
        chans = [float(x_noisy[ch, f, r, c]) for ch in range(C)] + [float(ref[ch, f, r, c]) for ch in range(C)]
        rows.append(_matvec(g["patch_w"], g["patch_b"], chans))
    x = np.array(rows)
    L = len(coords)
    for k in range(cfg.blocks):
        x = block_tokens(W, k, x, audio, sigma, range(L))
    v = np.empty((C, F, H, Wd))
    for n, (f, r, c) in enumerate(coords):
        hn = [a * (1.0 + sc) + sh for a, sc, sh in zip(_rms(list(x[n]), eps), scale, shift)]
        vn = _matvec(g["head_w"], g["head_b"], hn)
        for ch in range(C):
            v[ch, f, r, c] = vn[ch]
    return v


def audio_tokens(AW, states, cfg, a):
    """Audio tokens [F, tokens, D] of one stream, in float64, frame by frame.

    states [S, layers, channels]. Written without ``oracle.model``: for latent frame j the
    video frames it covers are listed (frame 0 alone; frames 8j - 7 .. 8j after it), each
    video frame t contributes the states within two of its position S - nv + t, the union
    of those positions is taken in increasing order and each is clamped into [0, S - 1];
    the selected states, flattened state by state, go through proj1 (frame 0) or proj1vf,
    a ReLU, proj2, a ReLU and proj3, and each of the 32 tokens through a LayerNorm with
    projNorm's weight and bias.
    """
    S = states.shape[0]
    F = cfg.frames
    nv = 1 + a.stride * (F - 1)
    half = a.window // 2
    out = np.empty((F, a.tokens, cfg.dim))
    for j in range(F):
        frames = [0] if j == 0 else list(range(a.stride * j - a.stride + 1, a.stride * j + 1))
        pos = sorted({S - nv + t + d for t in frames for d in range(-half, half + 1)})
        vec = []
        for p in pos:
            p = min(max(p, 0), S - 1)
            vec.extend(float(v) for v in np.asarray(states[p], dtype=np.float64).reshape(-1))
        w, b = (AW["proj1_w"], AW["proj1_b"]) if j == 0 else (AW["proj1vf_w"], AW["proj1vf_b"])
        h = [max(0.0, v) for v in _matvec(w, b, vec)]
        h = [max(0.0, v) for v in _matvec(AW["proj2_w"], AW["proj2_b"], h)]
        t = _matvec(AW["proj3_w"], AW["proj3_b"], h)
        for n in range(a.tokens):
            tok = list(t[n * cfg.dim:(n + 1) * cfg.dim])
            ln = _layer_norm(tok, cfg.eps)
            out[j, n] = [v * g + c for v, g, c in zip(ln, AW["projnorm_w"], AW["projnorm_b"])]
    return out
