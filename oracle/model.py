"""Vectorised numpy oracle of the FlashHead Lite DiT and its 4-step sampler.

TEST INFRASTRUCTURE ONLY (see the package docstring).

What the pages fix, and where:
  * gizai:flashhead (gizstack API reference), opening paragraph: the picture's
    reference latent is 5 frames of 16 x 16; each slice's audio becomes 5 latent
    frames of 32 audio tokens; a Wan-style transformer of 30 blocks of width 1536
    with 12 heads and rotary embeddings over frame, row and column predicts, in 4
    steps, the flow of the noisy latent, whose first latent frames carry the motion
    of the previous slice.
  * gizai:flashhead, Types > FlashHead: ``patch`` and ``head`` are Linear layers;
    ``headMods`` holds, at each step, the output norm's shift and scale [2, 1536];
    ``cos``/``sin`` are [1280, 768] with pair d of head h at column h*64 + d.
  * SoulX-FlashHead (audio-cpp model doc), Generate / Variant boundaries: 4
    inference steps; distilled Lite checkpoints use a re-noising update, non
    distilled ones Euler. The benchmark contract fixes Euler (reading R12).
  * The configurations define widths, FFN 8960 tanh-GELU, the 44/42/42 rotary
    split with theta 1e4, six adaLN vectors, per-frame cross-attention to 32
    audio tokens, output RMSNorm, patch Linear 256 -> 1536, head 1536 -> 128,
    bf16 weights/activations with fp32 accumulation, and the sampler sigmas.

Readings where the pages are silent (the same readings bind the CUDA library):
  R1  block: Wan order (shift, scale, gate) x (self-attn, FFN); h = LN(x)(1+scale)+shift
      with a non-affine LayerNorm; gated residuals.
  R2  eps 1e-6 for every LayerNorm/RMSNorm; LayerNorm uses the biased variance.
  R3  rotary pairs are adjacent dims (2d, 2d+1); pairs 0-21 rotate with the frame
      index, 22-42 with the row, 43-63 with the column; within an axis of n dims,
      pair j turns at theta^(-2j/n) rad per position; positions start at 0 and the
      motion frames count; every head uses the same table.
  R4  Q/K RMSNorm runs over the full width D with a learned gain of length D,
      before the head split.
  R5  self-attention is non-causal over all L tokens; cross-attention lets a token
      of latent frame f attend to that frame's 32 audio tokens only.
  R6  attention scale 1/sqrt(head_dim); softmax in float64 here.
  R7  the norm before cross-attention is a LayerNorm with learned affine, no modulation.
  R8  the cross-attention residual is ungated.
  R9  output norm: RMSNorm without gain, then (1 + scale) + shift (headMods).
  R10 timestep: tau = 1000 t; 256-dim sinusoid [cos(tau w_k) | sin(tau w_k)],
      w_k = 10000^(-k/128); e = Linear(SiLU(Linear(sinusoid))); e0 = Linear(SiLU(e))
      gives 6 x D; block mods = table_k + e0; head mods = head table + e.
  R11 every Linear has a bias.
  R12 sampler update is Euler x += (sigma' - sigma) v (the benchmark contract). The
      re-noising update the audio-cpp doc names for distilled checkpoints, which it does
      not define, is read as x0 = x - sigma v, then x = (1 - sigma') x0 + sigma' eps with
      a fresh N(0, 1) draw eps per step (``renoise_update``, ``sample_slice_renoise``).
  R14 frames 0-1 are overwritten with the motion latent before every network call
      and once more on the output.
  R15 the initial state at sigma = 1 is the noise for frames 2-4.
  R16 patch input channels: the noisy latent's 128 first, then the reference's 128.
  R19-R21 the audio projection (``audio_projection``): which encoder states each latent
      frame reads, and proj1 / proj1vf / proj2 / proj3 / projNorm as a ReLU MLP and a
      LayerNorm; stated where the functions are defined.

Precision modes (``prec``):
  'f64'  everything in float64 (used by the pins against the brute force);
  'f32'  float32 storage and matmuls, norms/softmax accumulated in float64 (the
         fp32 block configuration);
  'bf16' as 'f32', and every matmul/attention operand that the bf16
         configurations declare bf16 (activations entering a Linear, q/k/v, the
         audio tokens; weights are bf16 values already) is rounded to bf16 first.

Parity status: every function here is pinned by tests/test_oracle_pins.py
(closed forms, invariants, the float64 brute force of ``brute``). With no trained
weights or published outputs, agreement with the real checkpoint is unpinned.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

import synth_inputs as si


@dataclass(frozen=True)
class Config:
    dim: int = 1536
    heads: int = 12
    head_dim: int = 128
    ffn: int = 8960
    blocks: int = 30
    latent_ch: int = 128
    frames: int = 5
    lat_h: int = 16
    lat_w: int = 16
    audio_tokens: int = 32
    bf16: bool = True
    rope_theta: float = 1e4
    rope_split: tuple = (44, 42, 42)
    eps: float = 1e-6
    time_freq_dim: int = 256

    @property
    def tokens(self) -> int:
        return self.frames * self.lat_h * self.lat_w


# The five benchmark configurations (widths, counts and precision as stated).
CFG0 = Config(dim=384, heads=3, ffn=1024, blocks=1, frames=2, lat_h=8, lat_w=8, bf16=False)
CFG1 = Config(blocks=1)
CFG2 = Config()
CFG3 = Config()
CFG4 = Config(lat_h=24, lat_w=24)

BLOCK_SLOTS = [
    # (slot, name, shape(cfg), kind, fan_in(cfg))
    (0, "mod", lambda c: (6, c.dim), "mod", lambda c: c.dim),
    (1, "wq", lambda c: (c.dim, c.dim), "lin", lambda c: c.dim),
    (2, "bq", lambda c: (c.dim,), "lin", lambda c: c.dim),
    (3, "wk", lambda c: (c.dim, c.dim), "lin", lambda c: c.dim),
    (4, "bk", lambda c: (c.dim,), "lin", lambda c: c.dim),
    (5, "wv", lambda c: (c.dim, c.dim), "lin", lambda c: c.dim),
    (6, "bv", lambda c: (c.dim,), "lin", lambda c: c.dim),
    (7, "wo", lambda c: (c.dim, c.dim), "lin", lambda c: c.dim),
    (8, "bo", lambda c: (c.dim,), "lin", lambda c: c.dim),
    (9, "gq", lambda c: (c.dim,), "gain", lambda c: c.dim),
    (10, "gk", lambda c: (c.dim,), "gain", lambda c: c.dim),
    (11, "ln3_w", lambda c: (c.dim,), "gain", lambda c: c.dim),
    (12, "ln3_b", lambda c: (c.dim,), "lnb", lambda c: c.dim),
    (13, "wcq", lambda c: (c.dim, c.dim), "lin", lambda c: c.dim),
    (14, "bcq", lambda c: (c.dim,), "lin", lambda c: c.dim),
    (15, "wck", lambda c: (c.dim, c.dim), "lin", lambda c: c.dim),
    (16, "bck", lambda c: (c.dim,), "lin", lambda c: c.dim),
    (17, "wcv", lambda c: (c.dim, c.dim), "lin", lambda c: c.dim),
    (18, "bcv", lambda c: (c.dim,), "lin", lambda c: c.dim),
    (19, "wco", lambda c: (c.dim, c.dim), "lin", lambda c: c.dim),
    (20, "bco", lambda c: (c.dim,), "lin", lambda c: c.dim),
    (21, "gcq", lambda c: (c.dim,), "gain", lambda c: c.dim),
    (22, "gck", lambda c: (c.dim,), "gain", lambda c: c.dim),
    (23, "w1", lambda c: (c.ffn, c.dim), "lin", lambda c: c.dim),
    (24, "b1", lambda c: (c.ffn,), "lin", lambda c: c.dim),
    (25, "w2", lambda c: (c.dim, c.ffn), "lin", lambda c: c.ffn),
    (26, "b2", lambda c: (c.dim,), "lin", lambda c: c.ffn),
]

GLOBAL_SLOTS = [
    (0, "patch_w", lambda c: (c.dim, 2 * c.latent_ch), "lin", lambda c: 2 * c.latent_ch),
    (1, "patch_b", lambda c: (c.dim,), "lin", lambda c: 2 * c.latent_ch),
    (2, "head_w", lambda c: (c.latent_ch, c.dim), "lin", lambda c: c.dim),
    (3, "head_b", lambda c: (c.latent_ch,), "lin", lambda c: c.dim),
    (4, "head_mod", lambda c: (2, c.dim), "mod", lambda c: c.dim),
    (5, "t_w1", lambda c: (c.dim, c.time_freq_dim), "lin", lambda c: c.time_freq_dim),
    (6, "t_b1", lambda c: (c.dim,), "lin", lambda c: c.time_freq_dim),
    (7, "t_w2", lambda c: (c.dim, c.dim), "lin", lambda c: c.dim),
    (8, "t_b2", lambda c: (c.dim,), "lin", lambda c: c.dim),
    (9, "t_wp", lambda c: (6 * c.dim, c.dim), "lin", lambda c: c.dim),
    (10, "t_bp", lambda c: (6 * c.dim,), "lin", lambda c: c.dim),
]


def block_tid(k: int, slot: int) -> int:
    return si.BLOCK_STRIDE * k + slot


def global_tid(slot: int) -> int:
    return si.GLOBAL_BASE + slot


@dataclass
class Weights:
    cfg: Config
    blocks: list = field(default_factory=list)   # list of dict name -> float32 array
    glob: dict = field(default_factory=dict)


def make_weights(cfg: Config, seed: int, blocks=None) -> Weights:
    """Regenerate the synthetic weights from the seeded generator (bf16-rounded for bf16 configs)."""
    W = Weights(cfg)
    ks = range(cfg.blocks) if blocks is None else blocks
    for k in range(cfg.blocks):
        if k not in ks:
            W.blocks.append(None)
            continue
        d = {}
        for slot, name, shp, kind, fan in BLOCK_SLOTS:
            d[name] = si.weight_value(seed, block_tid(k, slot), shp(cfg), kind, fan(cfg), cfg.dim, cfg.bf16)
        W.blocks.append(d)
    for slot, name, shp, kind, fan in GLOBAL_SLOTS:
        W.glob[name] = si.weight_value(seed, global_tid(slot), shp(cfg), kind, fan(cfg), cfg.dim, cfg.bf16)
    return W


def param_count(cfg: Config) -> int:
    n = 0
    for _, _, shp, _, _ in BLOCK_SLOTS:
        n += int(np.prod(shp(cfg)))
    n *= cfg.blocks
    for _, _, shp, _, _ in GLOBAL_SLOTS:
        n += int(np.prod(shp(cfg)))
    return n


# ---------------------------------------------------------------------------
# elementary operations
# ---------------------------------------------------------------------------
def _dt(prec):
    return np.float64 if prec == "f64" else np.float32


def _operand(x, prec):
    """A matmul/attention operand in the precision the mode declares."""
    x = np.asarray(x, dtype=_dt(prec))
    return si.to_bf16(x) if prec == "bf16" else x


def linear(x, w, b, prec):
    """y = x W^T + b, operands in the mode's precision, accumulation float32/float64."""
    dt = _dt(prec)
    return (_operand(x, prec) @ np.asarray(w, dtype=dt).T + np.asarray(b, dtype=dt)).astype(dt)


def layer_norm(x, eps):
    """Non-affine LayerNorm over the last axis, biased variance (R2), float64 statistics."""
    x64 = np.asarray(x, dtype=np.float64)
    mu = x64.mean(axis=-1, keepdims=True)
    var = ((x64 - mu) ** 2).mean(axis=-1, keepdims=True)
    return (x64 - mu) / np.sqrt(var + eps)


def rms_norm(x, eps):
    """RMSNorm without gain over the last axis, float64 statistics."""
    x64 = np.asarray(x, dtype=np.float64)
    return x64 / np.sqrt((x64 * x64).mean(axis=-1, keepdims=True) + eps)


def silu(x):
    return x / (1.0 + np.exp(-x))


def gelu_tanh(x):
    """tanh approximation of GELU (the FFN activation the configurations name)."""
    x64 = np.asarray(x, dtype=np.float64)
    return 0.5 * x64 * (1.0 + np.tanh(math.sqrt(2.0 / math.pi) * (x64 + 0.044715 * x64 ** 3)))


def softmax(s, axis=-1):
    s64 = np.asarray(s, dtype=np.float64)
    m = s64.max(axis=axis, keepdims=True)
    p = np.exp(s64 - m)
    return p / p.sum(axis=axis, keepdims=True)


# ---------------------------------------------------------------------------
# timestep conditioning (R10) and rotary tables (R3)
# ---------------------------------------------------------------------------
def timestep_sinusoid(t, dim=256):
    """[cos(tau w_k) | sin(tau w_k)], tau = 1000 t, w_k = 10000^(-k/(dim/2))."""
    t = np.atleast_1d(np.asarray(t, dtype=np.float64))
    half = dim // 2
    w = 10000.0 ** (-np.arange(half, dtype=np.float64) / half)
    ang = (1000.0 * t)[:, None] * w[None, :]
    return np.concatenate([np.cos(ang), np.sin(ang)], axis=1)


def time_conditioning(W: Weights, t, prec):
    """Per-stream conditioning: e [B, D] and e0 [B, 6, D] for timesteps t [B].

    The conditioning MLP keeps float32 activations in the bf16 mode as well (its
    weights are bf16 values); only the token path's operands are bf16.
    """
    g = W.glob
    prec = "f32" if prec == "bf16" else prec
    dt = _dt(prec)
    sin = timestep_sinusoid(t, W.cfg.time_freq_dim).astype(dt)
    hid = silu(linear(sin, g["t_w1"], g["t_b1"], prec).astype(np.float64)).astype(dt)
    e = linear(hid, g["t_w2"], g["t_b2"], prec)
    e0 = linear(silu(e.astype(np.float64)).astype(dt), g["t_wp"], g["t_bp"], prec)
    return e.astype(np.float64), e0.astype(np.float64).reshape(-1, 6, W.cfg.dim)


def rope_angles(cfg: Config):
    """Rotation angle of every (token, pair) [L, head_dim/2], float64 (R3)."""
    nf, nh, nw = cfg.rope_split
    pf, ph, pw = nf // 2, nh // 2, nw // 2
    assert pf + ph + pw == cfg.head_dim // 2
    f = np.arange(cfg.frames)
    h = np.arange(cfg.lat_h)
    w = np.arange(cfg.lat_w)
    F, Hh, Ww = np.meshgrid(f, h, w, indexing="ij")
    pos = [F.reshape(-1), Hh.reshape(-1), Ww.reshape(-1)]
    cols = []
    for axis, (npairs, ndim) in enumerate(((pf, nf), (ph, nh), (pw, nw))):
        freq = cfg.rope_theta ** (-2.0 * np.arange(npairs, dtype=np.float64) / ndim)
        cols.append(pos[axis][:, None].astype(np.float64) * freq[None, :])
    return np.concatenate(cols, axis=1)


def apply_rope(x, ang):
    """Rotate adjacent pairs (2d, 2d+1) of x [..., L, NH, hd] by ang [L, hd/2]."""
    c = np.cos(ang)[:, None, :]
    s = np.sin(ang)[:, None, :]
    x0 = x[..., 0::2]
    x1 = x[..., 1::2]
    out = np.empty_like(x)
    out[..., 0::2] = x0 * c - x1 * s
    out[..., 1::2] = x0 * s + x1 * c
    return out


# ---------------------------------------------------------------------------
# the transformer block
# ---------------------------------------------------------------------------
def self_attention(q, k, v, scale):
    """Non-causal softmax attention per (stream, head). q,k,v [B, L, NH, hd] -> [B, L, NH, hd]."""
    B, L, NH, hd = q.shape
    out = np.empty((B, L, NH, hd), dtype=np.float64)
    for b in range(B):
        for h in range(NH):
            s = (q[b, :, h, :].astype(np.float64) @ k[b, :, h, :].astype(np.float64).T) * scale
            out[b, :, h, :] = softmax(s) @ v[b, :, h, :].astype(np.float64)
    return out


def frame_cross_attention(q, k, v, frames, scale):
    """Token of latent frame f attends to frame f's audio tokens only (R5).

    q [B, L, NH, hd]; k, v [B, F, A, NH, hd] -> [B, L, NH, hd].
    """
    B, L, NH, hd = q.shape
    per = L // frames
    qf = q.reshape(B, frames, per, NH, hd).astype(np.float64)
    s = np.einsum("bfinh,bfanh->bfnia", qf, k.astype(np.float64)) * scale
    p = softmax(s, axis=-1)
    o = np.einsum("bfnia,bfanh->bfinh", p, v.astype(np.float64))
    return o.reshape(B, L, NH, hd)


def cross_kv(W: Weights, k: int, audio, prec):
    """Cross-attention keys (RMS-normalised with gain, R4) and values of block k."""
    cfg = W.cfg
    p = W.blocks[k]
    B, F, A, D = audio.shape
    a = audio.reshape(B, F * A, D)
    kc = rms_norm(linear(a, p["wck"], p["bck"], prec), cfg.eps) * p["gck"].astype(np.float64)
    vc = linear(a, p["wcv"], p["bcv"], prec).astype(np.float64)
    shp = (B, F, A, cfg.heads, cfg.head_dim)
    return kc.reshape(shp), vc.reshape(shp)


def block_forward(W: Weights, k: int, x, audio, e0, prec, ang=None, kv=None):
    """One DiT block. x [B, L, D] residual stream; audio [B, F, A, D]; e0 [B, 6, D].

    Follows: adaLN self-attention with 3D rotary (R1-R6), LayerNorm-affine
    cross-attention to the frame's audio tokens (R7, R8), adaLN tanh-GELU FFN.
    """
    cfg = W.cfg
    p = W.blocks[k]
    dt = _dt(prec)
    B, L, D = x.shape
    NH, hd = cfg.heads, cfg.head_dim
    if ang is None:
        ang = rope_angles(cfg)
    mods = p["mod"].astype(np.float64)[None] + e0                      # [B, 6, D]
    sh1, sc1, g1, sh2, sc2, g2 = (mods[:, i, None, :] for i in range(6))
    scale = 1.0 / math.sqrt(hd)
    x = np.asarray(x, dtype=np.float64)

    # self-attention branch
    h = (layer_norm(x, cfg.eps) * (1.0 + sc1) + sh1).astype(dt)
    q = linear(h, p["wq"], p["bq"], prec)
    kk = linear(h, p["wk"], p["bk"], prec)
    v = linear(h, p["wv"], p["bv"], prec)
    q = rms_norm(q, cfg.eps) * p["gq"].astype(np.float64)
    kk = rms_norm(kk, cfg.eps) * p["gk"].astype(np.float64)
    q = apply_rope(q.reshape(B, L, NH, hd), ang)
    kk = apply_rope(kk.reshape(B, L, NH, hd), ang)
    v = v.astype(np.float64).reshape(B, L, NH, hd)
    o = self_attention(_operand(q, prec), _operand(kk, prec), _operand(v, prec), scale)
    y = linear(o.reshape(B, L, D).astype(dt), p["wo"], p["bo"], prec)
    x = x + g1 * y

    # audio cross-attention branch
    hc = layer_norm(x, cfg.eps) * p["ln3_w"].astype(np.float64) + p["ln3_b"].astype(np.float64)
    qc = rms_norm(linear(hc.astype(dt), p["wcq"], p["bcq"], prec), cfg.eps) * p["gcq"].astype(np.float64)
    if kv is None:
        kv = cross_kv(W, k, audio, prec)
    kc, vc = kv
    oc = frame_cross_attention(_operand(qc.reshape(B, L, NH, hd), prec), _operand(kc, prec),
                               _operand(vc, prec), cfg.frames, scale)
    x = x + linear(oc.reshape(B, L, D).astype(dt), p["wco"], p["bco"], prec)

    # FFN branch
    h2 = (layer_norm(x, cfg.eps) * (1.0 + sc2) + sh2).astype(dt)
    u = gelu_tanh(linear(h2, p["w1"], p["b1"], prec)).astype(dt)
    x = x + g2 * linear(u, p["w2"], p["b2"], prec)
    return x.astype(dt)


# ---------------------------------------------------------------------------
# flow prediction and sampler
# ---------------------------------------------------------------------------
def patchify(lat):
    """[B, C, F, H, W] -> token-major [B, L, C], token n = f*H*W + h*W + w."""
    B, C, F, H, Wd = lat.shape
    return lat.reshape(B, C, F * H * Wd).transpose(0, 2, 1)


def unpatchify(tok, cfg: Config):
    B, L, C = tok.shape
    return tok.transpose(0, 2, 1).reshape(B, C, cfg.frames, cfg.lat_h, cfg.lat_w)


def patch_embed(W: Weights, x_noisy, ref, prec):
    """Residual stream entering block 0: the patch Linear (gizai:flashhead, Types > FlashHead,
    ``patch``) over each token's channels, the noisy latent's first, then the reference's (R16)."""
    dt = _dt(prec)
    tok = np.concatenate([patchify(x_noisy), patchify(ref)], axis=2)
    return linear(tok.astype(dt), W.glob["patch_w"], W.glob["patch_b"], prec)


def head_mods(W: Weights, e):
    """Per-stream (shift, scale) of the output norm, [B, 2, D]: the head's modulation table
    plus the conditioning vector e (reading R10; ``headMods``, gizai:flashhead, Types > FlashHead)."""
    return W.glob["head_mod"].astype(np.float64)[None] + e[:, None, :]


def output_head(W: Weights, x, hm, prec):
    """Velocity tokens [B, L, C]: RMSNorm without gain, then (1 + scale) + shift (R9), then the
    head Linear (gizai:flashhead, Types > FlashHead, ``head``)."""
    cfg = W.cfg
    dt = _dt(prec)
    shift, scl = hm[:, 0, None, :], hm[:, 1, None, :]
    hn = (rms_norm(x, cfg.eps) * (1.0 + scl) + shift).astype(dt)
    return linear(hn, W.glob["head_w"], W.glob["head_b"], prec)


def predict_flow(W: Weights, x_noisy, ref, audio, sigma, prec, kvs=None, ang=None):
    """v = head(RMSNorm(blocks(patch([x_noisy | ref]))) ...) for one sigma; [B, C, F, H, W]."""
    cfg = W.cfg
    dt = _dt(prec)
    B = x_noisy.shape[0]
    if ang is None:
        ang = rope_angles(cfg)
    x = patch_embed(W, x_noisy, ref, prec)
    e, e0 = time_conditioning(W, np.full((B,), sigma, dtype=np.float64), prec)
    for k in range(cfg.blocks):
        kv = None if kvs is None else kvs[k]
        x = block_forward(W, k, x, audio, e0, prec, ang=ang, kv=kv)
    v = output_head(W, x, head_mods(W, e), prec)
    return unpatchify(v, cfg).astype(dt)


def pin_motion(x, motion):
    """Overwrite latent frames 0..1 with the motion latent (R14)."""
    x = x.copy()
    x[:, :, 0:motion.shape[2]] = motion
    return x


def sample_slice(W: Weights, noise, ref, motion, audio, sigmas, prec):
    """Euler flow sampling of one slice over the given sigmas (R12, R14, R15)."""
    dt = _dt(prec)
    kvs = [cross_kv(W, k, audio, prec) for k in range(W.cfg.blocks)]
    ang = rope_angles(W.cfg)
    x = np.asarray(noise, dtype=dt)
    for s in range(len(sigmas) - 1):
        x = pin_motion(x, motion)
        v = predict_flow(W, x, ref, audio, sigmas[s], prec, kvs=kvs, ang=ang)
        x = (x + np.asarray(sigmas[s + 1] - sigmas[s], dtype=dt) * v).astype(dt)
    return pin_motion(x, motion)


def renoise_update(x, v, sigma, sigma_next, eps):
    """One re-noising step (reading R12 of the update that SoulX-FlashHead (audio-cpp model
    doc), Generate / Variant boundaries, names for distilled checkpoints): the flow's clean
    estimate x0 = x - sigma v is put back on the noise path at sigma_next with fresh noise,
    x' = (1 - sigma_next) x0 + sigma_next eps. At sigma_next = 0 it is the Euler step."""
    dt = x.dtype
    x0 = (x - np.asarray(sigma, dtype=dt) * v).astype(dt)
    return (np.asarray(1.0 - sigma_next, dtype=dt) * x0 + np.asarray(sigma_next, dtype=dt) * eps).astype(dt)


def sample_slice_renoise(W: Weights, noise, ref, motion, audio, sigmas, eps, prec):
    """The slice sampler with the re-noising update (R12, R14, R15); eps [steps, B, C, F, H, W]
    holds the fresh draw of each step (its frames 0..1 are overwritten by the motion pin)."""
    dt = _dt(prec)
    kvs = [cross_kv(W, k, audio, prec) for k in range(W.cfg.blocks)]
    ang = rope_angles(W.cfg)
    x = np.asarray(noise, dtype=dt)
    for s in range(len(sigmas) - 1):
        x = pin_motion(x, motion)
        v = predict_flow(W, x, ref, audio, sigmas[s], prec, kvs=kvs, ang=ang)
        x = renoise_update(x, v, sigmas[s], sigmas[s + 1], np.asarray(eps[s], dtype=dt))
    return pin_motion(x, motion)


# ---------------------------------------------------------------------------
# audio projection: speech-encoder states -> the latent frames' audio tokens
# ---------------------------------------------------------------------------
# gizai:flashhead, opening paragraph: for each slice the last 8 s of speech go through
# wav2vec 2.0 base, its 12 layers' states taken at 200 frames, and 5 states around each of
# the slice's 33 frames make 5 latent frames of 32 audio tokens; Types > FlashHead lists the
# projection as proj1, proj1vf, proj2, proj3 (Linear layers) and projNorm (tensors).
# Readings (the pages give no widths or formulas):
#   R19 the slice's video frames are the last of the 200 states: video frame t (of 33)
#       sits at state 200 - 33 + t; its 5 states are that one and two either side,
#       indices clamped to [0, 199].
#   R20 33 = 1 + 4 x 8 (the video VAE's temporal stride 8): latent frame 0 is video frame 0
#       alone; latent frame j >= 1 is video frames 8j - 7 .. 8j, whose 5-state windows
#       together span 12 consecutive states.
#   R21 latent frame 0: a = relu(proj1(its 5 states x 12 layers x 768, state-major));
#       later frames: a = relu(proj1vf(their 12 states x 12 x 768)); then
#       b = relu(proj2(a)), 32 tokens of width D from proj3(b), and projNorm a LayerNorm
#       with learned affine (weight, bias) over each token, eps as R2. Hidden width 512.
@dataclass(frozen=True)
class AudioConfig:
    states: int = 200       # encoder frames in the 8 s window
    layers: int = 12
    channels: int = 768
    window: int = 5         # states around each video frame
    stride: int = 8         # video frames per latent frame after the first
    hidden: int = 512
    tokens: int = 32

    def video_frames(self, latent_frames: int) -> int:
        return 1 + self.stride * (latent_frames - 1)

    def group_states(self) -> int:
        return self.stride + self.window - 1


AUDIO = AudioConfig()

AUDIO_SLOTS = [
    (0, "proj1_w", lambda c, a: (a.hidden, a.window * a.layers * a.channels), "lin",
     lambda c, a: a.window * a.layers * a.channels),
    (1, "proj1_b", lambda c, a: (a.hidden,), "lin", lambda c, a: a.window * a.layers * a.channels),
    (2, "proj1vf_w", lambda c, a: (a.hidden, a.group_states() * a.layers * a.channels), "lin",
     lambda c, a: a.group_states() * a.layers * a.channels),
    (3, "proj1vf_b", lambda c, a: (a.hidden,), "lin", lambda c, a: a.group_states() * a.layers * a.channels),
    (4, "proj2_w", lambda c, a: (a.hidden, a.hidden), "lin", lambda c, a: a.hidden),
    (5, "proj2_b", lambda c, a: (a.hidden,), "lin", lambda c, a: a.hidden),
    (6, "proj3_w", lambda c, a: (a.tokens * c.dim, a.hidden), "lin", lambda c, a: a.hidden),
    (7, "proj3_b", lambda c, a: (a.tokens * c.dim,), "lin", lambda c, a: a.hidden),
    (8, "projnorm_w", lambda c, a: (c.dim,), "gain", lambda c, a: c.dim),
    (9, "projnorm_b", lambda c, a: (c.dim,), "lnb", lambda c, a: c.dim),
]
AUDIO_BASE = 32   # audio projection tensors: tid = GLOBAL_BASE + AUDIO_BASE + slot


def make_audio_weights(cfg: Config, seed: int, a: AudioConfig = AUDIO) -> dict:
    """The audio projection's synthetic weights (bf16-rounded matrices for bf16 configs)."""
    return {name: si.weight_value(seed, global_tid(AUDIO_BASE + slot), shp(cfg, a), kind, fan(cfg, a), cfg.dim,
                                  cfg.bf16)
            for slot, name, shp, kind, fan in AUDIO_SLOTS}


def audio_windows(states, latent_frames: int, a: AudioConfig = AUDIO):
    """(first [B, window, layers, channels], later [B, F-1, group_states, layers, channels]):
    the states each latent frame's projection reads (R19, R20)."""
    nv = a.video_frames(latent_frames)
    s0 = a.states - nv                       # state of video frame 0
    half = a.window // 2
    idx0 = np.clip(np.arange(s0 - half, s0 + half + 1), 0, a.states - 1)
    first = states[:, idx0]
    later = []
    for j in range(1, latent_frames):
        lo = s0 + a.stride * j - (a.stride - 1) - half
        idx = np.clip(np.arange(lo, lo + a.group_states()), 0, a.states - 1)
        later.append(states[:, idx])
    return first, np.stack(later, axis=1)


def audio_projection(AW: dict, states, cfg: Config, prec, a: AudioConfig = AUDIO):
    """Audio tokens [B, F, tokens, D] from the speech-encoder states [B, states, layers,
    channels] (R19-R21). The projection's activations stay float32 in the bf16 mode too (its
    weights are bf16 values); the tokens it returns are what the blocks' cross-attention reads."""
    prec = "f32" if prec == "bf16" else prec
    dt = _dt(prec)
    B = states.shape[0]
    F = cfg.frames
    first, later = audio_windows(np.asarray(states, dtype=dt), F, a)
    h0 = linear(first.reshape(B, -1), AW["proj1_w"], AW["proj1_b"], prec)              # [B, hidden]
    hv = linear(later.reshape(B * (F - 1), -1), AW["proj1vf_w"], AW["proj1vf_b"], prec)
    h = np.concatenate([h0[:, None], hv.reshape(B, F - 1, -1)], axis=1)                # [B, F, hidden]
    h = np.maximum(h, 0).astype(dt)
    h = np.maximum(linear(h.reshape(B * F, -1), AW["proj2_w"], AW["proj2_b"], prec), 0).astype(dt)
    t = linear(h, AW["proj3_w"], AW["proj3_b"], prec).reshape(B, F, a.tokens, cfg.dim)
    y = layer_norm(t, cfg.eps) * AW["projnorm_w"].astype(np.float64) + AW["projnorm_b"].astype(np.float64)
    return y.astype(dt)
