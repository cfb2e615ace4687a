"""Seeded synthetic inputs for the FlashHead Lite DiT hot path.

This module is the one piece of code that both the CPU oracle (``oracle/``) and
the GPU-side tests and benchmark import. It holds no arithmetic of the method:
only a counter-based random generator and the recipes that turn it into the
synthetic tensors (weights, latents, audio tokens, timesteps) the pages'
workloads stand in for. No trained weights or real audio are used.

Generator. SplitMix64 (Steele, Lea and Flood, "Fast splittable pseudorandom
number generators", OOPSLA 2014) is used as a hash of a 64-bit counter: the
counter is advanced by the golden-gamma constant and passed through the
variant-13 finaliser. For tensor ``tid`` under ``seed``, element ``i`` (row-major
flat index) draws the two counters ``base + 2i`` and ``base + 2i + 1`` with
``base = seed XOR (tid << 40)``. A 53-bit uniform is taken from the top bits of
each hash, ``u = (z >> 11) * 2**-53``. A normal value is one Box-Muller output,
``sqrt(-2 ln(1 - u1)) * cos(2 pi u2)``, in float64. A U(0,1) value is ``u1``.

The CUDA library implements the same generator independently (for its weights)
from the same published definition; the GPU tests compare the two.
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

MASK64 = (1 << 64) - 1
GOLDEN_GAMMA = np.uint64(0x9E3779B97F4A7C15)
_MIX1 = np.uint64(0xBF58476D1CE4E5B9)
_MIX2 = np.uint64(0x94D049BB133111EB)
_CHUNK = 1 << 20


def splitmix64(counter: np.ndarray) -> np.ndarray:
    """SplitMix64 output for each uint64 counter (wrapping arithmetic)."""
    with np.errstate(over="ignore"):
        z = counter + GOLDEN_GAMMA
        z = (z ^ (z >> np.uint64(30))) * _MIX1
        z = (z ^ (z >> np.uint64(27))) * _MIX2
        return z ^ (z >> np.uint64(31))


def _base(seed: int, tid: int) -> np.uint64:
    return np.uint64((int(seed) ^ (int(tid) << 40)) & MASK64)


def _uniform_pair(seed: int, tid: int, start: int, n: int):
    idx = np.arange(start, start + n, dtype=np.uint64)
    base = _base(seed, tid)
    with np.errstate(over="ignore"):
        c1 = base + np.uint64(2) * idx
        c2 = c1 + np.uint64(1)
    scale = 2.0 ** -53
    u1 = (splitmix64(c1) >> np.uint64(11)).astype(np.float64) * scale
    u2 = (splitmix64(c2) >> np.uint64(11)).astype(np.float64) * scale
    return u1, u2


_POOL = None


def _pool():
    global _POOL
    if _POOL is None:
        _POOL = ThreadPoolExecutor(max_workers=max(1, min(32, len(os.sched_getaffinity(0)))))
    return _POOL


def normal(seed: int, tid: int, shape) -> np.ndarray:
    """float64 N(0,1) tensor of ``shape`` for tensor id ``tid``."""
    n = int(np.prod(shape, dtype=np.int64))
    out = np.empty(n, dtype=np.float64)

    def fill(s):
        m = min(_CHUNK, n - s)
        u1, u2 = _uniform_pair(seed, tid, s, m)
        out[s:s + m] = np.sqrt(-2.0 * np.log1p(-u1)) * np.cos(2.0 * np.pi * u2)

    starts = range(0, n, _CHUNK)
    if n > _CHUNK:
        list(_pool().map(fill, starts))
    else:
        for s in starts:
            fill(s)
    return out.reshape(shape)


def uniform(seed: int, tid: int, shape) -> np.ndarray:
    """float64 U(0,1) tensor of ``shape`` for tensor id ``tid``."""
    n = int(np.prod(shape, dtype=np.int64))
    u1, _ = _uniform_pair(seed, tid, 0, n)
    return u1.reshape(shape)


def to_bf16(x: np.ndarray) -> np.ndarray:
    """Round to the nearest bfloat16 (ties to even); returned as float32 values."""
    f = np.ascontiguousarray(x, dtype=np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    u = (u + np.uint64(0x7FFF) + ((u >> np.uint64(16)) & np.uint64(1))) & np.uint64(0xFFFF0000)
    return u.astype(np.uint32).view(np.float32).reshape(f.shape)


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """uint16 bit patterns of float32 values that are already bf16-representable."""
    f = np.ascontiguousarray(x, dtype=np.float32)
    return (f.view(np.uint32) >> np.uint32(16)).astype(np.uint16)


# ---------------------------------------------------------------------------
# Weight tensors. Ids and init kinds are part of the library's public contract
# (declared in include/fh.h); each side builds its own table from it.
#   block k, slot s  ->  tid = 64*k + s          global slot g -> tid = 4096 + g
# init kinds: 'lin'  N(0,1)/sqrt(fan_in)   (matrices and their biases)
#             'mod'  N(0,1)/sqrt(dim)      (modulation tables)
#             'gain' 1 + 0.1 N(0,1)        (norm gains)
#             'lnb'  0.1 N(0,1)            (LayerNorm bias)
# ---------------------------------------------------------------------------
BLOCK_STRIDE = 64
GLOBAL_BASE = 4096


def weight_value(seed: int, tid: int, shape, kind: str, fan_in: int, dim: int,
                 bf16: bool) -> np.ndarray:
    """The synthetic value of one weight tensor as float32 (bf16-rounded when asked)."""
    z = normal(seed, tid, shape)
    if kind == "lin":
        w = z / np.sqrt(float(fan_in))
    elif kind == "mod":
        w = z / np.sqrt(float(dim))
    elif kind == "gain":
        w = 1.0 + 0.1 * z
    elif kind == "lnb":
        w = 0.1 * z
    else:
        raise ValueError(kind)
    w = w.astype(np.float32)
    return to_bf16(w) if bf16 else w


# ---------------------------------------------------------------------------
# Activation inputs. Input tensor ids live above every weight id.
# ---------------------------------------------------------------------------
IN_X = 1 << 20          # block input x [B, L, D]
IN_AUDIO = IN_X + 1     # audio tokens [B, F, A, D]
IN_T = IN_X + 2         # timestep t [B]
IN_NOISE = IN_X + 3     # initial noise [B, C, F, H, W]
IN_REF = IN_X + 4       # reference latent [B, C, F, H, W]
IN_MOTION = IN_X + 5    # motion latent [B, C, 2, H, W]
IN_LATENT = IN_X + 6    # noisy latent for one prediction [B, C, F, H, W]
IN_RENOISE = IN_X + 7   # fresh noise of the re-noising sampler, one draw per step [S, B, C, F, H, W]
IN_STATES = IN_X + 8    # speech-encoder states of the audio window [B, frames, layers, channels]


def config_seed(index: int) -> int:
    """Seed of the c-th benchmark configuration: 0 for the fp32 block, 1000 + c otherwise."""
    return 0 if index == 0 else 1000 + index


def block_inputs(seed: int, batch: int, tokens: int, dim: int, frames: int,
                 audio_tokens: int, bf16: bool):
    """x [B,L,D] f32, audio [B,F,A,D] (bf16-rounded f32 when bf16), t [B] f64 in (0,1)."""
    x = normal(seed, IN_X, (batch, tokens, dim)).astype(np.float32)
    a = normal(seed, IN_AUDIO, (batch, frames, audio_tokens, dim)).astype(np.float32)
    if bf16:
        a = to_bf16(a)
    t = uniform(seed, IN_T, (batch,))
    return x, a, t


def latent(seed: int, tid: int, batch: int, ch: int, frames: int, h: int, w: int) -> np.ndarray:
    return normal(seed, tid, (batch, ch, frames, h, w)).astype(np.float32)


def audio_tokens(seed: int, batch: int, frames: int, tokens: int, dim: int, bf16: bool) -> np.ndarray:
    a = normal(seed, IN_AUDIO, (batch, frames, tokens, dim)).astype(np.float32)
    return to_bf16(a) if bf16 else a


def renoise_draws(seed: int, steps: int, batch: int, ch: int, frames: int, h: int, w: int) -> np.ndarray:
    """The fresh N(0, 1) draws of a re-noising sampler slice, [steps, B, C, F, H, W] float32."""
    return normal(seed, IN_RENOISE, (steps, batch, ch, frames, h, w)).astype(np.float32)


def slice_inputs(seed: int, batch: int, ch: int, frames: int, h: int, w: int,
                 audio_tokens_per_frame: int, dim: int, bf16: bool, slice_index: int = 0):
    """Inputs of one sampler slice: noise, ref, motion fixed by ``seed``; audio seeded ``seed + slice``."""
    noise = latent(seed, IN_NOISE, batch, ch, frames, h, w)
    ref = latent(seed, IN_REF, batch, ch, frames, h, w)
    motion = latent(seed, IN_MOTION, batch, ch, 2, h, w)
    audio = audio_tokens(seed + slice_index, batch, frames, audio_tokens_per_frame, dim, bf16)
    return noise, ref, motion, audio


def speech_states(seed: int, batch: int, frames: int = 200, layers: int = 12, channels: int = 768) -> np.ndarray:
    """Synthetic stand-in for the speech encoder's hidden states over one audio window,
    [B, frames, layers, channels] float32 N(0, 1) (8 s at 25 states/s of a 12-layer,
    768-wide encoder in the pages' pipeline)."""
    return normal(seed, IN_STATES, (batch, frames, layers, channels)).astype(np.float32)
