"""Python binding of the FlashHead Lite DiT library (``libfh.so``, C ABI in include/fh.h).

Argument marshalling only: every step of the hot path runs in the library's CUDA
kernels. PyTorch supplies device memory and streams. There is no CPU fallback:
if the shared library is missing, importing the binding's entry points raises.

Typical use::

    import torch, audio_driven_talking_b200 as fh
    m = fh.DiT(fh.LITE, seed=1003)
    ws = m.workspace(batch=1)
    x = m.sample_slice(noise, ref, motion, audio, [1.0, 0.75, 0.5, 0.25, 0.0], ws)
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass, field, asdict

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfh.so")

FH_OK, FH_ERR_ARG, FH_ERR_SHAPE, FH_ERR_CUDA, FH_ERR_OOM, FH_ERR_TIMEOUT, FH_ERR_UNSUPPORTED = 0, -1, -2, -3, -4, -5, -6
FH_F32, FH_BF16 = 0, 1
ERROR_NAMES = {0: "FH_OK", -1: "FH_ERR_ARG", -2: "FH_ERR_SHAPE", -3: "FH_ERR_CUDA", -4: "FH_ERR_OOM",
               -5: "FH_ERR_TIMEOUT", -6: "FH_ERR_UNSUPPORTED"}


class FHError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"{ERROR_NAMES.get(code, code)}: {msg}")
        self.code = code


class _Config(ctypes.Structure):
    _fields_ = [("dim", ctypes.c_int), ("heads", ctypes.c_int), ("head_dim", ctypes.c_int), ("ffn", ctypes.c_int),
                ("blocks", ctypes.c_int), ("latent_ch", ctypes.c_int), ("frames", ctypes.c_int),
                ("lat_h", ctypes.c_int), ("lat_w", ctypes.c_int), ("audio_tokens", ctypes.c_int),
                ("max_batch", ctypes.c_int), ("dtype", ctypes.c_int), ("rope_theta", ctypes.c_float),
                ("rope_split", ctypes.c_int * 3), ("eps", ctypes.c_float), ("device", ctypes.c_int)]


@dataclass(frozen=True)
class ModelConfig:
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
    max_batch: int = 1
    dtype: int = FH_BF16
    rope_theta: float = 1e4
    rope_split: tuple = (44, 42, 42)
    eps: float = 1e-6

    @property
    def tokens(self) -> int:
        return self.frames * self.lat_h * self.lat_w

    def replace(self, **kw) -> "ModelConfig":
        d = asdict(self)
        d.update(kw)
        return ModelConfig(**d)


# The Lite network (gizai:flashhead: 30 blocks of 1536, 12 heads, 5 latent frames of
# 16 x 16, 32 audio tokens per latent frame) and the benchmark's other shapes.
LITE = ModelConfig()
FP32_BLOCK = ModelConfig(dim=384, heads=3, ffn=1024, blocks=1, frames=2, lat_h=8, lat_w=8, dtype=FH_F32)
ONE_BLOCK = ModelConfig(blocks=1)
LITE_768_X3 = ModelConfig(lat_h=24, lat_w=24, max_batch=3)

_lib = None


def load_library() -> ctypes.CDLL:
    """Load libfh.so (built in-tree by ``python -m audio_driven_talking_b200.build``)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python -m audio_driven_talking_b200.build`; "
                          "there is no fallback implementation")
    lib = ctypes.CDLL(LIB_PATH)
    P, I, F, Z, U64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t, ctypes.c_uint64
    sig = {
        "fh_dit_create": (I, [ctypes.POINTER(_Config), U64, P, ctypes.POINTER(P)]),
        "fh_dit_destroy": (I, [P]),
        "fh_dit_workspace_bytes": (Z, [P, I]),
        "fh_dit_block_forward": (I, [P, I, P, P, P, P, I, P, P]),
        "fh_dit_predict_flow": (I, [P, P, P, P, F, P, I, P, P]),
        "fh_sample_slice": (I, [P, P, P, P, P, P, I, P, I, P, P]),
        "fh_sample_slice_renoise": (I, [P, P, P, P, P, P, I, P, P, I, P, P]),
        "fh_sample_slice_host": (I, [P, P, P, P, P, P, I, P, I, P, P]),
        "fh_dit_get_weight": (I, [P, I, P, Z]),
        "fh_audio_project": (I, [P, P, P, I, P, P]),
        "fh_dit_sync": (I, [P, P]),
        "fh_dit_last_launch_count": (I, [P]),
        "fh_dit_set_timing": (I, [P, I]),
        "fh_dit_get_timing": (I, [P, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(I)]),
        "fh_last_error": (ctypes.c_char_p, []),
        "fh_op_linear": (I, [P, P, P, P, I, I, I, I, P]),
        "fh_dit_block_forward_noalloc": (I, [P, I, P, P, P, P, I, P]),
        "fh_dit_probe_wait_timeout": (I, [P, P]),
        "fh_op_attention": (I, [P, P, P, P, P, I, I, I, F, I, P]),
        "fh_op_cross_attention": (I, [P, P, P, P, P, I, I, I, I, I, F, I, P]),
        "fh_op_row_norm": (I, [P, P, I, I, I, P, P, ctypes.c_long, I, F, I, P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def _check(code: int):
    if code != FH_OK:
        raise FHError(code, load_library().fh_last_error().decode())


def _ptr(t) -> int:
    import torch
    if not isinstance(t, torch.Tensor):
        raise TypeError("expected a torch tensor")
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return t.data_ptr()


def _stream(stream) -> int:
    import torch
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _farr(vals):
    vals = [float(v) for v in vals]
    return (ctypes.c_float * len(vals))(*vals)


class DiT:
    """A FlashHead Lite DiT with seeded synthetic weights on one GPU."""

    def __init__(self, cfg: ModelConfig, seed: int, device: int | None = None, stream=None):
        import torch
        lib = load_library()
        self.cfg = cfg
        self.device = torch.cuda.current_device() if device is None else int(device)
        self.model_dtype = torch.bfloat16 if cfg.dtype == FH_BF16 else torch.float32
        c = _Config(cfg.dim, cfg.heads, cfg.head_dim, cfg.ffn, cfg.blocks, cfg.latent_ch, cfg.frames, cfg.lat_h,
                    cfg.lat_w, cfg.audio_tokens, cfg.max_batch, cfg.dtype, cfg.rope_theta,
                    (ctypes.c_int * 3)(*cfg.rope_split), cfg.eps, self.device)
        h = ctypes.c_void_p()
        with torch.cuda.device(self.device):
            _check(lib.fh_dit_create(ctypes.byref(c), ctypes.c_uint64(seed), _stream(stream), ctypes.byref(h)))
        self._h = h

    def close(self):
        if getattr(self, "_h", None):
            load_library().fh_dit_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    # ---------------------------------------------------------------- memory
    def workspace_bytes(self, batch: int) -> int:
        return int(load_library().fh_dit_workspace_bytes(self._h, batch))

    def workspace(self, batch: int):
        import torch
        n = self.workspace_bytes(batch)
        if n == 0:
            raise FHError(FH_ERR_SHAPE, f"batch {batch} not supported")
        return torch.empty(n, dtype=torch.uint8, device=f"cuda:{self.device}")

    # ---------------------------------------------------------------- compute
    def block_forward(self, block: int, x, audio, t, ws, out=None, stream=None):
        import torch
        B = x.shape[0]
        out = torch.empty_like(x) if out is None else out
        _check(load_library().fh_dit_block_forward(self._h, block, _ptr(x), _ptr(out), _ptr(audio), _farr(t), B,
                                                   _ptr(ws), _stream(stream)))
        return out

    def block_forward_noalloc(self, block: int, x, audio, t, out=None, stream=None):
        """block_forward on the library's static scratch (no workspace, no allocation by the library)."""
        import torch
        B = x.shape[0]
        out = torch.empty_like(x) if out is None else out
        _check(load_library().fh_dit_block_forward_noalloc(self._h, block, _ptr(x), _ptr(out), _ptr(audio),
                                                           _farr(t), B, _stream(stream)))
        return out

    def predict_flow(self, x_noisy, ref, audio, sigma: float, ws, out=None, stream=None):
        import torch
        B = x_noisy.shape[0]
        out = torch.empty_like(x_noisy) if out is None else out
        _check(load_library().fh_dit_predict_flow(self._h, _ptr(x_noisy), _ptr(ref), _ptr(audio),
                                                  ctypes.c_float(sigma), _ptr(out), B, _ptr(ws), _stream(stream)))
        return out

    def sample_slice(self, noise, ref, motion, audio, sigmas, ws, out=None, stream=None):
        import torch
        B = noise.shape[0]
        out = torch.empty_like(noise) if out is None else out
        _check(load_library().fh_sample_slice(self._h, _ptr(noise), _ptr(ref), _ptr(motion), _ptr(audio),
                                              _farr(sigmas), len(sigmas) - 1, _ptr(out), B, _ptr(ws),
                                              _stream(stream)))
        return out

    def sample_slice_renoise(self, noise, ref, motion, audio, sigmas, eps, ws, out=None, stream=None):
        """The sampler with the re-noising update; eps [steps, B, C, F, H, W] float32 on the device."""
        import torch
        B = noise.shape[0]
        out = torch.empty_like(noise) if out is None else out
        _check(load_library().fh_sample_slice_renoise(self._h, _ptr(noise), _ptr(ref), _ptr(motion), _ptr(audio),
                                                      _farr(sigmas), len(sigmas) - 1, _ptr(eps), _ptr(out), B,
                                                      _ptr(ws), _stream(stream)))
        return out

    def sample_slice_host(self, noise, ref, motion, audio, sigmas, ws, out, stream=None):
        """Host-buffer sampler: inputs/outputs are host torch tensors (pinned for async copies)."""
        B = noise.shape[0]
        _check(load_library().fh_sample_slice_host(self._h, noise.data_ptr(), ref.data_ptr(), motion.data_ptr(),
                                                   audio.data_ptr(), _farr(sigmas), len(sigmas) - 1,
                                                   out.data_ptr(), B, _ptr(ws), _stream(stream)))
        return out

    def audio_project(self, states, ws, out=None, stream=None):
        """Audio tokens [B, frames, 32, dim] (model dtype) from speech-encoder states
        [B, 200, 12, 768] float32 on the device (see include/fh.h, fh_audio_project)."""
        import torch
        B = states.shape[0]
        c = self.cfg
        if out is None:
            out = torch.empty((B, c.frames, c.audio_tokens, c.dim), dtype=self.model_dtype, device=states.device)
        _check(load_library().fh_audio_project(self._h, _ptr(states), _ptr(out), B, _ptr(ws), _stream(stream)))
        return out

    def sync(self, stream=None):
        _check(load_library().fh_dit_sync(self._h, _stream(stream)))

    def probe_wait_timeout(self, stream=None):
        """Make one bounded kernel wait run out (test of the failure-detection path)."""
        _check(load_library().fh_dit_probe_wait_timeout(self._h, _stream(stream)))

    @property
    def last_launch_count(self) -> int:
        return int(load_library().fh_dit_last_launch_count(self._h))

    def set_timing(self, kernel_class: int):
        _check(load_library().fh_dit_set_timing(self._h, kernel_class))

    def get_timing(self):
        us = ctypes.c_double()
        n = ctypes.c_int()
        _check(load_library().fh_dit_get_timing(self._h, ctypes.byref(us), ctypes.byref(n)))
        return us.value, n.value

    def get_weight(self, tensor_id: int, shape) -> np.ndarray:
        out = np.empty(shape, dtype=np.float32)
        _check(load_library().fh_dit_get_weight(self._h, tensor_id, out.ctypes.data, out.nbytes))
        return out


# ------------------------------------------------------------------ operators
def linear(A, W, bias, stream=None):
    """out = A @ W^T + bias via the library's GEMM (bf16 tensor cores or fp32 CUDA cores)."""
    import torch
    M, K = A.shape
    N = W.shape[0]
    dt = FH_BF16 if A.dtype == torch.bfloat16 else FH_F32
    out = torch.empty((M, N), dtype=torch.float32, device=A.device)
    _check(load_library().fh_op_linear(_ptr(A), _ptr(W), _ptr(bias), _ptr(out), M, N, K, dt, _stream(stream)))
    return out


def cross_attention(q, ssq_q, kv, ssq_k, frames, eps=1e-6, stream=None):
    """Per-frame audio cross-attention (see include/fh_ops.h): q [B, frames*hw, heads*128],
    kv [B, frames, 32, 2*heads*128] (keys then values), ssq_q/ssq_k float32 per-head sums."""
    import torch
    B, L, D = q.shape
    A = kv.shape[2]
    dt = FH_BF16 if q.dtype == torch.bfloat16 else FH_F32
    out = torch.empty_like(q)
    _check(load_library().fh_op_cross_attention(_ptr(q), _ptr(ssq_q), _ptr(kv), _ptr(ssq_k), _ptr(out), B, D // 128,
                                                frames, L // frames, A, ctypes.c_float(eps), dt, _stream(stream)))
    return out


def row_norm(x, mode, a, c, bstride=0, rows_per_batch=None, out_dtype=None, eps=1e-6, out=None, stream=None):
    """Row norm and modulation (see include/fh_ops.h, fh_op_row_norm): x float32 [M, D]."""
    import torch
    M, D = x.shape
    out_dtype = out_dtype or torch.bfloat16
    dt = FH_BF16 if out_dtype == torch.bfloat16 else FH_F32
    out = torch.empty((M, D), dtype=out_dtype, device=x.device) if out is None else out
    _check(load_library().fh_op_row_norm(_ptr(x), _ptr(out), M, D, mode, _ptr(a), _ptr(c), int(bstride),
                                         rows_per_batch or M, ctypes.c_float(eps), dt, _stream(stream)))
    return out


def attention(q, k, v, ssq, eps=1e-6, stream=None):
    """Self-attention with full-width RMS factors from ssq (see include/fh_ops.h)."""
    import torch
    B, NH, L, hd = q.shape
    dt = FH_BF16 if q.dtype == torch.bfloat16 else FH_F32
    out = torch.empty((B * L, NH * hd), dtype=q.dtype, device=q.device)
    _check(load_library().fh_op_attention(_ptr(q), _ptr(k), _ptr(v), _ptr(ssq), _ptr(out), B, NH, L,
                                          ctypes.c_float(eps), dt, _stream(stream)))
    return out


__all__ = ["DiT", "ModelConfig", "LITE", "FP32_BLOCK", "ONE_BLOCK", "LITE_768_X3", "FHError", "load_library",
           "linear", "attention", "cross_attention", "row_norm", "FH_F32", "FH_BF16"]
