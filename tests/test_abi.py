"""C-ABI checks that need no GPU: the library builds, loads, exports every symbol
the public headers declare, and rejects bad arguments on the host before any
device work."""
import ctypes
import glob
import os
import re

import pytest

import audio_driven_talking_b200 as fh
from audio_driven_talking_b200 import build as fhbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    fhbuild.build()
    return fh.load_library()


def declared_functions():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        for m in re.finditer(r"\b(fh_\w+)\s*\(", text):
            if not m.group(1).startswith("FH_"):
                names.add(m.group(1))
    return sorted(names)


def test_headers_declare_the_boundary():
    names = declared_functions()
    for required in ["fh_dit_create", "fh_dit_destroy", "fh_dit_workspace_bytes", "fh_dit_block_forward",
                     "fh_dit_predict_flow", "fh_sample_slice", "fh_sample_slice_host", "fh_dit_get_weight",
                     "fh_last_error", "fh_op_linear", "fh_op_attention"]:
        assert required in names


def test_library_exports_every_declared_symbol(lib):
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing


def test_library_targets_sm100a_only():
    """Every object is compiled for sm_100a (the build flags); no other arch is requested."""
    assert fhbuild.ARCH == ["-gencode", "arch=compute_100a,code=sm_100a"]


def test_null_and_shape_errors_on_host(lib):
    assert lib.fh_dit_workspace_bytes(None, 1) == 0
    out = ctypes.c_void_p()
    assert lib.fh_dit_create(None, 0, None, ctypes.byref(out)) == fh.FH_ERR_ARG
    assert b"null" in lib.fh_last_error()
    # head_dim must be 128
    cfg = fh.LITE
    bad = fh._Config(cfg.dim, cfg.heads, 64, cfg.ffn, cfg.blocks, cfg.latent_ch, cfg.frames, cfg.lat_h, cfg.lat_w,
                     cfg.audio_tokens, 1, cfg.dtype, cfg.rope_theta, (ctypes.c_int * 3)(*cfg.rope_split), cfg.eps, 0)
    assert lib.fh_dit_create(ctypes.byref(bad), 0, None, ctypes.byref(out)) == fh.FH_ERR_SHAPE
    # rotary split must sum to head_dim with even parts
    bad2 = fh._Config(cfg.dim, cfg.heads, 128, cfg.ffn, cfg.blocks, cfg.latent_ch, cfg.frames, cfg.lat_h, cfg.lat_w,
                      cfg.audio_tokens, 1, cfg.dtype, cfg.rope_theta, (ctypes.c_int * 3)(44, 43, 41), cfg.eps, 0)
    assert lib.fh_dit_create(ctypes.byref(bad2), 0, None, ctypes.byref(out)) == fh.FH_ERR_SHAPE
    # batch above the supported maximum
    bad3 = fh._Config(cfg.dim, cfg.heads, 128, cfg.ffn, cfg.blocks, cfg.latent_ch, cfg.frames, cfg.lat_h, cfg.lat_w,
                      cfg.audio_tokens, 9, cfg.dtype, cfg.rope_theta, (ctypes.c_int * 3)(*cfg.rope_split), cfg.eps, 0)
    assert lib.fh_dit_create(ctypes.byref(bad3), 0, None, ctypes.byref(out)) == fh.FH_ERR_SHAPE
    assert lib.fh_dit_sync(None, None) == fh.FH_ERR_ARG
    assert lib.fh_dit_get_weight(None, 0, None, 0) == fh.FH_ERR_ARG
    # the samplers reject a null model before touching a device
    sig = (ctypes.c_float * 5)(1.0, 0.75, 0.5, 0.25, 0.0)
    assert lib.fh_sample_slice(None, None, None, None, None, sig, 4, None, 1, None, None) == fh.FH_ERR_ARG
    assert lib.fh_sample_slice_renoise(None, None, None, None, None, sig, 4, None, None, 1, None, None) == fh.FH_ERR_ARG
    assert b"null" in lib.fh_last_error()


def test_no_device_is_rejected_not_substituted(lib):
    torch = pytest.importorskip("torch")
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    cfg = fh.FP32_BLOCK
    c = fh._Config(cfg.dim, cfg.heads, 128, cfg.ffn, cfg.blocks, cfg.latent_ch, cfg.frames, cfg.lat_h, cfg.lat_w,
                   cfg.audio_tokens, 1, cfg.dtype, cfg.rope_theta, (ctypes.c_int * 3)(*cfg.rope_split), cfg.eps, 0)
    out = ctypes.c_void_p()
    assert lib.fh_dit_create(ctypes.byref(c), 0, None, ctypes.byref(out)) == fh.FH_ERR_UNSUPPORTED
    assert not out.value


def test_binding_has_no_oracle_dependency():
    """The product path never imports the CPU oracle."""
    src = ""
    for p in glob.glob(os.path.join(ROOT, "audio_driven_talking_b200", "**", "*.*"), recursive=True):
        if p.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
            src += open(p).read()
    assert "oracle" not in re.sub(r"#.*|//.*", "", src).replace("the oracle", "")
