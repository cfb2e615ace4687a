"""Shared helpers of the GPU parity tests (test infrastructure).

Maps each benchmark configuration to the library's ModelConfig and the oracle's
Config, builds seeded inputs, and caches the oracle's regenerated weights.
"""
from __future__ import annotations

import functools

import numpy as np

import synth_inputs as si
from oracle import model as om

# Tolerances against the plain fp32 oracle, max |gpu - oracle| <= TOL * RMS(oracle) per
# output tensor: 2e-2 for the bf16 paths, 1e-4 for the fp32 path.
TOL_BF16 = 2e-2
TOL_F32 = 1e-4
# The oracle's precision for the comparison: the bf16 paths are checked against its plain
# float32 mode (its bf16-operand mode differs from float32 by ~2e-2 on the 30-block network
# itself, so it is no closer a reference); the fp32 block against float64.
ORACLE_PREC_BF16 = "f32"
SIGMAS = [1.0, 0.75, 0.5, 0.25, 0.0]

# Network seeds: config 0 and 1 have their own; configs 2-4 share the Lite network of
# config 2 (their inputs keep their own seeds).
NET_SEED = {0: 0, 1: 1001, 2: 1002, 3: 1002, 4: 1002}


def record(name: str, **vals):
    """Append a measured parity figure to $FH_PARITY_REPORT (a JSON-lines file), if set."""
    import json
    import os
    p = os.environ.get("FH_PARITY_REPORT")
    if p:
        with open(p, "a") as f:
            f.write(json.dumps({"case": name, **vals}) + "\n")


def rel_rms(gpu, ref) -> float:
    g = np.asarray(gpu, dtype=np.float64)
    r = np.asarray(ref, dtype=np.float64)
    return float(np.sqrt(np.mean((g - r) ** 2)) / np.sqrt(np.mean(r * r)))


def check(name: str, gpu, ref, tol: float):
    e, er = rel_err(gpu, ref), rel_rms(gpu, ref)
    record(name, max_err_over_rms=e, rms_err_over_rms=er, tol=tol)
    assert e < tol, f"{name}: max|err|/RMS = {e:.3e} (rms err {er:.3e}) above {tol}"


def expected(case: str):
    """A stored oracle output written by tests/golden/make_expected.py."""
    import os
    p = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", f"expected_{case}.npz")
    d = np.load(p)
    return d["out"]


def rel_err(gpu, ref) -> float:
    g = np.asarray(gpu, dtype=np.float64)
    r = np.asarray(ref, dtype=np.float64)
    return float(np.max(np.abs(g - r)) / np.sqrt(np.mean(r * r)))


def lib_config(c: int):
    import audio_driven_talking_b200 as fh
    return {0: fh.FP32_BLOCK, 1: fh.ONE_BLOCK, 2: fh.LITE, 3: fh.LITE, 4: fh.LITE_768_X3}[c]


def oracle_config(c: int):
    return {0: om.CFG0, 1: om.CFG1, 2: om.CFG2, 3: om.CFG3, 4: om.CFG4}[c]


@functools.lru_cache(maxsize=3)
def _network(c: int):
    return om.make_weights(oracle_config(c), NET_SEED[c])


def oracle_weights(c: int):
    """The oracle's own regeneration of the weights (configs 3 and 4 reuse config 2's network)."""
    base = _network(2 if c in (2, 3, 4) else c)
    return om.Weights(cfg=oracle_config(c), blocks=base.blocks, glob=base.glob)


def to_dev(x, dtype=None):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x)).cuda()
    return t.to(dtype) if dtype is not None else t
