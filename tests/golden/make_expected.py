"""Write the oracle's outputs for the full-size configurations to tests/golden/.

Calls only ``oracle/`` and the seeded input generator; nothing here touches the
CUDA library. The GPU parity tests compare the library against these files; a CPU
test checks that the oracle source they were made with is the current one.

  python tests/golden/make_expected.py            # all cases (tens of minutes on 8 cores)
  python tests/golden/make_expected.py cfg2       # one case
  python tests/golden/make_expected.py --restamp  # after a change of the oracle's source that
      # leaves its arithmetic alone: recompute cfg2, and only if it is bitwise the stored
      # output, stamp every stored file with the current source hash

Cases (the oracle in plain float32, its fp32 mode, as the parity reference of the
bf16 paths):
  cfg2          one flow prediction at sigma 0.75, batch 1, 5x16x16 latent
  cfg2_in2002, cfg2_in3002  the same prediction on inputs drawn with seeds 2002 and 3002
                (the margin of the 30-block parity is checked on three input draws)
  cfg3_s0/s19   the 4-step slice sampler, slices 0 and 19 (fresh audio per slice)
  cfg4_b0       the 4-step sampler at 5x24x24 (2880 tokens), stream 0 of the 3-stream batch
  cfg3_renoise_s0  the 4-step slice sampler with the re-noising update (reading R12), slice 0,
                its fresh draws from si.renoise_draws(seed of slice 0, 4, ...)
"""
from __future__ import annotations

import hashlib
import os
import sys
import time

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
sys.path.insert(0, ROOT)

import synth_inputs as si  # noqa: E402
from oracle import model as om  # noqa: E402

SIGMAS = [1.0, 0.75, 0.5, 0.25, 0.0]
NET_SEED = 1002


def oracle_hash() -> str:
    h = hashlib.sha256()
    for f in ("model.py",):
        h.update(open(os.path.join(ROOT, "oracle", f), "rb").read())
    h.update(open(os.path.join(ROOT, "synth_inputs.py"), "rb").read())
    return h.hexdigest()[:16]


def path(case: str) -> str:
    return os.path.join(HERE, f"expected_{case}.npz")


def make(case: str, W2=None):
    t0 = time.time()
    if case == "cfg2" or case.startswith("cfg2_in"):
        cfg = om.CFG2
        seed = si.config_seed(2) if case == "cfg2" else int(case[len("cfg2_in"):])
        W = W2 or om.make_weights(cfg, NET_SEED)
        x = si.latent(seed, si.IN_LATENT, 1, cfg.latent_ch, cfg.frames, cfg.lat_h, cfg.lat_w)
        ref = si.latent(seed, si.IN_REF, 1, cfg.latent_ch, cfg.frames, cfg.lat_h, cfg.lat_w)
        audio = si.audio_tokens(seed, 1, cfg.frames, cfg.audio_tokens, cfg.dim, True)
        out = om.predict_flow(W, x, ref, audio, 0.75, "f32")
    elif case.startswith("cfg3_s"):
        j = int(case[len("cfg3_s"):])
        cfg, seed = om.CFG3, si.config_seed(3)
        W = W2 or om.make_weights(cfg, NET_SEED)
        noise, ref, motion, audio = si.slice_inputs(seed, 1, cfg.latent_ch, cfg.frames, cfg.lat_h, cfg.lat_w,
                                                    cfg.audio_tokens, cfg.dim, True, j)
        out = om.sample_slice(W, noise, ref, motion, audio, SIGMAS, "f32")
    elif case == "cfg3_renoise_s0":
        cfg, seed = om.CFG3, si.config_seed(3)
        W = W2 or om.make_weights(cfg, NET_SEED)
        noise, ref, motion, audio = si.slice_inputs(seed, 1, cfg.latent_ch, cfg.frames, cfg.lat_h, cfg.lat_w,
                                                    cfg.audio_tokens, cfg.dim, True, 0)
        eps = si.renoise_draws(seed, len(SIGMAS) - 1, 1, cfg.latent_ch, cfg.frames, cfg.lat_h, cfg.lat_w)
        out = om.sample_slice_renoise(W, noise, ref, motion, audio, SIGMAS, eps, "f32")
    elif case == "cfg4_b0":
        cfg, seed = om.CFG4, si.config_seed(4)
        base = W2 or om.make_weights(om.CFG2, NET_SEED)
        W = om.Weights(cfg=cfg, blocks=base.blocks, glob=base.glob)
        noise, ref, motion, audio = si.slice_inputs(seed, 3, cfg.latent_ch, cfg.frames, cfg.lat_h, cfg.lat_w,
                                                    cfg.audio_tokens, cfg.dim, True)
        out = om.sample_slice(W, noise[:1], ref[:1], motion[:1], audio[:1], SIGMAS, "f32")
    else:
        raise ValueError(case)
    np.savez(path(case), out=out.astype(np.float32), oracle_hash=oracle_hash(), prec="f32")
    print(f"{case}: {time.time() - t0:.1f} s, rms {float(np.sqrt(np.mean(out.astype(np.float64) ** 2))):.4f}",
          flush=True)


CASES = ["cfg2", "cfg2_in2002", "cfg2_in3002", "cfg3_s0", "cfg3_s19", "cfg4_b0", "cfg3_renoise_s0"]

def restamp():
    W2 = om.make_weights(om.CFG2, NET_SEED)
    old = np.load(path("cfg2"))["out"]
    cfg, seed = om.CFG2, si.config_seed(2)
    x = si.latent(seed, si.IN_LATENT, 1, cfg.latent_ch, cfg.frames, cfg.lat_h, cfg.lat_w)
    ref = si.latent(seed, si.IN_REF, 1, cfg.latent_ch, cfg.frames, cfg.lat_h, cfg.lat_w)
    audio = si.audio_tokens(seed, 1, cfg.frames, cfg.audio_tokens, cfg.dim, True)
    new = om.predict_flow(W2, x, ref, audio, 0.75, "f32").astype(np.float32)
    if not np.array_equal(old, new):
        raise SystemExit("cfg2 differs from the stored output: the arithmetic changed, regenerate every case")
    for case in CASES:
        if os.path.exists(path(case)):
            d = np.load(path(case))
            np.savez(path(case), out=d["out"], oracle_hash=oracle_hash(), prec=str(d["prec"]))
            print(f"{case}: stamped {oracle_hash()}")


if __name__ == "__main__":
    if sys.argv[1:] == ["--restamp"]:
        restamp()
        sys.exit(0)
    cases = sys.argv[1:] or CASES
    W2 = om.make_weights(om.CFG2, NET_SEED)
    for c in cases:
        make(c, W2)
