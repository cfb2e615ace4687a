"""The audio projection (fh_audio_project) against the CPU oracle on the same seeded
speech-encoder states and weights: readings R19-R21 of gizai:flashhead's opening paragraph
(5 states around each of the slice's 33 frames make 5 latent frames of 32 audio tokens;
proj1, proj1vf, proj2, proj3, projNorm in Types > FlashHead)."""
import numpy as np
import pytest

import synth_inputs as si
from oracle import model as om
from gpu_helpers import rel_err, to_dev

torch = pytest.importorskip("torch")
pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

import audio_driven_talking_b200 as fh  # noqa: E402

SMALL_LIB = dict(dim=384, heads=3, ffn=1024, blocks=1, frames=3, lat_h=4, lat_w=4)
CASES = {
    # name: (library config, oracle config, network seed, batch)
    "lite": (fh.LITE.replace(blocks=1), om.Config(blocks=1), 1002, 1),
    "small_bf16_batch2": (fh.ModelConfig(max_batch=2, **SMALL_LIB), om.Config(**SMALL_LIB), 61, 2),
    "fp32": (fh.FP32_BLOCK, om.CFG0, 62, 1),
}


def bf16_out_err(gpu, ref) -> float:
    """Error beyond the output's own bf16 rounding (half an ulp, <= 2^-9 |ref|), over RMS(ref)."""
    g = np.asarray(gpu, dtype=np.float64)
    r = np.asarray(ref, dtype=np.float64)
    excess = np.maximum(np.abs(g - r) - 2.0 ** -8 * np.abs(r), 0.0)
    return float(np.max(excess) / np.sqrt(np.mean(r * r)))


@pytest.mark.parametrize("name", list(CASES))
def test_audio_projection_matches_oracle(name):
    lib_cfg, orc_cfg, seed, B = CASES[name]
    m = fh.DiT(lib_cfg, seed)
    states = si.speech_states(seed + 7, B)
    ws = m.workspace(B)
    got = m.audio_project(to_dev(states), ws)
    again = m.audio_project(to_dev(states), ws)
    m.sync()
    assert torch.equal(got, again)                      # a fixed order of the partial sums
    AW = om.make_audio_weights(orc_cfg, seed)
    for slot, tname in [(0, "proj1_w"), (3, "proj1vf_b"), (6, "proj3_w"), (8, "projnorm_w"), (9, "projnorm_b")]:
        # the same generator on both sides: equal except where a float64 libm result differs by an
        # ulp right at a rounding boundary (rare: a handful in tens of millions of values)
        mismatch = np.count_nonzero(m.get_weight(fh_audio_tid(slot), AW[tname].shape) != AW[tname])
        assert mismatch <= max(2, AW[tname].size // 10**7), (tname, mismatch)
    want = om.audio_projection(AW, states, orc_cfg, "f32")
    g = got.float().cpu().numpy()
    assert g.shape == want.shape == (B, orc_cfg.frames, 32, orc_cfg.dim)
    if lib_cfg.dtype == fh.FH_BF16:
        # float32 sums of bf16-exact products; beyond the bf16 rounding of the stored tokens only
        # the summation order remains
        assert bf16_out_err(g, want) < 1e-3
    else:
        assert rel_err(g, want) < 1e-4
    m.close()


def fh_audio_tid(slot: int) -> int:
    return 4096 + om.AUDIO_BASE + slot


def test_audio_projection_feeds_the_sampler():
    """Tokens from the projection drive a sampler slice like tokens given directly."""
    lib_cfg = fh.ModelConfig(**SMALL_LIB)
    m = fh.DiT(lib_cfg, 63)
    ws = m.workspace(1)
    states = to_dev(si.speech_states(64, 1))
    tok = m.audio_project(states, ws)
    noise, ref, motion, _ = si.slice_inputs(65, 1, 128, 3, 4, 4, 32, 384, True)
    args = [to_dev(noise), to_dev(ref), to_dev(motion)]
    a = m.sample_slice(*args, tok, [1.0, 0.5, 0.0], ws).cpu().numpy()
    b = m.sample_slice(*args, tok.clone(), [1.0, 0.5, 0.0], ws).cpu().numpy()
    m.sync()
    assert np.array_equal(a, b) and np.all(np.isfinite(a))
    m.close()
