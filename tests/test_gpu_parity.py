"""Model-level parity of the CUDA library (through the C ABI) with the CPU oracle on
the same seeded inputs, for the five benchmark configurations, plus ragged shapes,
batch independence, determinism, motion pinning and argument errors.

Tolerances (max |gpu - oracle| over RMS(oracle) per output tensor): 1e-4 for the fp32
block (oracle in float64), 2e-2 for the bf16 paths (oracle in plain float32). The
full-size outputs of configurations 2-4 come from tests/golden/make_expected.py,
which runs the oracle only."""
import numpy as np
import pytest

import synth_inputs as si
from oracle import model as om
from gpu_helpers import (NET_SEED, ORACLE_PREC_BF16, SIGMAS, TOL_BF16, TOL_F32, check, expected, lib_config,
                         oracle_config, oracle_weights, record, to_dev)

torch = pytest.importorskip("torch")
pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

import audio_driven_talking_b200 as fh  # noqa: E402

_models = {}


def model(c, cfg=None, seed=None):
    key = (c, cfg, seed)
    if key not in _models:
        _models[key] = fh.DiT(cfg or lib_config(c), NET_SEED[c] if seed is None else seed)
    return _models[key]


def _block_case(c, batch=1):
    ocfg = oracle_config(c)
    seed = si.config_seed(c)
    return si.block_inputs(seed, batch, ocfg.tokens, ocfg.dim, ocfg.frames, ocfg.audio_tokens, ocfg.bf16)


def _gpu_block(m, k, x, a, t):
    ws = m.workspace(x.shape[0])
    adt = m.model_dtype
    out = m.block_forward(k, to_dev(x), to_dev(a, adt), list(t), ws)
    m.sync()
    return out.cpu().numpy()


# ---------------------------------------------------------------------------- weights
@pytest.mark.parametrize("c,tids", [(0, [0, 1, 9, 11, 12, 23, 26, 4096, 4100, 4105]),
                                    (1, [0, 3, 10, 15, 17, 22, 25, 4096, 4098, 4104])])
def test_weights_follow_the_seeded_generator(c, tids):
    m = model(c)
    W = oracle_weights(c)
    names = {s: n for s, n, *_ in om.BLOCK_SLOTS}
    gnames = {s: n for s, n, *_ in om.GLOBAL_SLOTS}
    for tid in tids:
        ref = W.glob[gnames[tid - 4096]] if tid >= 4096 else W.blocks[tid // 64][names[tid % 64]]
        got = m.get_weight(tid, ref.shape)
        # same generator on both sides: equal except where float64 libm results differ by an ulp
        # right at a rounding boundary (none expected at these sizes)
        mismatch = np.count_nonzero(got != ref)
        assert mismatch <= 2, (tid, mismatch)


# ---------------------------------------------------------------------------- config 0
def test_cfg0_fp32_block_matches_oracle():
    m = model(0)
    W = oracle_weights(0)
    x, a, t = _block_case(0)
    got = _gpu_block(m, 0, x, a, t)
    _, e0 = om.time_conditioning(W, t, "f64")
    ref = om.block_forward(W, 0, x, a, e0, "f64")
    check("cfg0_fp32_block", got, ref, TOL_F32)


# ---------------------------------------------------------------------------- config 1
def test_cfg1_bf16_block_matches_oracle():
    m = model(1)
    W = oracle_weights(1)
    x, a, t = _block_case(1)
    got = _gpu_block(m, 0, x, a, t)
    _, e0 = om.time_conditioning(W, t, ORACLE_PREC_BF16)
    ref = om.block_forward(W, 0, x, a, e0, ORACLE_PREC_BF16)
    check("cfg1_bf16_block", got, ref, TOL_BF16)


# ---------------------------------------------------------------------------- ragged small bf16 network
RAGGED_LIB = None


def _ragged():
    # 3 latent frames of 12 x 12 = 432 tokens (ragged against 128-row tiles), 2 blocks, width 384
    lib = fh.ModelConfig(dim=384, heads=3, ffn=1024, blocks=2, frames=3, lat_h=12, lat_w=12, max_batch=2)
    orc = om.Config(dim=384, heads=3, ffn=1024, blocks=2, frames=3, lat_h=12, lat_w=12)
    return lib, orc


def test_ragged_bf16_sampler_matches_oracle():
    lib, orc = _ragged()
    m = model("ragged", lib, 77)
    W = om.make_weights(orc, 77)
    noise, ref, motion, audio = si.slice_inputs(78, 2, orc.latent_ch, orc.frames, orc.lat_h, orc.lat_w,
                                                orc.audio_tokens, orc.dim, True)
    ws = m.workspace(2)
    out = m.sample_slice(to_dev(noise), to_dev(ref), to_dev(motion), to_dev(audio, torch.bfloat16), SIGMAS, ws)
    m.sync()
    got = out.cpu().numpy()
    expect = om.sample_slice(W, noise, ref, motion, audio, SIGMAS, ORACLE_PREC_BF16)
    assert np.array_equal(got[:, :, :2], motion)
    check("ragged_432tok_b2_sampler", got, expect, TOL_BF16)
    # predict_flow on its own
    v = m.predict_flow(to_dev(noise), to_dev(ref), to_dev(audio, torch.bfloat16), 0.6, ws)
    m.sync()
    vref = om.predict_flow(W, noise, ref, audio, 0.6, ORACLE_PREC_BF16)
    check("ragged_432tok_b2_predict", v.cpu().numpy(), vref, TOL_BF16)


def _renoise_case(orc, seed, batch, steps):
    return si.renoise_draws(seed, steps, batch, orc.latent_ch, orc.frames, orc.lat_h, orc.lat_w)


def test_ragged_bf16_renoise_sampler_matches_oracle():
    """The re-noising sampler (reading R12) on the ragged network against the oracle's."""
    lib, orc = _ragged()
    m = model("ragged", lib, 77)
    W = om.make_weights(orc, 77)
    noise, ref, motion, audio = si.slice_inputs(78, 2, orc.latent_ch, orc.frames, orc.lat_h, orc.lat_w,
                                                orc.audio_tokens, orc.dim, True)
    eps = _renoise_case(orc, 79, 2, len(SIGMAS) - 1)
    ws = m.workspace(2)
    out = m.sample_slice_renoise(to_dev(noise), to_dev(ref), to_dev(motion), to_dev(audio, torch.bfloat16), SIGMAS,
                                 to_dev(eps), ws)
    m.sync()
    got = out.cpu().numpy()
    expect = om.sample_slice_renoise(W, noise, ref, motion, audio, SIGMAS, eps, ORACLE_PREC_BF16)
    assert np.array_equal(got[:, :, :2], motion)
    check("ragged_432tok_b2_renoise", got, expect, TOL_BF16)


def test_renoise_final_step_is_the_euler_step_bitwise():
    """A single step to sigma 0 puts no weight on the draw: the re-noising sampler's output
    equals the Euler sampler's bit for bit, for two different draws."""
    lib, orc = _ragged()
    m = model("ragged", lib, 77)
    noise, ref, motion, audio = si.slice_inputs(80, 2, orc.latent_ch, orc.frames, orc.lat_h, orc.lat_w,
                                                orc.audio_tokens, orc.dim, True)
    args = (to_dev(noise), to_dev(ref), to_dev(motion), to_dev(audio, torch.bfloat16))
    sig = [0.6, 0.0]
    ws = m.workspace(2)
    euler = m.sample_slice(*args, sig, ws).cpu().numpy()
    for seed in (81, 82):
        got = m.sample_slice_renoise(*args, sig, to_dev(_renoise_case(orc, seed, 2, 1)), ws).cpu().numpy()
        assert np.array_equal(got, euler)
    # with more steps the draws matter
    sig3 = [1.0, 0.5, 0.0]
    a = m.sample_slice_renoise(*args, sig3, to_dev(_renoise_case(orc, 83, 2, 2)), ws).cpu().numpy()
    b = m.sample_slice_renoise(*args, sig3, to_dev(_renoise_case(orc, 84, 2, 2)), ws).cpu().numpy()
    assert not np.array_equal(a[:, :, 2:], b[:, :, 2:])
    with pytest.raises(fh.FHError) as e:
        lib_h = fh.load_library()
        fh._check(lib_h.fh_sample_slice_renoise(m._h, fh._ptr(args[0]), fh._ptr(args[1]), fh._ptr(args[2]),
                                                fh._ptr(args[3]), fh._farr(sig), 1, None, fh._ptr(args[0]), 2,
                                                fh._ptr(ws), None))
    assert e.value.code == fh.FH_ERR_ARG


# ---------------------------------------------------------------------------- config 2
@pytest.mark.parametrize("case", ["cfg2", "cfg2_in2002", "cfg2_in3002"])
def test_cfg2_predict_flow_matches_oracle(case):
    """One 30-block prediction on three input draws (the configuration's own seed and two
    more), so that the margin under the bound is seen to hold beyond one draw."""
    m = model(2)
    ocfg = oracle_config(2)
    seed = si.config_seed(2) if case == "cfg2" else int(case[len("cfg2_in"):])
    x = si.latent(seed, si.IN_LATENT, 1, ocfg.latent_ch, ocfg.frames, ocfg.lat_h, ocfg.lat_w)
    ref = si.latent(seed, si.IN_REF, 1, ocfg.latent_ch, ocfg.frames, ocfg.lat_h, ocfg.lat_w)
    audio = si.audio_tokens(seed, 1, ocfg.frames, ocfg.audio_tokens, ocfg.dim, True)
    ws = m.workspace(1)
    v = m.predict_flow(to_dev(x), to_dev(ref), to_dev(audio, torch.bfloat16), 0.75, ws)
    m.sync()
    check(f"{case}_predict_flow", v.cpu().numpy(), expected(case), TOL_BF16)


# ---------------------------------------------------------------------------- config 3
@pytest.mark.parametrize("slice_index", [0, 19])
def test_cfg3_sampler_slice_matches_oracle(slice_index):
    m = model(3)
    ocfg = oracle_config(3)
    seed = si.config_seed(3)
    noise, ref, motion, audio = si.slice_inputs(seed, 1, ocfg.latent_ch, ocfg.frames, ocfg.lat_h, ocfg.lat_w,
                                                ocfg.audio_tokens, ocfg.dim, True, slice_index)
    ws = m.workspace(1)
    out = m.sample_slice(to_dev(noise), to_dev(ref), to_dev(motion), to_dev(audio, torch.bfloat16), SIGMAS, ws)
    m.sync()
    got = out.cpu().numpy()
    assert np.array_equal(got[:, :, :2], motion)
    check(f"cfg3_slice{slice_index}", got, expected(f"cfg3_s{slice_index}"), TOL_BF16)


def test_cfg3_renoise_slice_matches_oracle():
    """The re-noising sampler (reading R12) on the full-size slice, slice 0's inputs and the
    draws si.renoise_draws(seed, 4, ...), against the stored oracle output."""
    m = model(3)
    ocfg = oracle_config(3)
    seed = si.config_seed(3)
    noise, ref, motion, audio = si.slice_inputs(seed, 1, ocfg.latent_ch, ocfg.frames, ocfg.lat_h, ocfg.lat_w,
                                                ocfg.audio_tokens, ocfg.dim, True, 0)
    eps = _renoise_case(ocfg, seed, 1, len(SIGMAS) - 1)
    ws = m.workspace(1)
    out = m.sample_slice_renoise(to_dev(noise), to_dev(ref), to_dev(motion), to_dev(audio, torch.bfloat16), SIGMAS,
                                 to_dev(eps), ws)
    m.sync()
    got = out.cpu().numpy()
    assert np.array_equal(got[:, :, :2], motion)
    check("cfg3_renoise_slice0", got, expected("cfg3_renoise_s0"), TOL_BF16)


def test_cfg3_host_buffer_entry_matches_device_entry():
    m = model(3)
    ocfg = oracle_config(3)
    noise, ref, motion, audio = si.slice_inputs(si.config_seed(3), 1, ocfg.latent_ch, ocfg.frames, ocfg.lat_h,
                                                ocfg.lat_w, ocfg.audio_tokens, ocfg.dim, True, 3)
    ws = m.workspace(1)
    dev = m.sample_slice(to_dev(noise), to_dev(ref), to_dev(motion), to_dev(audio, torch.bfloat16), SIGMAS, ws)
    m.sync()
    host_out = torch.empty(noise.shape, dtype=torch.float32).pin_memory()
    pin = lambda a, dt=None: (torch.from_numpy(a).to(dt) if dt else torch.from_numpy(a)).pin_memory()
    m.sample_slice_host(pin(noise), pin(ref), pin(motion), pin(audio, torch.bfloat16), SIGMAS, ws, host_out)
    assert torch.equal(host_out, dev.cpu())


def test_sampler_is_deterministic():
    m = model(3)
    ocfg = oracle_config(3)
    noise, ref, motion, audio = si.slice_inputs(5, 1, ocfg.latent_ch, ocfg.frames, ocfg.lat_h, ocfg.lat_w,
                                                ocfg.audio_tokens, ocfg.dim, True)
    ws = m.workspace(1)
    args = (to_dev(noise), to_dev(ref), to_dev(motion), to_dev(audio, torch.bfloat16), SIGMAS, ws)
    a = m.sample_slice(*args).clone()
    b = m.sample_slice(*args)
    m.sync()
    assert torch.equal(a, b)


# ---------------------------------------------------------------------------- config 4
def test_cfg4_batch3_768_stream0_matches_oracle_and_streams_are_independent():
    m = model(4)
    ocfg = oracle_config(4)
    seed = si.config_seed(4)
    noise, ref, motion, audio = si.slice_inputs(seed, 3, ocfg.latent_ch, ocfg.frames, ocfg.lat_h, ocfg.lat_w,
                                                ocfg.audio_tokens, ocfg.dim, True)
    ws3 = m.workspace(3)
    out3 = m.sample_slice(to_dev(noise), to_dev(ref), to_dev(motion), to_dev(audio, torch.bfloat16), SIGMAS, ws3)
    m.sync()
    got3 = out3.cpu().numpy()
    assert np.array_equal(got3[:, :, :2], motion)
    # every stream of the batch equals a batch-1 run of that stream (bitwise: the kernels are row-independent)
    ws1 = m.workspace(1)
    for b in range(3):
        sl = slice(b, b + 1)
        o1 = m.sample_slice(to_dev(noise[sl]), to_dev(ref[sl]), to_dev(motion[sl]),
                            to_dev(audio[sl], torch.bfloat16), SIGMAS, ws1)
        m.sync()
        assert np.array_equal(o1.cpu().numpy()[0], got3[b])
    # stream 0 against the oracle (2880 tokens, 30 blocks, 4 steps)
    check("cfg4_stream0", got3[:1], expected("cfg4_b0"), TOL_BF16)


# ---------------------------------------------------------------------------- argument errors
def test_argument_errors_are_reported_not_run():
    m = model(1)
    ws = m.workspace(1)
    x, a, t = _block_case(1)
    xd, ad = to_dev(x), to_dev(a, torch.bfloat16)
    with pytest.raises(fh.FHError) as e:
        m.block_forward(1, xd, ad, list(t), ws)          # block index out of range
    assert e.value.code == fh.FH_ERR_ARG
    with pytest.raises(fh.FHError) as e:
        m.block_forward(0, torch.cat([xd, xd]), torch.cat([ad, ad]), list(t) * 2, ws)   # batch > max_batch
    assert e.value.code == fh.FH_ERR_SHAPE
    with pytest.raises(fh.FHError) as e:
        m.block_forward(0, xd, ad, list(t), ws[1:])       # misaligned workspace
    assert e.value.code == fh.FH_ERR_ARG
    assert m.workspace_bytes(0) == 0 and m.workspace_bytes(2) == 0
