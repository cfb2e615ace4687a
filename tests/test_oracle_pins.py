"""Pins of the CPU oracle against what the pages and the mathematics fix.

Every check here runs on the CPU (no GPU marker). They are chosen so that a
plausible mistake in the oracle (a dropped term, a wrong sign or index, a
transposed operand) fails at least one of them:
  * the float64 brute force (per-token loops, complex rotation) on the fp32
    block configuration, to 1e-10 relative;
  * rotary closed forms and invariants (identity at position 0, unit-frequency
    first pair of each axis, norm preservation, relative-position invariance);
  * attention invariants (rows sum to one, single key, per-frame locality,
    permutation of a frame's audio tokens);
  * norm/modulation special cases (LayerNorm moments, scale = -1, zero gates);
  * the Euler sampler's telescoping sum for a constant velocity, motion pinning;
  * the tanh-GELU against the exact erf form, the timestep sinusoid at t = 0;
  * the sizes the pages state (tests/golden/page_facts.json);
  * mutation checks: mistakes planted in the oracle make the brute-force pin fail.
"""
import json
import math
import os

import numpy as np
import pytest

import synth_inputs as si
from oracle import model as om
from oracle import brute

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "page_facts.json")


def rel(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.max(np.abs(a - b)) / np.sqrt(np.mean(b * b)))


@pytest.fixture(scope="module")
def cfg0_case():
    cfg = om.CFG0
    seed = si.config_seed(0)
    W = om.make_weights(cfg, seed)
    x, a, t = si.block_inputs(seed, 1, cfg.tokens, cfg.dim, cfg.frames, cfg.audio_tokens, False)
    return cfg, W, x, a, t


# ---------------------------------------------------------------------------
# generator and rounding helpers (input side)
# ---------------------------------------------------------------------------
def test_generator_moments():
    z = si.normal(7, 3, (200000,))
    assert abs(z.mean()) < 5 / math.sqrt(z.size)
    assert abs(z.var() - 1.0) < 5 * math.sqrt(2.0 / z.size)
    u = si.uniform(7, 3, (200000,))
    assert 0.0 <= u.min() and u.max() < 1.0
    assert abs(u.mean() - 0.5) < 5 * math.sqrt(1 / 12 / u.size)
    # different tensor ids / seeds give unrelated streams
    assert abs(np.corrcoef(si.normal(7, 3, (50000,)), si.normal(7, 4, (50000,)))[0, 1]) < 0.03
    assert abs(np.corrcoef(si.normal(7, 3, (50000,)), si.normal(8, 3, (50000,)))[0, 1]) < 0.03


def test_generator_chunking_is_positional():
    """Element i depends on (seed, tid, i) only, not on how many are drawn."""
    a = si.normal(11, 5, (3 * (1 << 22) + 17,))
    b = si.normal(11, 5, (1000,))
    assert np.array_equal(a[:1000], b)


def test_bf16_rounding_matches_torch():
    torch = pytest.importorskip("torch")
    x = si.normal(3, 9, (100000,)).astype(np.float32) * 37.0
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float32).numpy()
    assert np.array_equal(si.to_bf16(x), ref)


# ---------------------------------------------------------------------------
# sizes stated on the pages
# ---------------------------------------------------------------------------
def test_page_facts():
    facts = json.load(open(GOLDEN))
    c = om.CFG3
    assert c.tokens == facts["tokens_per_slice"]["value"]
    assert c.frames == facts["latent_frames"]["value"]
    assert [c.lat_h, c.lat_w] == facts["latent_hw"]["value"]
    assert c.blocks == facts["blocks"]["value"]
    assert c.dim == facts["width"]["value"]
    assert c.heads == facts["heads"]["value"]
    assert c.audio_tokens == facts["audio_tokens_per_latent_frame"]["value"]
    ang = om.rope_angles(c)
    assert ang.shape[1] == facts["pairs_per_head"]["value"]
    table = np.tile(ang, (1, c.heads))          # pair d of head h at column h*64 + d
    assert list(table.shape) == facts["rope_table_shape"]["value"]
    assert [2, c.dim] == facts["head_mods_shape"]["value"]
    # 24 frames at 25 fps = 0.96 s = 15360 samples at 16 kHz
    assert facts["frames_per_slice"]["value"] * facts["sample_rate"]["value"] \
        == facts["samples_per_slice"]["value"] * facts["fps"]["value"]
    # the 1.3B-parameter model: the synthetic network has the same order of size
    n = om.param_count(c)
    assert 1.25e9 < n < 1.45e9, n
    # 512 x 512 picture, 16 x 16 latent: spatial stride 32 (the LTX VAE)
    assert facts["picture_side"]["value"] // c.lat_h == 32


# ---------------------------------------------------------------------------
# rotary embedding
# ---------------------------------------------------------------------------
def test_rope_position_zero_is_identity():
    ang = om.rope_angles(om.CFG3)
    assert np.all(ang[0] == 0.0)


def test_rope_first_pair_of_each_axis_turns_one_radian_per_step():
    c = om.CFG3
    ang = om.rope_angles(c)
    hw = c.lat_h * c.lat_w
    n = 3 * hw + 5 * c.lat_w + 11          # frame 3, row 5, column 11
    pf, ph = c.rope_split[0] // 2, c.rope_split[1] // 2
    assert ang[n, 0] == 3.0
    assert ang[n, pf] == 5.0
    assert ang[n, pf + ph] == 11.0
    # frequencies fall monotonically inside each axis and stay in (0, 1]
    for lo, hi, pos in ((0, pf, 3.0), (pf, pf + ph, 5.0), (pf + ph, 64, 11.0)):
        f = ang[n, lo:hi] / pos
        assert np.all(np.diff(f) < 0) and f[0] == 1.0 and f[-1] > 0


def test_rope_preserves_norm_and_depends_on_offset_only():
    c = om.CFG3
    ang = om.rope_angles(c)
    rng_q = si.normal(1, 1, (c.tokens, c.heads, c.head_dim))
    rq = om.apply_rope(rng_q[None], ang)[0]
    assert np.allclose(np.linalg.norm(rq, axis=-1), np.linalg.norm(rng_q, axis=-1), rtol=1e-12)
    hw = c.lat_h * c.lat_w

    def tok(f, r, w):
        return f * hw + r * c.lat_w + w

    q = si.normal(2, 1, (c.heads, c.head_dim))
    k = si.normal(2, 2, (c.heads, c.head_dim))
    allq = np.broadcast_to(q, (c.tokens, c.heads, c.head_dim)).copy()
    allk = np.broadcast_to(k, (c.tokens, c.heads, c.head_dim)).copy()
    RQ = om.apply_rope(allq[None], ang)[0]
    RK = om.apply_rope(allk[None], ang)[0]
    d1 = np.einsum("hd,hd->h", RQ[tok(1, 2, 3)], RK[tok(0, 7, 1)])
    d2 = np.einsum("hd,hd->h", RQ[tok(4, 6, 13)], RK[tok(3, 11, 11)])   # both shifted by (3, 4, 10)
    assert np.allclose(d1, d2, rtol=1e-10, atol=1e-10)
    d3 = np.einsum("hd,hd->h", RQ[tok(4, 6, 12)], RK[tok(3, 11, 11)])   # a different offset
    assert not np.allclose(d1, d3, rtol=1e-3)


# ---------------------------------------------------------------------------
# attention, norms, conditioning
# ---------------------------------------------------------------------------
def test_attention_rows_sum_to_one_and_single_key():
    q = si.normal(5, 1, (1, 40, 2, 16))
    k = si.normal(5, 2, (1, 40, 2, 16))
    ones = np.ones((1, 40, 2, 16))
    assert np.allclose(om.self_attention(q, k, ones, 0.25), 1.0, atol=1e-14)
    v1 = si.normal(5, 3, (1, 1, 2, 16))
    o = om.self_attention(q[:, :1], k[:, :1], v1, 0.25)
    assert np.allclose(o, v1, atol=1e-14)
    # one audio token per frame returns that frame's value for every token
    kf = si.normal(5, 4, (1, 4, 1, 2, 16))
    vf = si.normal(5, 5, (1, 4, 1, 2, 16))
    oc = om.frame_cross_attention(q, kf, vf, frames=4, scale=0.25)
    assert np.allclose(oc.reshape(1, 4, 10, 2, 16), vf.reshape(1, 4, 1, 2, 16), atol=1e-14)


def test_softmax_shift_invariance():
    s = si.normal(6, 1, (7, 33))
    assert np.allclose(om.softmax(s), om.softmax(s + 123.25), atol=1e-15)


def test_cross_attention_audio_permutation_invariant():
    q = si.normal(9, 1, (1, 20, 2, 16))
    k = si.normal(9, 2, (1, 2, 8, 2, 16))
    v = si.normal(9, 3, (1, 2, 8, 2, 16))
    perm = np.array([3, 1, 7, 0, 6, 2, 5, 4])
    o1 = om.frame_cross_attention(q, k, v, 2, 0.25)
    o2 = om.frame_cross_attention(q, k[:, :, perm], v[:, :, perm], 2, 0.25)
    assert np.allclose(o1, o2, atol=1e-13)


def test_layer_norm_moments():
    x = si.normal(4, 1, (5, 384)) * 3.0 + 2.0
    y = om.layer_norm(x, 1e-6)
    assert np.allclose(y.mean(-1), 0.0, atol=1e-12)
    assert np.allclose(y.var(-1), 1.0, atol=1e-5)
    r = om.rms_norm(x, 0.0)
    assert np.allclose((r * r).mean(-1), 1.0, atol=1e-12)


def test_gelu_tanh_close_to_exact_gelu():
    xs = np.linspace(-8, 8, 4001)
    exact = np.array([0.5 * a * (1.0 + math.erf(a / math.sqrt(2.0))) for a in xs])
    err = np.max(np.abs(om.gelu_tanh(xs) - exact))
    assert err < 5e-4, err


def test_timestep_sinusoid_closed_forms():
    e = om.timestep_sinusoid(np.array([0.0, 0.25]))
    assert np.all(e[0, :128] == 1.0) and np.all(e[0, 128:] == 0.0)
    assert math.isclose(e[1, 0], math.cos(250.0), abs_tol=1e-15)
    assert math.isclose(e[1, 128], math.sin(250.0), abs_tol=1e-15)
    assert math.isclose(e[1, 127], math.cos(250.0 * 10000.0 ** (-127 / 128)), abs_tol=1e-15)


# ---------------------------------------------------------------------------
# whole block: brute force, special cases, locality
# ---------------------------------------------------------------------------
def _block(W, x, a, t, prec="f64"):
    _, e0 = om.time_conditioning(W, t, prec)
    return om.block_forward(W, 0, x, a, e0, prec)


def test_block_matches_float64_brute_force(cfg0_case):
    cfg, W, x, a, t = cfg0_case
    y = _block(W, x, a, t)
    toks = list(range(0, cfg.tokens, 9)) + [cfg.tokens - 1]
    yb = brute.block_tokens(W, 0, x[0], a[0], float(t[0]), toks)
    assert rel(y[0, toks], yb) < 1e-10


def test_block_f32_and_bf16_modes_close_to_f64(cfg0_case):
    cfg, W, x, a, t = cfg0_case
    y64 = _block(W, x, a, t, "f64")
    assert rel(_block(W, x, a, t, "f32"), y64) < 1e-5
    assert rel(_block(W, x, a, t, "bf16"), y64) < 2e-2


def test_block_batch_rows_independent(cfg0_case):
    cfg, W, x, a, t = cfg0_case
    x2, a2, t2 = si.block_inputs(99, 1, cfg.tokens, cfg.dim, cfg.frames, cfg.audio_tokens, False)
    xb = np.concatenate([x, x2])
    ab = np.concatenate([a, a2])
    tb = np.concatenate([t, t2])
    yb = _block(W, xb, ab, tb)
    assert np.allclose(yb[0], _block(W, x, a, t)[0], rtol=0, atol=1e-12)
    assert np.allclose(yb[1], _block(W, x2, a2, t2)[0], rtol=0, atol=1e-12)


def test_block_audio_locality(cfg0_case):
    """Perturbing frame f's audio changes only the rows of latent frame f."""
    cfg, W, x, a, t = cfg0_case
    y = _block(W, x, a, t)
    a2 = a.copy()
    a2[0, 1] += 0.5
    y2 = _block(W, x, a2, t)
    hw = cfg.lat_h * cfg.lat_w
    assert np.array_equal(y[0, :hw], y2[0, :hw])
    assert np.max(np.abs(y[0, hw:] - y2[0, hw:])) > 1e-3


def _with(W, k, **repl):
    import copy
    W2 = copy.deepcopy(W)
    for name, val in repl.items():
        W2.blocks[k][name] = val
    return W2


def test_block_zero_gates_and_zero_cross_is_identity(cfg0_case):
    """gate = 0 removes the self-attention and FFN branches; zero cross-O removes the last."""
    cfg, W, x, a, t = cfg0_case
    _, e0 = om.time_conditioning(W, t, "f64")
    mod = W.blocks[0]["mod"].astype(np.float64).copy()
    mod[2] = -e0[0, 2]
    mod[5] = -e0[0, 5]
    D = cfg.dim
    W2 = _with(W, 0, mod=mod, wco=np.zeros((D, D)), bco=np.zeros(D))
    y = om.block_forward(W2, 0, x, a, e0, "f64")
    assert np.max(np.abs(y - x)) < 1e-12


def test_block_scale_minus_one_gives_shift(cfg0_case):
    """(1 + scale) = 0 makes h = shift for every token: the self-attention branch is a constant."""
    cfg, W, x, a, t = cfg0_case
    _, e0 = om.time_conditioning(W, t, "f64")
    D = cfg.dim
    p = W.blocks[0]
    mod = p["mod"].astype(np.float64).copy()
    mod[1] = -1.0 - e0[0, 1]          # scale_msa = -1
    mod[2] = 1.0 - e0[0, 2]           # gate_msa = 1
    mod[5] = -e0[0, 5]                # FFN off
    W2 = _with(W, 0, mod=mod, wco=np.zeros((D, D)), bco=np.zeros(D))
    y = om.block_forward(W2, 0, x, a, e0, "f64")
    shift = mod[0] + e0[0, 0]
    v = p["wv"].astype(np.float64) @ shift + p["bv"]
    branch = p["wo"].astype(np.float64) @ v + p["bo"]
    assert np.max(np.abs(y[0] - x[0] - branch[None])) < 1e-10


# ---------------------------------------------------------------------------
# sampler
# ---------------------------------------------------------------------------
TINY = om.Config(dim=256, heads=2, ffn=512, blocks=2, latent_ch=16, frames=5, lat_h=4, lat_w=4,
                 audio_tokens=8, bf16=False)


def test_sampler_constant_velocity_is_exact_and_pins_motion():
    cfg = TINY
    W = om.make_weights(cfg, 5)
    c = si.normal(5, 77, (cfg.latent_ch,)).astype(np.float32)
    W.glob["head_w"] = np.zeros_like(W.glob["head_w"])
    W.glob["head_b"] = c
    noise, ref, motion, audio = si.slice_inputs(5, 1, cfg.latent_ch, cfg.frames, cfg.lat_h,
                                                cfg.lat_w, cfg.audio_tokens, cfg.dim, False)
    sig = [1.0, 0.75, 0.5, 0.25, 0.0]
    out = om.sample_slice(W, noise, ref, motion, audio, sig, "f64")
    assert np.array_equal(out[:, :, :2], motion)
    expect = noise[:, :, 2:] - c[None, :, None, None, None].astype(np.float64)
    assert np.max(np.abs(out[:, :, 2:] - expect)) < 1e-12


def test_sampler_matches_manual_euler_steps():
    cfg = TINY
    W = om.make_weights(cfg, 6)
    noise, ref, motion, audio = si.slice_inputs(6, 1, cfg.latent_ch, cfg.frames, cfg.lat_h,
                                                cfg.lat_w, cfg.audio_tokens, cfg.dim, False)
    sig = [1.0, 0.6, 0.0]
    out = om.sample_slice(W, noise, ref, motion, audio, sig, "f64")
    x = noise.astype(np.float64).copy()
    for s in range(2):
        x[:, :, :2] = motion
        v = om.predict_flow(W, x, ref, audio, sig[s], "f64")
        x = x + (sig[s + 1] - sig[s]) * v
    x[:, :, :2] = motion
    assert np.max(np.abs(out - x)) < 1e-12


def test_renoise_with_the_current_noise_estimate_is_the_euler_step():
    """On the linear noise path x = (1 - s) x0 + s e the velocity is v = e - x0, so the
    noise the flow implies is e_hat = x0_hat + v. Re-noising with e_hat must land exactly
    where the Euler step x + (s' - s) v does: a dropped term, a flipped sign or swapped
    sigmas in the re-noising update breaks this."""
    rng = np.random.default_rng(11)
    x = rng.standard_normal((3, 7, 5))
    v = rng.standard_normal((3, 7, 5))
    for s, s2 in [(1.0, 0.75), (0.75, 0.5), (0.5, 0.25), (0.3, 0.0)]:
        e_hat = (x - s * v) + v
        got = om.renoise_update(x, v, s, s2, e_hat)
        assert np.allclose(got, x + (s2 - s) * v, rtol=0, atol=1e-12)


def test_renoise_with_the_exact_velocity_returns_a_fresh_point_of_the_path():
    """For x on the path between a clean sample x0 and noise e at level s, and the exact
    velocity e - x0, the update recovers x0 and re-noises it with the fresh draw: the
    result is (1 - s') x0 + s' e_fresh, whatever e was."""
    rng = np.random.default_rng(12)
    x0, e, e_fresh = (rng.standard_normal((4, 9)) for _ in range(3))
    for s, s2 in [(1.0, 0.75), (0.6, 0.2), (0.25, 0.0)]:
        x = (1 - s) * x0 + s * e
        got = om.renoise_update(x, e - x0, s, s2, e_fresh)
        assert np.allclose(got, (1 - s2) * x0 + s2 * e_fresh, rtol=0, atol=1e-12)


def test_renoise_sampler_single_final_step_is_euler_and_ignores_the_draw():
    """With sigmas (s, 0) the re-noising sampler takes one step to sigma 0, which puts no
    weight on the fresh draw: the output equals the Euler sampler's for any draw,
    bitwise in float64, and the motion frames are the motion latent."""
    W = om.make_weights(TINY, 31)
    noise, ref, motion, audio = si.slice_inputs(32, 1, TINY.latent_ch, TINY.frames, TINY.lat_h, TINY.lat_w,
                                                TINY.audio_tokens, TINY.dim, False)
    sig = [0.6, 0.0]
    euler = om.sample_slice(W, noise, ref, motion, audio, sig, "f64")
    for seed in (1, 2):
        eps = si.renoise_draws(seed, 1, 1, TINY.latent_ch, TINY.frames, TINY.lat_h, TINY.lat_w)
        got = om.sample_slice_renoise(W, noise, ref, motion, audio, sig, eps, "f64")
        assert np.array_equal(got, euler)
        assert np.array_equal(got[:, :, :2], motion)


def test_renoise_sampler_matches_manual_steps():
    """The sampler applies the update after each network call with that step's own draw
    (eps[s] at step s, not another step's), pinning the motion frames before each call."""
    W = om.make_weights(TINY, 33)
    noise, ref, motion, audio = si.slice_inputs(34, 1, TINY.latent_ch, TINY.frames, TINY.lat_h, TINY.lat_w,
                                                TINY.audio_tokens, TINY.dim, False)
    sig = [1.0, 0.7, 0.3, 0.0]
    eps = si.renoise_draws(35, 3, 1, TINY.latent_ch, TINY.frames, TINY.lat_h, TINY.lat_w)
    e64 = eps.astype(np.float64)
    x = noise.astype(np.float64)
    for s in range(3):
        x = om.pin_motion(x, motion)
        v = om.predict_flow(W, x, ref, audio, sig[s], "f64")
        x = (1 - sig[s + 1]) * (x - sig[s] * v) + sig[s + 1] * e64[s]
    want = om.pin_motion(x, motion)
    got = om.sample_slice_renoise(W, noise, ref, motion, audio, sig, eps, "f64")
    assert np.allclose(got, want, rtol=0, atol=1e-12)
    # a different draw for the middle step changes the result
    eps2 = eps.copy()
    eps2[1] = -eps2[1]
    assert not np.allclose(om.sample_slice_renoise(W, noise, ref, motion, audio, sig, eps2, "f64"), want)


@pytest.mark.parametrize("mistake", ["dropped_keep_factor", "swapped_sigmas", "plus_sigma_v"])
def test_planted_renoise_mistakes_are_caught(mistake):
    """Each plausible slip in the re-noising update, planted in a copy of it, breaks the
    Euler identity that the pins above check."""
    def wrong(x, v, s, s2, e):
        if mistake == "dropped_keep_factor":
            return (x - s * v) + s2 * e
        if mistake == "swapped_sigmas":
            return (1 - s) * (x - s2 * v) + s * e
        return (1 - s2) * (x + s * v) + s2 * e
    rng = np.random.default_rng(13)
    x, v = rng.standard_normal((2, 6, 4))
    s, s2 = 0.75, 0.5
    e_hat = (x - s * v) + v
    euler = x + (s2 - s) * v
    assert np.allclose(om.renoise_update(x, v, s, s2, e_hat), euler, rtol=0, atol=1e-12)
    assert not np.allclose(wrong(x, v, s, s2, e_hat), euler, rtol=0, atol=1e-6)


def test_predict_flow_token_order():
    """Patchify / unpatchify are inverse and use token n = f*H*W + h*W + w."""
    lat = si.normal(3, 3, (2, 4, 3, 2, 5))
    tok = om.patchify(lat)
    assert tok.shape == (2, 30, 4)
    assert tok[1, 1 * 10 + 1 * 5 + 3, 2] == lat[1, 2, 1, 1, 3]
    cfg = om.Config(latent_ch=4, frames=3, lat_h=2, lat_w=5)
    assert np.array_equal(om.unpatchify(tok, cfg), lat)


# ---------------------------------------------------------------------------
# mutation checks: plausible mistakes planted in the oracle fail the pins
# ---------------------------------------------------------------------------
def test_planted_rope_half_split_is_caught(cfg0_case, monkeypatch):
    cfg, W, x, a, t = cfg0_case

    def half_split(xx, ang):
        c = np.cos(ang)[:, None, :]
        s = np.sin(ang)[:, None, :]
        h = xx.shape[-1] // 2
        out = np.empty_like(xx)
        out[..., :h] = xx[..., :h] * c - xx[..., h:] * s
        out[..., h:] = xx[..., :h] * s + xx[..., h:] * c
        return out

    monkeypatch.setattr(om, "apply_rope", half_split)
    y = _block(W, x, a, t)
    yb = brute.block_tokens(W, 0, x[0], a[0], float(t[0]), [5, 77])
    assert rel(y[0, [5, 77]], yb) > 1e-4


def test_planted_per_head_qk_norm_is_caught(cfg0_case, monkeypatch):
    cfg, W, x, a, t = cfg0_case
    orig = om.rms_norm

    def per_head(xx, eps):
        xx = np.asarray(xx, dtype=np.float64)
        if xx.shape[-1] == cfg.dim:
            s = xx.reshape(*xx.shape[:-1], cfg.heads, cfg.head_dim)
            return orig(s, eps).reshape(xx.shape)
        return orig(xx, eps)

    monkeypatch.setattr(om, "rms_norm", per_head)
    y = _block(W, x, a, t)
    yb = brute.block_tokens(W, 0, x[0], a[0], float(t[0]), [5, 77])
    assert rel(y[0, [5, 77]], yb) > 1e-4


def test_planted_cross_frame_leak_is_caught(cfg0_case, monkeypatch):
    cfg, W, x, a, t = cfg0_case

    def all_frames(q, k, v, frames, scale):
        B, L, NH, hd = q.shape
        kk = k.reshape(B, -1, NH, hd)
        vv = v.reshape(B, -1, NH, hd)
        return om.self_attention(q, kk, vv, scale)

    monkeypatch.setattr(om, "frame_cross_attention", all_frames)
    y = _block(W, x, a, t)
    yb = brute.block_tokens(W, 0, x[0], a[0], float(t[0]), [5, 77])
    assert rel(y[0, [5, 77]], yb) > 1e-4


# ---------------------------------------------------------------------------
# flow prediction: patch embed, output norm with the head mods, head Linear
# ---------------------------------------------------------------------------
PRED = om.Config(dim=256, heads=2, ffn=512, blocks=2, latent_ch=16, frames=3, lat_h=4, lat_w=4,
                 audio_tokens=8, bf16=False)
PRED_SIGMA = 0.6


@pytest.fixture(scope="module")
def pred_case():
    W = om.make_weights(PRED, 41)
    noise, ref, _, audio = si.slice_inputs(42, 1, PRED.latent_ch, PRED.frames, PRED.lat_h, PRED.lat_w,
                                           PRED.audio_tokens, PRED.dim, False)
    vb = brute.predict_flow(W, noise[0], ref[0], audio[0], PRED_SIGMA)
    return W, noise, ref, audio, vb


def _pred(W, noise, ref, audio):
    return om.predict_flow(W, noise, ref, audio, PRED_SIGMA, "f64")[0]


def test_conditioning_matches_brute_force(pred_case):
    W = pred_case[0]
    e, e0 = om.time_conditioning(W, np.array([PRED_SIGMA]), "f64")
    eb, e0b = brute._conditioning(W, PRED_SIGMA)
    assert rel(e[0], eb) < 1e-12
    assert rel(e0[0], e0b) < 1e-12


def test_predict_flow_matches_float64_brute_force(pred_case):
    """The whole prediction (patch embed over [noisy | ref], two blocks, RMSNorm with the
    head mods = head table + e, head Linear, token order) against the per-token brute force."""
    W, noise, ref, audio, vb = pred_case
    assert rel(_pred(W, noise, ref, audio), vb) < 1e-10


def _head_variant(kind):
    """A copy of the oracle's output head with one plausible slip planted in it."""
    def head(W, x, hm, prec):
        dt = om._dt(prec)
        shift, scl = hm[:, 0, None, :], hm[:, 1, None, :]
        if kind == "layer_norm":
            hn = om.layer_norm(x, W.cfg.eps) * (1.0 + scl) + shift
        elif kind == "dropped_one":
            hn = om.rms_norm(x, W.cfg.eps) * scl + shift
        elif kind == "swapped_shift_scale":
            hn = om.rms_norm(x, W.cfg.eps) * (1.0 + shift) + scl
        elif kind == "shift_before_norm":
            hn = om.rms_norm(x + shift, W.cfg.eps) * (1.0 + scl)
        else:
            raise ValueError(kind)
        return om.linear(hn.astype(dt), W.glob["head_w"], W.glob["head_b"], prec)
    return head


@pytest.mark.parametrize("kind", ["layer_norm", "dropped_one", "swapped_shift_scale", "shift_before_norm"])
def test_planted_output_head_mistakes_are_caught(pred_case, monkeypatch, kind):
    W, noise, ref, audio, vb = pred_case
    monkeypatch.setattr(om, "output_head", _head_variant(kind))
    assert rel(_pred(W, noise, ref, audio), vb) > 1e-4


def test_planted_reversed_concat_is_caught(pred_case, monkeypatch):
    W, noise, ref, audio, vb = pred_case

    def ref_first(W_, x_noisy, ref_, prec):
        tok = np.concatenate([om.patchify(ref_), om.patchify(x_noisy)], axis=2)
        return om.linear(tok.astype(om._dt(prec)), W_.glob["patch_w"], W_.glob["patch_b"], prec)

    monkeypatch.setattr(om, "patch_embed", ref_first)
    assert rel(_pred(W, noise, ref, audio), vb) > 1e-4


def test_planted_e0_for_e_in_head_mods_is_caught(pred_case, monkeypatch):
    """The head mods taking the block conditioning e0 (its first row) instead of e."""
    W, noise, ref, audio, vb = pred_case
    orig = om.time_conditioning

    def e0_as_e(W_, t, prec):
        e, e0 = orig(W_, t, prec)
        return e0[:, 0, :].copy(), e0

    monkeypatch.setattr(om, "time_conditioning", e0_as_e)
    assert rel(_pred(W, noise, ref, audio), vb) > 1e-4


# ---------------------------------------------------------------------------
# audio projection (readings R19-R21)
# ---------------------------------------------------------------------------
ACFG = om.Config(dim=256, heads=2, ffn=512, blocks=1, frames=5, lat_h=2, lat_w=2, bf16=False)
AUD = om.AudioConfig(states=60, layers=3, channels=16, hidden=24, tokens=4)


@pytest.fixture(scope="module")
def audio_case():
    AW = om.make_audio_weights(ACFG, 51, AUD)
    st = si.speech_states(52, 2, AUD.states, AUD.layers, AUD.channels)
    yb = brute.audio_tokens(AW, st[1], ACFG, AUD)
    return AW, st, yb


def test_audio_page_facts():
    """33 video frames per slice make 5 latent frames (1 + 4 x 8); the last video frame is the
    last of the 200 encoder states, 8 s at 25 per second; 5 states per video frame."""
    facts = json.load(open(GOLDEN))
    a = om.AUDIO
    assert a.video_frames(om.CFG3.frames) == facts["decoded_frames_per_slice"]["value"]
    assert a.states == facts["speech_encoder_states"]["value"]
    assert a.states == facts["audio_window_s"]["value"] * facts["fps"]["value"]
    assert a.layers == facts["speech_encoder_layers"]["value"]
    assert a.window == facts["states_per_video_frame"]["value"]
    assert a.tokens == om.CFG3.audio_tokens
    first, later = om.audio_windows(np.arange(a.states, dtype=np.float64).reshape(1, a.states, 1, 1), 5)
    assert list(first.reshape(-1)) == [165, 166, 167, 168, 169]
    assert later.shape[1:3] == (4, 12)
    assert list(later[0, 3].reshape(-1)) == [190, 191, 192, 193, 194, 195, 196, 197, 198, 199, 199, 199]


def test_audio_projection_matches_float64_brute_force(audio_case):
    AW, st, yb = audio_case
    y = om.audio_projection(AW, st, ACFG, "f64", AUD)
    assert y.shape == (2, ACFG.frames, AUD.tokens, ACFG.dim)
    assert rel(y[1], yb) < 1e-10


def test_audio_projection_zero_proj3_gives_the_norm_bias(audio_case):
    """A token of zeros normalises to zero, so the output is projNorm's bias."""
    AW, st, _ = audio_case
    AW2 = dict(AW, proj3_w=np.zeros_like(AW["proj3_w"]), proj3_b=np.zeros_like(AW["proj3_b"]))
    y = om.audio_projection(AW2, st, ACFG, "f64", AUD)
    assert np.max(np.abs(y - AW["projnorm_b"].astype(np.float64))) < 1e-12


def test_audio_projection_reads_only_its_window(audio_case):
    """States before every window change nothing; a state near the end changes only the latent
    frames whose windows hold it (frames 3 and 4 of 5 for the state two before the last)."""
    AW, st, _ = audio_case
    y = om.audio_projection(AW, st, ACFG, "f64", AUD)
    nv = AUD.video_frames(ACFG.frames)
    st2 = st.copy()
    st2[:, :AUD.states - nv - 2] += 3.0
    assert np.array_equal(om.audio_projection(AW, st2, ACFG, "f64", AUD), y)
    st3 = st.copy()
    st3[:, AUD.states - 3] += 1.0
    y3 = om.audio_projection(AW, st3, ACFG, "f64", AUD)
    assert np.array_equal(y3[:, :3], y[:, :3])
    assert np.max(np.abs(y3[:, 3:] - y[:, 3:])) > 1e-6


def _audio_variant(kind):
    """A copy of the oracle's projection with one plausible slip planted in it."""
    def windows(states, F, a=om.AUDIO):
        nv = a.video_frames(F)
        s0 = a.states - nv + (1 if kind == "window_off_by_one" else 0)
        half = a.window // 2
        first = states[:, np.clip(np.arange(s0 - half, s0 + half + 1), 0, a.states - 1)]
        later = []
        for j in range(1, F):
            lo = s0 + a.stride * j - (0 if kind == "group_shift" else a.stride - 1) - half
            later.append(states[:, np.clip(np.arange(lo, lo + a.group_states()), 0, a.states - 1)])
        return first, np.stack(later, axis=1)

    def proj(AW, states, cfg, prec, a=om.AUDIO):
        B, F = states.shape[0], cfg.frames
        first, later = windows(np.asarray(states, dtype=np.float64), F, a)
        h0 = om.linear(first.reshape(B, -1), AW["proj1_w"], AW["proj1_b"], "f64")
        hv = om.linear(later.reshape(B * (F - 1), -1), AW["proj1vf_w"], AW["proj1vf_b"], "f64")
        h = np.concatenate([h0[:, None], hv.reshape(B, F - 1, -1)], axis=1)
        act = (lambda v: v) if kind == "no_relu" else (lambda v: np.maximum(v, 0))
        h = act(h)
        h = act(om.linear(h.reshape(B * F, -1), AW["proj2_w"], AW["proj2_b"], "f64"))
        t = om.linear(h, AW["proj3_w"], AW["proj3_b"], "f64").reshape(B, F, a.tokens, cfg.dim)
        y = om.layer_norm(t, cfg.eps)
        if kind != "norm_without_affine":
            y = y * AW["projnorm_w"] + AW["projnorm_b"]
        return y
    return proj


@pytest.mark.parametrize("kind", ["window_off_by_one", "group_shift", "no_relu", "norm_without_affine"])
def test_planted_audio_projection_mistakes_are_caught(audio_case, kind):
    AW, st, yb = audio_case
    y = _audio_variant(kind)(AW, st, ACFG, "f64", AUD)
    assert rel(y[1], yb) > 1e-4
