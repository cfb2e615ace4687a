"""The no-allocation block forward (fh_dit_block_forward_noalloc) against the
workspace entry point it mirrors.

This entry point is for callers that cannot allocate device memory where they run a
block (plugins inside a host framework that owns all device memory, real-time threads
that must not take the allocator's locks). It runs the same kernels on a static
scratch array inside the library; these tests check, through the C ABI, that two
calls in a row give bitwise what fh_dit_block_forward gives with a caller-allocated
workspace (the kernels are deterministic, so any difference is stale or overlapping
scratch), and that a model too large for the static scratch is refused with a clear
error. The file sorts last so a run that stops at the first failure has run every
other test first; it also passes alone in a fresh process.
"""
import pytest

import synth_inputs as si

torch = pytest.importorskip("torch")
pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

import audio_driven_talking_b200 as fh  # noqa: E402


@pytest.mark.parametrize("which", ["fp32_block", "bf16_small"])
def test_noalloc_block_matches_workspace_entry_twice(which):
    if which == "fp32_block":
        cfg, adt = fh.FP32_BLOCK, torch.float32
    else:
        cfg = fh.ModelConfig(dim=384, heads=3, ffn=1024, blocks=2, frames=3, lat_h=12, lat_w=12)
        adt = torch.bfloat16
    m = fh.DiT(cfg, seed=21)
    assert 0 < m.workspace_bytes(1) <= 16 << 20
    x, a, t = si.block_inputs(22, 1, cfg.tokens, cfg.dim, cfg.frames, cfg.audio_tokens, cfg.dtype == fh.FH_BF16)
    xd, ad = torch.from_numpy(x).cuda(), torch.from_numpy(a).cuda().to(adt)
    ws = m.workspace(1)
    k = cfg.blocks - 1
    ref = m.block_forward(k, xd, ad, list(t), ws)
    m.sync()
    assert torch.isfinite(ref).all() and not torch.equal(ref, xd)
    for _ in range(2):
        got = m.block_forward_noalloc(k, xd, ad, list(t))
        m.sync()
        assert torch.equal(got, ref)
    m.close()


def test_noalloc_refuses_a_model_beyond_the_static_scratch():
    m = fh.DiT(fh.ONE_BLOCK, seed=23)
    assert m.workspace_bytes(1) > 16 << 20
    x = torch.zeros((1, fh.ONE_BLOCK.tokens, 1536), device="cuda")
    a = torch.zeros((1, 5, 32, 1536), device="cuda", dtype=torch.bfloat16)
    with pytest.raises(fh.FHError) as e:
        m.block_forward_noalloc(0, x, a, [0.5])
    assert e.value.code == fh.FH_ERR_SHAPE and "static scratch" in str(e.value)
    m.close()
