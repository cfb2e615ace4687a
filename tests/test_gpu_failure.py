"""Failure detection without a GPU fault: a kernel wait that nothing satisfies runs out
its bound, the error is latched and reported on the host, and the context stays usable."""
import time

import numpy as np
import pytest

import synth_inputs as si

torch = pytest.importorskip("torch")
pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

import audio_driven_talking_b200 as fh  # noqa: E402


def test_bounded_wait_runs_out_and_is_reported_once():
    m = fh.DiT(fh.FP32_BLOCK, seed=0)
    ws = m.workspace(1)
    x, a, t = si.block_inputs(0, 1, fh.FP32_BLOCK.tokens, 384, 2, 32, False)
    xd, ad = torch.from_numpy(x).cuda(), torch.from_numpy(a).cuda()
    before = m.block_forward(0, xd, ad, list(t), ws)
    m.sync()
    t0 = time.time()
    m.probe_wait_timeout()
    with pytest.raises(fh.FHError) as e:
        m.sync()
    assert e.value.code == fh.FH_ERR_TIMEOUT
    assert 0.5 < time.time() - t0 < 30.0          # about the 1 s bound, not a hang
    m.sync()                                        # reported once, then cleared
    after = m.block_forward(0, xd, ad, list(t), ws)  # the context still works
    m.sync()
    assert torch.equal(before, after)
    m.close()
