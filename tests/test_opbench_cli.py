"""The operator benchmark's command line, on the CPU (no GPU is touched by parsing)."""
import pytest

import audio_driven_talking_b200.opbench as ob


def test_defaults_are_the_models_shapes():
    a = ob.parser().parse_args(["linear"])
    assert (a.m, a.n, a.k) == (1280, 1536, 1536)          # 1280 tokens, width 1536
    a = ob.parser().parse_args(["attention"])
    assert (a.batch, a.heads, a.tokens) == (1, 12, 1280)  # 12 heads over one slice's latent
    a = ob.parser().parse_args(["row_norm"])
    assert a.rows * a.dim * 4 > 3 * 126 * 2 ** 20         # the HBM sweep's input is beyond the 126 MB L2
    assert not a.graph


@pytest.mark.parametrize("op", ["row_norm", "attention", "linear", "cross_attention", "slice", "slice_kernels"])
def test_every_operator_is_accepted(op):
    assert ob.parser().parse_args([op]).op == op


def test_unknown_operator_is_rejected():
    with pytest.raises(SystemExit):
        ob.parser().parse_args(["no_such_op"])
