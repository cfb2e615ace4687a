"""The stored full-size oracle outputs (tests/golden/expected_*.npz) were written by
tests/golden/make_expected.py from the current oracle and input generator."""
import glob
import importlib.util
import os

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))


def _maker():
    spec = importlib.util.spec_from_file_location("make_expected", os.path.join(HERE, "golden", "make_expected.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_stored_oracle_outputs_match_current_oracle_source():
    mk = _maker()
    files = sorted(glob.glob(os.path.join(HERE, "golden", "expected_*.npz")))
    assert files, "no stored oracle outputs"
    for f in files:
        d = np.load(f)
        assert str(d["oracle_hash"]) == mk.oracle_hash(), f"{os.path.basename(f)} is stale: rerun make_expected.py"
        assert str(d["prec"]) == "f32"
        assert np.all(np.isfinite(d["out"]))


def test_every_case_is_stored():
    mk = _maker()
    for case in mk.CASES:
        assert os.path.exists(mk.path(case)), case
