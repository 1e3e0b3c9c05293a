"""The oracle against its committed snapshot (tests/golden/tiny_fp32_round.json).

The snapshot was written by tests/golden/make_tiny_round.py from the oracle
alone; this is a regression guard for the oracle (its pins are in
test_oracle_pins.py): tokens and lengths must match exactly, the fp64 values to
1e-9 relative (summation order of the BLAS build only).
"""
import importlib.util
import json
import os

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))


def _load_maker():
    spec = importlib.util.spec_from_file_location("make_tiny_round", os.path.join(HERE, "golden", "make_tiny_round.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_oracle_reproduces_tiny_round_snapshot():
    with open(os.path.join(HERE, "golden", "tiny_fp32_round.json")) as fh:
        want = json.load(fh)
    got = _load_maker().tiny_round()
    for key in ("anchors", "tokens", "lengths", "logits_top5_index"):
        assert got[key] == want[key], key
    for key in ("conf", "logits_top5_value", "logits_row_sum", "k_ctx_layer0_row0", "v_ctx_layer0_row0"):
        np.testing.assert_allclose(np.asarray(got[key]), np.asarray(want[key]), rtol=1e-9, atol=1e-12, err_msg=key)
