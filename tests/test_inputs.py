"""The router-gap input rule (CPU): every token's 2nd-vs-3rd fp64 logit gap exceeds 1e-3."""
import numpy as np

import oracle
from helpers import GAP, gap_inputs, workload


def test_gap_rule_tiny_and_decode():
    for name in ("tiny", "v01_decode"):
        wl = workload(name)
        inp = gap_inputs(wl)
        _, _, z = oracle.route(inp["x"], inp["wr"], inp["bias"], want_logits=True)
        zs = -np.sort(-z, axis=1)
        assert np.all(zs[:, 1] - zs[:, 2] > GAP)
        assert np.array_equal(inp["attempts"] > 0, inp["attempts"] != 0)


def test_gap_rule_skewed_bias():
    wl = workload("skewed", T=2048)
    inp = gap_inputs(wl)
    ids, _ = oracle.route(inp["x"], inp["wr"], inp["bias"])
    share = np.mean(np.isin(ids, [3, 11]))
    assert 0.4 < share < 0.7  # the +2.0 bias pulls about half of all assignments onto experts 3 and 11
