"""The oracle reproduces its frozen outputs (tests/golden/oracle_small.json)."""

import json
import os

import numpy as np

from oracle import kivi, params as P, qjl

GOLD = os.path.join(os.path.dirname(__file__), "golden", "oracle_small.json")


def test_oracle_matches_frozen_fixture():
    data = json.load(open(GOLD))
    for c in data["cases"]:
        proj = P.make_projection(c["seed"], c["d"], c["m"], c["kind"])
        K = np.array(c["keys"], dtype=np.float32)
        words, norms, _ = qjl.quantize_keys(proj, K, c["first_token"])
        assert words.tolist() == c["words"]
        assert np.allclose(norms, c["norms"], rtol=1e-15)
        sq = qjl.project_queries(proj, np.array(c["queries"], dtype=np.float32))
        assert np.allclose(sq, c["sq"], rtol=1e-13, atol=1e-13)
        est = qjl.scores(proj, words[None], norms[None], sq[None])[0]
        assert np.allclose(est, c["scores"], rtol=1e-13, atol=1e-13)
    v = data["values"]
    codes, scale, zero = kivi.quantize_values_2bit(np.array(v["v"], dtype=np.float32))
    assert codes.tolist() == v["codes"]
    assert scale.astype(np.float64).tolist() == v["scale"]
    assert zero.astype(np.float64).tolist() == v["zero"]
