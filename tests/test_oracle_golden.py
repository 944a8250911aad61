"""The oracle reproduces its frozen outputs (tests/golden/oracle_small.json)."""

import json
import os

import numpy as np

from oracle import attention, kivi, params as P, qjl

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



def test_kivi_keys_and_prefill_match_frozen_fixture():
    data = json.load(open(GOLD))
    k = data["kivi_keys"]
    codes, scale, zero = kivi.quantize_keys_per_channel(np.array(k["k"], dtype=np.float32))
    assert codes.astype(np.int64).tolist() == k["codes"]
    assert scale.astype(np.float64).tolist() == k["scale"]
    assert zero.astype(np.float64).tolist() == k["zero"]
    sc = kivi.key_scores(codes, scale, zero, np.array(k["q"], dtype=np.float64))
    assert np.allclose(sc, k["scores"], rtol=1e-13, atol=1e-13)
    p = data["prefill"]
    out, _ = attention.prefill_attention(np.array(p["est"]), np.array(p["vhat"]), p["scale"])
    assert np.allclose(out, p["out"], rtol=1e-13, atol=1e-13)
