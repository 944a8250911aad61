"""Write tests/golden/oracle_small.json from the oracle alone.

The pages print no worked example of any step: no sketch, no estimate, no
value code. This fixture freezes the oracle's own outputs on tiny seeded
inputs, so that a later change to the oracle's arithmetic shows up as a
diff. The commit that makes such a change must name the passage that
justifies it. Run from the repository root:  python tests/golden/make_golden.py
"""

import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

from oracle import attention, kivi, params as P, qjl  # noqa: E402

OUT = os.path.join(os.path.dirname(os.path.abspath(__file__)), "oracle_small.json")


def case(kind, d, m, seed, n=5, nq=2, first_token=0):
    rng = np.random.default_rng(1000 + seed)
    K = rng.standard_normal((n, d)).astype(np.float32)
    Q = rng.standard_normal((nq, d)).astype(np.float32)
    proj = P.make_projection(seed, d, m, kind)
    words, norms, Y = qjl.quantize_keys(proj, K, first_token)
    sq = qjl.project_queries(proj, Q)
    est = qjl.scores(proj, words[None], norms[None], sq[None])[0]
    return {
        "kind": kind, "d": d, "m": m, "seed": seed, "first_token": first_token,
        "keys": K.tolist(), "queries": Q.tolist(),
        "words": [[int(w) for w in row] for row in words],
        "norms": norms.tolist(), "sq": sq.tolist(), "scores": est.tolist(),
        "min_abs_presign_over_norm": float(np.min(np.abs(Y) / norms[:, None])),
    }


def main():
    rng = np.random.default_rng(7)
    V = rng.standard_normal((3, 64)).astype(np.float32)
    codes, scale, zero = kivi.quantize_values_2bit(V)
    # KIVI per-channel keys: one 32-token block and a ragged block of 8
    Kk = (rng.standard_normal((1, 40, 32)) * 2).astype(np.float32)
    kc, ks, kz = kivi.quantize_keys_per_channel(Kk)
    Qk = rng.standard_normal((1, 2, 32)).astype(np.float32)
    ksc = kivi.key_scores(kc, ks, kz, Qk.astype(np.float64))
    # causal prefill over given scores and values
    est = rng.standard_normal((1, 6, 6)) * 2
    vh = rng.standard_normal((1, 6, 4))
    pout, _ = attention.prefill_attention(est, vh, 0.5)
    data = {
        "note": "oracle outputs on tiny seeded inputs; written by make_golden.py",
        "cases": [case(P.KIND_DENSE, 8, 32, 1), case(P.KIND_DFQJL, 8, 32, 2, first_token=40),
                  case(P.KIND_PFQJL, 16, 64, 3)],
        "values": {"v": V.tolist(), "codes": [[int(w) for w in r] for r in codes],
                   "scale": scale.astype(np.float64).tolist(), "zero": zero.astype(np.float64).tolist()},
        "kivi_keys": {"k": Kk.tolist(), "q": Qk.tolist(), "codes": kc.astype(np.int64).tolist(),
                      "scale": ks.astype(np.float64).tolist(), "zero": kz.astype(np.float64).tolist(),
                      "scores": ksc.tolist()},
        "prefill": {"est": est.tolist(), "vhat": vh.tolist(), "scale": 0.5, "out": pout.tolist()},
    }
    with open(OUT, "w") as f:
        json.dump(data, f, indent=1)


if __name__ == "__main__":
    main()
