"""The oracle against a worked example derived by hand (tests/golden/*.json).

The pages print no numeric example, so the fixture is worked out by hand from
the definitions it cites: logits with and without the forget gate, and the
decode cache after the last position. Its H factors do not commute, so a
reversed product order, a dropped gate term or a wrong sign changes an exact
value. Outputs are checked against softmax of the hand-derived logits.
"""
import json
import math
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        g = json.load(f)
    arr = lambda key: np.array(g[key], dtype=np.float64)[None, None]
    return g, arr


def tri(rows):
    return np.array([[-np.inf if x is None else x for x in r] for r in rows])


def softmax_rows(z, v):
    out = np.zeros((z.shape[0], v.shape[1]))
    lse = np.zeros(z.shape[0])
    for i, row in enumerate(z):
        m = max(x for x in row if x != -np.inf)
        s = math.fsum(math.exp(x - m) for x in row if x != -np.inf)
        lse[i] = m + math.log(s)
        for j, x in enumerate(row):
            if x != -np.inf:
                out[i] += math.exp(x - lse[i]) * v[j]
    return out, lse


@pytest.mark.parametrize("gated", [False, True])
def test_hand_worked_logits_and_outputs(orc, gated):
    g, arr = load("hand_worked_d2_l3.json")
    q, k, v, w = arr("q"), arr("k"), arr("v"), arr("w")
    beta = arr("beta")
    log_f = arr("log_f") if gated else None
    z = orc.scores(q, k, w, beta, log_f, scale=g["scale"])[0, 0]
    ref = tri(g["logits_gated" if gated else "logits"])
    np.testing.assert_allclose(z, ref, rtol=0, atol=1e-14)
    out, lse = orc.fwd(q, k, v, w, beta, log_f, scale=g["scale"])
    ro, rl = softmax_rows(ref, np.array(g["v"], dtype=np.float64))
    np.testing.assert_allclose(out[0, 0], ro, rtol=1e-14, atol=1e-15)
    np.testing.assert_allclose(lse[0, 0], rl, rtol=1e-14, atol=1e-15)


def test_hand_worked_prefill_cache(orc):
    g, arr = load("hand_worked_d2_l3.json")
    kc, vc, gc = orc.prefill_cache(arr("k"), arr("v"), arr("w"), arr("beta"), arr("log_f"))
    np.testing.assert_allclose(kc[0, 0], np.array(g["k_cache"], dtype=np.float64), rtol=0,
                               atol=1e-14)
    np.testing.assert_array_equal(vc[0, 0], np.array(g["v"], dtype=np.float64))
    np.testing.assert_allclose(gc[0, 0], np.array(g["g_cache"], dtype=np.float64), rtol=0,
                               atol=1e-14)
