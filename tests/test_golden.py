"""The oracle still reproduces its stored regression fixture (CPU only)."""
import json
import os

import numpy as np

import oracle

HERE = os.path.dirname(os.path.abspath(__file__))


def test_oracle_regression_fixture():
    with open(os.path.join(HERE, "golden", "oracle_small.json")) as f:
        fx = json.load(f)
    x = {n: np.array(a) for n, a in fx["inputs"].items()}
    o, ST = oracle.forward(x["q"], x["k"], x["v"], x["log_alpha"], x["b"], x["w"], S0=x["S0"])
    np.testing.assert_allclose(o, np.array(fx["o"]), rtol=0, atol=1e-13)
    np.testing.assert_allclose(ST, np.array(fx["S_T"]), rtol=0, atol=1e-13)
    g = oracle.backward(x["q"], x["k"], x["v"], x["log_alpha"], x["b"], x["w"], x["dO"], S0=x["S0"])
    for n, a in fx["grads"].items():
        np.testing.assert_allclose(g[n], np.array(a), rtol=0, atol=1e-12, err_msg=n)
