"""Write ``oracle_small.json``: a regression fixture for the fp64 oracle.

The pages print no worked numeric example of the Gated Delta Rule-2, so the
only stored values here are the oracle's own, written by this script (which
calls nothing but ``oracle/``). The fixture guards against unintended changes
to the oracle's arithmetic; the pins in ``tests/oracle_pins.py`` are what tie
the oracle to the pages.

Run from the repository root:  python tests/golden/make_golden.py
"""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)
import oracle  # noqa: E402


def case():
    rng = np.random.default_rng(20260525)
    B, T, H, dk, dv = 1, 10, 2, 4, 3
    q = rng.standard_normal((B, T, H, dk))
    k = rng.standard_normal((B, T, H, dk))
    q /= np.linalg.norm(q, axis=-1, keepdims=True)
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((B, T, H, dv))
    la = -np.log1p(np.exp(rng.standard_normal((B, T, H, dk))))
    b = 1 / (1 + np.exp(-rng.standard_normal((B, T, H, dk))))
    w = 1 / (1 + np.exp(-rng.standard_normal((B, T, H, dv))))
    S0 = rng.standard_normal((B, H, dk, dv)) * 0.5
    dO = rng.standard_normal((B, T, H, dv))
    return dict(q=q, k=k, v=v, log_alpha=la, b=b, w=w, S0=S0, dO=dO)


def main():
    x = case()
    o, ST = oracle.forward(x["q"], x["k"], x["v"], x["log_alpha"], x["b"], x["w"], S0=x["S0"])
    g = oracle.backward(x["q"], x["k"], x["v"], x["log_alpha"], x["b"], x["w"], x["dO"], S0=x["S0"])
    out = {"source": "oracle/ (fp64), tests/golden/make_golden.py",
           "inputs": {n: a.tolist() for n, a in x.items()},
           "o": o.tolist(), "S_T": ST.tolist(), "grads": {n: a.tolist() for n, a in g.items()}}
    with open(os.path.join(os.path.dirname(os.path.abspath(__file__)), "oracle_small.json"), "w") as f:
        json.dump(out, f)


if __name__ == "__main__":
    main()
