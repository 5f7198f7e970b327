"""Mutation test of the oracle's pins (CPU only).

Each mutant is a copy of ``oracle/gdr2_oracle.c`` with one plausible mistake
planted in it (a dropped term, a wrong sign, a wrong index or operand, a gate
left out). The pin suite must reject every mutant; a mutant that survives
means the pins would not notice that mistake in the real oracle.
"""
import os

import pytest

import oracle
import oracle_pins as P

SRC = os.path.join(os.path.dirname(oracle.__file__), "gdr2_oracle.c")

# (name, exact text in the oracle, replacement)
MUTANTS = [
    ("erase along e (b squared)",
     "S[(size_t)c * dv + j] += k[c] * (z[j] - r[j]);",
     "S[(size_t)c * dv + j] += k[c] * z[j] - e[c] * r[j];"),
    ("decay dropped",
     "for (int j = 0; j < dv; ++j) S[(size_t)c * dv + j] *= a[c];",
     "for (int j = 0; j < dv; ++j) S[(size_t)c * dv + j] *= 1.0;"),
    ("erase sign flipped", "k[c] * (z[j] - r[j]);", "k[c] * (z[j] + r[j]);"),
    ("decay exponent halved",
     "        a[c] = exp(la[c]);\n        e[c] = b[c] * k[c];",
     "        a[c] = exp(0.5 * la[c]);\n        e[c] = b[c] * k[c];"),
    ("erase gate dropped", "        e[c] = b[c] * k[c];\n    }\n    for (int j = 0; j < dv; ++j) z[j]",
     "        e[c] = k[c];\n    }\n    for (int j = 0; j < dv; ++j) z[j]"),
    ("write gate dropped", "for (int j = 0; j < dv; ++j) z[j] = w[j] * v[j];",
     "for (int j = 0; j < dv; ++j) z[j] = v[j];"),
    ("output read with k", "for (int c = 0; c < dk; ++c) acc += S[(size_t)c * dv + j] * q[c];",
     "for (int c = 0; c < dk; ++c) acc += S[(size_t)c * dv + j] * k[c];"),
    ("read uses a wrong index", "for (int c = 0; c < dk; ++c) acc += S[(size_t)c * dv + j] * e[c];",
     "for (int c = 0; c < dk; ++c) acc += S[(size_t)c * dv + j] * e[j % dk];"),
    ("initial state ignored", "if (S0) memcpy(S, S0 + (size_t)bh * SS, sizeof(double) * SS);",
     "if (0) memcpy(S, S0 + (size_t)bh * SS, sizeof(double) * SS);"),
    ("bwd: erase-gradient sign", "de[c] = -acc;", "de[c] = acc;"),
    ("bwd: decay gradient dropped", "dlat[c] = acc;", "dlat[c] = 0.0 * acc;"),
    ("bwd: key gradient via gate dropped", "dkt[c] += de[c] * bt[c];", "dkt[c] += 0.0 * bt[c];"),
    ("bwd: decay not applied to dS",
     "dS[(size_t)c * dv + j] = a[c] * dSb[(size_t)c * dv + j];",
     "dS[(size_t)c * dv + j] = dSb[(size_t)c * dv + j];"),
    ("bwd: write-gate gradient uses w", "dwt[j] = ddelta[j] * vt[j];", "dwt[j] = ddelta[j] * wt[j];"),
    ("bwd: dq from the previous state", "acc += Scur[(size_t)c * dv + j] * dOt[j];",
     "acc += Sprev[(size_t)c * dv + j] * dOt[j];"),
    ("bwd: erase term left out of dSb", "const double g = dS[(size_t)c * dv + j] - e[c] * ddelta[j];",
     "const double g = dS[(size_t)c * dv + j];"),
]

SUITE = P.ALL_PINS + [P.check_decode_matches_forward]


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(tmp_path, name, old, new):
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor for '{name}' must occur exactly once"
    mpath = tmp_path / "mutant.c"
    mpath.write_text(src.replace(old, new))
    lib = oracle.OracleLib(oracle.compile_library(str(mpath), str(tmp_path / "libmutant.so")))
    caught = []
    for pin in SUITE:
        try:
            pin(lib)
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"mutant '{name}' passed every pin"


# Mistakes planted in the block epilogue (oracle/block.py); pin P12 must reject each.
BLOCK_MUTANTS = [
    ("rms over the sum, not the mean", "np.mean(y * y, axis=-1, keepdims=True)", "np.sum(y * y, axis=-1, keepdims=True)"),
    ("epsilon dropped", "np.sqrt(ms + eps)", "np.sqrt(ms)"),
    ("epsilon outside the root", "np.sqrt(ms + eps)", "(np.sqrt(ms) + eps)"),
    ("sigmoid gate instead of silu", "return x / (1.0 + np.exp(-x))", "return 1.0 / (1.0 + np.exp(-x))"),
    ("gate sign flipped", "y = y * silu(g)", "y = y * silu(-np.asarray(g))"),
    ("weight inside the norm", "y = y / np.sqrt(ms + eps) * np.asarray(weight, dtype=np.float64)",
     "y = y * np.asarray(weight, dtype=np.float64) / np.sqrt(np.mean((y * weight) ** 2, axis=-1, keepdims=True) + eps)"),
]


@pytest.mark.parametrize("name,old,new", BLOCK_MUTANTS, ids=[m[0] for m in BLOCK_MUTANTS])
def test_block_mutant_is_caught(tmp_path, name, old, new):
    import importlib.util

    import oracle_pins as P

    src = open(os.path.join(os.path.dirname(oracle.__file__), "block.py")).read()
    assert src.count(old) == 1, f"mutation site not found: {old}"
    mpath = tmp_path / "block_mutant.py"
    mpath.write_text(src.replace(old, new))
    spec = importlib.util.spec_from_file_location("block_mutant", mpath)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    with pytest.raises(AssertionError):
        P.pin_output_norm_gate(OB=mod)


PROLOGUE_MUTANTS = [
    ("taps reversed", "y += wgt[:, i] * xp[..., i:i + T, :]", "y += wgt[:, W - 1 - i] * xp[..., i:i + T, :]"),
    ("state read newest first",
     "pad = np.zeros(lead + (W - 1, x.shape[-1])) if state is None else np.asarray(state, dtype=np.float64)",
     "pad = np.zeros(lead + (W - 1, x.shape[-1])) if state is None else np.asarray(state, dtype=np.float64)[..., ::-1, :]"),
    ("SiLU dropped", "        y = silu(causal_conv(x, weight, state))", "        y = causal_conv(x, weight, state)"),
    ("L2 epsilon outside the root", "x / np.sqrt(np.sum(x * x, axis=-1, keepdims=True) + eps)",
     "x / (np.sqrt(np.sum(x * x, axis=-1, keepdims=True)) + eps)"),
    ("L2 over all heads together", "y.reshape(sh[:-1] + (heads, sh[-1] // heads))", "y.reshape(sh[:-1] + (1, sh[-1]))"),
    ("softplus of the wrong sign", "-(np.maximum(x, 0.0) + np.log1p(np.exp(-np.abs(x))))",
     "-(np.maximum(-x, 0.0) + np.log1p(np.exp(-np.abs(x))))"),
    ("convolution runs across packed sequences", "y[:, s:e] = silu(causal_conv(x[:, s:e], weight, si))",
     "y[:, s:e] = silu(causal_conv(x, weight, None)[:, s:e])"),
    ("state after a short call ignores the old state",
     "    return np.concatenate([pad, x], axis=-2)[..., x.shape[-2]:, :]",
     "    return np.concatenate([np.zeros_like(pad), x], axis=-2)[..., x.shape[-2]:, :]"),
]


@pytest.mark.parametrize("name,old,new", PROLOGUE_MUTANTS, ids=[m[0] for m in PROLOGUE_MUTANTS])
def test_prologue_mutant_is_caught(tmp_path, name, old, new):
    import importlib.util

    import oracle_pins as P

    src = open(os.path.join(os.path.dirname(oracle.__file__), "block.py")).read()
    assert src.count(old) == 1, f"mutation site not found: {old}"
    mpath = tmp_path / "block_mutant.py"
    mpath.write_text(src.replace(old, new))
    spec = importlib.util.spec_from_file_location("block_mutant", mpath)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    with pytest.raises(AssertionError):
        P.pin_block_prologue(OB=mod)
