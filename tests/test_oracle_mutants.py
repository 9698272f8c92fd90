"""Plant plausible mistakes in a copy of the oracle and check the pins catch each one.

The mistakes go into a temporary copy of oracle/ssm_oracle.c, built on the CPU;
the real oracle is untouched.
"""
import os
import subprocess

import pytest

import oracle
from bwd_pins import BWD_PINS
from conv1d_pins import CONV_PINS
from oracle_pins import ALL_PINS

SRC = os.path.join(os.path.dirname(oracle.__file__), "ssm_oracle.c")

# (name, exact text in the oracle, replacement)
MUTANTS = [
    ("drop dt from input term", "dt * Bg[n * L + t] * u[t]", "Bg[n * L + t] * u[t]"),
    ("wrong sign in discretisation", "exp(dt * a)", "exp(-dt * a)"),
    ("B and C swapped in readout", "y += Cg[n * L + t] * h[n];", "y += Bg[n * L + t] * h[n];"),
    ("readout before the update", "h[n] = dA * h[n] + dt * Bg[n * L + t] * u[t];\n            y += Cg[n * L + t] * h[n];",
     "y += Cg[n * L + t] * h[n];\n            h[n] = dA * h[n] + dt * Bg[n * L + t] * u[t];"),
    ("dropped D skip", "y += Dd * u[t];", ""),
    ("D skip uses gate input", "y += Dd * u[t];", "y += Dd * (z ? z[t] : u[t]);"),
    ("softplus without log1p", "return log1p(exp(x));", "return exp(x);"),
    ("bias dropped", "double x = dl[t] + bias;", "double x = dl[t];"),
    ("gate is sigmoid", "return z / (1.0 + exp(-z));", "return 1.0 / (1.0 + exp(-z));"),
    ("A index transposed", "j->A[d * N + n]", "j->A[n * Dm + d % N]"),
    ("head index from modulo", "hd = d / (Dm / H)", "hd = d % H"),
    ("group index from modulo", "g = d / (Dm / G)", "g = d % G"),
    ("B time index off by one", "Bg[n * L + t] * u[t]", "Bg[n * L + (t ? t - 1 : 0)] * u[t]"),
    ("initial state ignored", "h[n] = j->h0 ? j->h0[row * N + n] : 0.0;", "h[n] = 0.0;"),
    ("state not decayed", "h[n] = dA * h[n] +", "h[n] = h[n] +"),
    ("u squared", "* u[t];\n            y +=", "* u[t] * u[t];\n            y +="),
    # the causal convolution
    ("conv taps reversed", "v += wr[k] * xr[s];", "v += wr[width - 1 - k] * xr[s];"),
    ("conv shifted by one step", "const int64_t s = t - (width - 1) + k;", "const int64_t s = t - width + k;"),
    ("conv not causal (centred)", "const int64_t s = t - (width - 1) + k;", "const int64_t s = t - (width - 1) / 2 + k;"),
    ("conv bias dropped", "double v = bias ? bias[d] : 0.0;", "double v = 0.0;"),
    ("conv activation sigmoid", "orow[t] = silu ? v / (1.0 + exp(-v)) : v;", "orow[t] = silu ? 1.0 / (1.0 + exp(-v)) : v;"),
    # the backward scan
    ("bwd dt drops the decay term", "ddt += gs[n] * Bg[n * L + t] * u[t] + gdA * a * dA;",
     "ddt += gs[n] * Bg[n * L + t] * u[t];"),
    ("bwd state gradient not decayed", "gs[n] = dA * gs[n];", ""),
    ("bwd decay gradient uses h_t", "const double gdA = gs[n] * hp[n];", "const double gdA = gs[n] * hc[n];"),
    ("bwd softplus derivative dropped", "const double sp = j->softplus ? sigmoid_f64(x) : 1.0;",
     "const double sp = 1.0;"),
    ("bwd dB without dt", "j->g.dB[bc] += gs[n] * dt * u[t];", "j->g.dB[bc] += gs[n] * u[t];"),
    ("bwd dC from the previous state", "j->g.dC[bc] += dy * hc[n];", "j->g.dC[bc] += dy * hp[n];"),
    ("bwd dz through silu itself", "j->g.dz[row * L + t] = go[t] * y * dsilu;",
     "j->g.dz[row * L + t] = go[t] * y * silu_f64(z[t]);"),
    ("bwd readout gradient not added", "gs[n] += dy * Cg[n * L + t];", ""),
    ("bwd dlast ignored", "gs[n] = j->dlast ? j->dlast[row * N + n] : 0.0;", "gs[n] = 0.0;"),
    ("bwd du misses the skip", "double du = dy * Dd,", "double du = 0.0 * Dd,"),
    ("bwd dA without dt", "j->g.dA[ai] += gdA * dt * dA;", "j->g.dA[ai] += gdA * dA;"),
    ("bwd gate gradient ungated", "const double dy = go[t] * gate;", "const double dy = go[t];"),
]


def _build_mutant(tmp_path, name, old, new):
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation site for '{name}' not found"
    mutated = src.replace(old, new, 1)
    assert mutated != src
    c = tmp_path / "mutant.c"
    so = tmp_path / "mutant.so"
    c.write_text(mutated)
    subprocess.check_call(["gcc", "-O1", "-fPIC", "-shared", "-ffp-contract=off", "-o", str(so), str(c),
                           "-lm", "-lpthread"])
    return oracle.load(str(so))


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(tmp_path, name, old, new):
    lib = _build_mutant(tmp_path, name, old, new)
    caught = []
    for pin in ALL_PINS + CONV_PINS + BWD_PINS:
        try:
            pin(lib)
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"no pin catches the mutant '{name}'"
