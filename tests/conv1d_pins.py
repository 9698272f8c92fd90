"""Pins of the fp64 causal-conv1d oracle against values and routines other than itself.

* a worked example by hand (tests/golden/conv1d_hand_worked.json);
* numpy's full discrete convolution, truncated to the first seqlen outputs
  (np.convolve(x, w reversed)[:L] is the causal convolution by its definition);
* the impulse response: a unit step at t0 gives w read backwards from t0 on;
* causality: changing x at t0 leaves every output before t0 unchanged;
* the activation: out(silu) = v / (1 + e^-v) with v = out(linear), elementwise.
"""
import json
import math
import os

import numpy as np

import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "conv1d_hand_worked.json")


def _conv(lib, x, w, b=None, silu=False):
    return oracle.causal_conv1d(x, w, b, silu=silu, lib=lib)


def pin_conv_hand_worked(lib):
    g = json.load(open(GOLDEN))
    x = np.array(g["inputs"]["x"], dtype=np.float64).reshape(1, 1, -1)
    w = np.array(g["inputs"]["w"], dtype=np.float64).reshape(1, -1)
    b = np.array([g["inputs"]["bias"]], dtype=np.float64)
    lin = _conv(lib, x, w, b, silu=False).ravel()
    exp_lin = np.array(g["expected_linear"])
    assert np.array_equal(lin, exp_lin), (lin, exp_lin)
    act = _conv(lib, x, w, b, silu=True).ravel()
    exp_act = np.array([v / (1.0 + math.exp(-v)) for v in exp_lin])
    assert np.allclose(act, exp_act, rtol=1e-15, atol=0), (act, exp_act)


def pin_conv_numpy_convolve(lib):
    rng = np.random.default_rng(31)
    for width in (1, 2, 3, 4, 6):
        x = rng.standard_normal((2, 5, 37))
        w = rng.standard_normal((5, width))
        b = rng.standard_normal(5)
        out = _conv(lib, x, w, b)
        for bi in range(2):
            for d in range(5):
                ref = np.convolve(x[bi, d], w[d, ::-1])[:37] + b[d]
                assert np.allclose(out[bi, d], ref, rtol=1e-13, atol=1e-13), (width, bi, d)


def pin_conv_impulse_response(lib):
    width, L, t0 = 4, 12, 5
    w = np.array([[0.1, -0.7, 1.3, 2.9]])
    x = np.zeros((1, 1, L))
    x[0, 0, t0] = 1.0
    out = _conv(lib, x, w).ravel()
    expect = np.zeros(L)
    for k in range(width):
        expect[t0 + k] = w[0, width - 1 - k]
    assert np.array_equal(out, expect), (out, expect)


def pin_conv_causality(lib):
    rng = np.random.default_rng(32)
    x = rng.standard_normal((1, 3, 20))
    w = rng.standard_normal((3, 4))
    b = rng.standard_normal(3)
    base = _conv(lib, x, w, b, silu=True)
    x2 = x.copy()
    x2[:, :, 9] += 5.0
    moved = _conv(lib, x2, w, b, silu=True)
    assert np.array_equal(base[:, :, :9], moved[:, :, :9])
    assert not np.allclose(base[:, :, 9:13], moved[:, :, 9:13])


def pin_conv_activation(lib):
    rng = np.random.default_rng(33)
    x = rng.standard_normal((2, 4, 15)) * 3
    w = rng.standard_normal((4, 4))
    b = rng.standard_normal(4)
    v = _conv(lib, x, w, b, silu=False)
    s = _conv(lib, x, w, b, silu=True)
    assert np.allclose(s, v / (1.0 + np.exp(-v)), rtol=1e-14, atol=1e-15)


CONV_PINS = [pin_conv_hand_worked, pin_conv_numpy_convolve, pin_conv_impulse_response, pin_conv_causality,
             pin_conv_activation]
