"""The kernels' softplus polynomial, pinned on the CPU.

The scan kernels compute softplus(x) = max(x, 0) + log1p(e) with e = 2^(-|x| log2 e)
in (0, 1], and log1p(e) as e * q(e), q a degree-7 polynomial for log1p(e)/e on [0, 1]
(the coefficients `kSoftplusQ` in csrc/scan_kernel.cuh, highest degree first).

How the coefficients were made: a Remez exchange for the minimax RELATIVE error of
log1p(e)/e on [0, 1] at degree 7 (the linear Remez system p(x_i) - f(x_i) =
(-1)^i E f(x_i) on n + 2 reference points, started from Chebyshev extrema and
re-seated on the alternating extrema of the error), in numpy fp64, each coefficient
then rounded to fp32.  This test repeats that fit, checks the committed constants
against it, and bounds the error of the float32 evaluation the kernel performs.
"""
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
KERNEL = os.path.join(ROOT, "selective_state_space_30_b200", "csrc", "scan_kernel.cuh")


def committed_coefficients():
    src = open(KERNEL).read()
    m = re.search(r"kSoftplusQ\[8\]\s*=\s*\{([^}]*)\}", src)
    assert m, "kSoftplusQ not found"
    vals = [float(v.strip().rstrip("f")) for v in m.group(1).split(",") if v.strip()]
    assert len(vals) == 8
    return np.array(vals, dtype=np.float32)


def f(x):
    """log1p(x)/x, 1 at x = 0."""
    x = np.asarray(x, dtype=np.float64)
    safe = np.where(x == 0, 1.0, x)
    return np.where(x == 0, 1.0, np.log1p(safe) / safe)


def remez_relative(deg, a=0.0, b=1.0, iters=30, grid_n=200001):
    """Minimax polynomial of degree `deg` for the relative error p/f - 1 on [a, b]."""
    n = deg + 2
    k = np.arange(n)
    x = (a + b) / 2 - (b - a) / 2 * np.cos(np.pi * k / (n - 1))
    grid = np.linspace(a, b, grid_n)
    fg = f(grid)
    c, E = None, None
    for _ in range(iters):
        fx = f(x)
        M = np.zeros((n, n))
        M[:, :deg + 1] = np.vander(x, deg + 1)
        M[:, deg + 1] = ((-1.0) ** k) * fx
        sol = np.linalg.solve(M, fx)
        c, E = sol[:deg + 1], abs(sol[deg + 1])
        err = np.polyval(c, grid) / fg - 1
        # one extremum per run of equal sign, then the n of them that alternate
        idx, start = [], 0
        sgn = np.sign(err)
        for i in range(1, grid_n + 1):
            if i == grid_n or sgn[i] != sgn[start]:
                seg = np.arange(start, i)
                idx.append(seg[np.argmax(np.abs(err[seg]))])
                start = i
        while len(idx) > n:
            idx = idx[1:] if abs(err[idx[0]]) < abs(err[idx[-1]]) else idx[:-1]
        if len(idx) < n:
            break
        x = grid[np.array(idx)]
    return c, E


def horner_f32(coef, e):
    """q(e) as the kernel evaluates it: float32 Horner with a fused multiply-add per step
    (the fp64 product-sum of two float32 values, rounded once to float32, is exact FMA rounding)."""
    q = np.full(e.shape, coef[0], dtype=np.float32)
    for c in coef[1:]:
        q = (q.astype(np.float64) * e.astype(np.float64) + np.float64(c)).astype(np.float32)
    return q


def test_remez_fit_converges_to_the_minimax_error():
    c, E = remez_relative(7)
    grid = np.linspace(0, 1, 100001)
    err = np.abs(np.polyval(c, grid) / f(grid) - 1)
    # equioscillation: the level E of the last exchange is the maximum error
    assert abs(err.max() - E) < 1e-3 * E
    assert 1.5e-7 < E < 2.5e-7


def test_committed_coefficients_are_the_remez_fit_rounded_to_fp32():
    q = committed_coefficients()
    c, E = remez_relative(7)
    assert np.max(np.abs(q.astype(np.float64) - c)) < 3e-7
    grid = np.linspace(0, 1, 400001)
    err = np.abs(np.polyval(q.astype(np.float64), grid) / f(grid) - 1)
    assert err.max() < 1.2 * E


def test_float32_evaluation_of_log1p_within_4e7_relative():
    q = committed_coefficients()
    e = np.concatenate([np.linspace(0, 1, 1000001, dtype=np.float32),
                        np.float32(2.0) ** -np.arange(1, 126, dtype=np.float32)])
    e = e[e > 0]
    lp = (e.astype(np.float64) * horner_f32(q, e).astype(np.float64)).astype(np.float32)
    ref = np.log1p(e.astype(np.float64))
    rel = np.abs(lp.astype(np.float64) / ref - 1)
    assert rel.max() <= 4e-7


def test_a_perturbed_coefficient_fails_the_bound():
    """The bound has teeth: moving one coefficient by 1e-5 breaks it."""
    q = committed_coefficients().copy()
    q[3] += np.float32(1e-5)
    e = np.linspace(1e-3, 1, 200001, dtype=np.float32)
    lp = (e.astype(np.float64) * horner_f32(q, e).astype(np.float64))
    rel = np.abs(lp / np.log1p(e.astype(np.float64)) - 1)
    assert rel.max() > 4e-7
