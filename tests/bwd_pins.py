"""Checks that pin the fp64 oracle's backward scan to facts other than itself.

Each `pin_bwd_*` takes an oracle library handle (the real build, or a broken copy
in the mutation tests) and raises AssertionError on a disagreement:

* central finite differences of the oracle's forward scan (itself pinned by
  oracle_pins.py): the gradient is the derivative of
  loss = sum(dout * out) + sum(dlast * last_state), element by element, for
  every input (S6 and per-head layouts, groups, h0 and dlast, softplus off,
  no gate / skip / bias);
* the one-step closed form (L = 1, with an initial state), written out from
  the recurrence by hand below;
* du as the transpose of the materialised semi-separable map u -> y
  ("Agent 229: SSM optimization patterns" page, section 2 "State Space
  Duality"): du = M^T dy + D dy with dy = dout * silu(z);
* linearity of every gradient in (dout, dlast), and magnitudes that bound
  the gradients;
* dz's magnitude covering an fp32 evaluation of dz where silu'(z) cancels.
"""
from __future__ import annotations

import numpy as np

import oracle
from oracle_pins import _close, _materialised, _rand_problem, _run, _silu, _softplus

FD_RTOL, FD_ATOL = 2e-6, 2e-7
INPUTS = ("u", "delta", "A", "B", "C", "D", "z", "delta_bias")
GRAD_OF = {"u": "du", "delta": "ddelta", "A": "dA", "B": "dB", "C": "dC", "D": "dD", "z": "dz",
           "delta_bias": "ddelta_bias", "h0": "dh0"}


def _bwd(lib, c, p, dout, dlast=None, h0=None, softplus=True):
    return oracle.selective_scan_bwd(c["batch"], c["dim"], c["L"], c["N"], p["u"], p["delta"], p["A"], p["B"],
                                     p["C"], dout, p["D"], p["z"], p["delta_bias"], softplus, c.get("nheads", 0),
                                     c.get("ngroups", 1), h0=h0, dlast=dlast, want_dh0=h0 is not None,
                                     nthreads=2, lib=lib)


def _loss(lib, c, p, dout, dlast, h0, softplus):
    out, last, _ = _run(lib, c["batch"], c["dim"], c["L"], c["N"], p, softplus=softplus,
                        nheads=c.get("nheads", 0), ngroups=c.get("ngroups", 1), h0=h0)
    s = float(np.sum(dout * out))
    if dlast is not None:
        s += float(np.sum(dlast * last))
    return s


def _sigmoid(x):
    return 0.5 * (1.0 + np.tanh(0.5 * x))


FD_CASES = [
    dict(batch=2, dim=4, L=5, N=3, ngroups=2, h0=True, dlast=True),
    dict(batch=1, dim=4, L=6, N=2, nheads=2, h0=True, dlast=False),
    dict(batch=2, dim=2, L=4, N=3, softplus=False),
    dict(batch=1, dim=3, L=5, N=2, plain=True, dlast=True),
]


def pin_bwd_finite_differences(lib):
    rng = np.random.default_rng(31)
    for c in FD_CASES:
        nh, ng = c.get("nheads", 0), c.get("ngroups", 1)
        plain = c.get("plain", False)
        p = _rand_problem(rng, c["batch"], c["dim"], c["L"], c["N"], nheads=nh, ngroups=ng, D=not plain,
                          z=not plain, bias=not plain)
        softplus = c.get("softplus", True)
        if not softplus:   # dt = delta + bias > 0 without softplus
            p["delta"] = np.abs(p["delta"]) * 0.2 + 0.05
            p["delta_bias"] = np.abs(p["delta_bias"]) * 0.1
        h0 = rng.standard_normal((c["batch"], c["dim"], c["N"])) if c.get("h0") else None
        dout = rng.standard_normal((c["batch"], c["dim"], c["L"]))
        dlast = rng.standard_normal((c["batch"], c["dim"], c["N"])) if c.get("dlast") else None
        grads, _ = _bwd(lib, c, p, dout, dlast, h0, softplus)
        q = dict(p, h0=h0)
        for name in INPUTS + ("h0",):
            if q[name] is None:
                continue
            base = np.array(q[name], dtype=np.float64)
            fd = np.zeros_like(base)
            for i in np.ndindex(base.shape):
                step = 1e-6 * max(1.0, abs(base[i]))
                vals = []
                for sgn in (1.0, -1.0):
                    pert = base.copy()
                    pert[i] += sgn * step
                    pp = dict(q, **{name: pert})
                    vals.append(_loss(lib, c, {k: pp[k] for k in INPUTS}, dout, dlast, pp["h0"], softplus))
                fd[i] = (vals[0] - vals[1]) / (2 * step)
            g = grads[GRAD_OF[name]]
            assert g is not None, f"no gradient for {name}"
            scale = 1.0 + np.max(np.abs(fd))
            _close(g, fd, rtol=FD_RTOL, atol=FD_ATOL * scale, what=f"finite differences d{name} {c}")


def pin_bwd_single_step(lib):
    """L = 1 with h0:  h = e^(dt a) h0 + dt B u,  y = C.h + D u,  out = y silu(z),  last = h."""
    rng = np.random.default_rng(32)
    batch, dim, N = 2, 3, 4
    c = dict(batch=batch, dim=dim, L=1, N=N)
    p = _rand_problem(rng, batch, dim, 1, N)
    h0 = rng.standard_normal((batch, dim, N))
    dout = rng.standard_normal((batch, dim, 1))
    dlast = rng.standard_normal((batch, dim, N))
    grads, _ = _bwd(lib, c, p, dout, dlast, h0)
    exp = {k: np.zeros_like(v) for k, v in grads.items() if v is not None}
    for b in range(batch):
        for d in range(dim):
            x = p["delta"][b, d, 0] + p["delta_bias"][d]
            dt, a = _softplus(x), p["A"][d]
            Bn, Cn, u, z = p["B"][b, 0, :, 0], p["C"][b, 0, :, 0], p["u"][b, d, 0], p["z"][b, d, 0]
            e = np.exp(dt * a)
            h = e * h0[b, d] + dt * Bn * u
            y = np.dot(Cn, h) + p["D"][d] * u
            s = _sigmoid(z)
            dy = dout[b, d, 0] * z * s
            gh = dy * Cn + dlast[b, d]          # dLoss/dh
            exp["du"][b, d, 0] = dy * p["D"][d] + np.sum(gh * dt * Bn)
            exp["dz"][b, d, 0] = dout[b, d, 0] * y * (s + z * s * (1.0 - s))
            exp["dB"][b, 0, :, 0] += gh * dt * u
            exp["dC"][b, 0, :, 0] += dy * h
            exp["dD"][d] += dy * u
            ddt = np.sum(gh * (a * e * h0[b, d] + Bn * u))
            exp["ddelta"][b, d, 0] = ddt * _sigmoid(x)
            exp["ddelta_bias"][d] += ddt * _sigmoid(x)
            exp["dA"][d] += gh * h0[b, d] * dt * e
            exp["dh0"][b, d] = gh * e
    for k, v in exp.items():
        _close(grads[k], v, rtol=1e-11, atol=1e-12, what=f"L=1 closed form {k}")


def pin_bwd_du_transpose(lib):
    """h0 = 0: u -> y is linear with the semi-separable matrix M (+ D), so du = M^T dy + D dy."""
    rng = np.random.default_rng(33)
    batch, dim, L, N = 1, 2, 16, 3
    c = dict(batch=batch, dim=dim, L=L, N=N)
    p = _rand_problem(rng, batch, dim, L, N)
    dout = rng.standard_normal((batch, dim, L))
    grads, _ = _bwd(lib, c, p, dout)
    for d in range(dim):
        # columns of M from the materialised forward with one-hot inputs and no gate, no skip
        q = dict(p, z=None, D=None)
        M = np.zeros((L, L))
        for s in range(L):
            e = np.zeros((batch, dim, L))
            e[0, d, s] = 1.0
            ys, _, _ = _materialised(dict(q, u=e), batch, dim, L, N)
            M[:, s] = ys[0, d]
        dy = dout[0, d] * _silu(p["z"][0, d])
        _close(grads["du"][0, d], M.T @ dy + p["D"][d] * dy, rtol=1e-10, atol=1e-12, what="du = M^T dy + D dy")


def pin_bwd_linear_in_dout(lib):
    rng = np.random.default_rng(34)
    c = dict(batch=2, dim=3, L=6, N=2, ngroups=1)
    p = _rand_problem(rng, 2, 3, 6, 2)
    h0 = rng.standard_normal((2, 3, 2))
    d1, d2 = rng.standard_normal((2, 3, 6)), rng.standard_normal((2, 3, 6))
    l1, l2 = rng.standard_normal((2, 3, 2)), rng.standard_normal((2, 3, 2))
    g1, m1 = _bwd(lib, c, p, d1, l1, h0)
    g2, _ = _bwd(lib, c, p, d2, l2, h0)
    g3, _ = _bwd(lib, c, p, 2.0 * d1 - 0.5 * d2, 2.0 * l1 - 0.5 * l2, h0)
    for k, v in g3.items():
        if v is None:
            continue
        _close(v, 2.0 * g1[k] - 0.5 * g2[k], rtol=1e-10, atol=1e-11, what=f"linearity {k}")
        assert np.all(m1[k] >= np.abs(g1[k]) * (1 - 1e-12) - 1e-15), f"magnitude below |grad| for {k}"


def pin_bwd_dz_magnitude_covers_fp32(lib):
    """dz = dout y silu'(z) evaluated in fp32 (numpy float32, from the rounded fp64 y) stays within
    1e-4 of the oracle's magnitude for dz, on a grid of z that runs through the root of
    silu'(z) = s (1 + z (1 - s)) near z = -1.278, where the factor cancels in fp32."""
    rng = np.random.default_rng(35)
    L, N = 400, 4
    c = dict(batch=1, dim=1, L=L, N=N)
    p = _rand_problem(rng, 1, 1, L, N)
    zg = np.concatenate([np.linspace(-1.30, -1.25, L // 2), np.linspace(-8.0, 6.0, L // 2)])
    p["z"] = zg.reshape(1, 1, L)
    dout = rng.standard_normal((1, 1, L))
    grads, mags = _bwd(lib, c, p, dout)
    # y without the gate, from the pinned forward
    y, _, _ = _run(lib, 1, 1, L, N, dict(p, z=None))
    s64 = 1.0 / (1.0 + np.exp(-zg))
    # the grid reaches the cancellation: |silu'| far below the sum of its terms' magnitudes
    assert np.min(np.abs(s64 * (1.0 + zg * (1.0 - s64))) / (s64 * (1.0 + np.abs(zg) * (1.0 - s64)))) < 1e-4
    f = np.float32
    with np.errstate(over="ignore", invalid="ignore"):   # a broken oracle's y may not fit fp32
        z32 = zg.astype(f)
        s32 = f(1.0) / (f(1.0) + np.exp(-z32))
        d32 = s32 * (f(1.0) + z32 * (f(1.0) - s32))
        dz32 = (dout[0, 0].astype(f) * y[0, 0].astype(f) * d32).astype(np.float64)
    err = np.abs(dz32 - grads["dz"][0, 0])
    tol = 1e-4 * mags["dz"][0, 0]
    assert np.all(err <= tol), f"fp32 dz outside 1e-4 * mag at z = {zg[np.argmax(err - tol)]!r}"


BWD_PINS = [pin_bwd_finite_differences, pin_bwd_single_step, pin_bwd_du_transpose, pin_bwd_linear_in_dout,
            pin_bwd_dz_magnitude_covers_fp32]
