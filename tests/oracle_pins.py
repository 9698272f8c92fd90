"""Checks that pin the fp64 oracle to facts other than itself.

Each `pin_*` takes an oracle library handle (the real build, or a deliberately
broken copy in the mutation tests) and raises AssertionError when the oracle
disagrees with an independent statement of the method:

* closed forms: one step (L=1), A = 0 (prefix sum), dA = 0 (memoryless),
  a worked example by hand (tests/golden/hand_worked_example.json);
* the fixed-parameter (LTI) special case as a convolution
  (Mamba "architecture-details" page, "How S6 Works": traditional SSM with
  fixed A, B, C; kernel K_k = sum_n C_n dA_n^k dt B_n);
* the materialised semi-separable matrix
  M[t,s] = sum_n C_t[n] (prod_{s<r<=t} dA_r[n]) dt_s B_s[n]
  ("Agent 229: SSM optimization patterns" page, sections 2 "State Space
  Duality" and 10 "Structured Matrices");
* an independent associative (Hillis-Steele) scan with the operator
  (a1, b1) o (a2, b2) = (a1 a2, a2 b1 + b2) (same page, sections 1 and 11);
* chunk-split invariance (same page, section 9 "Chunked Computation");
* structure: linearity in u, causality, head / group broadcasting.

None of these reuse the oracle's code: softplus comes from numpy.logaddexp,
exponentials from numpy, the recurrence from explicit products or scans.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np

import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
RTOL = 1e-11


def _close(a, b, rtol=RTOL, atol=1e-12, what=""):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    assert a.shape == b.shape, f"{what}: shape {a.shape} vs {b.shape}"
    err = np.abs(a - b)
    tol = atol + rtol * np.abs(b)
    bad = err > tol
    assert not bad.any(), f"{what}: max err {err.max():.3e} (worst at {np.unravel_index(np.argmax(err - tol), err.shape)})"


def _softplus(x):
    return np.logaddexp(0.0, x)  # library routine, not the oracle's formula


def _silu(z):
    return z * (0.5 * (1.0 + np.tanh(0.5 * z)))  # sigmoid via tanh: another route than 1/(1+e^-z)


def _rand_problem(rng, batch, dim, L, N, nheads=0, ngroups=1, D=True, z=True, bias=True):
    H = nheads or dim
    p = {
        "u": rng.standard_normal((batch, dim, L)),
        "delta": rng.standard_normal((batch, H, L)) * 0.5,
        "A": (-rng.uniform(0.5, 3.0, (dim, N))) if H == dim else -rng.uniform(0.5, 3.0, H),
        "B": rng.standard_normal((batch, ngroups, N, L)),
        "C": rng.standard_normal((batch, ngroups, N, L)),
        "D": rng.standard_normal(dim) if D else None,
        "z": rng.standard_normal((batch, dim, L)) if z else None,
        "delta_bias": rng.uniform(-4.0, 1.0, H) if bias else None,
    }
    return p


def _run(lib, batch, dim, L, N, p, softplus=True, nheads=0, ngroups=1, h0=None, channels=None):
    return oracle.selective_scan(batch, dim, L, N, p["u"], p["delta"], p["A"], p["B"], p["C"], p["D"], p["z"],
                                 p["delta_bias"], softplus, nheads, ngroups, h0=h0, channels=channels,
                                 nthreads=2, lib=lib)


def _dt(p, b, hd, t, softplus):
    x = p["delta"][b, hd, t] + (p["delta_bias"][hd] if p["delta_bias"] is not None else 0.0)
    return _softplus(x) if softplus else x


def _materialised(p, batch, dim, L, N, softplus=True, nheads=0, ngroups=1, h0=None):
    """y = M u (+ initial-state term) + D u, gated, from the semi-separable matrix."""
    H = nheads or dim
    out = np.zeros((batch, dim, L))
    last = np.zeros((batch, dim, N))
    mag = np.zeros((batch, dim, L))
    for b in range(batch):
        for d in range(dim):
            hd, g = d // (dim // H), d // (dim // ngroups)
            a = p["A"][d] if H == dim else np.full(N, p["A"][hd])
            dt = np.array([_dt(p, b, hd, t, softplus) for t in range(L)])
            dA = np.exp(np.outer(dt, a))                       # (L, N)
            Bm, Cm = p["B"][b, g].T, p["C"][b, g].T            # (L, N)
            u = p["u"][b, d]
            # decay[t, s, n] = prod_{s<r<=t} dA[r, n]
            M = np.zeros((L, L))
            H_ts = np.zeros((L, L, N))  # contribution of step s to h_t
            for t in range(L):
                for s in range(t + 1):
                    decay = np.prod(dA[s + 1:t + 1], axis=0) if t > s else np.ones(N)
                    H_ts[t, s] = decay * dt[s] * Bm[s] * u[s]
                    M[t, s] = np.sum(Cm[t] * decay * dt[s] * Bm[s])
            h = H_ts.sum(axis=1)                              # (L, N) states after each step
            if h0 is not None:
                for t in range(L):
                    h[t] += np.prod(dA[:t + 1], axis=0) * h0[b, d]
            y = M @ u
            if h0 is not None:
                y = np.sum(Cm * h, axis=1)
            Dd = p["D"][d] if p["D"] is not None else 0.0
            y = y + Dd * u
            gate = _silu(p["z"][b, d]) if p["z"] is not None else np.ones(L)
            out[b, d] = y * gate
            last[b, d] = h[L - 1] if L else (h0[b, d] if h0 is not None else 0.0)
            mag[b, d] = np.abs(gate) * (np.sum(np.abs(Cm * h), axis=1) + np.abs(Dd * u))
    return out, last, mag


# ---------------------------------------------------------------- the pins


def pin_hand_worked_example(lib):
    with open(os.path.join(GOLDEN, "hand_worked_example.json")) as f:
        g = json.load(f)
    env = {"ln2": math.log(2.0), "ln3": math.log(3.0)}
    ev = lambda s: float(eval(s, {"__builtins__": {}}, env))  # noqa: E731 (expressions from the fixture)
    i = g["inputs"]
    p = {"u": np.array(i["u"]).reshape(1, 1, 3), "delta": np.array(i["delta"]).reshape(1, 1, 3),
         "A": np.array(i["A"]).reshape(1, 2), "B": np.array(i["B"]).reshape(1, 1, 2, 3),
         "C": np.array(i["C"]).reshape(1, 1, 2, 3), "D": np.array(i["D"]),
         "z": np.array([ev(s) for s in i["z"]]).reshape(1, 1, 3), "delta_bias": np.array(i["delta_bias"])}
    out, last, _ = _run(lib, 1, 1, 3, 2, p, softplus=i["softplus"])
    _close(out.ravel(), [ev(s) for s in g["expected"]["out"]], what="hand example out")
    _close(last.ravel(), [ev(s) for s in g["expected"]["last_state"]], what="hand example last_state")
    p["z"] = None
    out, _, _ = _run(lib, 1, 1, 3, 2, p, softplus=i["softplus"])
    _close(out.ravel(), [ev(s) for s in g["expected"]["y_no_gate"]], what="hand example y")


def pin_single_step(lib):
    """L = 1: h = dt*B*u, y = C.h + D*u, out = y*silu(z)  (softplus on and off)."""
    rng = np.random.default_rng(11)
    for softplus in (True, False):
        p = _rand_problem(rng, 2, 5, 1, 6)
        if not softplus:
            p["delta_bias"] = np.abs(p["delta_bias"]) + 0.1
            p["delta"] = np.abs(p["delta"])
        out, last, mag = _run(lib, 2, 5, 1, 6, p, softplus=softplus)
        for b in range(2):
            for d in range(5):
                x = p["delta"][b, d, 0] + p["delta_bias"][d]
                dt = _softplus(x) if softplus else x
                h = dt * p["B"][b, 0, :, 0] * p["u"][b, d, 0]
                y = np.dot(p["C"][b, 0, :, 0], h) + p["D"][d] * p["u"][b, d, 0]
                _close(last[b, d], h, what="L=1 state")
                _close(out[b, d, 0], y * _silu(p["z"][b, d, 0]), what="L=1 out")


def pin_lti_convolution(lib):
    """Constant dt, B, C along t: y = K * u + D u with K_k = sum_n C_n dA_n^k dt B_n."""
    rng = np.random.default_rng(12)
    batch, dim, L, N = 2, 3, 40, 5
    p = _rand_problem(rng, batch, dim, L, N)
    p["delta"] = np.repeat(rng.standard_normal((batch, dim, 1)) * 0.5, L, axis=2)
    p["B"] = np.repeat(rng.standard_normal((batch, 1, N, 1)), L, axis=3)
    p["C"] = np.repeat(rng.standard_normal((batch, 1, N, 1)), L, axis=3)
    out, last, _ = _run(lib, batch, dim, L, N, p)
    for b in range(batch):
        for d in range(dim):
            dt = _softplus(p["delta"][b, d, 0] + p["delta_bias"][d])
            dA = np.exp(dt * p["A"][d])
            Bn, Cn = p["B"][b, 0, :, 0], p["C"][b, 0, :, 0]
            K = np.array([np.sum(Cn * dA ** k * dt * Bn) for k in range(L)])
            y = np.convolve(K, p["u"][b, d])[:L] + p["D"][d] * p["u"][b, d]
            _close(out[b, d], y * _silu(p["z"][b, d]), rtol=1e-10, what="LTI convolution")
            hL = np.array([np.sum(dA[n] ** np.arange(L - 1, -1, -1) * dt * Bn[n] * p["u"][b, d]) for n in range(N)])
            _close(last[b, d], hL, rtol=1e-10, what="LTI last state")


def pin_semiseparable(lib):
    """Selective case against the materialised semi-separable matrix (S6 layout, heads, groups)."""
    rng = np.random.default_rng(13)
    cases = [dict(batch=2, dim=3, L=12, N=4), dict(batch=1, dim=4, L=9, N=3, nheads=2),
             dict(batch=2, dim=4, L=7, N=2, ngroups=2), dict(batch=1, dim=6, L=8, N=3, nheads=3, ngroups=3)]
    for c in cases:
        nh, ng = c.get("nheads", 0), c.get("ngroups", 1)
        p = _rand_problem(rng, c["batch"], c["dim"], c["L"], c["N"], nheads=nh, ngroups=ng)
        out, last, mag = _run(lib, c["batch"], c["dim"], c["L"], c["N"], p, nheads=nh, ngroups=ng)
        ro, rl, rm = _materialised(p, c["batch"], c["dim"], c["L"], c["N"], nheads=nh, ngroups=ng)
        _close(out, ro, rtol=1e-10, what=f"semi-separable out {c}")
        _close(last, rl, rtol=1e-10, what=f"semi-separable last {c}")
        _close(mag, rm, rtol=1e-10, what=f"semi-separable mag {c}")


def _assoc_scan(a, b):
    """Inclusive Hillis-Steele scan of pairs with (a1,b1) o (a2,b2) = (a1 a2, a2 b1 + b2), along axis 0."""
    a, b = a.copy(), b.copy()
    L = a.shape[0]
    k = 1
    while k < L:
        a_prev, b_prev = a[:-k].copy(), b[:-k].copy()
        b[k:] = a[k:] * b_prev + b[k:]
        a[k:] = a[k:] * a_prev
        k *= 2
    return a, b


def pin_associative_scan(lib):
    rng = np.random.default_rng(14)
    batch, dim, L, N = 2, 3, 37, 4
    p = _rand_problem(rng, batch, dim, L, N, z=False, D=False)
    out, last, _ = _run(lib, batch, dim, L, N, p)
    for b in range(batch):
        for d in range(dim):
            dt = _softplus(p["delta"][b, d] + p["delta_bias"][d])            # (L,)
            dA = np.exp(np.outer(dt, p["A"][d]))                              # (L, N)
            x = dt[:, None] * p["B"][b, 0].T * p["u"][b, d][:, None]           # (L, N)
            _, h = _assoc_scan(dA, x)
            y = np.sum(p["C"][b, 0].T * h, axis=1)
            _close(out[b, d], y, rtol=1e-10, what="associative scan")
            _close(last[b, d], h[-1], rtol=1e-10, what="associative scan state")


def pin_chunk_split(lib):
    """Running [0, L1) then [L1, L) from the carried state equals one run."""
    rng = np.random.default_rng(15)
    batch, dim, L, N = 2, 4, 50, 5
    p = _rand_problem(rng, batch, dim, L, N)
    out, last, _ = _run(lib, batch, dim, L, N, p)
    for L1 in (1, 17, 49):
        p1 = dict(p, u=p["u"][..., :L1], delta=p["delta"][..., :L1], z=p["z"][..., :L1],
                  B=p["B"][..., :L1], C=p["C"][..., :L1])
        p2 = dict(p, u=p["u"][..., L1:], delta=p["delta"][..., L1:], z=p["z"][..., L1:],
                  B=p["B"][..., L1:], C=p["C"][..., L1:])
        o1, s1, _ = _run(lib, batch, dim, L1, N, {k: (np.ascontiguousarray(v) if isinstance(v, np.ndarray) else v)
                                                  for k, v in p1.items()})
        o2, s2, _ = _run(lib, batch, dim, L - L1, N, {k: (np.ascontiguousarray(v) if isinstance(v, np.ndarray) else v)
                                                      for k, v in p2.items()}, h0=s1)
        _close(np.concatenate([o1, o2], axis=2), out, rtol=1e-12, what=f"chunk split at {L1}")
        _close(s2, last, rtol=1e-12, what=f"chunk split state at {L1}")
    # the carried state also matches the materialised form with an initial state
    h0 = rng.standard_normal((batch, dim, N))
    o, s, _ = _run(lib, batch, dim, 9, N, {k: (np.ascontiguousarray(v[..., :9]) if k in ("u", "delta", "z", "B", "C")
                                               else v) for k, v in p.items()}, h0=h0)
    q = {k: (v[..., :9] if k in ("u", "delta", "z", "B", "C") else v) for k, v in p.items()}
    ro, rl, _ = _materialised(q, batch, dim, 9, N, h0=h0)
    _close(o, ro, rtol=1e-10, what="initial state")
    _close(s, rl, rtol=1e-10, what="initial state, last")


def pin_a_zero_prefix_sum(lib):
    """A = 0: dA = 1 and h_n(t) = sum_{s<=t} dt_s B_n(s) u_s."""
    rng = np.random.default_rng(16)
    batch, dim, L, N = 1, 3, 25, 4
    p = _rand_problem(rng, batch, dim, L, N)
    p["A"] = np.zeros((dim, N))
    out, last, _ = _run(lib, batch, dim, L, N, p)
    for d in range(dim):
        dt = _softplus(p["delta"][0, d] + p["delta_bias"][d])
        h = np.cumsum(dt[:, None] * p["B"][0, 0].T * p["u"][0, d][:, None], axis=0)
        y = np.sum(p["C"][0, 0].T * h, axis=1) + p["D"][d] * p["u"][0, d]
        _close(out[0, d], y * _silu(p["z"][0, d]), rtol=1e-10, what="A=0 prefix sum")
        _close(last[0, d], h[-1], rtol=1e-10, what="A=0 last")


def pin_memoryless(lib):
    """A -> -inf: dA = 0, y_t = dt u (C_t . B_t) + D u."""
    rng = np.random.default_rng(17)
    batch, dim, L, N = 2, 2, 10, 3
    p = _rand_problem(rng, batch, dim, L, N)
    p["A"] = np.full((dim, N), -1e300)
    out, last, _ = _run(lib, batch, dim, L, N, p)
    for b in range(batch):
        for d in range(dim):
            dt = _softplus(p["delta"][b, d] + p["delta_bias"][d])
            cb = np.sum(p["C"][b, 0] * p["B"][b, 0], axis=0)
            y = dt * p["u"][b, d] * cb + p["D"][d] * p["u"][b, d]
            _close(out[b, d], y * _silu(p["z"][b, d]), rtol=1e-12, what="memoryless")
            _close(last[b, d], dt[-1] * p["B"][b, 0, :, -1] * p["u"][b, d, -1], rtol=1e-12, what="memoryless last")


def pin_linearity_causality(lib):
    rng = np.random.default_rng(18)
    batch, dim, L, N = 1, 3, 30, 4
    p = _rand_problem(rng, batch, dim, L, N, z=False)
    u1, u2 = rng.standard_normal((batch, dim, L)), rng.standard_normal((batch, dim, L))
    o1, s1, _ = _run(lib, batch, dim, L, N, dict(p, u=u1))
    o2, s2, _ = _run(lib, batch, dim, L, N, dict(p, u=u2))
    o3, s3, _ = _run(lib, batch, dim, L, N, dict(p, u=2.0 * u1 - 3.0 * u2))
    _close(o3, 2.0 * o1 - 3.0 * o2, rtol=1e-10, atol=1e-10, what="linearity in u")
    _close(s3, 2.0 * s1 - 3.0 * s2, rtol=1e-10, atol=1e-10, what="linearity in u (state)")
    t0 = 13
    u4 = u1.copy()
    u4[..., t0] += 5.0
    o4, _, _ = _run(lib, batch, dim, L, N, dict(p, u=u4))
    _close(o4[..., :t0], o1[..., :t0], rtol=0, atol=0, what="causality")
    assert np.all(np.abs(o4[..., t0] - o1[..., t0]) > 0), "perturbation at t0 must reach y(t0)"


def pin_head_mode_broadcast(lib):
    """Scalar A / delta / bias per head equals the per-channel layout with those values broadcast."""
    rng = np.random.default_rng(19)
    batch, dim, L, N, H = 2, 6, 11, 4, 3
    p = _rand_problem(rng, batch, dim, L, N, nheads=H)
    out, last, _ = _run(lib, batch, dim, L, N, p, nheads=H)
    P = dim // H
    q = dict(p, A=np.repeat(np.repeat(p["A"], P)[:, None], N, axis=1),
             delta=np.repeat(p["delta"], P, axis=1), delta_bias=np.repeat(p["delta_bias"], P))
    o2, s2, _ = _run(lib, batch, dim, L, N, q)
    _close(out, o2, rtol=1e-13, what="head mode")
    _close(last, s2, rtol=1e-13, what="head mode state")


def pin_groups(lib):
    """ngroups = G equals G independent problems, each with its own B, C."""
    rng = np.random.default_rng(20)
    batch, dim, L, N, G = 2, 6, 9, 3, 3
    p = _rand_problem(rng, batch, dim, L, N, ngroups=G)
    out, last, _ = _run(lib, batch, dim, L, N, p, ngroups=G)
    P = dim // G
    for g in range(G):
        sl = slice(g * P, (g + 1) * P)
        q = {"u": p["u"][:, sl].copy(), "delta": p["delta"][:, sl].copy(), "A": p["A"][sl].copy(),
             "B": p["B"][:, g:g + 1].copy(), "C": p["C"][:, g:g + 1].copy(), "D": p["D"][sl].copy(),
             "z": p["z"][:, sl].copy(), "delta_bias": p["delta_bias"][sl].copy()}
        o, s, _ = _run(lib, batch, P, L, N, q)
        _close(out[:, sl], o, rtol=1e-13, what="groups")
        _close(last[:, sl], s, rtol=1e-13, what="groups state")


def pin_row_mode(lib):
    """Row mode (a subset of channels) returns the same rows as the full run."""
    rng = np.random.default_rng(21)
    batch, dim, L, N, H = 2, 6, 13, 4, 3
    p = _rand_problem(rng, batch, dim, L, N, nheads=H)
    out, last, mag = _run(lib, batch, dim, L, N, p, nheads=H)
    ch = [0, 5, 7, 11, 3]
    P = dim // H
    q = dict(p, u=np.stack([p["u"][c // dim, c % dim] for c in ch]),
             z=np.stack([p["z"][c // dim, c % dim] for c in ch]),
             delta=np.stack([p["delta"][c // dim, (c % dim) // P] for c in ch]))
    o, s, m = _run(lib, batch, dim, L, N, q, nheads=H, channels=ch)
    for k, c in enumerate(ch):
        _close(o[k], out[c // dim, c % dim], rtol=0, atol=0, what="row mode out")
        _close(s[k], last[c // dim, c % dim], rtol=0, atol=0, what="row mode state")
        _close(m[k], mag[c // dim, c % dim], rtol=0, atol=0, what="row mode mag")


ALL_PINS = [pin_hand_worked_example, pin_single_step, pin_lti_convolution, pin_semiseparable,
            pin_associative_scan, pin_chunk_split, pin_a_zero_prefix_sum, pin_memoryless,
            pin_linearity_causality, pin_head_mode_broadcast, pin_groups, pin_row_mode]
