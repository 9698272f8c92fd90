"""The wiring of selective_scan_fn (the torch autograd Function over the forward
and backward entry points), on CPU.

The two library calls it makes are replaced, in this test only, by the fp64
oracle on float64 tensors; torch.autograd.gradcheck then compares the gradients
that the Function hands back, input by input, with finite differences of its
forward.  A gradient returned for the wrong input, a dropped optional gradient
(D, bias, h0) or a wrong incoming-gradient pairing (dout, dlast) fails here.
The numbers the CUDA path computes are checked on the GPU
(test_autograd_gpu.py).
"""
import numpy as np
import pytest
import torch

import oracle
import selective_state_space_30_b200 as ssm


def _np(t):
    return None if t is None else t.detach().cpu().numpy()


def _fake_fwd(u, delta, A, B, C, D=None, z=None, delta_bias=None, softplus=True, h0=None, **_):
    batch, dim, L = u.shape
    ngroups, N = B.shape[1], B.shape[2]
    out, last, _mag = oracle.selective_scan(batch, dim, L, N, _np(u), _np(delta), _np(A), _np(B), _np(C), _np(D),
                                            _np(z), _np(delta_bias), softplus, delta.shape[1], ngroups,
                                            h0=_np(h0), nthreads=1)
    return torch.from_numpy(out), torch.from_numpy(last)


def _fake_bwd(u, delta, A, B, C, dout, D=None, z=None, delta_bias=None, softplus=True, h0=None, dlast=None,
              want_dh0=False, **_):
    batch, dim, L = u.shape
    ngroups, N = B.shape[1], B.shape[2]
    g, _mags = oracle.selective_scan_bwd(batch, dim, L, N, _np(u), _np(delta), _np(A), _np(B), _np(C), _np(dout),
                                         _np(D), _np(z), _np(delta_bias), softplus, delta.shape[1], ngroups,
                                         h0=_np(h0), dlast=_np(dlast), want_dh0=want_dh0, nthreads=1)
    res = {k: (torch.from_numpy(np.ascontiguousarray(v)) if v is not None else None) for k, v in g.items()}
    # the library's front end always forms dD and ddelta_bias
    if res.get("dD") is None:
        res["dD"] = torch.zeros(dim, dtype=torch.float64)
    if res.get("ddelta_bias") is None:
        res["ddelta_bias"] = torch.zeros(delta.shape[1], dtype=torch.float64)
    return res


@pytest.fixture
def oracle_backed(monkeypatch):
    monkeypatch.setattr(ssm, "selective_scan_fwd", _fake_fwd)
    monkeypatch.setattr(ssm, "selective_scan_bwd", _fake_bwd)


def _problem(rng, batch, dim, L, N, ngroups=1, full=True, with_h0=True):
    t = lambda *s: torch.from_numpy(rng.standard_normal(s))  # noqa: E731
    p = dict(u=t(batch, dim, L), delta=t(batch, dim, L) * 0.5, A=-torch.rand(dim, N, dtype=torch.float64) - 0.5,
             B=t(batch, ngroups, N, L), C=t(batch, ngroups, N, L))
    p.update(D=t(dim) if full else None, z=t(batch, dim, L) if full else None,
             delta_bias=t(dim) * 0.3 if full else None, h0=t(batch, dim, N) if with_h0 else None)
    return {k: (v.requires_grad_() if v is not None else None) for k, v in p.items()}


ORDER = ("u", "delta", "A", "B", "C", "D", "z", "delta_bias", "h0")


@pytest.mark.parametrize("full,with_h0,ngroups", [(True, True, 1), (False, False, 1), (True, False, 2)])
def test_gradients_reach_their_inputs(oracle_backed, full, with_h0, ngroups):
    rng = np.random.default_rng(7)
    p = _problem(rng, 2, 4, 5, 3, ngroups=ngroups, full=full, with_h0=with_h0)
    names = [k for k in ORDER if p[k] is not None]

    def f(*xs):
        kw = dict(zip(names, xs))
        return ssm.selective_scan_fn(kw["u"], kw["delta"], kw["A"], kw["B"], kw["C"], kw.get("D"), kw.get("z"),
                                     kw.get("delta_bias"), True, kw.get("h0"))

    assert torch.autograd.gradcheck(f, tuple(p[k] for k in names), eps=1e-6, atol=1e-6, rtol=1e-5)


def test_unused_last_state_and_unwanted_h0(oracle_backed):
    """Only out feeds the loss (last_state's incoming gradient is zero); h0 does not
    require a gradient, so none is formed for it."""
    rng = np.random.default_rng(8)
    p = _problem(rng, 1, 2, 4, 2)
    p["h0"] = p["h0"].detach()
    out, _ = ssm.selective_scan_fn(*(p[k] for k in ORDER[:8]), True, p["h0"])
    w = torch.from_numpy(rng.standard_normal(out.shape))
    (out * w).sum().backward()
    g, _ = oracle.selective_scan_bwd(1, 2, 4, 2, *(_np(p[k]) for k in ("u", "delta", "A", "B", "C")), _np(w),
                                     *(_np(p[k]) for k in ("D", "z", "delta_bias")), True, 2, 1, h0=_np(p["h0"]),
                                     nthreads=1)
    for k, name in (("u", "du"), ("B", "dB"), ("D", "dD"), ("delta_bias", "ddelta_bias")):
        np.testing.assert_allclose(_np(p[k].grad), g[name], rtol=1e-12, atol=1e-14)
    assert p["h0"].grad is None


@pytest.mark.parametrize("store_states", [True, False])
def test_states_stored_only_when_asked(monkeypatch, store_states):
    """On a shape the tiled backward covers (S6 layout, dstate 16, 32 channels), the forward
    is handed a state buffer of ckpt_shape and the backward the same buffer; with
    store_states False neither gets one (the backward recomputes the states)."""
    seen = {}

    def fwd(*a, ckpt=None, **kw):
        seen["fwd"] = ckpt
        return _fake_fwd(*a, **kw)

    def bwd(*a, ckpt=None, **kw):
        seen["bwd"] = ckpt
        return _fake_bwd(*a, **kw)

    monkeypatch.setattr(ssm, "selective_scan_fwd", fwd)
    monkeypatch.setattr(ssm, "selective_scan_bwd", bwd)
    p = _problem(np.random.default_rng(9), 1, 32, 6, 16)
    out, last = ssm.selective_scan_fn(*(p[k] for k in ORDER[:8]), True, p["h0"], store_states=store_states)
    (out.sum() + last.sum()).backward()
    if store_states:
        assert tuple(seen["fwd"].shape) == ssm.ckpt_shape(1, 32, 6, 16) and seen["bwd"] is seen["fwd"]
    else:
        assert seen["fwd"] is None and seen["bwd"] is None
