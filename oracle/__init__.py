"""fp64 CPU oracle for the selective-SSM (S6) forward scan, its gradient (the
backward scan) and the causal convolution in front of it.

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the bench's CPU
baseline may import this package; the product path never does.  It shares no
code with the CUDA library (the only common dependency is the seeded input
generator in `ssm_inputs`, which holds none of the scan's arithmetic).

The arithmetic lives in `ssm_oracle.c` (plain fp64 loop; see its header for the
passages it follows).  This wrapper only converts the generated tensors exactly
to float64 and marshals pointers.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Sequence, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ssm_oracle.c")
_LIB_PATH = os.path.join(_HERE, "_oracle.so")
_lib = None


class _Dims(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int64), ("dim", ctypes.c_int64), ("seqlen", ctypes.c_int64),
                ("dstate", ctypes.c_int64), ("nheads", ctypes.c_int64), ("ngroups", ctypes.c_int64)]


GRAD_NAMES = ("du", "ddelta", "dA", "dB", "dC", "dD", "dz", "ddelta_bias", "dh0")


class _Grads(ctypes.Structure):
    _fields_ = [(k, ctypes.POINTER(ctypes.c_double)) for k in GRAD_NAMES]


def build(force: bool = False) -> str:
    """Compile the oracle with plain gcc: fp64, no FMA contraction, no fast-math."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math",
                               "-o", tmp, _SRC, "-lm", "-lpthread"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def load(path: Optional[str] = None):
    """Load the oracle library (optionally another build of it, e.g. in a test)."""
    lib = ctypes.CDLL(path or build())
    p = ctypes.POINTER(ctypes.c_double)
    lib.oracle_selective_scan_f64.restype = ctypes.c_int
    lib.oracle_selective_scan_f64.argtypes = [
        ctypes.POINTER(_Dims), p, p, p, p, p, p, p, p, ctypes.c_int, p,
        ctypes.POINTER(ctypes.c_int64), ctypes.c_int64, p, p, p, ctypes.c_int]
    lib.oracle_selective_scan_bwd_f64.restype = ctypes.c_int
    lib.oracle_selective_scan_bwd_f64.argtypes = [
        ctypes.POINTER(_Dims), p, p, p, p, p, p, p, p, ctypes.c_int, p, p, p,
        ctypes.POINTER(_Grads), ctypes.POINTER(_Grads), ctypes.c_int]
    i64 = ctypes.c_int64
    lib.oracle_causal_conv1d_f64.restype = ctypes.c_int
    lib.oracle_causal_conv1d_f64.argtypes = [i64, i64, i64, i64, p, p, p, ctypes.c_int, p]
    return lib


def _get_lib():
    global _lib
    if _lib is None:
        _lib = load()
    return _lib


def _nthreads() -> int:
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def _f64(a) -> Optional[np.ndarray]:
    """Exact float64 copy of a tensor given as float64/float32 or bf16 bits (uint16)."""
    if a is None:
        return None
    a = np.asarray(a)
    if a.dtype == np.uint16:
        b = a.astype(np.uint32) << 16
        return np.ascontiguousarray(b.view(np.float32).astype(np.float64))
    return np.ascontiguousarray(a.astype(np.float64))


def _ptr(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def selective_scan(batch: int, dim: int, seqlen: int, dstate: int, u, delta, A, B, C, D=None, z=None,
                   delta_bias=None, softplus: bool = True, nheads: int = 0, ngroups: int = 1,
                   h0=None, channels: Optional[Sequence[int]] = None, nthreads: Optional[int] = None,
                   lib=None) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Run the fp64 oracle.

    Returns (out, last_state, mag) in float64.  Full mode: out/mag (batch, dim, L),
    last_state (batch, dim, N).  Row mode (`channels` = flat ids b*dim + d; u, z,
    delta and h0 given as the matching rows): out/mag (nch, L), last_state (nch, N).
    """
    H = nheads if nheads else dim
    dims = _Dims(batch, dim, seqlen, dstate, H, ngroups)
    uu, dd, AA, BB, CC = _f64(u), _f64(delta), _f64(A), _f64(B), _f64(C)
    DD, zz, bb, hh = _f64(D), _f64(z), _f64(delta_bias), _f64(h0)
    if channels is None:
        rows = batch * dim
        ch = None
        nch = 0
    else:
        ch = np.ascontiguousarray(np.asarray(channels, dtype=np.int64))
        rows = nch = int(ch.size)
    # size checks (the C side trusts these)
    exp_u = rows * seqlen
    exp_delta = (batch * H if channels is None else rows) * seqlen
    if uu.size != exp_u or dd.size != exp_delta:
        raise ValueError("u / delta size does not match the problem")
    if zz is not None and zz.size != exp_u:
        raise ValueError("z size does not match the problem")
    if BB.size != batch * ngroups * dstate * seqlen or CC.size != BB.size:
        raise ValueError("B / C size does not match the problem")
    if AA.size != (dim * dstate if H == dim else H):
        raise ValueError("A size does not match the problem")
    if DD is not None and DD.size != dim:
        raise ValueError("D size does not match the problem")
    if bb is not None and bb.size != H:
        raise ValueError("delta_bias size does not match the problem")
    if hh is not None and hh.size != rows * dstate:
        raise ValueError("h0 size does not match the problem")
    out = np.empty(rows * seqlen, dtype=np.float64)
    mag = np.empty(rows * seqlen, dtype=np.float64)
    last = np.empty(rows * dstate, dtype=np.float64)
    lib = lib or _get_lib()
    rc = lib.oracle_selective_scan_f64(
        ctypes.byref(dims), _ptr(uu), _ptr(dd), _ptr(AA), _ptr(BB), _ptr(CC), _ptr(DD), _ptr(zz), _ptr(bb),
        1 if softplus else 0, _ptr(hh),
        ch.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)) if ch is not None else None, nch,
        _ptr(out), _ptr(last), _ptr(mag), nthreads or _nthreads())
    if rc != 0:
        raise ValueError("oracle rejected its arguments")
    if channels is None:
        return (out.reshape(batch, dim, seqlen), last.reshape(batch, dim, dstate),
                mag.reshape(batch, dim, seqlen))
    return out.reshape(rows, seqlen), last.reshape(rows, dstate), mag.reshape(rows, seqlen)


def run_inputs(dims, inputs: dict, channels=None, h0=None, nthreads=None, lib=None):
    """Convenience: run on a dict produced by `ssm_inputs.make_inputs`."""
    return selective_scan(dims.batch, dims.dim, dims.seqlen, dims.dstate, inputs["u"], inputs["delta"],
                          inputs["A"], inputs["B"], inputs["C"], inputs.get("D"), inputs.get("z"),
                          inputs.get("delta_bias"), bool(inputs.get("softplus", True)), dims.nheads,
                          dims.ngroups, h0=h0, channels=channels, nthreads=nthreads, lib=lib)


def causal_conv1d(x, w, bias=None, silu: bool = True, lib=None) -> np.ndarray:
    """The causal depthwise convolution (see `oracle_causal_conv1d_f64`) in fp64.

    x: (batch, dim, seqlen) as float64/float32 or bf16 bits; w: (dim, width);
    bias: (dim) or None.  Returns out (batch, dim, seqlen) float64.
    """
    xx, ww, bb = _f64(x), _f64(w), _f64(bias)
    xs = np.asarray(x).shape
    if len(xs) != 3:
        raise ValueError("x must be (batch, dim, seqlen)")
    batch, dim, seqlen = xs
    if ww.ndim != 2 or ww.shape[0] != dim:
        raise ValueError("w must be (dim, width)")
    width = ww.shape[1]
    if bb is not None and bb.size != dim:
        raise ValueError("bias must be (dim)")
    out = np.empty(batch * dim * seqlen, dtype=np.float64)
    lib = lib or _get_lib()
    rc = lib.oracle_causal_conv1d_f64(batch, dim, seqlen, width, _ptr(xx), _ptr(ww), _ptr(bb),
                                      1 if silu else 0, _ptr(out))
    if rc != 0:
        raise ValueError("oracle rejected its arguments")
    return out.reshape(batch, dim, seqlen)


def selective_scan_bwd(batch: int, dim: int, seqlen: int, dstate: int, u, delta, A, B, C, dout, D=None, z=None,
                       delta_bias=None, softplus: bool = True, nheads: int = 0, ngroups: int = 1, h0=None,
                       dlast=None, want_dh0: bool = False, nthreads: Optional[int] = None, lib=None):
    """Gradients of the forward scan (see `oracle_selective_scan_bwd_f64`) in fp64.

    dout has out's shape (batch, dim, L); dlast (optional) last_state's (batch, dim, N).
    Returns (grads, mags): dicts name -> float64 array over GRAD_NAMES, shaped
    du, dz (batch, dim, L); ddelta (batch, nheads, L); dA like A; dB, dC
    (batch, ngroups, N, L); dD (dim); ddelta_bias (nheads); dh0 (batch, dim, N).
    dz is None without z, dh0 unless want_dh0.  mags hold the magnitude sums
    used by the tolerance checks.
    """
    H = nheads if nheads else dim
    dims = _Dims(batch, dim, seqlen, dstate, H, ngroups)
    arrs = {k: _f64(v) for k, v in dict(u=u, delta=delta, A=A, B=B, C=C, D=D, z=z, bias=delta_bias, h0=h0,
                                          dout=dout, dlast=dlast).items()}
    rows = batch * dim
    if arrs["u"].size != rows * seqlen or arrs["dout"].size != rows * seqlen:
        raise ValueError("u / dout size does not match the problem")
    if arrs["delta"].size != batch * H * seqlen:
        raise ValueError("delta size does not match the problem")
    if arrs["z"] is not None and arrs["z"].size != rows * seqlen:
        raise ValueError("z size does not match the problem")
    nbc = batch * ngroups * dstate * seqlen
    if arrs["B"].size != nbc or arrs["C"].size != nbc:
        raise ValueError("B / C size does not match the problem")
    nA = dim * dstate if H == dim else H
    if arrs["A"].size != nA:
        raise ValueError("A size does not match the problem")
    if arrs["D"] is not None and arrs["D"].size != dim:
        raise ValueError("D size does not match the problem")
    if arrs["bias"] is not None and arrs["bias"].size != H:
        raise ValueError("delta_bias size does not match the problem")
    for k in ("h0", "dlast"):
        if arrs[k] is not None and arrs[k].size != rows * dstate:
            raise ValueError(f"{k} size does not match the problem")
    shapes = dict(du=(batch, dim, seqlen), ddelta=(batch, H, seqlen), dA=(dim, dstate) if H == dim else (H,),
                  dB=(batch, ngroups, dstate, seqlen), dC=(batch, ngroups, dstate, seqlen), dD=(dim,),
                  dz=(batch, dim, seqlen), ddelta_bias=(H,), dh0=(batch, dim, dstate))
    grads, mags = {}, {}
    for k in GRAD_NAMES:
        want = (k != "dz" or arrs["z"] is not None) and (k != "dh0" or want_dh0)
        grads[k] = np.zeros(shapes[k], dtype=np.float64) if want else None
        mags[k] = np.zeros(shapes[k], dtype=np.float64) if want else None
    gs = _Grads(*[_ptr(grads[k]) for k in GRAD_NAMES])
    ms = _Grads(*[_ptr(mags[k]) for k in GRAD_NAMES])
    lib = lib or _get_lib()
    rc = lib.oracle_selective_scan_bwd_f64(
        ctypes.byref(dims), _ptr(arrs["u"]), _ptr(arrs["delta"]), _ptr(arrs["A"]), _ptr(arrs["B"]), _ptr(arrs["C"]),
        _ptr(arrs["D"]), _ptr(arrs["z"]), _ptr(arrs["bias"]), 1 if softplus else 0, _ptr(arrs["h0"]),
        _ptr(arrs["dout"]), _ptr(arrs["dlast"]), ctypes.byref(gs), ctypes.byref(ms), nthreads or _nthreads())
    if rc != 0:
        raise ValueError("oracle rejected its arguments")
    return grads, mags


def run_inputs_bwd(dims, inputs: dict, dout, dlast=None, h0=None, want_dh0=False, nthreads=None, lib=None):
    """Convenience: the backward on a dict produced by `ssm_inputs.make_inputs`."""
    return selective_scan_bwd(dims.batch, dims.dim, dims.seqlen, dims.dstate, inputs["u"], inputs["delta"],
                              inputs["A"], inputs["B"], inputs["C"], dout, inputs.get("D"), inputs.get("z"),
                              inputs.get("delta_bias"), bool(inputs.get("softplus", True)), dims.nheads,
                              dims.ngroups, h0=h0, dlast=dlast, want_dh0=want_dh0, nthreads=nthreads, lib=lib)
