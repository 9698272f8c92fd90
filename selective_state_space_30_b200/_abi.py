"""ctypes binding of libssmscan.so: the C ABI of include/ssm_scan.h, same names.

Argument marshalling only -- every step of the scan runs in the library's
CUDA kernels.  Pointer arguments take either a plain integer address or
anything with a `data_ptr()` method (a torch tensor); None means NULL.
There is no fallback: if the library is not built, loading raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Any, Optional

_HERE = os.path.dirname(os.path.abspath(__file__))
# SSM_SCAN_LIBRARY names another build of the same library (the debug build, say)
LIB_PATH = os.environ.get("SSM_SCAN_LIBRARY") or os.path.join(_HERE, "libssmscan.so")

SSM_OK = 0
SSM_ERR_INVALID_ARG = 1
SSM_ERR_UNSUPPORTED = 2
SSM_ERR_CUDA = 3
SSM_ERR_TIMEOUT = 4
SSM_ERR_BOUNDS = 5
SSM_F32 = 0
SSM_BF16 = 1

# every exported symbol declared in include/ssm_scan.h
EXPORTS = ("ssm_scan_plan", "ssm_selective_scan_fwd", "ssm_selective_scan_fwd_h0",
           "ssm_selective_scan_fwd_ckpt", "ssm_selective_scan_fwd_host", "ssm_selective_scan_fwd_noalloc",
           "ssm_selective_scan_noalloc_device_status", "ssm_selective_scan_noalloc_test_hooks",
           "ssm_selective_state_update",
           "ssm_causal_conv1d_fwd", "ssm_selective_scan_bwd_workspace_size", "ssm_selective_scan_bwd",
           "ssm_selective_scan_bwd_ckpt", "ssm_selective_scan_bwd_device_status", "ssm_selective_scan_bwd_test_hooks",
           "ssm_scan_set_option",
           "ssm_scan_plan_schedule", "ssm_scan_destroy",
           "ssm_scan_device_status", "ssm_status_string", "ssm_scan_plan_info", "ssm_probe_ex2")

SSM_OPT_SPIN_LIMIT = 1
SSM_OPT_INJECT_STALL = 2
SSM_OPT_SEG_LEN = 3
SSM_OPT_CONSUMER_WARPS = 4
SSM_OPT_WORKERS = 5
SSM_OPT_STATES_PER_LANE = 6
SSM_OPT_SSD = 7
SSM_OPT_TIME_LANES = 8
SSM_OPT_TENSOR_MEMORY = 9


class SsmError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} (status {status})")


class ssm_dims_t(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int64), ("dim", ctypes.c_int64), ("seqlen", ctypes.c_int64),
                ("dstate", ctypes.c_int64), ("nheads", ctypes.c_int64), ("ngroups", ctypes.c_int64),
                ("io_dtype", ctypes.c_int32), ("reserved", ctypes.c_int32)]


class ssm_grads_t(ctypes.Structure):
    _fields_ = [("du", ctypes.c_void_p), ("ddelta", ctypes.c_void_p), ("dA", ctypes.c_void_p),
                ("dB", ctypes.c_void_p), ("dC", ctypes.c_void_p), ("dD", ctypes.c_void_p),
                ("dz", ctypes.c_void_p), ("ddelta_bias", ctypes.c_void_p), ("dh0", ctypes.c_void_p)]


GRAD_NAMES = tuple(f[0] for f in ssm_grads_t._fields_)

_lib = None


def load_library(path: Optional[str] = None):
    """Load libssmscan.so (raises if it has not been built)."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise RuntimeError(f"{p} is missing: build it with `python -m selective_state_space_30_b200.build` "
                           "(there is no CPU fallback)")
    lib = ctypes.CDLL(p)
    vp, i32, i64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64
    dims_p = ctypes.POINTER(ssm_dims_t)
    fwd_args = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i32, dims_p]
    lib.ssm_scan_plan.argtypes = [ctypes.POINTER(vp), dims_p, i32]
    lib.ssm_selective_scan_fwd.argtypes = fwd_args + [vp, vp, vp]
    lib.ssm_selective_scan_fwd_h0.argtypes = fwd_args + [vp, vp, vp, vp]
    lib.ssm_selective_scan_fwd_ckpt.argtypes = fwd_args + [vp, vp, vp, vp, vp]
    lib.ssm_selective_scan_fwd_host.argtypes = fwd_args + [vp, vp, vp]
    lib.ssm_selective_scan_fwd_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, i32, dims_p, vp, vp, vp]
    lib.ssm_selective_scan_noalloc_device_status.argtypes = [vp]
    lib.ssm_selective_scan_noalloc_test_hooks.argtypes = [i32, i64]
    lib.ssm_selective_state_update.argtypes = [dims_p, vp, vp, vp, vp, vp, vp, vp, vp, vp, i32, vp, vp]
    lib.ssm_causal_conv1d_fwd.argtypes = [i64, i64, i64, i32, i32, vp, vp, vp, i32, vp, vp]
    lib.ssm_selective_scan_bwd_workspace_size.argtypes = [dims_p, ctypes.POINTER(ctypes.c_size_t)]
    lib.ssm_selective_scan_bwd.argtypes = [dims_p, vp, vp, vp, vp, vp, vp, vp, vp, i32, vp, vp, vp,
                                           ctypes.POINTER(ssm_grads_t), vp, ctypes.c_size_t, vp]
    lib.ssm_selective_scan_bwd_ckpt.argtypes = [dims_p, vp, vp, vp, vp, vp, vp, vp, vp, i32, vp, vp, vp, vp,
                                                ctypes.POINTER(ssm_grads_t), vp, ctypes.c_size_t, vp]
    lib.ssm_selective_scan_bwd_device_status.argtypes = [vp, vp]
    lib.ssm_selective_scan_bwd_test_hooks.argtypes = [i32, i64]
    lib.ssm_scan_destroy.argtypes = [vp]
    lib.ssm_scan_device_status.argtypes = [vp, vp]
    lib.ssm_status_string.argtypes = [i32]
    lib.ssm_status_string.restype = ctypes.c_char_p
    lib.ssm_scan_plan_info.argtypes = [vp, ctypes.POINTER(i32), ctypes.POINTER(i32), ctypes.POINTER(i32),
                                       ctypes.POINTER(i32), ctypes.POINTER(ctypes.c_char_p)]
    lib.ssm_probe_ex2.argtypes = [vp, i32, i32, vp]
    lib.ssm_scan_set_option.argtypes = [vp, i32, i64]
    lib.ssm_scan_plan_schedule.argtypes = [vp] + [ctypes.POINTER(i32)] * 5
    for name in EXPORTS:
        if name != "ssm_status_string":
            getattr(lib, name).restype = i32
    if path is None:
        _lib = lib
    return lib


def _ptr(x: Any) -> Optional[int]:
    if x is None:
        return None
    if isinstance(x, int):
        return x
    if hasattr(x, "data_ptr"):
        return int(x.data_ptr())
    if hasattr(x, "ctypes"):  # numpy array (host entry point)
        return int(x.ctypes.data)
    raise TypeError(f"cannot take a device pointer of {type(x)!r}")


def _stream(s: Any) -> Optional[int]:
    if s is None:
        return None
    if isinstance(s, int):
        return s or None
    return int(getattr(s, "cuda_stream", s)) or None


def _check(rc: int, where: str) -> int:
    if rc != SSM_OK:
        raise SsmError(rc, where)
    return rc


def make_dims(batch: int, dim: int, seqlen: int, dstate: int, nheads: int = 0, ngroups: int = 1,
              io_dtype: int = SSM_BF16) -> ssm_dims_t:
    return ssm_dims_t(batch, dim, seqlen, dstate, nheads or dim, ngroups, io_dtype, 0)


def status_string(status: int) -> str:
    return load_library().ssm_status_string(int(status)).decode()


ssm_status_string = status_string


def ssm_scan_plan(dims: ssm_dims_t, device: int = 0) -> int:
    plan = ctypes.c_void_p()
    _check(load_library().ssm_scan_plan(ctypes.byref(plan), ctypes.byref(dims), int(device)), "ssm_scan_plan")
    return int(plan.value)


def ssm_selective_scan_fwd(plan: int, u, delta, A, B, C, D, z, delta_bias, softplus: bool, dims: ssm_dims_t,
                           out, last_state, stream=None, check: bool = True) -> int:
    rc = load_library().ssm_selective_scan_fwd(
        plan, _ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z), _ptr(delta_bias),
        1 if softplus else 0, ctypes.byref(dims), _ptr(out), _ptr(last_state), _stream(stream))
    return _check(rc, "ssm_selective_scan_fwd") if check else rc


def ssm_selective_scan_fwd_h0(plan: int, u, delta, A, B, C, D, z, delta_bias, softplus: bool, dims: ssm_dims_t,
                              h0, out, last_state, stream=None, check: bool = True) -> int:
    rc = load_library().ssm_selective_scan_fwd_h0(
        plan, _ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z), _ptr(delta_bias),
        1 if softplus else 0, ctypes.byref(dims), _ptr(h0), _ptr(out), _ptr(last_state), _stream(stream))
    return _check(rc, "ssm_selective_scan_fwd_h0") if check else rc


def ssm_selective_scan_fwd_ckpt(plan: int, u, delta, A, B, C, D, z, delta_bias, softplus: bool, dims: ssm_dims_t,
                                h0, out, last_state, ckpt, stream=None, check: bool = True) -> int:
    rc = load_library().ssm_selective_scan_fwd_ckpt(
        plan, _ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z), _ptr(delta_bias),
        1 if softplus else 0, ctypes.byref(dims), _ptr(h0), _ptr(out), _ptr(last_state), _ptr(ckpt), _stream(stream))
    return _check(rc, "ssm_selective_scan_fwd_ckpt") if check else rc


def ssm_selective_scan_fwd_host(plan: int, u, delta, A, B, C, D, z, delta_bias, softplus: bool,
                                dims: ssm_dims_t, out, last_state, stream=None, check: bool = True) -> int:
    rc = load_library().ssm_selective_scan_fwd_host(
        plan, _ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z), _ptr(delta_bias),
        1 if softplus else 0, ctypes.byref(dims), _ptr(out), _ptr(last_state), _stream(stream))
    return _check(rc, "ssm_selective_scan_fwd_host") if check else rc


def ssm_selective_scan_fwd_noalloc(u, delta, A, B, C, D, z, delta_bias, softplus: bool, dims: ssm_dims_t,
                                   out, last_state, stream=None, check: bool = True) -> int:
    """The forward scan without a plan or any device allocation (see include/ssm_scan.h)."""
    rc = load_library().ssm_selective_scan_fwd_noalloc(
        _ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z), _ptr(delta_bias),
        1 if softplus else 0, ctypes.byref(dims), _ptr(out), _ptr(last_state), _stream(stream))
    return _check(rc, "ssm_selective_scan_fwd_noalloc") if check else rc


def ssm_selective_scan_noalloc_device_status(stream=None) -> int:
    """Kernel-side status of the last allocation-free call on the current device (syncs, clears it)."""
    return int(load_library().ssm_selective_scan_noalloc_device_status(_stream(stream)))


def ssm_selective_scan_noalloc_test_hooks(stall: bool, spin_limit: int = 0) -> int:
    """Allocation-free entry point's test hooks (see include/ssm_scan.h)."""
    return _check(load_library().ssm_selective_scan_noalloc_test_hooks(1 if stall else 0, int(spin_limit)),
                  "ssm_selective_scan_noalloc_test_hooks")


def ssm_selective_state_update(dims: ssm_dims_t, state, u, delta, A, B, C, D, z, delta_bias, softplus: bool,
                               out, stream=None, check: bool = True) -> int:
    """One recurrence step with the state updated in place (see include/ssm_scan.h)."""
    rc = load_library().ssm_selective_state_update(
        ctypes.byref(dims), _ptr(state), _ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z),
        _ptr(delta_bias), 1 if softplus else 0, _ptr(out), _stream(stream))
    return _check(rc, "ssm_selective_state_update") if check else rc


def ssm_causal_conv1d_fwd(batch: int, dim: int, seqlen: int, width: int, io_dtype: int, x, w, bias,
                          silu: bool, out, stream=None, check: bool = True) -> int:
    """The causal depthwise convolution (see include/ssm_scan.h)."""
    rc = load_library().ssm_causal_conv1d_fwd(int(batch), int(dim), int(seqlen), int(width), int(io_dtype), _ptr(x),
                                              _ptr(w), _ptr(bias), 1 if silu else 0, _ptr(out), _stream(stream))
    return _check(rc, "ssm_causal_conv1d_fwd") if check else rc


def ssm_selective_scan_bwd_workspace_size(dims: ssm_dims_t, check: bool = True) -> int:
    """Bytes of device scratch ssm_selective_scan_bwd needs for `dims` (see include/ssm_scan.h)."""
    n = ctypes.c_size_t()
    rc = load_library().ssm_selective_scan_bwd_workspace_size(ctypes.byref(dims), ctypes.byref(n))
    if check:
        _check(rc, "ssm_selective_scan_bwd_workspace_size")
    return int(n.value) if rc == SSM_OK else -rc


def ssm_selective_scan_bwd(dims: ssm_dims_t, u, delta, A, B, C, D, z, delta_bias, softplus: bool, h0, dout,
                           dlast, grads: dict, workspace, workspace_bytes: int, stream=None,
                           check: bool = True) -> int:
    """Gradients of the forward scan (see include/ssm_scan.h); `grads` maps GRAD_NAMES to outputs or None."""
    g = ssm_grads_t(*[_ptr(grads.get(k)) for k in GRAD_NAMES])
    rc = load_library().ssm_selective_scan_bwd(
        ctypes.byref(dims), _ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z), _ptr(delta_bias),
        1 if softplus else 0, _ptr(h0), _ptr(dout), _ptr(dlast), ctypes.byref(g), _ptr(workspace),
        int(workspace_bytes), _stream(stream))
    return _check(rc, "ssm_selective_scan_bwd") if check else rc


def ssm_selective_scan_bwd_ckpt(dims: ssm_dims_t, u, delta, A, B, C, D, z, delta_bias, softplus: bool, h0, dout,
                                dlast, ckpt, grads: dict, workspace, workspace_bytes: int, stream=None,
                                check: bool = True) -> int:
    """ssm_selective_scan_bwd given the forward's stored states (ckpt; None = recompute them)."""
    g = ssm_grads_t(*[_ptr(grads.get(k)) for k in GRAD_NAMES])
    rc = load_library().ssm_selective_scan_bwd_ckpt(
        ctypes.byref(dims), _ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z), _ptr(delta_bias),
        1 if softplus else 0, _ptr(h0), _ptr(dout), _ptr(dlast), _ptr(ckpt), ctypes.byref(g), _ptr(workspace),
        int(workspace_bytes), _stream(stream))
    return _check(rc, "ssm_selective_scan_bwd_ckpt") if check else rc


def ssm_selective_scan_bwd_device_status(workspace, stream=None) -> int:
    """Kernel-side status of the last backward call on `workspace` (syncs the stream, clears it)."""
    return int(load_library().ssm_selective_scan_bwd_device_status(_ptr(workspace), _stream(stream)))


def ssm_selective_scan_bwd_test_hooks(stall: bool, wait_budget_us: int = 0) -> int:
    """Backward test hooks (see include/ssm_scan.h): make chained waits run out; shorten their limit."""
    return _check(load_library().ssm_selective_scan_bwd_test_hooks(1 if stall else 0, int(wait_budget_us)),
                  "ssm_selective_scan_bwd_test_hooks")


def ssm_scan_destroy(plan: Optional[int]) -> int:
    return _check(load_library().ssm_scan_destroy(plan), "ssm_scan_destroy")


def ssm_scan_device_status(plan: int, stream=None) -> int:
    return int(load_library().ssm_scan_device_status(plan, _stream(stream)))


def ssm_scan_plan_info(plan: int) -> dict:
    g, b, s, n = ctypes.c_int(), ctypes.c_int(), ctypes.c_int(), ctypes.c_int()
    name = ctypes.c_char_p()
    _check(load_library().ssm_scan_plan_info(plan, ctypes.byref(g), ctypes.byref(b), ctypes.byref(s),
                                             ctypes.byref(n), ctypes.byref(name)), "ssm_scan_plan_info")
    return {"grid": g.value, "block": b.value, "smem_bytes": s.value, "launches_per_call": n.value,
            "variant": name.value.decode()}


def ssm_scan_set_option(plan: int, option: int, value: int) -> int:
    return _check(load_library().ssm_scan_set_option(plan, int(option), int(value)), "ssm_scan_set_option")


def ssm_scan_plan_schedule(plan: int) -> dict:
    v = [ctypes.c_int() for _ in range(5)]
    _check(load_library().ssm_scan_plan_schedule(plan, *[ctypes.byref(x) for x in v]), "ssm_scan_plan_schedule")
    return dict(zip(("consumer_warps", "seg_len", "n_tiles", "n_seg", "n_ctas"), (x.value for x in v)))


def ssm_probe_ex2(sink, blocks: int, iters: int, stream=None) -> int:
    return _check(load_library().ssm_probe_ex2(_ptr(sink), int(blocks), int(iters), _stream(stream)),
                  "ssm_probe_ex2")
