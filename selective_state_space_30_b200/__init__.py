"""B200-native selective-SSM (S6) forward scan.

The product is the CUDA library `libssmscan.so` (C ABI: include/ssm_scan.h).
This package binds it with ctypes (`_abi`, same names as the C entry points)
and adds a small torch-tensor front end:

    out, last_state = selective_scan_fwd(u, delta, A, B, C, D, z, delta_bias, softplus=True)
    out, last_state = selective_scan_fn(...)   # the same, differentiable (torch autograd)

PyTorch is only used for device memory and streams; the scan runs in the
library's kernels.  There is no CPU or PyTorch fallback.
"""
from __future__ import annotations

import threading
from typing import Dict, Optional, Tuple

from . import _abi
from ._abi import (SSM_BF16, SSM_ERR_BOUNDS, SSM_ERR_CUDA, SSM_ERR_INVALID_ARG, SSM_ERR_TIMEOUT,  # noqa: F401
                   SSM_ERR_UNSUPPORTED, SSM_F32, SSM_OK, SSM_OPT_CONSUMER_WARPS, SSM_OPT_INJECT_STALL,
                   SSM_OPT_SEG_LEN, SSM_OPT_SPIN_LIMIT, SSM_OPT_SSD, SSM_OPT_STATES_PER_LANE, SSM_OPT_WORKERS,
                   SSM_OPT_TIME_LANES, SSM_OPT_TENSOR_MEMORY,
                   SsmError, load_library, make_dims,
                   ssm_dims_t, ssm_probe_ex2, ssm_scan_destroy, ssm_scan_device_status, ssm_scan_plan,
                   ssm_scan_plan_info, ssm_scan_plan_schedule, ssm_scan_set_option, ssm_selective_scan_fwd,
                   ssm_selective_scan_fwd_h0, ssm_selective_scan_fwd_ckpt, ssm_selective_scan_fwd_host,
                   ssm_selective_scan_fwd_noalloc,
                   ssm_selective_scan_noalloc_device_status, ssm_selective_scan_noalloc_test_hooks,
                   ssm_selective_state_update, ssm_causal_conv1d_fwd, ssm_selective_scan_bwd,
                   ssm_selective_scan_bwd_ckpt,
                   ssm_selective_scan_bwd_workspace_size, ssm_selective_scan_bwd_device_status,
                   ssm_selective_scan_bwd_test_hooks, ssm_grads_t,
                   GRAD_NAMES,
                   ssm_status_string)

__all__ = ["selective_scan_fwd", "selective_scan_fwd_host", "selective_scan_fn", "Plan", "get_plan", "ssm_scan_plan",
           "ssm_selective_scan_fwd", "ssm_selective_scan_fwd_h0", "ssm_selective_scan_fwd_ckpt",
           "ssm_selective_scan_fwd_host", "ckpt_shape", "bwd_covers",
           "ssm_selective_scan_fwd_noalloc", "ssm_selective_scan_noalloc_device_status",
           "ssm_selective_scan_noalloc_test_hooks", "ssm_selective_state_update", "ssm_causal_conv1d_fwd",
           "selective_scan_bwd", "ssm_selective_scan_bwd", "ssm_selective_scan_bwd_ckpt",
           "ssm_selective_scan_bwd_workspace_size",
           "ssm_selective_scan_bwd_device_status", "ssm_selective_scan_bwd_test_hooks",
           "ssm_scan_destroy", "ssm_scan_device_status", "ssm_status_string", "ssm_scan_plan_info",
           "ssm_scan_set_option", "ssm_scan_plan_schedule",
           "ssm_probe_ex2", "make_dims", "SsmError", "load_library"]


class Plan:
    """Owns one ssm_plan_t (a problem shape on one device)."""

    def __init__(self, batch, dim, seqlen, dstate, nheads=0, ngroups=1, io_dtype=SSM_BF16, device=0):
        self.dims = make_dims(batch, dim, seqlen, dstate, nheads, ngroups, io_dtype)
        self.device = int(device)
        self.handle = ssm_scan_plan(self.dims, self.device)

    def info(self) -> dict:
        return ssm_scan_plan_info(self.handle)

    def device_status(self, stream=None) -> int:
        return ssm_scan_device_status(self.handle, stream)

    def close(self) -> None:
        if self.handle:
            ssm_scan_destroy(self.handle)
            self.handle = 0

    def __del__(self):  # pragma: no cover - interpreter shutdown order varies
        try:
            self.close()
        except Exception:
            pass


_plans: Dict[tuple, Plan] = {}
_plans_lock = threading.Lock()


def get_plan(batch, dim, seqlen, dstate, nheads=0, ngroups=1, io_dtype=SSM_BF16, device=0, stream=None) -> Plan:
    """The cached plan of a shape on a device, one per stream: a plan's workspace
    (ticket counter, carry flags and buffers) serves one call at a time, and the
    calls on one stream run in order."""
    key = (batch, dim, seqlen, dstate, nheads or dim, ngroups, io_dtype, device, _abi._stream(stream) or 0)
    with _plans_lock:
        p = _plans.get(key)
        if p is None:
            p = Plan(batch, dim, seqlen, dstate, nheads, ngroups, io_dtype, device)
            _plans[key] = p
        return p


def _shapes(u, delta, A, B):
    import torch
    if u.dim() != 3 or delta.dim() != 3 or B.dim() != 4:
        raise ValueError("u, delta: (batch, dim|nheads, seqlen); B, C: (batch, ngroups, dstate, seqlen)")
    batch, dim, seqlen = u.shape
    nheads = delta.shape[1]
    ngroups, dstate = B.shape[1], B.shape[2]
    if u.dtype == torch.bfloat16:
        io = SSM_BF16
    elif u.dtype == torch.float32:
        io = SSM_F32
    else:
        raise ValueError("u must be bfloat16 or float32")
    return batch, dim, seqlen, dstate, nheads, ngroups, io


def ckpt_shape(batch: int, dim: int, seqlen: int, dstate: int) -> Tuple[int, int, int, int]:
    """Shape of the state checkpoints ssm_selective_scan_fwd_ckpt stores (fp32): the state
    entering every 8-step window."""
    return (batch, dim, (seqlen + 7) // 8, dstate)


def bwd_covers(u, delta, A, B) -> bool:
    """Whether ssm_selective_scan_bwd covers these inputs' shape (the per-channel layout,
    dstate 16, dim / ngroups a multiple of 32)."""
    if u.dim() != 3 or delta.dim() != 3 or B.dim() != 4:
        return False
    dim, nheads, ngroups, dstate = u.shape[1], delta.shape[1], B.shape[1], B.shape[2]
    return nheads == dim and dstate == 16 and ngroups > 0 and (dim // ngroups) % 32 == 0


def selective_scan_fwd(u, delta, A, B, C, D=None, z=None, delta_bias=None, softplus: bool = True,
                       h0=None, return_last_state: bool = True, out=None, last_state=None,
                       stream=None, ckpt=None) -> Tuple[object, Optional[object]]:
    """Forward scan on CUDA tensors (layouts as in include/ssm_scan.h).

    Returns (out, last_state); last_state is None when return_last_state is False.
    Output tensors are allocated with torch on u's device unless given.  With `ckpt`
    (fp32, ckpt_shape(...)) the call is ssm_selective_scan_fwd_ckpt, which also stores
    the states the backward walks from.
    """
    import torch
    batch, dim, seqlen, dstate, nheads, ngroups, io = _shapes(u, delta, A, B)
    for name, t in (("u", u), ("delta", delta), ("A", A), ("B", B), ("C", C), ("D", D), ("z", z),
                    ("delta_bias", delta_bias), ("h0", h0)):
        if t is not None:
            if not t.is_cuda:
                raise ValueError(f"{name} must be a CUDA tensor")
            if not t.is_contiguous():
                raise ValueError(f"{name} must be contiguous")
    dev = u.device.index if u.device.index is not None else torch.cuda.current_device()
    if stream is None:
        stream = torch.cuda.current_stream(u.device).cuda_stream
    plan = get_plan(batch, dim, seqlen, dstate, nheads, ngroups, io, dev, stream)
    if out is None:
        out = torch.empty_like(u)
    if return_last_state and last_state is None:
        last_state = torch.empty((batch, dim, dstate), dtype=torch.float32, device=u.device)
    if ckpt is not None:
        if not (ckpt.is_cuda and ckpt.is_contiguous() and ckpt.dtype == torch.float32 and
                tuple(ckpt.shape) == ckpt_shape(batch, dim, seqlen, dstate)):
            raise ValueError("ckpt must be a contiguous fp32 CUDA tensor of ckpt_shape(batch, dim, seqlen, dstate)")
        ssm_selective_scan_fwd_ckpt(plan.handle, u, delta, A, B, C, D, z, delta_bias, softplus, plan.dims, h0, out,
                                    last_state if return_last_state else None, ckpt, stream)
    else:
        ssm_selective_scan_fwd_h0(plan.handle, u, delta, A, B, C, D, z, delta_bias, softplus, plan.dims, h0, out,
                                  last_state if return_last_state else None, stream)
    return out, (last_state if return_last_state else None)


def selective_scan_fwd_host(u, delta, A, B, C, D=None, z=None, delta_bias=None, softplus: bool = True,
                            out=None, last_state=None, return_last_state: bool = True, device: int = 0,
                            stream=None):
    """End-to-end call on HOST tensors (pinned for asynchronous copies): the library
    copies the inputs to the device, runs the scan and copies the results back."""
    import torch
    batch, dim, seqlen, dstate, nheads, ngroups, io = _shapes(u, delta, A, B)
    if stream is None:
        stream = torch.cuda.current_stream(device).cuda_stream
    plan = get_plan(batch, dim, seqlen, dstate, nheads, ngroups, io, device, stream)
    if out is None:
        out = torch.empty_like(u, pin_memory=True)
    if return_last_state and last_state is None:
        last_state = torch.empty((batch, dim, dstate), dtype=torch.float32, pin_memory=True)
    ssm_selective_scan_fwd_host(plan.handle, u, delta, A, B, C, D, z, delta_bias, softplus, plan.dims, out,
                                last_state if return_last_state else None, stream)
    return out, (last_state if return_last_state else None)


def selective_scan_bwd(u, delta, A, B, C, dout, D=None, z=None, delta_bias=None, softplus: bool = True,
                       h0=None, dlast=None, want_dh0: bool = False, workspace=None, stream=None, ckpt=None) -> dict:
    """Gradients of the forward scan on CUDA tensors (see include/ssm_scan.h,
    ssm_selective_scan_bwd).  Returns a dict over GRAD_NAMES: du, ddelta, dz in
    u's dtype; dA, dB, dC, dD, ddelta_bias, dh0 fp32 (dz None without z, dh0
    only with want_dh0; dD and ddelta_bias are the gradients at D = 0 / bias = 0
    when those are not given).  The workspace is allocated with torch unless
    given (uint8, at least ssm_selective_scan_bwd_workspace_size bytes).  `ckpt`: the
    states selective_scan_fwd stored for the same inputs (the backward then skips
    recomputing them), or None."""
    import torch
    batch, dim, seqlen, dstate, nheads, ngroups, io = _shapes(u, delta, A, B)
    for name, t in (("u", u), ("delta", delta), ("A", A), ("B", B), ("C", C), ("dout", dout), ("D", D),
                    ("z", z), ("delta_bias", delta_bias), ("h0", h0), ("dlast", dlast), ("ckpt", ckpt)):
        if t is not None:
            if not t.is_cuda:
                raise ValueError(f"{name} must be a CUDA tensor")
            if not t.is_contiguous():
                raise ValueError(f"{name} must be contiguous")
    dims = make_dims(batch, dim, seqlen, dstate, nheads, ngroups, io)
    nbytes = ssm_selective_scan_bwd_workspace_size(dims)
    if workspace is None:
        workspace = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=u.device)
    f32 = dict(dtype=torch.float32, device=u.device)
    g = {"du": torch.empty_like(u), "ddelta": torch.empty_like(delta), "dA": torch.empty(A.shape, **f32),
         "dB": torch.empty(B.shape, **f32), "dC": torch.empty(C.shape, **f32),
         "dD": torch.empty((dim,), **f32), "dz": torch.empty_like(z) if z is not None else None,
         "ddelta_bias": torch.empty((nheads,), **f32),
         "dh0": torch.empty((batch, dim, dstate), **f32) if want_dh0 else None}
    if stream is None:
        stream = torch.cuda.current_stream(u.device).cuda_stream
    ssm_selective_scan_bwd_ckpt(dims, u, delta, A, B, C, D, z, delta_bias, softplus, h0, dout, dlast, ckpt, g,
                                workspace, workspace.numel() * workspace.element_size(), stream)
    return g


_fn_cls = None


def _selective_scan_function():
    """The torch.autograd.Function over the forward and backward entry points (built
    on first use, so that importing the package does not import torch)."""
    global _fn_cls
    if _fn_cls is not None:
        return _fn_cls
    import torch

    class SelectiveScanFn(torch.autograd.Function):
        @staticmethod
        def forward(ctx, u, delta, A, B, C, D, z, delta_bias, h0, softplus, store_states):
            # where the backward covers the shape, the forward stores the states it walks from
            ck = None
            if store_states and any(ctx.needs_input_grad) and bwd_covers(u, delta, A, B) and u.numel() > 0:
                ck = torch.empty(ckpt_shape(u.shape[0], u.shape[1], u.shape[2], B.shape[2]),
                                 dtype=torch.float32, device=u.device)
            out, last = selective_scan_fwd(u, delta, A, B, C, D, z, delta_bias, softplus, h0=h0, ckpt=ck)
            ctx.save_for_backward(u, delta, A, B, C, D, z, delta_bias, h0, ck)
            ctx.softplus = softplus
            return out, last

        @staticmethod
        def backward(ctx, dout, dlast):
            u, delta, A, B, C, D, z, delta_bias, h0, ck = ctx.saved_tensors
            want_dh0 = h0 is not None and ctx.needs_input_grad[8]
            g = selective_scan_bwd(u, delta, A, B, C, dout.contiguous(), D, z, delta_bias, ctx.softplus, h0=h0,
                                   dlast=dlast.contiguous() if dlast is not None else None, want_dh0=want_dh0,
                                   ckpt=ck)
            return (g["du"], g["ddelta"], g["dA"], g["dB"].to(B.dtype), g["dC"].to(C.dtype),
                    g["dD"] if D is not None else None, g["dz"], g["ddelta_bias"] if delta_bias is not None else None,
                    g["dh0"], None, None)

    _fn_cls = SelectiveScanFn
    return _fn_cls


def selective_scan_fn(u, delta, A, B, C, D=None, z=None, delta_bias=None, softplus: bool = True, h0=None,
                      store_states: bool = True):
    """The forward scan as a differentiable torch operation: returns (out, last_state),
    and the backward runs ssm_selective_scan_bwd (dstate 8 to 128, both layouts).  On the
    shapes its tiled kernel takes, the forward also stores the states the backward walks
    back from (ckpt_shape: B*D*L*N/2 bytes) unless store_states is False; the backward then
    recomputes them.  dB and dC are formed in fp32 and returned in B's and C's dtype."""
    return _selective_scan_function().apply(u, delta, A, B, C, D, z, delta_bias, h0, softplus, store_states)
