"""Shared helpers of the parity tests: tolerances, device transfer, C-ABI runs.

Tolerances (written out here, used by every test):
  * fp32 outputs and every last_state:      |gpu - ref| <= 1e-4 * (1 + |ref|)
  * bf16 outputs, the stated bound:         |gpu - ref| <= ulp_bf16(ref) + 2e-3 * |ref|
    gated bound (what the test enforces):   the stated bound + 1e-4 * mag
    where mag = |silu(z)| * (sum_n |C_n h_n| + |D u|) is the oracle's fp64 size of
    the terms summed into y.  The kernel sums them in fp32, so where they cancel
    the fp32 rounding of the sum (about N * 2^-24 * mag) can exceed a bound
    relative to |ref|; 1e-4 * mag is ~100x that rounding and still far below
    any real error (a wrong term moves the result by O(mag)).  Tests report how
    many outputs meet the stated bound alone.
ulp_bf16(ref) is the spacing of bf16 numbers at bf16(ref): 2^(floor(log2|bf16(ref)|) - 7).
"""
from __future__ import annotations

import numpy as np

import oracle
import ssm_inputs as si


def bf16_round_f64(x: np.ndarray) -> np.ndarray:
    import torch
    return torch.from_numpy(np.asarray(x, dtype=np.float64)).to(torch.bfloat16).to(torch.float64).numpy()


def bf16_ulp(ref: np.ndarray) -> np.ndarray:
    r = np.abs(bf16_round_f64(ref))
    e = np.floor(np.log2(np.maximum(r, 2.0 ** -126)))
    return 2.0 ** (e - 7)


def check_out(gpu: np.ndarray, ref: np.ndarray, mag: np.ndarray, dtype: str, what: str = "out") -> dict:
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert gpu.shape == ref.shape, (gpu.shape, ref.shape)
    assert np.all(np.isfinite(gpu)), f"{what}: non-finite GPU values"
    err = np.abs(gpu - ref)
    if dtype == "f32":
        tol = 1e-4 * (1.0 + np.abs(ref))
        strict = err <= tol
        ok = strict
    else:
        stated = bf16_ulp(ref) + 2e-3 * np.abs(ref)
        strict = err <= stated
        ok = err <= stated + 1e-4 * mag
    n = err.size
    rep = {"n": int(n), "strict_pass": int(strict.sum()), "pass": int(ok.sum()),
           "max_err": float(err.max()) if n else 0.0}
    if n and not ok.all():
        k = int(np.argmax(~ok.ravel()))
        raise AssertionError(f"{what}: {n - int(ok.sum())} of {n} outside tolerance; first at flat {k}: "
                             f"gpu={gpu.ravel()[k]!r} ref={ref.ravel()[k]!r} mag={mag.ravel()[k]!r}")
    return rep


def check_state(gpu: np.ndarray, ref: np.ndarray, what: str = "last_state") -> dict:
    gpu = np.asarray(gpu, dtype=np.float64)
    err = np.abs(gpu - ref)
    ok = err <= 1e-4 * (1.0 + np.abs(ref))
    if gpu.size and not ok.all():
        k = int(np.argmax(~ok.ravel()))
        raise AssertionError(f"{what}: {int((~ok).sum())} of {ok.size} outside 1e-4*(1+|ref|); first at {k}: "
                             f"gpu={gpu.ravel()[k]!r} ref={ref.ravel()[k]!r}")
    return {"n": int(gpu.size), "max_err": float(err.max()) if gpu.size else 0.0}


# ------------------------------------------------------------- device side

def to_device(arr, device="cuda"):
    """numpy (fp32, or bf16 bits as uint16) -> torch CUDA tensor of the same bits."""
    import torch
    if arr is None:
        return None
    a = np.ascontiguousarray(arr)
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(device)
    return torch.from_numpy(a).to(device)


def to_host_f64(t) -> np.ndarray:
    import torch
    if t.dtype == torch.bfloat16:
        return t.float().cpu().numpy().astype(np.float64)
    return t.cpu().numpy().astype(np.float64)


OPTION_CODES = {"spin_limit": 1, "inject_stall": 2, "seg_len": 3, "warps": 4, "ctas": 5, "states_per_lane": 6,
                "ssd": 7, "time_lanes": 8, "tensor_memory": 9}


def run_gpu(dims: si.Dims, inp: dict, h0=None, with_state=True, device="cuda", stream=None, opts=None,
            expect_status=0):
    """Run the CUDA path through the C ABI (plan, options, forward, device status, destroy)."""
    import torch
    import selective_state_space_30_b200 as ssm
    io = ssm.SSM_BF16 if dims.dtype == "bf16" else ssm.SSM_F32
    d = ssm.make_dims(dims.batch, dims.dim, dims.seqlen, dims.dstate, dims.H, dims.ngroups, io)
    dev = {k: to_device(inp.get(k), device) for k in ("u", "delta", "A", "B", "C", "D", "z", "delta_bias")}
    out = torch.empty_like(dev["u"])
    last = torch.full((dims.batch, dims.dim, dims.dstate), float("nan"), dtype=torch.float32,
                      device=device) if with_state else None
    h0d = to_device(np.ascontiguousarray(h0, dtype=np.float32), device) if h0 is not None else None
    plan = ssm.ssm_scan_plan(d, torch.device(device).index or 0)
    try:
        for k, v in (opts or {}).items():
            ssm.ssm_scan_set_option(plan, OPTION_CODES[k], v)
        ssm.ssm_selective_scan_fwd_h0(plan, dev["u"], dev["delta"], dev["A"], dev["B"], dev["C"], dev["D"],
                                      dev["z"], dev["delta_bias"], bool(inp.get("softplus", True)), d, h0d, out,
                                      last, stream)
        st = ssm.ssm_scan_device_status(plan, stream)
        assert st == expect_status, f"device status {st}, expected {expect_status}"
        torch.cuda.synchronize()
    finally:
        ssm.ssm_scan_destroy(plan)
    return out, last


def oracle_rows(dims: si.Dims, inp: dict, channels, h0=None):
    """The oracle on a subset of channels (rows of u, z, delta taken from the full tensors)."""
    H = dims.H
    P = dims.dim // H
    u = np.stack([inp["u"][c // dims.dim, c % dims.dim] for c in channels])
    z = np.stack([inp["z"][c // dims.dim, c % dims.dim] for c in channels]) if inp.get("z") is not None else None
    dl = np.stack([inp["delta"][c // dims.dim, (c % dims.dim) // P] for c in channels])
    h0r = np.stack([h0[c // dims.dim, c % dims.dim] for c in channels]) if h0 is not None else None
    rows = dict(inp, u=u, z=z, delta=dl)
    return oracle.run_inputs(dims, rows, channels=channels, h0=h0r)


def sample_channels(dims: si.Dims, k: int, seed: int = 1234):
    """k flat channel ids: the first and last channel of every batch row plus a seeded spread."""
    total = dims.batch * dims.dim
    rng = np.random.default_rng(seed)
    fixed = set()
    for b in range(dims.batch):
        fixed.update({b * dims.dim, b * dims.dim + dims.dim - 1})
    rest = rng.choice(total, size=min(total, k), replace=False)
    ch = sorted(fixed.union(int(x) for x in rest))
    return ch
