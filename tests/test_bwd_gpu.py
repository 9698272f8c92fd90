"""The backward scan (ssm_selective_scan_bwd) against the fp64 oracle's gradients.

Tolerance, per gradient element, from the oracle's magnitude sums (mag: the same
sum with every term and the carried state / state gradient replaced by their
absolute values; see oracle_selective_scan_bwd_f64):

    |gpu - ref| <= 1e-4 * mag + 2^-126 * G  (+ ulp_bf16(ref) for the bf16 outputs du, ddelta, dz)

The kernel forms every gradient in fp32 with the forward's approximations
(ex2.approx for exp, a polynomial softplus, rcp.approx in the sigmoids), so its
error is a small multiple of 2^-22 of the terms it sums, grown along the state
and gradient recurrences; 1e-4 * mag is the forward's gating bound.  A wrong
term moves a gradient by O(mag).  The floor: the kernel forms each decay
exp(dt A) in fp32 (ex2.approx.ftz), where a decay below 2^-126, the smallest normal
fp32 number, is zero, while the fp64 oracle keeps it.  Such a decay changes a
gradient by at most 2^-126 times the state gradient it multiplies; G bounds that state
gradient (1 by default; grad_scale() bounds it from the inputs for the shapes whose
states damp that fast).  Needs a B200.
"""
import numpy as np
import pytest
import torch

import oracle
import ssm_inputs as si
from parity import bf16_ulp, to_device, to_host_f64

pytestmark = pytest.mark.gpu

BF16_OUT = ("du", "ddelta", "dz")


def _recipe(kind):
    if kind == "c2":   # the mamba-130m recipe: delta ~ N(0, 0.5), D ~ N(0, 1)
        return si.Recipe(d_init="normal", delta_init="normal_half")
    if kind == "plain":
        return si.Recipe(has_D=False, has_z=False, has_bias=False, delta_init="normal_half")
    return si.Recipe()


def run_bwd(dims, inp, gin, want_dh0=False, softplus=True):
    import selective_state_space_30_b200 as ssm
    dev = {k: to_device(inp.get(k)) for k in ("u", "delta", "A", "B", "C", "D", "z", "delta_bias")}
    io = ssm.SSM_BF16 if dims.dtype == "bf16" else ssm.SSM_F32
    d = ssm.make_dims(dims.batch, dims.dim, dims.seqlen, dims.dstate, dims.H, dims.ngroups, io)
    ws = torch.empty(max(ssm.ssm_selective_scan_bwd_workspace_size(d), 1), dtype=torch.uint8, device="cuda")
    g = ssm.selective_scan_bwd(dev["u"], dev["delta"], dev["A"], dev["B"], dev["C"], to_device(gin["dout"]),
                               dev["D"], dev["z"], dev["delta_bias"], softplus, h0=to_device(gin.get("h0")),
                               dlast=to_device(gin.get("dlast")), want_dh0=want_dh0, workspace=ws)
    assert ssm.ssm_selective_scan_bwd_device_status(ws) == ssm.SSM_OK
    torch.cuda.synchronize()
    return g


def grad_scale(inp, gin, seqlen):
    """An upper bound on any state gradient: |dlast| + L * max|dy| * max|C|, with
    |dy| = |dout silu(z)| <= |dout| * max(|z|, 0.28) (every decay is at most 1)."""
    def f(a):
        if a is None:
            return 0.0
        a = np.asarray(a)
        if a.dtype == np.uint16:   # bf16 bits
            a = (a.astype(np.uint32) << 16).view(np.float32)
        return float(np.max(np.abs(a.astype(np.float64))))
    zmax = max(f(inp.get("z")), 0.28) if inp.get("z") is not None else 1.0
    return 1.0 + f(gin.get("dlast")) + seqlen * f(gin["dout"]) * zmax * f(inp["C"])


def check_grads(g, ref, mag, dtype, what="", bf16_out=BF16_OUT, gscale=1.0):
    for k, r in ref.items():
        if r is None:
            assert g.get(k) is None, f"{what}{k}: expected no output"
            continue
        got = to_host_f64(g[k]).reshape(r.shape)
        assert np.all(np.isfinite(got)), f"{what}{k}: non-finite values"
        err = np.abs(got - r)
        tol = 1e-4 * mag[k] + 2.0 ** -126 * gscale   # decays below fp32's smallest normal number are zero
        if dtype == "bf16" and k in bf16_out:
            tol = tol + bf16_ulp(r)
        bad = err > tol
        if bad.any():
            i = int(np.argmax(bad.ravel()))
            raise AssertionError(f"{what}{k}: {int(bad.sum())} of {bad.size} outside tolerance; first at flat {i}: "
                                 f"gpu={got.ravel()[i]!r} ref={r.ravel()[i]!r} mag={mag[k].ravel()[i]!r}")


CASES = [
    # (dims, recipe, dlast, h0, softplus)
    (si.Dims(2, 64, 100, 16, dtype="bf16"), "c2", True, True, True),       # ragged tail, h0 and dlast
    (si.Dims(1, 32, 64, 16, dtype="f32"), "default", False, False, True),  # two whole blocks
    (si.Dims(2, 64, 77, 16, dtype="f32"), "c2", True, False, True),        # L not a multiple of 4: element loads
    (si.Dims(2, 128, 96, 16, ngroups=2, dtype="bf16"), "c2", False, True, True),   # two groups
    (si.Dims(1, 96, 33, 16, dtype="bf16"), "plain", True, False, True),    # no z, D, bias; 33 = a block + 1
    (si.Dims(3, 32, 8, 16, dtype="bf16"), "default", False, False, True),  # shorter than a block
    (si.Dims(2, 32, 200, 16, dtype="f32"), "default", False, False, False),  # softplus off; 2 segments
    (si.Dims(1, 32, 1000, 16, dtype="bf16"), "c2", True, True, True),      # one tile: 8 chained segments
    (si.Dims(2, 64, 777, 16, dtype="f32"), "c2", True, False, True),       # 7 segments, ragged, element loads
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"{c[0].batch}x{c[0].dim}x{c[0].seqlen}g{c[0].ngroups}"
                                                      f"{c[0].dtype}-{c[1]}{'-sp' if c[4] else '-nosp'}")
def test_bwd_matches_oracle(case):
    dims, kind, dlast, h0, softplus = case
    inp = si.make_inputs(dims, _recipe(kind), 41)
    if not softplus:   # dt = delta + bias is dt itself and must be >= 0 (the caller's contract)
        inp["delta"] = (np.abs(si.make_inputs(dims, _recipe("c2"), 41)["delta"]) * np.float32(0.05)).astype(np.float32)
        inp["delta_bias"] = np.zeros_like(inp["delta_bias"])
    inp["softplus"] = softplus
    gin = si.make_grad_inputs(dims, 42, dlast=dlast, h0=h0)
    ref, mag = oracle.run_inputs_bwd(dims, inp, gin["dout"], dlast=gin["dlast"], h0=gin["h0"], want_dh0=True)
    g = run_bwd(dims, inp, gin, want_dh0=True, softplus=softplus)
    check_grads(g, ref, mag, dims.dtype)


def test_bwd_is_deterministic():
    """Every gradient but dB and dC repeats bit for bit; dB and dC are sums of atomic adds
    over the channels of a group, so between calls they may differ only by the rounding of
    the order of those adds (a few fp32 ulps of their terms' size)."""
    dims = si.Dims(2, 64, 130, 16, dtype="bf16")
    inp = si.make_inputs(dims, _recipe("c2"), 43)
    gin = si.make_grad_inputs(dims, 44, dlast=True)
    a = run_bwd(dims, inp, gin)
    b = run_bwd(dims, inp, gin)
    for k in a:
        if a[k] is None:
            continue
        if k in ("dB", "dC"):
            scale = float(torch.max(torch.abs(a[k]))) + 1.0
            assert float(torch.max(torch.abs(a[k] - b[k]))) <= 1e-5 * scale, f"{k} differs beyond rounding"
        else:
            assert torch.equal(a[k], b[k]), f"{k} differs between two identical calls"


def test_bwd_no_steps():
    """seqlen 0: every gradient is zero and dh0 = dlast."""
    dims = si.Dims(2, 32, 0, 16, dtype="bf16")
    inp = si.make_inputs(dims, _recipe("c2"), 45)
    gin = si.make_grad_inputs(dims, 46, dlast=True)
    g = run_bwd(dims, inp, gin, want_dh0=True)
    assert torch.equal(g["dh0"].cpu(), torch.from_numpy(gin["dlast"]))
    for k in ("dA", "dD", "ddelta_bias"):
        assert torch.count_nonzero(g[k]) == 0


def test_bwd_argument_checks():
    import selective_state_space_30_b200 as ssm
    x = torch.zeros(1 << 16, device="cuda")
    y = torch.zeros(1 << 16, device="cuda")
    ws = torch.zeros(1 << 20, dtype=torch.uint8, device="cuda")
    grads = {k: y for k in ("du", "ddelta", "dA", "dB", "dC")}

    def call(dims, z=None, g=grads, nbytes=ws.numel()):
        return ssm.ssm_selective_scan_bwd(dims, x, x, x, x, x, None, z, None, True, None, x, None, g, ws, nbytes,
                                          check=False)
    ok = ssm.make_dims(1, 32, 16, 16, 0, 1, ssm.SSM_BF16)
    assert ssm.ssm_selective_scan_bwd_workspace_size(ok) <= ws.numel()
    # shapes outside the tiled kernel run on the generic backward
    assert call(ssm.make_dims(1, 32, 16, 128, 0, 1, ssm.SSM_BF16)) == ssm.SSM_OK                 # dstate 128
    assert call(ssm.make_dims(1, 64, 16, 16, 2, 1, ssm.SSM_BF16)) == ssm.SSM_OK                  # per-head layout
    assert call(ssm.make_dims(1, 48, 16, 16, 0, 1, ssm.SSM_BF16)) == ssm.SSM_OK                  # dim not x32
    assert call(ssm.make_dims(1, 32, 16, 24, 0, 1, ssm.SSM_BF16)) == ssm.SSM_ERR_UNSUPPORTED     # dstate 24
    assert call(ok, z=x) == ssm.SSM_ERR_INVALID_ARG                                              # z without dz
    assert call(ok, nbytes=16) == ssm.SSM_ERR_INVALID_ARG                                        # workspace too small
    assert call(ok, g=dict(grads, dB=None)) == ssm.SSM_ERR_INVALID_ARG                           # missing output
    assert call(ok) == ssm.SSM_OK


def test_bwd_full_size_mamba_130m():
    """The bench workload (mamba-130m: 8 x 1536 x 2048, N = 16, bf16), every gradient against
    the full fp64 oracle backward: the recomputing call, and the call with the states the
    forward stored (both in the bench's launch configuration: 8-warp CTAs)."""
    import selective_state_space_30_b200 as ssm
    w = si.workload("mamba-130m")
    dims = w.dims
    inp = si.make_inputs(dims, w.recipe, w.seed)
    gin = si.make_grad_inputs(dims, 1)
    ref, mag = oracle.run_inputs_bwd(dims, inp, gin["dout"])
    g = run_bwd(dims, inp, gin)
    check_grads(g, ref, mag, dims.dtype, what="mamba-130m ")
    del g
    _, _, ck = _fwd_ckpt(dims, inp)
    dev = {k: to_device(inp.get(k)) for k in ("u", "delta", "A", "B", "C", "D", "z", "delta_bias")}
    d = ssm.make_dims(dims.batch, dims.dim, dims.seqlen, dims.dstate, dims.H, dims.ngroups, ssm.SSM_BF16)
    ws = torch.empty(ssm.ssm_selective_scan_bwd_workspace_size(d), dtype=torch.uint8, device="cuda")
    g = ssm.selective_scan_bwd(dev["u"], dev["delta"], dev["A"], dev["B"], dev["C"], to_device(gin["dout"]),
                               dev["D"], dev["z"], dev["delta_bias"], True, workspace=ws, ckpt=ck)
    assert ssm.ssm_selective_scan_bwd_device_status(ws) == ssm.SSM_OK
    torch.cuda.synchronize()
    check_grads(g, ref, mag, dims.dtype, what="mamba-130m, stored states ")


def test_bwd_wait_timeout_reports_and_recovers():
    """A chained wait that runs out (test hook: the flag it waits for is never written) ends
    the call with SSM_ERR_TIMEOUT, without a fault; the next call on the same context and
    workspace runs normally and matches the oracle."""
    import selective_state_space_30_b200 as ssm
    dims = si.Dims(1, 32, 1000, 16, dtype="bf16")          # one tile, 8 chained segments
    inp = si.make_inputs(dims, _recipe("c2"), 47)
    gin = si.make_grad_inputs(dims, 48)
    d = ssm.make_dims(1, 32, 1000, 16, 32, 1, ssm.SSM_BF16)
    ws = torch.empty(ssm.ssm_selective_scan_bwd_workspace_size(d), dtype=torch.uint8, device="cuda")
    dev = {k: to_device(inp.get(k)) for k in ("u", "delta", "A", "B", "C", "D", "z", "delta_bias")}
    try:
        ssm.ssm_selective_scan_bwd_test_hooks(True, 20000)   # 20 ms per wait
        ssm.selective_scan_bwd(dev["u"], dev["delta"], dev["A"], dev["B"], dev["C"], to_device(gin["dout"]),
                               dev["D"], dev["z"], dev["delta_bias"], True, workspace=ws)
        assert ssm.ssm_selective_scan_bwd_device_status(ws) == ssm.SSM_ERR_TIMEOUT
    finally:
        ssm.ssm_selective_scan_bwd_test_hooks(False, 0)
    g = ssm.selective_scan_bwd(dev["u"], dev["delta"], dev["A"], dev["B"], dev["C"], to_device(gin["dout"]),
                               dev["D"], dev["z"], dev["delta_bias"], True, workspace=ws)
    assert ssm.ssm_selective_scan_bwd_device_status(ws) == ssm.SSM_OK
    ref, mag = oracle.run_inputs_bwd(dims, inp, gin["dout"])
    check_grads(g, ref, mag, dims.dtype)


# ------------------------------------------------- the forward's stored states

def _prefix_states(dims, inp, h0):
    """The oracle's state entering every 8-step window: h0 (or zero) for window 0, else the
    last state of the oracle run over the first 8k steps."""
    nwin = (dims.seqlen + 7) // 8
    ref = np.zeros((dims.batch, dims.dim, nwin, dims.dstate))
    ref[:, :, 0] = h0 if h0 is not None else 0.0
    for k in range(1, nwin):
        t = 8 * k
        dk = si.Dims(dims.batch, dims.dim, t, dims.dstate, dims.nheads, dims.ngroups, dims.dtype)
        pre = dict(inp)
        for key in ("u", "delta", "z", "B", "C"):
            if pre.get(key) is not None:
                pre[key] = np.ascontiguousarray(pre[key][..., :t])
        _, last, _ = oracle.run_inputs(dk, pre, h0=h0)
        ref[:, :, k] = last
    return ref


def _fwd_ckpt(dims, inp, h0=None, opts=None):
    """ssm_selective_scan_fwd_ckpt through the C ABI on a plan with the given options;
    returns (out, last_state, ckpt) and the plain forward's (out, last_state)."""
    import selective_state_space_30_b200 as ssm
    from parity import OPTION_CODES
    io = ssm.SSM_BF16 if dims.dtype == "bf16" else ssm.SSM_F32
    d = ssm.make_dims(dims.batch, dims.dim, dims.seqlen, dims.dstate, dims.H, dims.ngroups, io)
    dev = {k: to_device(inp.get(k)) for k in ("u", "delta", "A", "B", "C", "D", "z", "delta_bias")}
    h0d = to_device(np.ascontiguousarray(h0, dtype=np.float32)) if h0 is not None else None
    nwin = (dims.seqlen + 7) // 8
    ck = torch.full((dims.batch, dims.dim, nwin, dims.dstate), float("nan"), device="cuda")
    res = []
    plan = ssm.ssm_scan_plan(d, 0)
    try:
        for k, v in (opts or {}).items():
            ssm.ssm_scan_set_option(plan, OPTION_CODES[k], v)
        for with_ckpt in (True, False):
            out = torch.empty_like(dev["u"])
            last = torch.empty((dims.batch, dims.dim, dims.dstate), dtype=torch.float32, device="cuda")
            args = (plan, dev["u"], dev["delta"], dev["A"], dev["B"], dev["C"], dev["D"], dev["z"],
                    dev["delta_bias"], True, d, h0d, out, last)
            if with_ckpt:
                ssm.ssm_selective_scan_fwd_ckpt(*args, ck)
            else:
                ssm.ssm_selective_scan_fwd_h0(*args)
            assert ssm.ssm_scan_device_status(plan) == ssm.SSM_OK
            res.append((out, last))
        torch.cuda.synchronize()
    finally:
        ssm.ssm_scan_destroy(plan)
    return res[0], res[1], ck


CKPT_CASES = [
    (si.Dims(2, 64, 300, 16, dtype="bf16"), None),                                   # the plan's layout
    (si.Dims(2, 64, 300, 16, dtype="bf16"), dict(tensor_memory=1, warps=8, states_per_lane=2)),   # per-lane rows
    (si.Dims(1, 32, 640, 16, dtype="bf16"), dict(tensor_memory=1, warps=8, states_per_lane=2, seg_len=128)),
    (si.Dims(2, 96, 200, 16, dtype="bf16"), dict(tensor_memory=1, warps=12, states_per_lane=4)),  # shuffles
    (si.Dims(1, 32, 100, 16, dtype="f32"), None),                                    # 32-step blocks
    (si.Dims(2, 64, 777, 16, dtype="f32"), dict(tensor_memory=1, warps=16, states_per_lane=2, seg_len=128)),
]


@pytest.mark.parametrize("case", CKPT_CASES, ids=lambda c: f"{c[0].batch}x{c[0].dim}x{c[0].seqlen}n{c[0].dstate}"
                                                           f"{c[0].dtype}-{'plan' if c[1] is None else c[1]['warps']}")
def test_forward_stores_window_states(case):
    """ssm_selective_scan_fwd_ckpt: outputs bit-equal to the plain forward, and every stored
    state (window k: the state entering step 8k) equal, within the forward's state bound,
    to the oracle's last state over the first 8k steps (window 0: h0)."""
    dims, opts = case
    inp = si.make_inputs(dims, _recipe("c2"), 51)
    h0 = si.make_grad_inputs(dims, 52, h0=True)["h0"]
    (out, last), (out0, last0), ck = _fwd_ckpt(dims, inp, h0, opts)
    assert torch.equal(out, out0) and torch.equal(last, last0)
    ref = _prefix_states(dims, inp, h0)
    from parity import check_state
    check_state(to_host_f64(ck), ref, what="stored states")


@pytest.mark.parametrize("dims,opts", [(si.Dims(2, 64, 256, 16, dtype="bf16"), dict(tensor_memory=2)),
                                       (si.Dims(2, 64, 129, 8, dtype="bf16"), None),
                                       (si.Dims(2, 64, 128, 16, nheads=4, dtype="bf16"), None)],
                         ids=["tensor-memory", "dstate8", "per-head"])
def test_forward_checkpoints_refused_outside_the_backward(dims, opts):
    """The states are stored where the backward can use them: the register kernel, the S6
    layout, dstate 16; elsewhere the call is refused (SSM_ERR_UNSUPPORTED)."""
    import selective_state_space_30_b200 as ssm
    recipe = si.Recipe(a_init="neg_uniform_1_16") if dims.head_mode else _recipe("c2")
    inp = si.make_inputs(dims, recipe, 53)
    with pytest.raises(ssm.SsmError):
        _fwd_ckpt(dims, inp, None, opts)


@pytest.mark.parametrize("case", [CASES[0], CASES[2], CASES[4], CASES[5], CASES[7], CASES[8],
                                  (si.Dims(2, 32, 5, 16, dtype="bf16"), "c2", True, True, True)],
                         ids=["2x64x100bf16", "2x64x77f32", "1x96x33bf16", "3x32x8bf16", "1x32x1000bf16",
                              "2x64x777f32", "2x32x5bf16"])
def test_bwd_with_forward_states(case):
    """ssm_selective_scan_bwd_ckpt with the states the forward stored: every gradient but dB
    and dC bit-equal to the backward that recomputes them (the same states, the same
    arithmetic), dB and dC within the rounding of their atomic sums, and all within the
    oracle's bound."""
    import selective_state_space_30_b200 as ssm
    dims, kind, dlast, h0, softplus = case
    inp = si.make_inputs(dims, _recipe(kind), 41)
    gin = si.make_grad_inputs(dims, 42, dlast=dlast, h0=h0)
    _, _, ck = _fwd_ckpt(dims, inp, gin.get("h0"))
    dev = {k: to_device(inp.get(k)) for k in ("u", "delta", "A", "B", "C", "D", "z", "delta_bias")}
    io = ssm.SSM_BF16 if dims.dtype == "bf16" else ssm.SSM_F32
    d = ssm.make_dims(dims.batch, dims.dim, dims.seqlen, dims.dstate, dims.H, dims.ngroups, io)
    ws = torch.empty(ssm.ssm_selective_scan_bwd_workspace_size(d), dtype=torch.uint8, device="cuda")
    g = ssm.selective_scan_bwd(dev["u"], dev["delta"], dev["A"], dev["B"], dev["C"], to_device(gin["dout"]),
                               dev["D"], dev["z"], dev["delta_bias"], True, h0=to_device(gin.get("h0")),
                               dlast=to_device(gin.get("dlast")), want_dh0=True, workspace=ws, ckpt=ck)
    assert ssm.ssm_selective_scan_bwd_device_status(ws) == ssm.SSM_OK
    torch.cuda.synchronize()
    g0 = run_bwd(dims, inp, gin, want_dh0=True)
    for k in g:
        if g[k] is None:
            continue
        if k in ("dB", "dC"):
            scale = float(torch.max(torch.abs(g0[k]))) + 1.0
            assert float(torch.max(torch.abs(g[k] - g0[k]))) <= 1e-5 * scale, f"{k} differs beyond rounding"
        else:
            assert torch.equal(g[k], g0[k]), f"{k} differs from the recomputing backward"
    ref, mag = oracle.run_inputs_bwd(dims, inp, gin["dout"], dlast=gin["dlast"], h0=gin["h0"], want_dh0=True)
    check_grads(g, ref, mag, dims.dtype)


def test_bwd_with_forward_states_8_byte_aligned():
    """Stored states at an address that is 8- but not 16-byte aligned take the element copies
    instead of the 16-byte ones: the same gradients (dB and dC within their rounding)."""
    import selective_state_space_30_b200 as ssm
    dims, kind, dlast, h0, softplus = CASES[0]
    inp = si.make_inputs(dims, _recipe(kind), 43)
    gin = si.make_grad_inputs(dims, 44, dlast=dlast, h0=h0)
    _, _, ck = _fwd_ckpt(dims, inp, gin.get("h0"))
    buf = torch.empty(ck.numel() + 2, dtype=torch.float32, device="cuda")
    ck8 = buf[2:].view(ck.shape)
    ck8.copy_(ck)
    assert ck8.data_ptr() % 16 == 8
    dev = {k: to_device(inp.get(k)) for k in ("u", "delta", "A", "B", "C", "D", "z", "delta_bias")}
    io = ssm.SSM_BF16 if dims.dtype == "bf16" else ssm.SSM_F32
    d = ssm.make_dims(dims.batch, dims.dim, dims.seqlen, dims.dstate, dims.H, dims.ngroups, io)
    ws = torch.empty(ssm.ssm_selective_scan_bwd_workspace_size(d), dtype=torch.uint8, device="cuda")
    res = []
    for c in (ck, ck8):
        res.append(ssm.selective_scan_bwd(dev["u"], dev["delta"], dev["A"], dev["B"], dev["C"],
                                          to_device(gin["dout"]), dev["D"], dev["z"], dev["delta_bias"], True,
                                          h0=to_device(gin.get("h0")), dlast=to_device(gin.get("dlast")),
                                          want_dh0=True, workspace=ws, ckpt=c))
        assert ssm.ssm_selective_scan_bwd_device_status(ws) == ssm.SSM_OK
    torch.cuda.synchronize()
    for k in res[0]:
        if res[0][k] is None:
            continue
        if k in ("dB", "dC"):
            scale = float(torch.max(torch.abs(res[0][k]))) + 1.0
            assert float(torch.max(torch.abs(res[1][k] - res[0][k]))) <= 1e-5 * scale, k
        else:
            assert torch.equal(res[0][k], res[1][k]), k


# ------------------------------------------ the generic backward (other layouts)

GENERIC_CASES = [
    # (dims, recipe kind, dlast, h0, softplus): shapes the tiled kernel does not take
    (si.Dims(2, 64, 100, 16, nheads=4, dtype="bf16"), "head", True, True, True),     # per-head, dstate 16
    (si.Dims(1, 128, 300, 128, nheads=2, dtype="bf16"), "head", True, True, True),   # the Mamba-2 shape, small
    (si.Dims(2, 64, 160, 64, nheads=8, ngroups=2, dtype="f32"), "head", False, False, True),   # heads and groups
    (si.Dims(2, 24, 77, 8, dtype="f32"), "c2", True, True, True),                    # dstate 8
    (si.Dims(2, 40, 260, 32, ngroups=2, dtype="bf16"), "c2", False, True, True),     # dstate 32, two groups
    (si.Dims(1, 16, 513, 64, dtype="f32"), "c2", True, False, True),                 # two segments and a step
    (si.Dims(2, 48, 90, 16, dtype="bf16"), "c2", True, True, True),                  # 48 channels: no 32-channel tile
    (si.Dims(1, 32, 70, 128, nheads=4, dtype="f32"), "plainhead", False, False, False),   # no z, D, bias; no softplus
    (si.Dims(1, 6, 70, 32, dtype="f32"), "c2", True, True, True),                     # 2 channels per CTA
    (si.Dims(2, 2, 50, 128, nheads=1, dtype="bf16"), "head", True, False, True),      # one head of 2 channels
    (si.Dims(1, 128, 256, 128, nheads=2, dtype="bf16"), "head", True, True, True),   # 16-byte B and C loads
    (si.Dims(2, 64, 96, 32, dtype="bf16"), "c2", True, False, True),                 # the same, dstate 32
    (si.Dims(1, 2, 70, 8, nheads=1, dtype="f32"), "head", True, True, True),         # 16 threads: fewer than the steps
    (si.Dims(2, 3, 45, 8, dtype="f32"), "c2", False, True, True),                    # 8 threads per CTA
]


def _generic_recipe(kind):
    if kind == "head":
        return si.Recipe(a_init="neg_uniform_1_16", d_init="normal", delta_init="normal_half")
    if kind == "plainhead":
        return si.Recipe(a_init="neg_uniform_1_16", has_D=False, has_z=False, has_bias=False,
                         delta_init="normal_half")
    if kind == "c2":
        return si.Recipe(a_init="neg_uniform_1_16", d_init="normal", delta_init="normal_half")
    raise ValueError(kind)


@pytest.mark.parametrize("case", GENERIC_CASES,
                         ids=lambda c: f"{c[0].batch}x{c[0].dim}x{c[0].seqlen}n{c[0].dstate}h{c[0].H}g{c[0].ngroups}"
                                       f"{c[0].dtype}-{c[1]}")
def test_generic_bwd_matches_oracle(case):
    """The per-head layout and dstate 8 to 128 run on the generic backward: every gradient
    against the oracle's, within the same bound as the tiled kernel."""
    dims, kind, dlast, h0, softplus = case
    inp = si.make_inputs(dims, _generic_recipe(kind), 61)
    if not softplus:
        inp["delta"] = (np.abs(si.make_inputs(dims, _generic_recipe("head"), 61)["delta"]) *
                        np.float32(0.05)).astype(np.float32)
        if dims.dtype == "bf16":
            raise AssertionError("the no-softplus case is fp32")
    inp["softplus"] = softplus
    gin = si.make_grad_inputs(dims, 62, dlast=dlast, h0=h0)
    ref, mag = oracle.run_inputs_bwd(dims, inp, gin["dout"], dlast=gin["dlast"], h0=gin["h0"], want_dh0=True)
    g = run_bwd(dims, inp, gin, want_dh0=True, softplus=softplus)
    check_grads(g, ref, mag, dims.dtype, what=f"{dims} ")


def test_generic_bwd_refuses_stored_states_and_odd_dstate():
    """The forward stores no states for these shapes, so a ckpt pointer is an argument
    error; a dstate outside {8, 16, 32, 64, 128} is unsupported."""
    import selective_state_space_30_b200 as ssm
    x = torch.zeros(1 << 16, device="cuda")
    ws = torch.zeros(1 << 20, dtype=torch.uint8, device="cuda")
    grads = {k: x for k in ("du", "ddelta", "dA", "dB", "dC")}
    head = ssm.make_dims(1, 64, 16, 16, 4, 1, ssm.SSM_BF16)
    assert ssm.ssm_selective_scan_bwd_ckpt(head, x, x, x, x, x, None, None, None, True, None, x, None, x, grads,
                                           ws, ws.numel(), check=False) == ssm.SSM_ERR_INVALID_ARG
    odd = ssm.make_dims(1, 32, 16, 12, 0, 1, ssm.SSM_BF16)
    assert ssm.ssm_selective_scan_bwd(odd, x, x, x, x, x, None, None, None, True, None, x, None, grads, ws,
                                      ws.numel(), check=False) == ssm.SSM_ERR_UNSUPPORTED
