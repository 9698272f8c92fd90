"""The single-step state update (ssm_selective_state_update) against the oracle.

One step from a given state is the scan with seqlen 1 and h0 = state, so the
oracle is oracle.run_inputs on seqlen-1 inputs with h0; a run of K steps, state
carried in place, must match the oracle's K-step scan step by step (needs a B200).
"""
import numpy as np
import pytest
import torch

import oracle
import ssm_inputs as si
from parity import check_out, check_state, to_device, to_host_f64

pytestmark = pytest.mark.gpu

SHAPES = [
    si.Dims(8, 1536, 1, 16, dtype="bf16"),                 # mamba-130m decode step
    si.Dims(3, 40, 1, 16, dtype="f32"),                    # ragged channel count
    si.Dims(2, 64, 1, 8, dtype="bf16"),
    si.Dims(2, 48, 1, 32, ngroups=3, dtype="f32"),
    si.Dims(2, 32, 1, 64, dtype="bf16"),
    si.Dims(4, 2048, 1, 128, nheads=32, dtype="bf16"),     # Mamba-2 decode step
    si.Dims(1, 7, 1, 16, dtype="bf16"),                    # fewer lanes than a warp
]


def _recipe(d):
    if d.head_mode or d.dstate != 16:
        return si.Recipe(a_init="neg_uniform_1_16", d_init="normal", delta_init="normal_half")
    return si.Recipe(d_init="normal", delta_init="normal_half")


def _step(dims, inp, state, z=True, softplus=True):
    import selective_state_space_30_b200 as ssm
    io = ssm.SSM_BF16 if dims.dtype == "bf16" else ssm.SSM_F32
    d = ssm.make_dims(dims.batch, dims.dim, 1, dims.dstate, dims.H, dims.ngroups, io)
    dev = {k: to_device(inp.get(k)) for k in ("u", "delta", "A", "B", "C", "D", "z", "delta_bias")}
    out = torch.empty_like(dev["u"])
    ssm.ssm_selective_state_update(d, state, dev["u"], dev["delta"], dev["A"], dev["B"], dev["C"], dev["D"],
                                   dev["z"] if z else None, dev["delta_bias"], softplus, out)
    torch.cuda.synchronize()
    return out


@pytest.mark.parametrize("dims", SHAPES, ids=lambda d: f"{d.batch}x{d.dim}x{d.dstate}h{d.H}g{d.ngroups}{d.dtype}")
def test_one_step_matches_oracle(dims):
    inp = si.make_inputs(dims, _recipe(dims), 21)
    h0 = np.random.default_rng(5).standard_normal((dims.batch, dims.dim, dims.dstate)).astype(np.float32)
    state = torch.from_numpy(h0.copy()).cuda()
    out = _step(dims, inp, state)
    ro, rl, rm = oracle.run_inputs(dims, inp, h0=h0)
    check_out(to_host_f64(out), ro, rm, dims.dtype)
    check_state(to_host_f64(state), rl)


def test_steps_carry_state_like_the_scan():
    """K steps with the state updated in place = the oracle's K-step scan, output by output."""
    K = 24
    full = si.Dims(2, 96, K, 16, dtype="bf16")
    inp = si.make_inputs(full, _recipe(full), 22)
    h0 = np.random.default_rng(6).standard_normal((2, 96, 16)).astype(np.float32)
    ro, rl, rm = oracle.run_inputs(full, inp, h0=h0)
    state = torch.from_numpy(h0.copy()).cuda()
    one = si.Dims(2, 96, 1, 16, dtype="bf16")
    for t in range(K):
        step = dict(inp)
        for k in ("u", "z", "delta", "B", "C"):
            step[k] = np.ascontiguousarray(inp[k][..., t:t + 1])
        out = _step(one, step, state)
        check_out(to_host_f64(out), ro[..., t:t + 1], rm[..., t:t + 1], "bf16", what=f"out step {t}")
    check_state(to_host_f64(state), rl)


def test_without_gate_and_softplus():
    """softplus off: delta + delta_bias is dt itself, so the inputs give dt >= 0 (the caller's
    contract; a very negative dt makes exp(dt*A) overflow in fp32 while the fp64 oracle does not)."""
    dims = si.Dims(2, 64, 1, 16, dtype="f32")
    inp = si.make_inputs(dims, _recipe(dims), 23)
    inp["delta"] = (np.abs(inp["delta"]) * np.float32(0.05)).astype(np.float32)
    inp["delta_bias"] = np.zeros_like(inp["delta_bias"])
    h0 = np.random.default_rng(8).standard_normal((2, 64, 16)).astype(np.float32)
    state = torch.from_numpy(h0.copy()).cuda()
    out = _step(dims, inp, state, z=False, softplus=False)
    ro, rl, rm = oracle.run_inputs(dims, dict(inp, z=None, softplus=False), h0=h0)
    check_out(to_host_f64(out), ro, rm, "f32")
    check_state(to_host_f64(state), rl)


def test_argument_checks():
    import selective_state_space_30_b200 as ssm
    d2 = ssm.make_dims(2, 64, 2, 16, 64, 1, ssm.SSM_BF16)     # seqlen must be 1
    x = torch.zeros(2 * 64 * 16, device="cuda")
    rc = ssm.ssm_selective_state_update(d2, x, x, x, x, x, x, None, None, None, True, x, check=False)
    assert rc == ssm.SSM_ERR_INVALID_ARG
    d1 = ssm.make_dims(2, 64, 1, 24, 64, 1, ssm.SSM_BF16)     # no kernel for N = 24
    rc = ssm.ssm_selective_state_update(d1, x, x, x, x, x, x, None, None, None, True, x, check=False)
    assert rc == ssm.SSM_ERR_UNSUPPORTED
    d1 = ssm.make_dims(2, 64, 1, 16, 64, 1, ssm.SSM_BF16)
    rc = ssm.ssm_selective_state_update(d1, x[1:], x, x, x, x, x, None, None, None, True, x, check=False)
    assert rc == ssm.SSM_ERR_UNSUPPORTED                       # state not 16-byte aligned
    rc = ssm.ssm_selective_state_update(d1, None, x, x, x, x, x, None, None, None, True, x, check=False)
    assert rc == ssm.SSM_ERR_INVALID_ARG
