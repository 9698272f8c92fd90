"""Seeded random shapes through the forward and the backward, each against the fp64
oracle.  The layout (per channel or per head), groups, dstate, I/O dtype, sequence
length (ragged, sometimes a multiple of the SSD chunk) and the optional inputs (D, z,
delta_bias, h0, dlast) are drawn together, so that combinations no hand-written case
names are covered as well.  Tolerances are those of the other parity tests.  Needs a
B200."""
import numpy as np
import pytest
import torch

import oracle
import ssm_inputs as si
from parity import check_out, check_state, run_gpu, to_device, to_host_f64
from test_bwd_gpu import check_grads, grad_scale

pytestmark = pytest.mark.gpu


def _draw(seed):
    """A random problem: (dims, recipe, h0, dlast)."""
    rng = np.random.default_rng(7000 + seed)
    N = int(rng.choice([8, 16, 32, 64, 128]))
    head = bool(rng.random() < 0.4)
    dtype = str(rng.choice(["bf16", "f32"]))
    if head:
        P = int(rng.choice([8, 16, 32, 64]))
        nh = int(rng.integers(1, 4))
        dim = P * nh
        ngroups = 2 if (nh % 2 == 0 and rng.random() < 0.5) else 1
    else:
        dim = int(rng.choice([16, 32, 48, 64, 96, 128]))
        nh = 0
        ngroups = 2 if rng.random() < 0.3 else 1
    batch = int(rng.integers(1, 3))
    L = int(rng.integers(1, 600))
    if head and N == 128 and dim % 64 == 0 and dtype == "bf16" and rng.random() < 0.5:
        L = 128 * int(rng.integers(1, 4))   # the chunked (SSD) path's shapes
    recipe = si.Recipe(a_init="neg_uniform_1_16" if head else "neg_n_plus_1", d_init="normal",
                       delta_init="normal_half", has_D=bool(rng.random() < 0.8), has_z=bool(rng.random() < 0.8),
                       has_bias=bool(rng.random() < 0.8))
    dims = si.Dims(batch, dim, L, N, nheads=nh, ngroups=ngroups, dtype=dtype)
    return dims, recipe, bool(rng.random() < 0.5), bool(rng.random() < 0.5)


@pytest.mark.parametrize("seed", range(64))
def test_fuzz_forward(seed):
    dims, recipe, with_h0, _ = _draw(seed)
    inp = si.make_inputs(dims, recipe, seed)
    h0 = si.make_grad_inputs(dims, seed, h0=True)["h0"] if with_h0 else None
    out, last = run_gpu(dims, inp, h0=h0)
    ref_out, ref_last, mag = oracle.run_inputs(dims, inp, h0=h0)
    check_out(to_host_f64(out), ref_out, mag, dims.dtype, what=f"{dims} out")
    check_state(to_host_f64(last), ref_last, what=f"{dims} last_state")


@pytest.mark.parametrize("seed", range(64))
def test_fuzz_backward(seed):
    import selective_state_space_30_b200 as ssm
    dims, recipe, with_h0, with_dlast = _draw(100 + seed)
    inp = si.make_inputs(dims, recipe, seed)
    gin = si.make_grad_inputs(dims, seed + 1, dlast=with_dlast, h0=with_h0)
    dev = {k: to_device(inp.get(k)) for k in ("u", "delta", "A", "B", "C", "D", "z", "delta_bias")}
    io = ssm.SSM_BF16 if dims.dtype == "bf16" else ssm.SSM_F32
    d = ssm.make_dims(dims.batch, dims.dim, dims.seqlen, dims.dstate, dims.H, dims.ngroups, io)
    ws = torch.empty(max(ssm.ssm_selective_scan_bwd_workspace_size(d), 1), dtype=torch.uint8, device="cuda")
    g = ssm.selective_scan_bwd(dev["u"], dev["delta"], dev["A"], dev["B"], dev["C"], to_device(gin["dout"]),
                               dev["D"], dev["z"], dev["delta_bias"], True, h0=to_device(gin.get("h0")),
                               dlast=to_device(gin.get("dlast")), want_dh0=with_h0, workspace=ws)
    assert ssm.ssm_selective_scan_bwd_device_status(ws) == ssm.SSM_OK
    torch.cuda.synchronize()
    ref, mag = oracle.run_inputs_bwd(dims, inp, gin["dout"], dlast=gin.get("dlast"), h0=gin.get("h0"),
                                     want_dh0=with_h0)
    check_grads(g, ref, mag, dims.dtype, what=f"{dims} ", gscale=grad_scale(inp, gin, dims.seqlen))


@pytest.mark.parametrize("seed", range(24))
def test_fuzz_backward_with_stored_states(seed):
    """The training path on random shapes the tiled backward covers (per channel, dstate 16,
    groups of whole 32-channel tiles): the forward stores its states, the backward reads them."""
    import selective_state_space_30_b200 as ssm
    rng = np.random.default_rng(9000 + seed)
    ngroups = 2 if rng.random() < 0.3 else 1
    dim = 32 * ngroups * int(rng.integers(1, 4))
    dims = si.Dims(int(rng.integers(1, 3)), dim, int(rng.integers(1, 700)), 16, ngroups=ngroups,
                   dtype=str(rng.choice(["bf16", "f32"])))
    recipe = si.Recipe(d_init="normal", delta_init="normal_half", has_D=bool(rng.random() < 0.8),
                       has_z=bool(rng.random() < 0.8), has_bias=bool(rng.random() < 0.8))
    with_h0, with_dlast = bool(rng.random() < 0.5), bool(rng.random() < 0.5)
    inp = si.make_inputs(dims, recipe, seed)
    gin = si.make_grad_inputs(dims, seed + 1, dlast=with_dlast, h0=with_h0)
    dev = {k: to_device(inp.get(k)) for k in ("u", "delta", "A", "B", "C", "D", "z", "delta_bias")}
    h0 = to_device(gin.get("h0"))
    ck = torch.empty(ssm.ckpt_shape(dims.batch, dims.dim, dims.seqlen, dims.dstate), dtype=torch.float32,
                     device="cuda")
    ssm.selective_scan_fwd(dev["u"], dev["delta"], dev["A"], dev["B"], dev["C"], dev["D"], dev["z"],
                           dev["delta_bias"], True, h0=h0, ckpt=ck)
    io = ssm.SSM_BF16 if dims.dtype == "bf16" else ssm.SSM_F32
    d = ssm.make_dims(dims.batch, dims.dim, dims.seqlen, dims.dstate, dims.H, dims.ngroups, io)
    ws = torch.empty(ssm.ssm_selective_scan_bwd_workspace_size(d), dtype=torch.uint8, device="cuda")
    g = ssm.selective_scan_bwd(dev["u"], dev["delta"], dev["A"], dev["B"], dev["C"], to_device(gin["dout"]),
                               dev["D"], dev["z"], dev["delta_bias"], True, h0=h0,
                               dlast=to_device(gin.get("dlast")), want_dh0=with_h0, workspace=ws, ckpt=ck)
    assert ssm.ssm_selective_scan_bwd_device_status(ws) == ssm.SSM_OK
    torch.cuda.synchronize()
    ref, mag = oracle.run_inputs_bwd(dims, inp, gin["dout"], dlast=gin.get("dlast"), h0=gin.get("h0"),
                                     want_dh0=with_h0)
    check_grads(g, ref, mag, dims.dtype, what=f"{dims}, stored states ")


@pytest.mark.parametrize("seed", [78, 138, 324, 360, 401])
def test_fuzz_backward_deep_decay(seed):
    """Seeds of the backward draw (dstate 64 or 128, A down to -128) whose decays fall
    below fp32's smallest normal number: the kernel's dh0 is zero where the fp64 oracle's
    is about 1e-38, within the tolerance's floor of 2^-126 times the state gradient bound."""
    test_fuzz_backward(seed)
