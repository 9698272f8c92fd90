"""selective_scan_fn, the forward and backward entry points as one torch autograd
operation, against the fp64 oracle's forward and gradients.

The incoming gradients are the seeded dout (in the I/O dtype) and dlast; the loss
is therefore sum(dout * out) + sum(dlast * last_state), the one the oracle's backward
differentiates.  Tolerances are those of the backward's own tests; dB and dC come
back in B's and C's dtype, so for bf16 they also take one bf16 ulp.  Needs a B200.
"""
import pytest
import torch

import oracle
import ssm_inputs as si
from parity import check_out, check_state, to_device, to_host_f64
from test_bwd_gpu import BF16_OUT, _recipe, check_grads

pytestmark = pytest.mark.gpu

INPUTS = ("u", "delta", "A", "B", "C", "D", "z", "delta_bias")
GRAD_OF = {"u": "du", "delta": "ddelta", "A": "dA", "B": "dB", "C": "dC", "D": "dD", "z": "dz",
           "delta_bias": "ddelta_bias"}


@pytest.mark.parametrize("dtype,store_states", [("bf16", True), ("f32", True), ("bf16", False)])
def test_autograd_matches_oracle(dtype, store_states):
    """store_states False: the forward stores nothing and the backward recomputes the states."""
    import selective_state_space_30_b200 as ssm
    dims = si.Dims(2, 64, 100, 16, dtype=dtype)
    inp = si.make_inputs(dims, _recipe("c2"), 51)
    inp["softplus"] = True
    gin = si.make_grad_inputs(dims, 52, dlast=True, h0=True)
    leaves = {k: to_device(inp[k]).requires_grad_() for k in INPUTS}
    h0 = to_device(gin["h0"]).requires_grad_()
    out, last = ssm.selective_scan_fn(*(leaves[k] for k in INPUTS), softplus=True, h0=h0, store_states=store_states)
    torch.autograd.backward([out, last], [to_device(gin["dout"]), to_device(gin["dlast"])])
    torch.cuda.synchronize()

    # the forward half: the same outputs as the oracle's forward from h0
    ref_out, ref_last, mag_out = oracle.run_inputs(dims, inp, h0=gin["h0"])
    check_out(to_host_f64(out.detach()), ref_out, mag_out, dtype)
    check_state(to_host_f64(last.detach()), ref_last)

    # the backward half: every leaf's gradient
    ref, mag = oracle.run_inputs_bwd(dims, inp, gin["dout"], dlast=gin["dlast"], h0=gin["h0"], want_dh0=True)
    got = {GRAD_OF[k]: leaves[k].grad for k in INPUTS}
    got["dh0"] = h0.grad
    for k in ("dB", "dC"):
        assert got[k].dtype == leaves[k[1:]].dtype
    check_grads(got, ref, mag, dtype, what="autograd ", bf16_out=BF16_OUT + ("dB", "dC"))


def test_autograd_without_optional_inputs():
    """No D, z or bias, no h0, and last_state unused (its incoming gradient is zero)."""
    import selective_state_space_30_b200 as ssm
    dims = si.Dims(1, 32, 40, 16, dtype="f32")
    inp = si.make_inputs(dims, si.Recipe(has_D=False, has_z=False, has_bias=False, delta_init="normal_half"), 53)
    inp["softplus"] = True
    gin = si.make_grad_inputs(dims, 54)
    leaves = {k: to_device(inp[k]).requires_grad_() for k in ("u", "delta", "A", "B", "C")}
    out, _ = ssm.selective_scan_fn(leaves["u"], leaves["delta"], leaves["A"], leaves["B"], leaves["C"])
    out.backward(to_device(gin["dout"]))
    ref, mag = oracle.run_inputs_bwd(dims, inp, gin["dout"])
    got = {GRAD_OF[k]: leaves[k].grad for k in leaves}
    check_grads(got, {k: ref[k] for k in got}, mag, "f32", what="autograd, no options ")


@pytest.mark.parametrize("dims", [si.Dims(2, 64, 130, 16, nheads=4, dtype="bf16"),
                                  si.Dims(1, 128, 200, 128, nheads=2, dtype="bf16")],
                         ids=["per-head-n16", "per-head-n128"])
def test_autograd_per_head_layout(dims):
    """The per-head (Mamba-2) layout through selective_scan_fn: the forward (the scan
    kernel, or the chunked tensor-core path for dstate 128) and the generic backward;
    every leaf's gradient against the oracle's, A and delta_bias per head."""
    import selective_state_space_30_b200 as ssm
    inp = si.make_inputs(dims, si.Recipe(a_init="neg_uniform_1_16", d_init="normal", delta_init="normal_half"), 55)
    inp["softplus"] = True
    gin = si.make_grad_inputs(dims, 56, dlast=True)
    leaves = {k: to_device(inp[k]).requires_grad_() for k in INPUTS}
    out, last = ssm.selective_scan_fn(*(leaves[k] for k in INPUTS), softplus=True)
    torch.autograd.backward([out, last], [to_device(gin["dout"]), to_device(gin["dlast"])])
    torch.cuda.synchronize()
    ref_out, ref_last, mag_out = oracle.run_inputs(dims, inp)
    check_out(to_host_f64(out.detach()), ref_out, mag_out, dims.dtype)
    ref, mag = oracle.run_inputs_bwd(dims, inp, gin["dout"], dlast=gin["dlast"])
    got = {GRAD_OF[k]: leaves[k].grad for k in INPUTS}
    check_grads(got, {k: ref[k] for k in got}, mag, dims.dtype, what="autograd, per head ",
                bf16_out=BF16_OUT + ("dB", "dC"))
