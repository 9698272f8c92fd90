"""The chunked tensor-core (SSD) path for the per-head layout, dstate 128, head dim 64
(bf16 I/O), against the fp64 oracle, and against the scan kernel (needs a B200).

Same tolerances as every bf16 parity test (tests/parity.py): outputs within
ulp + 2e-3|ref| + 1e-4 mag, last_state within 1e-4 (1 + |ref|).
"""
import numpy as np
import pytest
import torch

import oracle
import ssm_inputs as si
from parity import check_out, check_state, run_gpu, to_host_f64

pytestmark = pytest.mark.gpu

SHAPES = [
    si.Dims(1, 128, 256, 128, nheads=2, dtype="bf16"),              # two chunks, two heads
    si.Dims(2, 256, 384, 128, nheads=4, ngroups=2, dtype="bf16"),   # heads in two B/C groups
    si.Dims(1, 64, 128, 128, nheads=1, dtype="bf16"),               # one chunk
    si.Dims(2, 128, 1024, 128, nheads=2, dtype="bf16"),             # eight chunks
]
RECIPE = si.Recipe(a_init="neg_uniform_1_16", d_init="normal", delta_init="normal_half")


def _variant(dims, opts=None):
    import selective_state_space_30_b200 as ssm
    from parity import OPTION_CODES
    d = ssm.make_dims(dims.batch, dims.dim, dims.seqlen, dims.dstate, dims.H, dims.ngroups, ssm.SSM_BF16)
    plan = ssm.ssm_scan_plan(d, 0)
    try:
        for k, v in (opts or {}).items():
            ssm.ssm_scan_set_option(plan, OPTION_CODES[k], v)
        return ssm.ssm_scan_plan_info(plan)["variant"]
    finally:
        ssm.ssm_scan_destroy(plan)


@pytest.mark.parametrize("dims", SHAPES, ids=lambda d: f"{d.batch}x{d.dim}x{d.seqlen}h{d.H}g{d.ngroups}")
def test_ssd_matches_oracle(dims):
    assert _variant(dims).startswith("ssd_")
    inp = si.make_inputs(dims, RECIPE, 51)
    out, last = run_gpu(dims, inp)
    ro, rl, rm = oracle.run_inputs(dims, inp)
    check_out(to_host_f64(out), ro, rm, "bf16")
    check_state(to_host_f64(last), rl)


def test_ssd_initial_state_and_no_gate():
    dims = si.Dims(2, 128, 256, 128, nheads=2, dtype="bf16")
    inp = si.make_inputs(dims, si.Recipe(a_init="neg_uniform_1_16", d_init="normal", delta_init="normal_half",
                                         has_z=False), 52)
    h0 = np.random.default_rng(9).standard_normal((2, 128, 128)).astype(np.float32)
    out, last = run_gpu(dims, inp, h0=h0)
    ro, rl, rm = oracle.run_inputs(dims, inp, h0=h0)
    check_out(to_host_f64(out), ro, rm, "bf16")
    check_state(to_host_f64(last), rl)


def test_ssd_agrees_with_the_scan_kernel():
    dims = si.Dims(2, 128, 512, 128, nheads=2, dtype="bf16")
    assert not _variant(dims, {"ssd": 1}).startswith("ssd_")
    inp = si.make_inputs(dims, RECIPE, 53)
    o1, l1 = run_gpu(dims, inp)
    o2, l2 = run_gpu(dims, inp, opts={"ssd": 1})
    ro, rl, rm = oracle.run_inputs(dims, inp)
    for o, l in ((o1, l1), (o2, l2)):
        check_out(to_host_f64(o), ro, rm, "bf16")
        check_state(to_host_f64(l), rl)
    # the two paths sum in different orders: close, not bitwise equal
    assert torch.allclose(l1, l2, rtol=1e-4, atol=1e-4)


def test_ssd_option_checks():
    import selective_state_space_30_b200 as ssm
    from selective_state_space_30_b200 import _abi
    lib = _abi.load_library()
    d = ssm.make_dims(1, 64, 200, 128, 1, 1, ssm.SSM_BF16)          # seqlen not a multiple of 128
    plan = ssm.ssm_scan_plan(d, 0)
    try:
        assert not ssm.ssm_scan_plan_info(plan)["variant"].startswith("ssd_")
        assert lib.ssm_scan_set_option(plan, ssm.SSM_OPT_SSD, 2) == ssm.SSM_ERR_UNSUPPORTED
        assert lib.ssm_scan_set_option(plan, ssm.SSM_OPT_SSD, 3) == ssm.SSM_ERR_INVALID_ARG
    finally:
        ssm.ssm_scan_destroy(plan)
