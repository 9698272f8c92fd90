"""The allocation-free entry point (needs a B200).

Callers that cannot allocate device memory -- code inside a framework that owns
all device memory through its own pre-reserved pool, or a hot path that must not
take an allocation -- call ssm_selective_scan_fwd_noalloc, which takes its
scratch from a fixed 8 MiB __device__ array instead of a plan's workspace.  This
test calls it through the C ABI twice in a row (the second call reuses the
array as the first left it) and checks each result against the plan-based
ssm_selective_scan_fwd within the parity tolerance; it also checks that a
problem too large for the array is refused before anything runs, pins the
size check at the array's limit (the largest batch that fits runs; one more row
is refused), reads the kernel-side status after a normal call, and makes a
bounded wait give up through the test hook to see that the status read reports
it.  The file is named to be collected last.
"""
import re

import numpy as np
import pytest
import torch

import ssm_inputs as si
from parity import check_out, check_state, to_device, to_host_f64

pytestmark = pytest.mark.gpu


def _run_plan(ssm, d, t, out, last):
    plan = ssm.ssm_scan_plan(d, 0)
    try:
        ssm.ssm_selective_scan_fwd(plan, t["u"], t["delta"], t["A"], t["B"], t["C"], t["D"], t["z"],
                                   t["delta_bias"], True, d, out, last, None)
        assert ssm.ssm_scan_device_status(plan) == ssm.SSM_OK
    finally:
        ssm.ssm_scan_destroy(plan)


@pytest.mark.parametrize("shape", [(2, 64, 512, 16, 0, "bf16"), (2, 80, 300, 16, 0, "bf16"),
                                   (2, 64, 384, 128, 4, "bf16"), (1, 48, 257, 16, 0, "f32")],
                         ids=lambda s: "x".join(map(str, s)))
def test_noalloc_matches_plan_path_twice(shape):
    import selective_state_space_30_b200 as ssm
    b, dm, L, N, H, dt = shape
    dims = si.Dims(b, dm, L, N, nheads=H, dtype=dt)
    recipe = si.Recipe(a_init="neg_uniform_1_16" if (dims.head_mode or N != 16) else "neg_n_plus_1",
                       d_init="normal", delta_init="normal_half")
    inp = si.make_inputs(dims, recipe, 21)
    io = ssm.SSM_BF16 if dt == "bf16" else ssm.SSM_F32
    d = ssm.make_dims(b, dm, L, N, dims.H, 1, io)
    t = {k: to_device(inp[k]) for k in ("u", "delta", "A", "B", "C", "D", "z", "delta_bias")}
    ref_out = torch.empty_like(t["u"])
    ref_last = torch.empty(b, dm, N, device="cuda")
    _run_plan(ssm, d, t, ref_out, ref_last)
    r_out, r_last = to_host_f64(ref_out), to_host_f64(ref_last)
    # the plan path's own sum sizes serve as the tolerance scale (same arithmetic)
    mag = np.abs(r_out) + 1.0
    for _ in range(2):
        out = torch.full_like(t["u"], float("nan"))
        last = torch.full((b, dm, N), float("nan"), device="cuda")
        ssm.ssm_selective_scan_fwd_noalloc(t["u"], t["delta"], t["A"], t["B"], t["C"], t["D"], t["z"],
                                           t["delta_bias"], True, d, out, last, None)
        torch.cuda.synchronize()
        assert ssm.ssm_selective_scan_noalloc_device_status() == ssm.SSM_OK
        check_out(to_host_f64(out), r_out, mag, dt, what="noalloc out")
        check_state(to_host_f64(last), r_last, what="noalloc last_state")


def test_noalloc_refuses_a_workspace_larger_than_its_scratch():
    import selective_state_space_30_b200 as ssm
    # 16 x 8192 channels x 128 states of carry (64 MiB) cannot fit the 8 MiB array;
    # the call must refuse before touching any of the (dummy) pointers
    d = ssm.make_dims(16, 8192, 1024, 128, 8192, 1, ssm.SSM_BF16)
    dummy = torch.empty(16, device="cuda")
    rc = ssm.ssm_selective_scan_fwd_noalloc(dummy, dummy, dummy, dummy, dummy, None, None, None, True, d,
                                            dummy, None, None, check=False)
    assert rc == ssm.SSM_ERR_UNSUPPORTED


SCRATCH_BYTES = 8 << 20


def _noalloc_need(ssm, d):
    """Workspace bytes of a call, computed as the entry point lays it out: a 64-byte header,
    one flag per channel tile (rounded up to 256 bytes), then CT x N fp32 carry states per
    tile.  The lane layout (and so CT) is the plan path's, which the entry point shares."""
    plan = ssm.ssm_scan_plan(d, 0)
    try:
        name = ssm.ssm_scan_plan_info(plan)["variant"]
        n_tiles = ssm.ssm_scan_plan_schedule(plan)["n_tiles"]
    finally:
        ssm.ssm_scan_destroy(plan)
    w, s, kt = (int(x) for x in re.search(r"_w(\d+)s(\d+)t(\d+)", name).groups())
    ct = w * 32 * s // (d.dstate * kt)
    carry_off = (64 + n_tiles * 4 + 255) // 256 * 256
    return carry_off + n_tiles * ct * d.dstate * 4


def test_noalloc_size_check_at_the_scratch_limit():
    """The largest batch whose workspace fits the 8 MiB array runs and matches the plan path;
    one more batch row is refused before anything runs."""
    import selective_state_space_30_b200 as ssm
    dim, L, N = 4096, 64, 16
    mk = lambda b: ssm.make_dims(b, dim, L, N, dim, 1, ssm.SSM_BF16)
    b = 1
    while _noalloc_need(ssm, mk(b + 1)) <= SCRATCH_BYTES:
        b += 1
    assert _noalloc_need(ssm, mk(b)) <= SCRATCH_BYTES < _noalloc_need(ssm, mk(b + 1))
    assert _noalloc_need(ssm, mk(b)) > SCRATCH_BYTES - 2 * 64 * 4096   # close to the limit
    # one more row: refused, nothing touched
    dummy = torch.empty(16, device="cuda")
    rc = ssm.ssm_selective_scan_fwd_noalloc(dummy, dummy, dummy, dummy, dummy, None, None, None, True, mk(b + 1),
                                            dummy, None, None, check=False)
    assert rc == ssm.SSM_ERR_UNSUPPORTED
    # the largest batch that fits: runs, and agrees with the plan path
    dims = si.Dims(b, dim, L, N, dtype="bf16")
    inp = si.make_inputs(dims, si.Recipe(d_init="normal", delta_init="normal_half"), 5)
    t = {k: to_device(inp[k]) for k in ("u", "delta", "A", "B", "C", "D", "z", "delta_bias")}
    d = mk(b)
    ref_out = torch.empty_like(t["u"])
    ref_last = torch.empty(b, dim, N, device="cuda")
    _run_plan(ssm, d, t, ref_out, ref_last)
    out = torch.full_like(t["u"], float("nan"))
    last = torch.full((b, dim, N), float("nan"), device="cuda")
    ssm.ssm_selective_scan_fwd_noalloc(t["u"], t["delta"], t["A"], t["B"], t["C"], t["D"], t["z"],
                                       t["delta_bias"], True, d, out, last, None)
    assert ssm.ssm_selective_scan_noalloc_device_status() == ssm.SSM_OK
    r_out = to_host_f64(ref_out)
    check_out(to_host_f64(out), r_out, np.abs(r_out) + 1.0, "bf16", what="noalloc out at the limit")
    check_state(to_host_f64(last), to_host_f64(ref_last), what="noalloc last_state at the limit")


def test_noalloc_timeout_is_reported_and_the_next_call_is_clean():
    """With the stall hook on, a chained wait gives up (bounded), the status read says
    SSM_ERR_TIMEOUT once, and after the hook is off the next call matches the plan path."""
    import selective_state_space_30_b200 as ssm
    b, dm, L, N = 1, 64, 4096, 16       # one tile row, many segments: chained waits happen
    dims = si.Dims(b, dm, L, N, dtype="bf16")
    inp = si.make_inputs(dims, si.Recipe(d_init="normal", delta_init="normal_half"), 9)
    t = {k: to_device(inp[k]) for k in ("u", "delta", "A", "B", "C", "D", "z", "delta_bias")}
    d = ssm.make_dims(b, dm, L, N, dm, 1, ssm.SSM_BF16)
    out = torch.empty_like(t["u"])
    last = torch.empty(b, dm, N, device="cuda")
    ssm.ssm_selective_scan_noalloc_test_hooks(True, 4000)     # about 1 ms per wait
    try:
        ssm.ssm_selective_scan_fwd_noalloc(t["u"], t["delta"], t["A"], t["B"], t["C"], t["D"], t["z"],
                                           t["delta_bias"], True, d, out, last, None)
        assert ssm.ssm_selective_scan_noalloc_device_status() == ssm.SSM_ERR_TIMEOUT
        assert ssm.ssm_selective_scan_noalloc_device_status() == ssm.SSM_OK   # read and cleared
    finally:
        ssm.ssm_selective_scan_noalloc_test_hooks(False, 0)
    ref_out = torch.empty_like(t["u"])
    ref_last = torch.empty(b, dm, N, device="cuda")
    _run_plan(ssm, d, t, ref_out, ref_last)
    ssm.ssm_selective_scan_fwd_noalloc(t["u"], t["delta"], t["A"], t["B"], t["C"], t["D"], t["z"],
                                       t["delta_bias"], True, d, out, last, None)
    assert ssm.ssm_selective_scan_noalloc_device_status() == ssm.SSM_OK
    r_out = to_host_f64(ref_out)
    check_out(to_host_f64(out), r_out, np.abs(r_out) + 1.0, "bf16", what="noalloc out after a timeout")
