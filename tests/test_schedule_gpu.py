"""The chained-carry scheduler on the GPU: results do not depend on the schedule
(segment length, channels per lane, worker count) and a wait that runs out is
reported as SSM_ERR_TIMEOUT without hanging the GPU (needs a B200)."""
import re
import numpy as np
import pytest
import torch

import oracle
import ssm_inputs as si
from parity import OPTION_CODES, check_out, check_state, run_gpu, to_host_f64

pytestmark = pytest.mark.gpu

SHAPES = [
    si.Dims(2, 80, 300, 16, dtype="bf16"),            # ragged L, partial channel tile, scalar loads
    si.Dims(2, 64, 512, 16, dtype="bf16"),            # vector path
    si.Dims(1, 48, 257, 16, dtype="f32"),
    si.Dims(2, 64, 384, 128, nheads=4, dtype="bf16"),  # scalar A per head, N = 128
    si.Dims(2, 32, 224, 64, ngroups=2, dtype="bf16"),
]
SCHEDULES = [dict(seg_len=32), dict(seg_len=64, warps=4), dict(seg_len=96, warps=8), dict(seg_len=32, ctas=1),
             dict(seg_len=64, ctas=3, warps=8), dict(ctas=5), dict(seg_len=160, ctas=7, warps=4)]
# N <= 16: the other lane layouts (consumer warps x states per lane); the same
# per-state arithmetic, so the results stay bit-identical
SCHEDULES_SMALL_N = [dict(warps=16, states_per_lane=2), dict(warps=8, states_per_lane=2, seg_len=64, ctas=3),
                     dict(warps=4, states_per_lane=2), dict(warps=16, states_per_lane=2, seg_len=32, ctas=1)]
SCHEDULES_N16 = [dict(warps=12, states_per_lane=4), dict(warps=12, states_per_lane=4, seg_len=32, ctas=2)]
# bf16, N = 16, A per channel: the register kernel forced (the default there is the
# tensor-memory kernel), and the tensor-memory kernel's layouts, among them the
# sequence-parallel blocks (lanes split each 32-step block in time and join their
# sub-chunks by an associative scan); bit-identical among themselves for the same
# (kernel, S, KT)
SCHEDULES_REGISTER = [dict(tensor_memory=1), dict(tensor_memory=1, warps=16, states_per_lane=2, seg_len=64, ctas=3),
                      dict(tensor_memory=1, warps=8, states_per_lane=4)]
SCHEDULES_TENSOR_MEMORY = [dict(tensor_memory=2, warps=16, states_per_lane=2, time_lanes=1, seg_len=32, ctas=1),
                           dict(tensor_memory=2, warps=8, states_per_lane=4, time_lanes=1),
                           dict(tensor_memory=2, warps=12, states_per_lane=4, time_lanes=1, seg_len=96, ctas=5),
                           dict(tensor_memory=2, warps=16, states_per_lane=2, time_lanes=2),
                           dict(tensor_memory=2, warps=16, states_per_lane=2, time_lanes=2, seg_len=64, ctas=3),
                           dict(tensor_memory=2, warps=8, states_per_lane=2, time_lanes=2),
                           dict(tensor_memory=2, warps=8, states_per_lane=2, time_lanes=2, seg_len=32, ctas=1)]


def _recipe(d):
    if d.head_mode or d.dstate != 16:
        return si.Recipe(a_init="neg_uniform_1_16", d_init="normal", delta_init="normal_half")
    return si.Recipe(d_init="normal", delta_init="normal_half")


def _lane_layout(plan_variant: str):
    """(kernel, S, KT) of a variant name <ws|tc>_<dtype>_n<N>_w<W>s<S>t<KT>...: the per-state
    arithmetic depends on the kernel, the states per lane and the time sub-chunks, not on the
    warps or the segments."""
    m = re.search(r"^(ws|tc)_.*_w(\d+)s(\d+)t(\d+)", plan_variant)
    return m.group(1), int(m.group(3)), int(m.group(4))


@pytest.mark.parametrize("dims", SHAPES, ids=lambda d: f"{d.batch}x{d.dim}x{d.seqlen}x{d.dstate}h{d.H}g{d.ngroups}{d.dtype}")
def test_schedule_invariance(dims):
    """Every schedule agrees with the oracle; schedules with the same states per lane run
    the same fp32 operations in the same order (segments and blocks are 32-step aligned),
    so their results are bit-identical."""
    import selective_state_space_30_b200 as ssm
    inp = si.make_inputs(dims, _recipe(dims), 11)
    ro, rl, rm = oracle.run_inputs(dims, inp)
    tc_shape = dims.dstate == 16 and dims.dtype == "bf16" and not dims.head_mode
    scheds = [None] + SCHEDULES + (SCHEDULES_SMALL_N if dims.dstate <= 16 else []) + \
        (SCHEDULES_N16 if dims.dstate == 16 and dims.dtype == "bf16" else []) + \
        (SCHEDULES_REGISTER + SCHEDULES_TENSOR_MEMORY if tc_shape else [])
    io = ssm.SSM_BF16 if dims.dtype == "bf16" else ssm.SSM_F32
    refs = {}
    for opts in scheds:
        d = ssm.make_dims(dims.batch, dims.dim, dims.seqlen, dims.dstate, dims.H, dims.ngroups, io)
        plan = ssm.ssm_scan_plan(d, 0)
        try:
            for k, v in (opts or {}).items():
                ssm.ssm_scan_set_option(plan, OPTION_CODES[k], v)
            spl = _lane_layout(ssm.ssm_scan_plan_info(plan)["variant"])
        finally:
            ssm.ssm_scan_destroy(plan)
        out, last = run_gpu(dims, inp, opts=opts)
        if spl not in refs:
            check_out(to_host_f64(out), ro, rm, dims.dtype)
            check_state(to_host_f64(last), rl)
            refs[spl] = (out, last)
            continue
        ref_out, ref_last = refs[spl]
        assert torch.equal(out, ref_out), f"output differs under schedule {opts}"
        assert torch.equal(last, ref_last), f"last_state differs under schedule {opts}"


def test_schedule_with_initial_state():
    dims = si.Dims(2, 64, 320, 16, dtype="bf16")
    inp = si.make_inputs(dims, _recipe(dims), 12)
    h0 = np.random.default_rng(3).standard_normal((2, 64, 16)).astype(np.float32)
    ro, rl, rm = oracle.run_inputs(dims, inp, h0=h0)
    for opts in (None, dict(seg_len=32), dict(seg_len=64, ctas=2)):
        out, last = run_gpu(dims, inp, h0=h0, opts=opts)
        check_out(to_host_f64(out), ro, rm, "bf16")
        check_state(to_host_f64(last), rl)


def test_wait_timeout_is_reported_and_context_survives():
    """A chained wait on a flag that nothing sets gives up after the spin limit,
    records SSM_ERR_TIMEOUT, and the next call on the same context is correct."""
    import selective_state_space_30_b200 as ssm
    from parity import to_device
    dims = si.Dims(2, 64, 256, 16, dtype="bf16")
    inp = si.make_inputs(dims, _recipe(dims), 13)
    d = ssm.make_dims(2, 64, 256, 16, 64, 1, ssm.SSM_BF16)
    t = {k: to_device(inp[k]) for k in ("u", "delta", "A", "B", "C", "D", "z", "delta_bias")}
    out = torch.empty_like(t["u"])
    last = torch.empty(2, 64, 16, device="cuda")
    plan = ssm.ssm_scan_plan(d, 0)
    try:
        ssm.ssm_scan_set_option(plan, ssm.SSM_OPT_SEG_LEN, 64)       # 4 chained segments per tile
        ssm.ssm_scan_set_option(plan, ssm.SSM_OPT_SPIN_LIMIT, 2000)  # a few ms of polling
        ssm.ssm_scan_set_option(plan, ssm.SSM_OPT_INJECT_STALL, 1)
        ssm.ssm_selective_scan_fwd(plan, t["u"], t["delta"], t["A"], t["B"], t["C"], t["D"], t["z"],
                                   t["delta_bias"], True, d, out, last, None)
        assert ssm.ssm_scan_device_status(plan) == ssm.SSM_ERR_TIMEOUT
        assert ssm.ssm_scan_device_status(plan) == ssm.SSM_OK          # reading clears it
        ssm.ssm_scan_set_option(plan, ssm.SSM_OPT_INJECT_STALL, 0)
        ssm.ssm_selective_scan_fwd(plan, t["u"], t["delta"], t["A"], t["B"], t["C"], t["D"], t["z"],
                                   t["delta_bias"], True, d, out, last, None)
        assert ssm.ssm_scan_device_status(plan) == ssm.SSM_OK
        torch.cuda.synchronize()
    finally:
        ssm.ssm_scan_destroy(plan)
    ro, rl, rm = oracle.run_inputs(dims, inp)
    check_out(to_host_f64(out), ro, rm, "bf16")
    check_state(to_host_f64(last), rl)


def test_option_errors():
    import selective_state_space_30_b200 as ssm
    d = ssm.make_dims(1, 32, 64, 16, 32, 1, ssm.SSM_BF16)
    plan = ssm.ssm_scan_plan(d, 0)
    try:
        with pytest.raises(ssm.SsmError):
            ssm.ssm_scan_set_option(plan, 99, 1)
        with pytest.raises(ssm.SsmError):
            ssm.ssm_scan_set_option(plan, ssm.SSM_OPT_CONSUMER_WARPS, 3)
        with pytest.raises(ssm.SsmError):
            ssm.ssm_scan_set_option(plan, ssm.SSM_OPT_SPIN_LIMIT, 0)
        sch = ssm.ssm_scan_plan_schedule(plan)
        assert sch["n_seg"] >= 1 and sch["seg_len"] % 32 == 0 and sch["consumer_warps"] in (4, 8)
    finally:
        ssm.ssm_scan_destroy(plan)


def test_layout_option_checks():
    import selective_state_space_30_b200 as ssm
    from selective_state_space_30_b200 import _abi
    lib = _abi.load_library()
    # 8 x 1536 channels, N = 16, bf16: sixteen warps with two states per lane fill the SMs
    d = ssm.make_dims(8, 1536, 256, 16, 1536, 1, ssm.SSM_BF16)
    plan = ssm.ssm_scan_plan(d, 0)
    try:
        assert ssm.ssm_scan_plan_info(plan)["variant"] == "ws_bf16_n16_w16s2t1_vec"
        assert ssm.ssm_scan_plan_schedule(plan)["n_tiles"] >= 148
        # the tensor-memory kernel on request
        assert lib.ssm_scan_set_option(plan, ssm.SSM_OPT_TENSOR_MEMORY, 2) == ssm.SSM_OK
        assert ssm.ssm_scan_plan_info(plan)["variant"] == "tc_bf16_n16_w16s2t1_vec"
        assert lib.ssm_scan_set_option(plan, ssm.SSM_OPT_TENSOR_MEMORY, 0) == ssm.SSM_OK
        assert lib.ssm_scan_set_option(plan, ssm.SSM_OPT_STATES_PER_LANE, 3) == ssm.SSM_ERR_INVALID_ARG
        assert lib.ssm_scan_set_option(plan, ssm.SSM_OPT_CONSUMER_WARPS, 6) == ssm.SSM_ERR_INVALID_ARG
        assert lib.ssm_scan_set_option(plan, ssm.SSM_OPT_TIME_LANES, 3) == ssm.SSM_ERR_INVALID_ARG
        assert lib.ssm_scan_set_option(plan, ssm.SSM_OPT_TENSOR_MEMORY, 3) == ssm.SSM_ERR_INVALID_ARG
        # the register kernel on request
        assert lib.ssm_scan_set_option(plan, ssm.SSM_OPT_TENSOR_MEMORY, 1) == ssm.SSM_OK
        assert ssm.ssm_scan_plan_info(plan)["variant"].startswith("ws_bf16_n16_")
        assert lib.ssm_scan_set_option(plan, ssm.SSM_OPT_STATES_PER_LANE, 4) == ssm.SSM_OK
        assert lib.ssm_scan_set_option(plan, ssm.SSM_OPT_CONSUMER_WARPS, 8) == ssm.SSM_OK
        assert ssm.ssm_scan_plan_info(plan)["variant"] == "ws_bf16_n16_w8s4t1_vec"
        # sixteen warps exist only with two states per lane: refused, previous schedule kept
        assert lib.ssm_scan_set_option(plan, ssm.SSM_OPT_CONSUMER_WARPS, 16) == ssm.SSM_ERR_UNSUPPORTED
        assert ssm.ssm_scan_plan_info(plan)["variant"] == "ws_bf16_n16_w8s4t1_vec"
        # time sub-chunks exist only in the tensor-memory kernel
        assert lib.ssm_scan_set_option(plan, ssm.SSM_OPT_TIME_LANES, 2) == ssm.SSM_ERR_UNSUPPORTED
    finally:
        ssm.ssm_scan_destroy(plan)
    # 4 x 4096 channels: sixteen warps with two states per lane fill the SMs; 1 x 5120
    # channels: eight warps with two states per lane keep a tile per SM
    for shape, name in (((4, 4096), "ws_bf16_n16_w16s2t1_vec"), ((1, 5120), "ws_bf16_n16_w8s2t1_vec")):
        plan = ssm.ssm_scan_plan(ssm.make_dims(shape[0], shape[1], 256, 16, shape[1], 1, ssm.SSM_BF16), 0)
        try:
            assert ssm.ssm_scan_plan_info(plan)["variant"] == name
        finally:
            ssm.ssm_scan_destroy(plan)
    # fp32 I/O and the per-head layout have no tensor-memory kernel
    for dd in (ssm.make_dims(2, 64, 256, 16, 64, 1, ssm.SSM_F32), ssm.make_dims(2, 64, 256, 16, 4, 1, ssm.SSM_BF16)):
        plan = ssm.ssm_scan_plan(dd, 0)
        try:
            assert ssm.ssm_scan_plan_info(plan)["variant"].startswith("ws_")
            assert lib.ssm_scan_set_option(plan, ssm.SSM_OPT_TENSOR_MEMORY, 2) == ssm.SSM_ERR_UNSUPPORTED
        finally:
            ssm.ssm_scan_destroy(plan)
    dh = ssm.make_dims(2, 64, 256, 128, 4, 1, ssm.SSM_BF16)
    plan = ssm.ssm_scan_plan(dh, 0)
    try:
        assert lib.ssm_scan_set_option(plan, ssm.SSM_OPT_STATES_PER_LANE, 2) == ssm.SSM_ERR_UNSUPPORTED
        assert ssm.ssm_scan_plan_info(plan)["variant"].endswith("s16t1_head_vec")
    finally:
        ssm.ssm_scan_destroy(plan)
