"""Runs in a child process whose SSM_SCAN_LIBRARY names the debug build of the
library (SSM_DEBUG: every scan kernel checks its indices against the buffers it
touches and records SSM_ERR_BOUNDS instead of an out-of-range access).  Each
shape must come back with the device status SSM_OK and match the oracle."""
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, HERE)
sys.path.insert(0, os.path.dirname(HERE))

import numpy as np  # noqa: E402

import oracle  # noqa: E402
import ssm_inputs as si  # noqa: E402
from parity import check_out, check_state, run_gpu, to_host_f64  # noqa: E402

# (batch, dim, L, N, nheads, ngroups, dtype, plan options): ragged and short sequences,
# partial channel tiles, groups, heads, every state size, both kernels
SHAPES = [
    (2, 80, 300, 16, 0, 1, "bf16", {}),
    (2, 80, 300, 16, 0, 1, "bf16", dict(tensor_memory=2, warps=16, states_per_lane=2)),
    (1, 40, 33, 16, 0, 1, "bf16", dict(tensor_memory=2, warps=12, states_per_lane=4)),
    (3, 32, 97, 16, 0, 1, "bf16", dict(tensor_memory=2, warps=16, states_per_lane=2, time_lanes=2, seg_len=32)),
    (2, 96, 200, 16, 0, 2, "bf16", dict(tensor_memory=1, warps=8, states_per_lane=4, seg_len=64, ctas=3)),
    (3, 40, 257, 16, 0, 1, "f32", {}),
    (2, 64, 200, 128, 4, 1, "bf16", {}),
    (2, 24, 120, 8, 0, 1, "bf16", {}),
    (2, 40, 88, 32, 0, 1, "bf16", {}),
    (1, 40, 72, 64, 0, 1, "f32", {}),
    (2, 64, 160, 64, 8, 2, "bf16", dict(seg_len=32)),
    (1, 17, 5, 16, 0, 1, "bf16", {}),
]


def main():
    import selective_state_space_30_b200 as ssm
    assert os.path.basename(ssm._abi.LIB_PATH) == "libssmscan_debug.so", ssm._abi.LIB_PATH
    for b, dm, L, N, H, G, dt, opts in SHAPES:
        dims = si.Dims(b, dm, L, N, nheads=H, ngroups=G, dtype=dt)
        head = dims.head_mode
        recipe = si.Recipe(a_init="neg_uniform_1_16" if (head or N != 16) else "neg_n_plus_1",
                           d_init="normal", delta_init="normal_half")
        inp = si.make_inputs(dims, recipe, 3 + L)
        # run_gpu asserts the device status (SSM_OK: no index left its buffer)
        out, last = run_gpu(dims, inp, opts=opts)
        ro, rl, rm = oracle.run_inputs(dims, inp)
        check_out(to_host_f64(out), ro, rm, dt, what=f"debug build {dims} {opts}")
        check_state(to_host_f64(last), rl, what=f"debug build last_state {dims} {opts}")
    # the forward variant that also stores the backward's states (S6 layout, N = 16)
    import torch
    from parity import OPTION_CODES, to_device
    for b, dm, L, dt, opts in [(2, 80, 300, "bf16", {}), (3, 40, 257, "f32", {}), (1, 17, 5, "bf16", {}),
                               (2, 64, 333, "bf16", dict(tensor_memory=1, warps=8, states_per_lane=2, seg_len=128))]:
        dims = si.Dims(b, dm, L, 16, dtype=dt)
        inp = si.make_inputs(dims, si.Recipe(d_init="normal", delta_init="normal_half"), 5 + L)
        out0, last0 = run_gpu(dims, inp, opts=opts)
        io = ssm.SSM_BF16 if dt == "bf16" else ssm.SSM_F32
        d = ssm.make_dims(b, dm, L, 16, dm, 1, io)
        dev = {k: to_device(inp.get(k)) for k in ("u", "delta", "A", "B", "C", "D", "z", "delta_bias")}
        out = torch.empty_like(dev["u"])
        last = torch.empty((b, dm, 16), dtype=torch.float32, device="cuda")
        ck = torch.empty((b, dm, (L + 7) // 8, 16), dtype=torch.float32, device="cuda")
        plan = ssm.ssm_scan_plan(d, 0)
        try:
            for k, v in opts.items():
                ssm.ssm_scan_set_option(plan, OPTION_CODES[k], v)
            ssm.ssm_selective_scan_fwd_ckpt(plan, dev["u"], dev["delta"], dev["A"], dev["B"], dev["C"], dev["D"],
                                            dev["z"], dev["delta_bias"], True, d, None, out, last, ck)
            assert ssm.ssm_scan_device_status(plan) == ssm.SSM_OK, f"stored-state forward {dims} {opts}"
            torch.cuda.synchronize()
        finally:
            ssm.ssm_scan_destroy(plan)
        assert torch.equal(out, out0) and torch.equal(last, last0), f"stored-state forward differs {dims} {opts}"
    print("debug build: all shapes SSM_OK and at parity")


if __name__ == "__main__":
    main()
