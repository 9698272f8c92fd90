"""CUDA path vs the fp64 oracle, element by element, through the C ABI (needs a B200)."""
import numpy as np
import pytest

import oracle
import ssm_inputs as si
from parity import check_out, check_state, oracle_rows, run_gpu, sample_channels, to_host_f64

pytestmark = pytest.mark.gpu


def _full_check(dims, recipe, seed=0, h0=None, inp=None):
    inp = inp if inp is not None else si.make_inputs(dims, recipe, seed)
    out, last = run_gpu(dims, inp, h0=h0)
    ro, rl, rm = oracle.run_inputs(dims, inp, h0=h0)
    rep = check_out(to_host_f64(out), ro, rm, dims.dtype)
    check_state(to_host_f64(last), rl)
    return rep


# --------------------------------------------------------------- the five workloads

def test_tiny_f32_full():
    w = si.WORKLOADS["tiny-f32"]
    rep = _full_check(w.dims, w.recipe, w.seed)
    assert rep["strict_pass"] == rep["n"]


@pytest.mark.parametrize("name", ["mamba-130m", "mamba-1.4b", "mamba-2.8b-long", "mamba2-n128"])
def test_workload_full_size_every_element(name):
    """Full-size run in the bench's launch configuration (a default plan); every output and
    every final state compared with the oracle, which runs over channel chunks so that its
    fp64 arrays stay small.  Reports how many outputs meet the stated bound alone."""
    w = si.WORKLOADS[name]
    d = w.dims
    inp = si.make_inputs(d, w.recipe, w.seed)
    out, last = run_gpu(d, inp)
    o = to_host_f64(out).reshape(d.batch * d.dim, d.seqlen)
    ls = last.cpu().numpy().reshape(d.batch * d.dim, d.dstate).astype(np.float64)
    del out, last
    total = d.batch * d.dim
    chunk = max(1, (1 << 26) // max(1, d.seqlen))      # about 64 M outputs per oracle run
    agg = {"n": 0, "strict_pass": 0, "pass": 0, "max_err": 0.0}
    for c0 in range(0, total, chunk):
        ch = list(range(c0, min(total, c0 + chunk)))
        ro, rl, rm = oracle_rows(d, inp, ch)
        rep = check_out(o[c0:c0 + len(ch)], ro, rm, d.dtype, what=f"{name} channels {c0}..")
        check_state(ls[c0:c0 + len(ch)], rl, what=f"{name} last_state channels {c0}..")
        for k in ("n", "strict_pass", "pass"):
            agg[k] += rep[k]
        agg["max_err"] = max(agg["max_err"], rep["max_err"])
    assert agg["n"] == total * d.seqlen
    print(name, agg)


# --------------------------------------------------------------- small shapes, many tiles, ragged

SMALL = [
    # (batch, dim, L, N, nheads, ngroups, dtype)
    (2, 80, 300, 16, 0, 1, "bf16"),     # partial channel tile, ragged L, unaligned rows (scalar loads)
    (2, 80, 304, 16, 0, 1, "bf16"),     # 16-byte rows, ragged last block
    (3, 40, 257, 16, 0, 1, "f32"),
    (2, 64, 260, 16, 0, 1, "f32"),
    (2, 96, 200, 16, 0, 2, "bf16"),     # two B/C groups
    (2, 64, 200, 128, 4, 1, "bf16"),    # scalar A per head, N = 128
    (1, 48, 96, 128, 3, 1, "f32"),
    (2, 64, 136, 128, 0, 1, "bf16"),    # per-channel A with N = 128
    (2, 24, 120, 8, 0, 1, "bf16"),
    (2, 40, 88, 32, 0, 1, "bf16"),
    (1, 40, 72, 64, 0, 1, "f32"),
    (2, 64, 160, 64, 8, 2, "bf16"),
]


@pytest.mark.parametrize("shape", SMALL, ids=lambda s: "x".join(map(str, s)))
def test_small_full(shape):
    b, dm, L, N, H, G, dt = shape
    dims = si.Dims(b, dm, L, N, nheads=H, ngroups=G, dtype=dt)
    head = dims.head_mode
    recipe = si.Recipe(a_init="neg_uniform_1_16" if (head or N != 16) else "neg_n_plus_1",
                       d_init="normal", delta_init="normal_half")
    if not head and N != 16:
        # per-channel A drawn per (d, n)
        recipe = si.Recipe(a_init="neg_uniform_1_16", d_init="normal", delta_init="normal_half")
    _full_check(dims, recipe, seed=3)


# the tensor-memory kernel (bf16, N = 16, A per channel) forced on small shapes: ragged and
# unaligned L (element copies into the boxes), short sequences, partial channel tiles, two
# B/C groups, an initial state, and each of its lane layouts
TC_SHAPES = [
    # (batch, dim, L, ngroups, h0, options)
    (2, 80, 300, 1, False, dict(warps=16, states_per_lane=2, time_lanes=1)),
    (2, 80, 304, 1, False, dict(warps=16, states_per_lane=2, time_lanes=1)),
    (2, 96, 200, 2, False, dict(warps=8, states_per_lane=4, time_lanes=1)),
    (1, 40, 33, 1, True, dict(warps=12, states_per_lane=4, time_lanes=1)),
    (2, 64, 512, 1, True, dict(warps=16, states_per_lane=2, time_lanes=2)),
    (2, 48, 250, 1, False, dict(warps=8, states_per_lane=2, time_lanes=2)),
    (1, 64, 1000, 2, True, dict(warps=8, states_per_lane=2, time_lanes=2, seg_len=128)),
    (3, 32, 7, 1, False, dict(warps=16, states_per_lane=2, time_lanes=2)),
]


@pytest.mark.parametrize("shape", TC_SHAPES, ids=lambda s: "x".join(map(str, s[:5])) + "_" +
                         "_".join(f"{k}{v}" for k, v in s[5].items()))
def test_tensor_memory_kernel(shape):
    b, dm, L, G, with_h0, opts = shape
    dims = si.Dims(b, dm, L, 16, ngroups=G, dtype="bf16")
    inp = si.make_inputs(dims, si.Recipe(d_init="normal", delta_init="normal_half"), 17 + L)
    h0 = np.random.default_rng(L).standard_normal((b, dm, 16)).astype(np.float32) if with_h0 else None
    out, last = run_gpu(dims, inp, h0=h0, opts=dict(opts, tensor_memory=2))
    ro, rl, rm = oracle.run_inputs(dims, inp, h0=h0)
    check_out(to_host_f64(out), ro, rm, "bf16", what=f"tensor-memory kernel {opts}")
    check_state(to_host_f64(last), rl, what=f"tensor-memory kernel last_state {opts}")


@pytest.mark.parametrize("softplus,has_D,has_z,has_bias", [(False, True, True, True), (True, False, True, True),
                                                         (True, True, False, True), (True, True, True, False),
                                                         (False, False, False, False)])
def test_optional_inputs(softplus, has_D, has_z, has_bias):
    dims = si.Dims(2, 40, 100, 16, dtype="bf16")
    r = si.Recipe(d_init="normal", delta_init="normal_half", softplus=softplus, has_D=has_D, has_z=has_z,
                  has_bias=has_bias)
    inp = si.make_inputs(dims, r, 5)
    if not softplus:
        # without softplus the step is delta + bias itself: keep it positive and small
        delta = np.abs(si.to_f64(inp["delta"])) * 0.05
        inp["delta"] = np.array([si.f64_to_bf16_bits(x) for x in delta.ravel()],
                                dtype=np.uint16).reshape(delta.shape)
        if has_bias:
            inp["delta_bias"] = np.logaddexp(0.0, inp["delta_bias"].astype(np.float64)).astype(np.float32)
    _full_check(dims, r, inp=inp)


@pytest.mark.parametrize("L", [1, 2, 7, 31, 32, 33, 64])
def test_short_sequences(L):
    for dt in ("bf16", "f32"):
        dims = si.Dims(2, 40, L, 16, dtype=dt)
        _full_check(dims, si.Recipe(d_init="normal", delta_init="normal_half"), seed=L)


def test_empty():
    import torch
    for dims in (si.Dims(0, 32, 64, 16), si.Dims(2, 32, 0, 16)):
        inp = si.make_inputs(dims, si.Recipe(), 0)
        out, last = run_gpu(dims, inp)
        assert out.numel() == dims.batch * dims.dim * dims.seqlen
        assert torch.all(last == 0)  # no steps: the state stays zero


def test_initial_state_and_chunk_split():
    """h0 input against the oracle, and [0,L1) + [L1,L) with the carried state equals one run."""
    dims = si.Dims(2, 64, 384, 16, dtype="bf16")
    r = si.Recipe(d_init="normal", delta_init="normal_half")
    inp = si.make_inputs(dims, r, 9)
    rng = np.random.default_rng(0)
    h0 = rng.standard_normal((dims.batch, dims.dim, dims.dstate)).astype(np.float32)
    _full_check(dims, r, inp=inp, h0=h0)
    out, last = run_gpu(dims, inp)
    for L1 in (128, 96, 100):
        d1 = si.Dims(2, 64, L1, 16, dtype="bf16")
        d2 = si.Dims(2, 64, dims.seqlen - L1, 16, dtype="bf16")
        cut = lambda k, a, lo, hi: np.ascontiguousarray(a[..., lo:hi]) if k in ("u", "delta", "z", "B", "C") else a
        i1 = {k: cut(k, v, 0, L1) for k, v in inp.items()}
        i2 = {k: cut(k, v, L1, dims.seqlen) for k, v in inp.items()}
        o1, s1 = run_gpu(d1, i1)
        o2, s2 = run_gpu(d2, i2, h0=s1.cpu().numpy())
        o12 = np.concatenate([to_host_f64(o1), to_host_f64(o2)], axis=2)
        if L1 % 32 == 0:
            # block boundaries line up: the same fp32 operations in the same order
            assert np.array_equal(o12, to_host_f64(out)), f"split at {L1} not bit-exact"
            assert np.array_equal(s2.cpu().numpy(), last.cpu().numpy())
        else:
            ro, rl, rm = oracle.run_inputs(dims, inp)
            check_out(o12, ro, rm, "bf16")
            check_state(s2.cpu().numpy().astype(np.float64), rl)


def test_misaligned_pointers_take_scalar_path():
    """Inputs at an odd 2-byte offset (not 16-byte aligned) give the same results as aligned ones."""
    import torch
    import selective_state_space_30_b200 as ssm
    from parity import to_device
    dims = si.Dims(2, 40, 96, 16, dtype="bf16")
    inp = si.make_inputs(dims, si.Recipe(d_init="normal", delta_init="normal_half"), 4)
    ref, ref_last = run_gpu(dims, inp)
    d = ssm.make_dims(2, 40, 96, 16, 40, 1, ssm.SSM_BF16)

    def shifted(a):
        t = to_device(a)
        buf = torch.empty(t.numel() + 1, dtype=t.dtype, device="cuda")
        v = buf[1:].view(t.shape)
        v.copy_(t)
        return v
    dev = {k: shifted(inp[k]) for k in ("u", "delta", "B", "C", "z")}
    A, D, bias = to_device(inp["A"]), to_device(inp["D"]), to_device(inp["delta_bias"])
    outbuf = torch.empty(2 * 40 * 96 + 1, dtype=torch.bfloat16, device="cuda")
    out = outbuf[1:].view(2, 40, 96)
    last = torch.empty(2, 40, 16, device="cuda")
    plan = ssm.ssm_scan_plan(d, 0)
    try:
        ssm.ssm_selective_scan_fwd(plan, dev["u"], dev["delta"], A, dev["B"], dev["C"], D, dev["z"], bias, True,
                                   d, out, last, None)
        torch.cuda.synchronize()
    finally:
        ssm.ssm_scan_destroy(plan)
    assert torch.equal(out, ref) and torch.equal(last, ref_last)


HOST_CASES = [
    si.Dims(2, 64, 256, 16, dtype="bf16"),                  # two chunks of one batch row
    si.Dims(6, 64, 200, 16, dtype="bf16"),                  # six chunks, ragged length
    si.Dims(1, 64, 256, 16, dtype="f32"),                   # one batch row, too short to split: no pipeline
    si.Dims(4, 128, 256, 128, nheads=2, dtype="bf16"),      # four chunks through the tensor-core path
    si.Dims(1, 96, 4096, 16, dtype="bf16"),                 # one batch row in four time chunks, chained states
    si.Dims(1, 64, 6144, 16, ngroups=2, dtype="f32"),       # six time chunks, two groups
    si.Dims(1, 128, 4096, 128, nheads=2, dtype="bf16"),     # time chunks through the tensor-core path
]


@pytest.mark.parametrize("dims", HOST_CASES, ids=lambda d: f"{d.batch}x{d.dim}x{d.seqlen}n{d.dstate}{d.dtype}")
def test_host_entry_point_matches_oracle(dims):
    """ssm_selective_scan_fwd_host (copies in, scan, copies out; pipelined over batch rows, or
    over stretches of the sequence for one batch row) against the oracle, and twice in a row
    on the same plan."""
    import torch
    import selective_state_space_30_b200 as ssm
    rec = si.Recipe(a_init="neg_uniform_1_16") if dims.head_mode else si.Recipe(d_init="normal",
                                                                                 delta_init="normal_half")
    inp = si.make_inputs(dims, rec, 6)
    io = ssm.SSM_BF16 if dims.dtype == "bf16" else ssm.SSM_F32
    d = ssm.make_dims(dims.batch, dims.dim, dims.seqlen, dims.dstate, dims.H, dims.ngroups, io)
    host = {k: np.ascontiguousarray(inp[k]) for k in ("u", "delta", "A", "B", "C", "D", "z", "delta_bias")}
    odt = np.uint16 if dims.dtype == "bf16" else np.float32
    ro, rl, rm = oracle.run_inputs(dims, inp)
    plan = ssm.ssm_scan_plan(d, 0)
    try:
        for _ in range(2):
            out = np.empty((dims.batch, dims.dim, dims.seqlen), dtype=odt)
            last = np.empty((dims.batch, dims.dim, dims.dstate), dtype=np.float32)
            ssm.ssm_selective_scan_fwd_host(plan, host["u"], host["delta"], host["A"], host["B"], host["C"],
                                            host["D"], host["z"], host["delta_bias"], True, d, out, last, None)
            torch.cuda.synchronize()
            assert ssm.ssm_scan_device_status(plan) == ssm.SSM_OK
            got = si.to_f64(out) if dims.dtype == "bf16" else out.astype(np.float64)
            check_out(got, ro, rm, dims.dtype)
            check_state(last.astype(np.float64), rl)
    finally:
        ssm.ssm_scan_destroy(plan)


def test_deterministic():
    w = si.WORKLOADS["mamba-130m"]
    d = si.Dims(2, 256, 512, 16, dtype="bf16")
    inp = si.make_inputs(d, w.recipe, 1)
    o1, s1 = run_gpu(d, inp)
    o2, s2 = run_gpu(d, inp)
    import torch
    assert torch.equal(o1, o2) and torch.equal(s1, s2)


def test_argument_errors_on_gpu():
    import selective_state_space_30_b200 as ssm
    import torch
    d = ssm.make_dims(1, 32, 64, 16, 32, 1, ssm.SSM_BF16)
    plan = ssm.ssm_scan_plan(d, 0)
    try:
        x = torch.zeros(1, 32, 64, dtype=torch.bfloat16, device="cuda")
        A = torch.zeros(32, 16, device="cuda")
        BC = torch.zeros(1, 1, 16, 64, dtype=torch.bfloat16, device="cuda")
        other = ssm.make_dims(1, 32, 65, 16, 32, 1, ssm.SSM_BF16)
        rc = ssm.ssm_selective_scan_fwd(plan, x, x, A, BC, BC, None, None, None, True, other, x, None, None,
                                        check=False)
        assert rc == ssm.SSM_ERR_INVALID_ARG
        rc = ssm.ssm_selective_scan_fwd(plan, None, x, A, BC, BC, None, None, None, True, d, x, None, None,
                                        check=False)
        assert rc == ssm.SSM_ERR_INVALID_ARG
        rc = ssm.ssm_selective_scan_fwd(plan, x, x, A, BC, BC, None, None, None, True, d, x, None, None,
                                        check=False)
        assert rc == ssm.SSM_OK
        assert ssm.ssm_scan_device_status(plan) == ssm.SSM_OK
    finally:
        ssm.ssm_scan_destroy(plan)
    with pytest.raises(ssm.SsmError):
        ssm.ssm_scan_plan(ssm.make_dims(1, 32, 64, 24, 32, 1, ssm.SSM_BF16), 0)  # N = 24: no kernel


def test_torch_front_end():
    import torch
    import selective_state_space_30_b200 as ssm
    from parity import to_device
    dims = si.Dims(2, 64, 128, 16, dtype="bf16")
    inp = si.make_inputs(dims, si.Recipe(d_init="normal", delta_init="normal_half"), 2)
    ref, ref_last = run_gpu(dims, inp)
    t = {k: to_device(inp[k]) for k in ("u", "delta", "A", "B", "C", "D", "z", "delta_bias")}
    out, last = ssm.selective_scan_fwd(t["u"], t["delta"], t["A"], t["B"], t["C"], t["D"], t["z"],
                                       t["delta_bias"], softplus=True)
    torch.cuda.synchronize()
    assert torch.equal(out, ref) and torch.equal(last, ref_last)
