"""The causal depthwise convolution (ssm_causal_conv1d_fwd) against the fp64 oracle (needs a B200).

Inputs: the seeded generator's u rows as x; taps and bias from seeded normals
scaled like a width-4 convolution's init (1/sqrt(width)).  Tolerances: the
fp32 rule 1e-4*(1+|ref|) for fp32 output; for bf16 output the stated bf16
bound ulp(ref) + 2e-3*|ref| plus 1e-4 * (|bias| + sum |w x|), the size of the
terms the fp32 sum adds up (see tests/parity.py).
"""
import numpy as np
import pytest
import torch

import oracle
import ssm_inputs as si
from parity import check_out, to_device, to_host_f64

pytestmark = pytest.mark.gpu

CASES = [
    # (batch, dim, seqlen, width, dtype, silu, bias)
    (2, 64, 128, 4, "bf16", True, True),      # 16-byte chunks
    (2, 40, 67, 4, "bf16", True, True),       # ragged length: one step per thread
    (1, 16, 64, 3, "f32", True, True),
    (3, 24, 96, 1, "f32", False, True),
    (2, 32, 256, 2, "bf16", False, False),
    (1, 8, 5, 4, "bf16", True, True),         # shorter than the taps
    (8, 1536, 2048, 4, "bf16", True, True),   # the mamba-130m layer's x
]


def _inputs(batch, dim, L, width, dtype, seed):
    d = si.Dims(batch, dim, L, 16, dtype=dtype)
    x = si.make_inputs(d, si.Recipe(), seed)["u"]
    rng = np.random.default_rng(seed)
    w = (rng.standard_normal((dim, width)) / np.sqrt(width)).astype(np.float32)
    b = (rng.standard_normal(dim) * 0.1).astype(np.float32)
    return x, w, b


def _run(batch, dim, L, width, dtype, x, w, b, silu):
    import selective_state_space_30_b200 as ssm
    xd = to_device(x)
    out = torch.empty_like(xd)
    io = ssm.SSM_BF16 if dtype == "bf16" else ssm.SSM_F32
    ssm.ssm_causal_conv1d_fwd(batch, dim, L, width, io, xd, to_device(w), to_device(b) if b is not None else None,
                              silu, out)
    torch.cuda.synchronize()
    return to_host_f64(out)


@pytest.mark.parametrize("case", CASES, ids=lambda c: "x".join(map(str, c)))
def test_conv1d_matches_oracle(case):
    batch, dim, L, width, dtype, silu, has_bias = case
    x, w, b = _inputs(batch, dim, L, width, dtype, 41)
    b = b if has_bias else None
    got = _run(batch, dim, L, width, dtype, x, w, b, silu)
    ref = oracle.causal_conv1d(x, w, b, silu=silu)
    # size of the summed terms, for the bf16 gate
    xf = oracle._f64(x)
    terms = np.zeros_like(ref) + (np.abs(b)[None, :, None] if b is not None else 0.0)
    for k in range(width):
        shift = width - 1 - k
        xs = np.zeros_like(xf)
        xs[:, :, shift:] = xf[:, :, :L - shift] if shift < L else 0.0
        terms += np.abs(w[:, k])[None, :, None] * np.abs(xs)
    if silu:
        terms = terms * np.abs(ref / np.where(ref == 0, 1, oracle.causal_conv1d(x, w, b, silu=False)))
    check_out(got, ref, terms, dtype)


def test_conv1d_feeds_the_scan():
    """conv1d then the scan equals the oracle's conv1d then the oracle's scan (bf16 between them)."""
    import selective_state_space_30_b200 as ssm
    from parity import check_state, run_gpu
    dims = si.Dims(2, 64, 192, 16, dtype="bf16")
    inp = si.make_inputs(dims, si.Recipe(d_init="normal", delta_init="normal_half"), 42)
    x, w, b = _inputs(2, 64, 192, 4, "bf16", 43)
    xd = to_device(x)
    ud = torch.empty_like(xd)
    ssm.ssm_causal_conv1d_fwd(2, 64, 192, 4, ssm.SSM_BF16, xd, to_device(w), to_device(b), True, ud)
    torch.cuda.synchronize()
    u_bits = ud.view(torch.int16).cpu().numpy().view(np.uint16)
    # the oracle's own conv1d, rounded to bf16 the way the kernel stores it, must give the same u
    ref_u = oracle.causal_conv1d(x, w, b, silu=True)
    from parity import bf16_round_f64
    assert np.max(np.abs(oracle._f64(u_bits) - bf16_round_f64(ref_u))) <= np.max(np.abs(ref_u)) * 2 ** -7
    scan_in = dict(inp, u=u_bits)
    out, last = run_gpu(dims, scan_in)
    ro, rl, rm = oracle.run_inputs(dims, scan_in)
    check_out(to_host_f64(out), ro, rm, "bf16")
    check_state(to_host_f64(last), rl)


def test_conv1d_argument_checks():
    import selective_state_space_30_b200 as ssm
    x = torch.zeros(64, device="cuda")
    f = ssm.ssm_causal_conv1d_fwd
    assert f(1, 4, 16, 5, ssm.SSM_F32, x, x, None, True, x, check=False) == ssm.SSM_ERR_UNSUPPORTED
    assert f(1, 4, 16, 0, ssm.SSM_F32, x, x, None, True, x, check=False) == ssm.SSM_ERR_UNSUPPORTED
    assert f(1, 4, 16, 4, 7, x, x, None, True, x, check=False) == ssm.SSM_ERR_INVALID_ARG
    assert f(1, 4, 16, 4, ssm.SSM_F32, None, x, None, True, x, check=False) == ssm.SSM_ERR_INVALID_ARG
    assert f(0, 4, 16, 4, ssm.SSM_F32, None, None, None, True, None, check=False) == ssm.SSM_OK
