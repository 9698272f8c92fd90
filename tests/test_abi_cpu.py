"""The C-ABI library on a machine without a GPU: it loads, exports every symbol
include/*.h declares, and rejects bad arguments on the host.  No compute calls."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    names = set()
    for f in os.listdir(os.path.join(ROOT, "include")):
        if not f.endswith(".h"):
            continue
        text = open(os.path.join(ROOT, "include", f)).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        for m in re.finditer(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\**\s*(ssm_[A-Za-z0-9_]+)\s*\(", text, re.M):
            names.add(m.group(1))
    return names


@pytest.fixture(scope="module")
def lib():
    from selective_state_space_30_b200 import build, _abi
    build.build()
    return _abi.load_library()


def test_every_declared_symbol_is_exported(lib):
    names = _declared_functions()
    assert {"ssm_scan_plan", "ssm_selective_scan_fwd", "ssm_scan_destroy"} <= names
    for n in sorted(names):
        assert hasattr(lib, n), f"{n} declared in include/ but not exported"
    from selective_state_space_30_b200 import _abi
    import selective_state_space_30_b200 as pkg
    assert names == set(_abi.EXPORTS), "binding and header disagree"
    for n in names:
        assert callable(getattr(pkg, n, None)), f"package does not expose {n}"


def test_status_strings(lib):
    import selective_state_space_30_b200 as ssm
    for code in range(6):
        s = ssm.ssm_status_string(code)
        assert s and s != "unknown status"
    assert ssm.ssm_status_string(99) == "unknown status"


def test_host_side_argument_checks(lib):
    import selective_state_space_30_b200 as ssm
    from selective_state_space_30_b200 import _abi
    good = ssm.make_dims(2, 32, 64, 16, 32, 1, ssm.SSM_BF16)
    # NULL out_plan
    assert lib.ssm_scan_plan(None, ctypes.byref(good), 0) == ssm.SSM_ERR_INVALID_ARG
    bad = [
        ssm.make_dims(2, 30, 64, 16, 4, 1, ssm.SSM_BF16),   # dim not a multiple of nheads
        ssm.make_dims(2, 32, 64, 16, 32, 3, ssm.SSM_BF16),  # dim not a multiple of ngroups
        ssm.make_dims(-1, 32, 64, 16, 32, 1, ssm.SSM_BF16),
        ssm.make_dims(2, 0, 64, 16, 32, 1, ssm.SSM_BF16),
        ssm.make_dims(2, 32, 64, 0, 32, 1, ssm.SSM_BF16),
        _abi.ssm_dims_t(2, 32, 64, 16, 32, 1, 7, 0),         # unknown dtype
        _abi.ssm_dims_t(2, 32, 64, 16, 32, 1, 1, 5),         # reserved != 0
    ]
    for d in bad:
        p = ctypes.c_void_p()
        assert lib.ssm_scan_plan(ctypes.byref(p), ctypes.byref(d), 0) == ssm.SSM_ERR_INVALID_ARG
        assert p.value is None
    p = ctypes.c_void_p()
    unsupported = ssm.make_dims(2, 32, 64, 24, 32, 1, ssm.SSM_BF16)   # N = 24: no kernel
    assert lib.ssm_scan_plan(ctypes.byref(p), ctypes.byref(unsupported), 0) == ssm.SSM_ERR_UNSUPPORTED
    # a NULL plan is rejected by every entry point that needs one
    assert lib.ssm_selective_scan_fwd(None, None, None, None, None, None, None, None, None, 1,
                                      ctypes.byref(good), None, None, None) == ssm.SSM_ERR_INVALID_ARG
    assert lib.ssm_scan_device_status(None, None) == ssm.SSM_ERR_INVALID_ARG
    assert lib.ssm_scan_plan_info(None, None, None, None, None, None) == ssm.SSM_ERR_INVALID_ARG
    assert lib.ssm_scan_destroy(None) == ssm.SSM_OK
    assert lib.ssm_probe_ex2(None, 1, 1, None) == ssm.SSM_ERR_INVALID_ARG


def test_state_update_host_checks(lib):
    """ssm_selective_state_update rejects bad arguments before touching the GPU."""
    import selective_state_space_30_b200 as ssm
    a, mis = 0x10000, 0x10004   # stand-in device addresses: 16-byte aligned, and not
    args = lambda st: (st, a, a, a, a, a, None, None, None, 1, a, None)  # noqa: E731
    f = lib.ssm_selective_state_update
    assert f(None, *args(a)) == ssm.SSM_ERR_INVALID_ARG
    assert f(ctypes.byref(ssm.make_dims(2, 64, 2, 16, 64, 1, ssm.SSM_BF16)), *args(a)) == ssm.SSM_ERR_INVALID_ARG
    assert f(ctypes.byref(ssm.make_dims(2, 64, 1, 24, 64, 1, ssm.SSM_BF16)), *args(a)) == ssm.SSM_ERR_UNSUPPORTED
    d = ssm.make_dims(2, 64, 1, 16, 64, 1, ssm.SSM_BF16)
    assert f(ctypes.byref(d), *args(None)) == ssm.SSM_ERR_INVALID_ARG
    assert f(ctypes.byref(d), *args(mis)) == ssm.SSM_ERR_UNSUPPORTED
    assert f(ctypes.byref(ssm.make_dims(0, 64, 1, 16, 64, 1, ssm.SSM_BF16)), *args(None)) == ssm.SSM_OK


def test_conv1d_host_checks(lib):
    """ssm_causal_conv1d_fwd rejects bad arguments before touching the GPU."""
    import selective_state_space_30_b200 as ssm
    a = 0x10000
    f = lib.ssm_causal_conv1d_fwd
    assert f(1, 4, 16, 5, ssm.SSM_F32, a, a, None, 1, a, None) == ssm.SSM_ERR_UNSUPPORTED
    assert f(1, 4, 16, 4, 9, a, a, None, 1, a, None) == ssm.SSM_ERR_INVALID_ARG
    assert f(1, 0, 16, 4, ssm.SSM_F32, a, a, None, 1, a, None) == ssm.SSM_ERR_INVALID_ARG
    assert f(1, 4, 16, 4, ssm.SSM_F32, None, a, None, 1, a, None) == ssm.SSM_ERR_INVALID_ARG
    assert f(0, 4, 16, 4, ssm.SSM_F32, None, None, None, 1, None, None) == ssm.SSM_OK


def test_bwd_host_checks(lib):
    """ssm_selective_scan_bwd and its workspace query reject bad shapes before touching the GPU."""
    import selective_state_space_30_b200 as ssm
    from selective_state_space_30_b200 import _abi
    n = ctypes.c_size_t()
    ws = lib.ssm_selective_scan_bwd_workspace_size
    assert ws(ctypes.byref(ssm.make_dims(2, 32, 64, 16, 0, 1, ssm.SSM_BF16)), None) == ssm.SSM_ERR_INVALID_ARG
    assert ws(None, ctypes.byref(n)) == ssm.SSM_ERR_INVALID_ARG
    generic = [
        ssm.make_dims(2, 64, 64, 16, 2, 1, ssm.SSM_BF16),     # per-head layout
        ssm.make_dims(2, 32, 64, 128, 0, 1, ssm.SSM_BF16),    # dstate 128
        ssm.make_dims(2, 48, 64, 16, 0, 1, ssm.SSM_BF16),     # 48 channels: not whole 32-channel tiles
        ssm.make_dims(2, 64, 64, 16, 0, 4, ssm.SSM_BF16),     # 16 channels per group
        ssm.make_dims(2, 32, 600, 8, 0, 1, ssm.SSM_F32),      # dstate 8, three 256-step segments
    ]
    for d in generic:   # the generic backward: header, ddelta sums, per-row partials, a state per segment
        assert ws(ctypes.byref(d), ctypes.byref(n)) == ssm.SSM_OK
        nseg = (d.seqlen + 255) // 256
        need = 256 + d.batch * d.nheads * d.seqlen * 4 + d.batch * d.dim * d.dstate * 4 + d.batch * d.dim * 4 + \
            d.batch * d.dim * nseg * d.dstate * 4
        assert need <= n.value <= need + 4 * 256
    for d in (ssm.make_dims(2, 32, 64, 24, 0, 1, ssm.SSM_BF16), ssm.make_dims(2, 32, 64, 256, 0, 1, ssm.SSM_BF16)):
        assert ws(ctypes.byref(d), ctypes.byref(n)) == ssm.SSM_ERR_UNSUPPORTED    # dstate 24, 256
    for d in (ssm.make_dims(2, 30, 64, 16, 0, 4, ssm.SSM_BF16), _abi.ssm_dims_t(2, 32, 64, 16, 32, 1, 7, 0)):
        assert ws(ctypes.byref(d), ctypes.byref(n)) == ssm.SSM_ERR_INVALID_ARG
    g = _abi.ssm_grads_t()
    f = lib.ssm_selective_scan_bwd
    d = ssm.make_dims(2, 32, 64, 24, 0, 1, ssm.SSM_BF16)
    assert f(ctypes.byref(d), *([None] * 8), 1, None, None, None, ctypes.byref(g), None, 0, None) == \
        ssm.SSM_ERR_UNSUPPORTED
    d = ssm.make_dims(2, 64, 64, 16, 2, 1, ssm.SSM_BF16)      # per-head: generic, but no dA output
    assert f(ctypes.byref(d), *([None] * 8), 1, None, None, None, ctypes.byref(g), None, 0, None) == \
        ssm.SSM_ERR_INVALID_ARG
    d = ssm.make_dims(2, 32, 64, 16, 0, 1, ssm.SSM_BF16)
    assert f(ctypes.byref(d), *([None] * 8), 1, None, None, None, None, None, 0, None) == ssm.SSM_ERR_INVALID_ARG
    assert f(ctypes.byref(d), *([None] * 8), 1, None, None, None, ctypes.byref(g), None, 0, None) == \
        ssm.SSM_ERR_INVALID_ARG                                # no dA output
    assert lib.ssm_selective_scan_bwd_device_status(None, None) == ssm.SSM_ERR_INVALID_ARG


def test_plan_without_a_gpu_reports_cuda_error(lib):
    import torch
    import selective_state_space_30_b200 as ssm
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    d = ssm.make_dims(2, 32, 64, 16, 32, 1, ssm.SSM_BF16)
    p = ctypes.c_void_p()
    assert lib.ssm_scan_plan(ctypes.byref(p), ctypes.byref(d), 0) == ssm.SSM_ERR_CUDA


def test_product_path_never_touches_the_oracle():
    """The package and its CUDA sources name neither the oracle nor the input generator."""
    pkg = os.path.join(ROOT, "selective_state_space_30_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, f)).read()
                assert not re.search(r"\b(import\s+oracle|from\s+oracle|ssm_oracle|oracle_selective)", text), f
                assert "ssm_inputs" not in text, f
    for f in os.listdir(os.path.join(ROOT, "oracle")):
        if f.endswith((".py", ".c")):
            text = open(os.path.join(ROOT, "oracle", f)).read()
            assert "selective_state_space_30_b200" not in text and "libssmscan" not in text, f


def test_missing_library_fails_loudly(tmp_path):
    from selective_state_space_30_b200 import _abi
    with pytest.raises(RuntimeError, match="no CPU fallback"):
        _abi.load_library(str(tmp_path / "libssmscan.so"))
