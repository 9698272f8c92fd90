"""Seeded synthetic inputs for the selective-scan (S6) forward workloads.

This module only draws numbers and rounds them to the storage dtype; it holds
none of the scan's arithmetic.  The fp64 oracle and the CUDA path both take
their inputs from here, so they see bit-identical tensors.

Shapes and value recipes follow the Mamba layer shapes the selective scan is
run on (Mamba "architecture-details" page: "Model Configuration",
"Layer Count Scaling" and "Initialization Strategy" sections):

* dt is log-uniform in [dt_min, dt_max] = [1e-3, 0.1] with floor 1e-4, one per
  channel (or per head), and enters through delta_bias = softplus^-1(dt);
* A is -(n+1) per state (or -U(1,16) per head for the large-state shape);
* u, z, B, C are N(0, 1);
* delta is 0 (or N(0,1)*0.5 for the 130M shape) and D is 1 (or N(0,1)).

Tensor layouts (contiguous, row-major):
  u, z, out      (batch, dim, seqlen)
  delta          (batch, nheads, seqlen)        nheads == dim for S6
  B, C           (batch, ngroups, dstate, seqlen)
  A              (dim, dstate) for S6, (nheads,) for scalar-A-per-head
  D              (dim,)
  delta_bias     (nheads,)
  last_state     (batch, dim, dstate)

bf16 tensors are carried as uint16 numpy arrays holding the bf16 bit pattern.
"""
from __future__ import annotations

import ctypes
import dataclasses
import os
import subprocess
from typing import Dict, Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gen.c")
_LIB_PATH = os.path.join(_HERE, "_gen.so")
_lib = None

# distribution codes (gen.c)
_NORMAL, _UNIFORM, _LOGUNIFORM, _CONST, _SPINV_LOGUNIFORM = 0, 1, 2, 3, 4
_F64, _F32, _BF16 = 0, 1, 2

# fixed stream ids: one independent stream per tensor, in this order
STREAMS = {"A": 0, "D": 1, "dt": 2, "u": 3, "delta": 4, "z": 5, "B": 6, "C": 7,
           "dout": 8, "dlast": 9, "h0": 10}


def build(force: bool = False) -> str:
    """Compile gen.c into _gen.so next to it (plain gcc, no vector math)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math",
                               "-o", tmp, _SRC, "-lm", "-lpthread"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _get_lib():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        lib.ssm_gen_fill.restype = ctypes.c_int
        lib.ssm_gen_fill.argtypes = [ctypes.c_uint64, ctypes.c_uint64, ctypes.c_int64, ctypes.c_int64,
                                     ctypes.c_int, ctypes.c_double, ctypes.c_double, ctypes.c_double,
                                     ctypes.c_int, ctypes.c_void_p, ctypes.c_int]
        lib.ssm_f64_to_bf16.restype = ctypes.c_uint16
        lib.ssm_f64_to_bf16.argtypes = [ctypes.c_double]
        lib.ssm_gen_mix64.restype = ctypes.c_uint64
        lib.ssm_gen_mix64.argtypes = [ctypes.c_uint64]
        lib.ssm_gen_raw64.restype = ctypes.c_uint64
        lib.ssm_gen_raw64.argtypes = [ctypes.c_uint64, ctypes.c_uint64, ctypes.c_uint64]
        _lib = lib
    return _lib


def _nthreads() -> int:
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def fill(seed: int, stream: int, offset: int, count: int, dist: int, p0: float, p1: float = 0.0,
         p2: float = 0.0, dtype: str = "f64") -> np.ndarray:
    """Elements offset..offset+count of one stream, as f64 / f32 / bf16-bits(uint16)."""
    code = {"f64": _F64, "f32": _F32, "bf16": _BF16}[dtype]
    npdt = {"f64": np.float64, "f32": np.float32, "bf16": np.uint16}[dtype]
    out = np.empty(count, dtype=npdt)
    rc = _get_lib().ssm_gen_fill(seed, stream, offset, count, dist, p0, p1, p2, code,
                                 out.ctypes.data if count else None, _nthreads())
    if rc != 0:
        raise ValueError("ssm_gen_fill rejected its arguments")
    return out


def f64_to_bf16_bits(x: float) -> int:
    """Round one fp64 value to bf16 (nearest, ties to even); returns the 16-bit pattern."""
    return int(_get_lib().ssm_f64_to_bf16(float(x)))


def mix64(x: int) -> int:
    return int(_get_lib().ssm_gen_mix64(x))


def raw64(seed: int, stream: int, i: int) -> int:
    return int(_get_lib().ssm_gen_raw64(seed, stream, i))


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float64."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def to_f64(arr: np.ndarray) -> np.ndarray:
    """Exact float64 view of a generated tensor (bf16 bits or fp32)."""
    if arr.dtype == np.uint16:
        return bf16_bits_to_f64(arr)
    return arr.astype(np.float64)


@dataclasses.dataclass(frozen=True)
class Dims:
    """Problem shape: B, D, L, N plus head / group structure and the I/O dtype."""
    batch: int
    dim: int
    seqlen: int
    dstate: int
    nheads: int = 0      # 0 -> dim (per-channel delta / A / bias, the S6 layout)
    ngroups: int = 1
    dtype: str = "bf16"  # dtype of u, delta, z, B, C, out; A, D, bias, state are fp32

    @property
    def H(self) -> int:
        return self.nheads if self.nheads else self.dim

    @property
    def head_mode(self) -> bool:
        return self.H != self.dim

    def validate(self) -> None:
        if min(self.batch, self.dim, self.seqlen, self.dstate, self.H, self.ngroups) < 0:
            raise ValueError("negative size")
        if self.H and self.dim % self.H:
            raise ValueError("dim must be a multiple of nheads")
        if self.ngroups and self.dim % self.ngroups:
            raise ValueError("dim must be a multiple of ngroups")
        if self.dtype not in ("f32", "bf16"):
            raise ValueError("dtype must be f32 or bf16")


@dataclasses.dataclass(frozen=True)
class Recipe:
    """How each tensor is drawn (see module docstring)."""
    a_init: str = "neg_n_plus_1"      # or "neg_uniform_1_16" (per head)
    d_init: str = "one"               # or "normal"
    delta_init: str = "zero"          # or "normal_half"
    dt_min: float = 1e-3
    dt_max: float = 0.1
    dt_floor: float = 1e-4
    softplus: bool = True
    has_D: bool = True
    has_z: bool = True
    has_bias: bool = True


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    dims: Dims
    recipe: Recipe
    seed: int = 0
    note: str = ""


# The five workload shapes of the selective-scan forward (names say what they are).
WORKLOADS: Dict[str, Workload] = {
    "tiny-f32": Workload(
        "tiny-f32", Dims(1, 16, 64, 16, dtype="f32"), Recipe(),
        note="tiny S6 scan, fp32: B=1, d_inner=16, L=64, N=16"),
    "mamba-130m": Workload(
        "mamba-130m", Dims(8, 1536, 2048, 16, dtype="bf16"),
        Recipe(d_init="normal", delta_init="normal_half"),
        note="Mamba-130M layer: B=8, d_inner=1536, L=2048, N=16, bf16 I/O"),
    "mamba-1.4b": Workload(
        "mamba-1.4b", Dims(4, 4096, 4096, 16, dtype="bf16"), Recipe(),
        note="Mamba-1.4B layer: B=4, d_inner=4096, L=4096, N=16, bf16 I/O"),
    "mamba-2.8b-long": Workload(
        "mamba-2.8b-long", Dims(1, 5120, 65536, 16, dtype="bf16"), Recipe(),
        note="Mamba-2.8B long context: B=1, d_inner=5120, L=65536, N=16, bf16 I/O"),
    "mamba2-n128": Workload(
        "mamba2-n128", Dims(4, 2048, 8192, 128, nheads=32, ngroups=1, dtype="bf16"),
        Recipe(a_init="neg_uniform_1_16"),
        note="Mamba-2 style: B=4, 32 heads x 64, L=8192, N=128, scalar A per head, bf16 I/O"),
}


def _gen_normal(seed, name, offset, count, dtype, scale=1.0):
    return fill(seed, STREAMS[name], offset, count, _NORMAL, scale, 0.0, 0.0, dtype)


def make_params(dims: Dims, recipe: Recipe, seed: int = 0) -> Dict[str, Optional[np.ndarray]]:
    """The small fp32 parameter tensors: A, D, delta_bias."""
    dims.validate()
    H, N = dims.H, dims.dstate
    if recipe.a_init == "neg_n_plus_1":
        if dims.head_mode:
            raise ValueError("A=-(n+1) is a per-channel init; head mode uses a scalar A per head")
        A = np.tile(-(np.arange(N, dtype=np.float32) + 1.0), (dims.dim, 1)).astype(np.float32)
    elif recipe.a_init == "neg_uniform_1_16":
        A = fill(seed, STREAMS["A"], 0, H if dims.head_mode else dims.dim * N, _UNIFORM, -1.0, -16.0, 0.0, "f32")
        if not dims.head_mode:
            A = A.reshape(dims.dim, N)
    else:
        raise ValueError(recipe.a_init)
    if not recipe.has_D:
        D = None
    elif recipe.d_init == "one":
        D = np.ones(dims.dim, dtype=np.float32)
    elif recipe.d_init == "normal":
        D = _gen_normal(seed, "D", 0, dims.dim, "f32")
    else:
        raise ValueError(recipe.d_init)
    bias = None
    if recipe.has_bias:
        bias = fill(seed, STREAMS["dt"], 0, H, _SPINV_LOGUNIFORM, recipe.dt_min, recipe.dt_max,
                    recipe.dt_floor, "f32")
    return {"A": A, "D": D, "delta_bias": bias}


def make_inputs(dims: Dims, recipe: Recipe, seed: int = 0,
                channels: Optional[Sequence[int]] = None) -> Dict[str, Optional[np.ndarray]]:
    """All tensors of one problem.

    channels=None gives full tensors.  Otherwise `channels` is a list of flat
    channel ids c = b*dim + d and u, z come back as (len(channels), L) rows,
    delta as the matching (len(channels), L) rows of its (batch, nheads, L)
    tensor (the row of channel d's head), and B, C in full (they are small).
    """
    dims.validate()
    Bt, Dm, L, N, H, G = dims.batch, dims.dim, dims.seqlen, dims.dstate, dims.H, dims.ngroups
    dt = dims.dtype
    out = make_params(dims, recipe, seed)

    def normal_rows(name, row_len, rows_total, rows, scale=1.0):
        if rows is None:
            return _gen_normal(seed, name, 0, rows_total * row_len, dt, scale).reshape(rows_total, row_len)
        return np.stack([_gen_normal(seed, name, r * row_len, row_len, dt, scale) for r in rows]) \
            if len(rows) else np.empty((0, row_len), dtype=np.uint16 if dt == "bf16" else np.float32)

    rows_u = None if channels is None else list(channels)
    u = normal_rows("u", L, Bt * Dm, rows_u)
    z = normal_rows("z", L, Bt * Dm, rows_u) if recipe.has_z else None
    if channels is None:
        rows_dl = None
    else:
        P = Dm // H
        rows_dl = [(c // Dm) * H + (c % Dm) // P for c in channels]
    if recipe.delta_init == "zero":
        nrow = Bt * H if rows_dl is None else len(rows_dl)
        delta = np.zeros((nrow, L), dtype=np.uint16 if dt == "bf16" else np.float32)
    elif recipe.delta_init == "normal_half":
        delta = normal_rows("delta", L, Bt * H, rows_dl, scale=0.5)
    else:
        raise ValueError(recipe.delta_init)
    Bm = _gen_normal(seed, "B", 0, Bt * G * N * L, dt).reshape(Bt, G, N, L)
    Cm = _gen_normal(seed, "C", 0, Bt * G * N * L, dt).reshape(Bt, G, N, L)
    if channels is None:
        u = u.reshape(Bt, Dm, L)
        z = z.reshape(Bt, Dm, L) if z is not None else None
        delta = delta.reshape(Bt, H, L)
    out.update({"u": u, "delta": delta, "z": z, "B": Bm, "C": Cm, "softplus": recipe.softplus})
    return out


def make_grad_inputs(dims: Dims, seed: int = 0, dlast: bool = False, h0: bool = False
                     ) -> Dict[str, Optional[np.ndarray]]:
    """The incoming gradients of a backward pass: dout (batch, dim, L) in the I/O
    dtype, N(0, 1); optionally dlast, the gradient of last_state, and an initial
    state h0, both (batch, dim, N) fp32 N(0, 1)."""
    dims.validate()
    Bt, Dm, L, N = dims.batch, dims.dim, dims.seqlen, dims.dstate
    out = {"dout": _gen_normal(seed, "dout", 0, Bt * Dm * L, dims.dtype).reshape(Bt, Dm, L),
           "dlast": None, "h0": None}
    if dlast:
        out["dlast"] = _gen_normal(seed, "dlast", 0, Bt * Dm * N, "f32").reshape(Bt, Dm, N)
    if h0:
        out["h0"] = _gen_normal(seed, "h0", 0, Bt * Dm * N, "f32").reshape(Bt, Dm, N)
    return out


def workload(name: str) -> Workload:
    return WORKLOADS[name]
