"""The seeded input generator (no GPU)."""
import fractions
import math

import numpy as np
import pytest

import ssm_inputs as si


def test_splitmix64_published_vectors():
    # SplitMix64 (Steele, Lea, Flood 2014): state += GAMMA; out = mix(state)
    G = 0x9E3779B97F4A7C15
    M = (1 << 64) - 1
    assert si.mix64(G) == 0xE220A8397B1DCDAF  # first output from state 0
    want = [6457827717110365317, 3203168211198807973, 9817491932198370423,
            4593380528125082431, 16408922859458223821]  # first outputs from state 1234567
    assert [si.mix64((1234567 + i * G) & M) for i in range(1, 6)] == want


def _bf16_value(bits):
    return float(si.bf16_bits_to_f64(np.array([bits], dtype=np.uint16))[0])


def _nearest_even_bf16(x: float) -> int:
    """Brute force: the bf16 pattern nearest to x in exact rational arithmetic, ties to even."""
    f32 = np.array([x], dtype=np.float32).view(np.uint32)[0]
    cand = set()
    base = int(f32) >> 16
    for k in range(base - 2, base + 3):
        if 0 <= k < 0x10000:
            cand.add(k)
    for k in list(cand):
        cand.add(k ^ 0x8000 if k == 0 else k)
    X = fractions.Fraction(x)
    best = None
    for k in cand:
        v = _bf16_value(k)
        if not math.isfinite(v):
            continue
        d = abs(fractions.Fraction(v) - X)
        key = (d, k & 1)
        if best is None or key < best[0]:
            best = (key, k)
    return best[1]


def test_bf16_rounding_is_nearest_even_from_f64():
    rng = np.random.default_rng(0)
    xs = list(rng.standard_normal(3000) * np.exp(rng.uniform(-20, 20, 3000)))
    # exact ties and near-ties between two bf16 neighbours (where rounding through fp32 would go wrong)
    for k in range(200):
        lo = _bf16_value(0x3F80 + k)
        hi = _bf16_value(0x3F80 + k + 1)
        mid = (lo + hi) / 2.0
        xs += [mid, math.nextafter(mid, 0), math.nextafter(mid, 10), -mid]
        xs += [mid + (hi - lo) * 2.0 ** -30]  # above the tie by less than fp32 resolves
    for x in xs:
        got = si.f64_to_bf16_bits(x)
        want = _nearest_even_bf16(x)
        # signed zero aside, the pattern must match
        assert got == want or (_bf16_value(got) == 0 and _bf16_value(want) == 0), (x, hex(got), hex(want))


def test_bf16_special_values():
    assert si.f64_to_bf16_bits(0.0) == 0x0000
    assert si.f64_to_bf16_bits(-0.0) == 0x8000
    assert si.f64_to_bf16_bits(1.0) == 0x3F80
    assert si.f64_to_bf16_bits(float("inf")) == 0x7F80
    assert si.f64_to_bf16_bits(3.5e38) == 0x7F80          # rounds past the largest finite bf16
    assert si.f64_to_bf16_bits(2.0 ** -133) == 0x0001     # smallest bf16 subnormal
    assert si.f64_to_bf16_bits(2.0 ** -134) == 0x0000     # a tie to even, down to zero
    assert si.f64_to_bf16_bits(3 * 2.0 ** -135) == 0x0001


def test_slices_regenerate_identically():
    full = si.fill(7, 3, 0, 300000, 0, 1.0, 0.0, 0.0, "bf16")
    for off, cnt in [(0, 5), (1, 7), (12345, 1000), (299990, 10), (131071, 3)]:
        part = si.fill(7, 3, off, cnt, 0, 1.0, 0.0, 0.0, "bf16")
        assert np.array_equal(part, full[off:off + cnt])
    f32 = si.fill(7, 3, 0, 1000, 0, 1.0, 0.0, 0.0, "f32")
    f64 = si.fill(7, 3, 0, 1000, 0, 1.0, 0.0, 0.0, "f64")
    assert np.array_equal(f32, f64.astype(np.float32))


def test_distributions():
    n = 400000
    x = si.fill(1, 3, 0, n, 0, 1.0, 0.0, 0.0, "f64")
    assert abs(x.mean()) < 0.01 and abs(x.std() - 1.0) < 0.01
    assert abs(np.mean(x ** 4) - 3.0) < 0.06                 # normal kurtosis
    assert abs(np.mean(np.abs(x) < 1.0) - 0.6827) < 0.005
    y = si.fill(1, 4, 0, n, 0, 0.5, 0.0, 0.0, "f64")
    assert abs(y.std() - 0.5) < 0.005
    u = si.fill(1, 0, 0, n, 1, -1.0, -16.0, 0.0, "f64")
    assert u.min() > -16.0 and u.max() < -1.0 and abs(u.mean() + 8.5) < 0.05
    dt = si.fill(1, 2, 0, n, 2, 1e-3, 0.1, 1e-4, "f64")
    assert dt.min() >= 1e-3 and dt.max() <= 0.1
    lg = np.log(dt)
    assert abs(lg.mean() - 0.5 * (math.log(1e-3) + math.log(0.1))) < 0.02
    bias = si.fill(1, 2, 0, n, 4, 1e-3, 0.1, 1e-4, "f64")
    np.testing.assert_allclose(np.logaddexp(0.0, bias), dt, rtol=1e-12)   # softplus(bias) == dt


def test_streams_are_independent():
    a = si.fill(0, 3, 0, 100000, 0, 1.0, 0.0, 0.0, "f64")
    b = si.fill(0, 5, 0, 100000, 0, 1.0, 0.0, 0.0, "f64")
    c = si.fill(1, 3, 0, 100000, 0, 1.0, 0.0, 0.0, "f64")
    assert abs(np.corrcoef(a, b)[0, 1]) < 0.02
    assert abs(np.corrcoef(a, c)[0, 1]) < 0.02


@pytest.mark.parametrize("name", list(si.WORKLOADS))
def test_workload_params_and_row_mode(name):
    w = si.WORKLOADS[name]
    d = w.dims
    prm = si.make_params(d, w.recipe, w.seed)
    if d.head_mode:
        assert prm["A"].shape == (d.H,) and np.all(prm["A"] < -1) and np.all(prm["A"] > -16)
    else:
        assert prm["A"].shape == (d.dim, d.dstate)
        assert np.array_equal(prm["A"][0], -(np.arange(d.dstate) + 1.0))
    assert prm["delta_bias"].shape == (d.H,)
    dt = np.logaddexp(0.0, prm["delta_bias"].astype(np.float64))
    assert dt.min() > 0.9e-3 and dt.max() < 0.11
    assert prm["D"].shape == (d.dim,)
    # row mode equals the matching rows of the full tensors (small shapes only)
    if d.batch * d.dim * d.seqlen <= 1 << 22:
        full = si.make_inputs(d, w.recipe, w.seed)
        ch = [0, d.batch * d.dim - 1, d.dim // 2]
        rows = si.make_inputs(d, w.recipe, w.seed, channels=ch)
        for k, c in enumerate(ch):
            b, dd = divmod(c, d.dim)
            assert np.array_equal(rows["u"][k], full["u"][b, dd])
            assert np.array_equal(rows["z"][k], full["z"][b, dd])
            assert np.array_equal(rows["delta"][k], full["delta"][b, dd // (d.dim // d.H)])


def test_empty_shapes():
    for d in (si.Dims(0, 32, 64, 16), si.Dims(2, 32, 0, 16)):
        x = si.make_inputs(d, si.Recipe(), 0)
        assert x["u"].shape == (d.batch, d.dim, d.seqlen)
        assert x["B"].shape == (d.batch, 1, d.dstate, d.seqlen)
