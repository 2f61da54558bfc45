"""The factored rotary tables' claim, on the CPU: cos / sin of row p = 16 r + l formed from the
cos / sin of a coarse angle (row 16 r; paired: position 32 r) and a fine one (row l, either half)
by the angle-addition formula in float64 and rounded once to float32 equal the float32 roundings
of the directly computed values except in the last bit next to float32 rounding midpoints. This
pins the reading that pha_rope_factor_tables and pha_rope_factored rely on (the GPU tests compare
the device's factor tables and rotations with the same definitions)."""
import numpy as np
import pytest


@pytest.mark.parametrize("paired", [False, True])
@pytest.mark.parametrize("hd", [16, 128])
def test_angle_addition_matches_direct_tables(paired, hd):
    rows, base, L = 70000, 10000.0, 16
    half = hd // 2
    inv = base ** (-2.0 * np.arange(half) / hd)
    p = np.arange(rows)
    hi, lo = p // L, p % L
    halves = (0, 1) if paired else (0,)
    for hf in halves:
        pos = (2 * p + hf) if paired else p
        ang = pos[:, None] * inv[None, :]
        c_dir, s_dir = np.cos(ang).astype(np.float32), np.sin(ang).astype(np.float32)
        a = ((2 * L * hi) if paired else (L * hi))[:, None] * inv[None, :]   # coarse angle
        b = ((2 * lo + hf) if paired else lo)[:, None] * inv[None, :]        # fine angle
        ca, sa, cb, sb = np.cos(a), np.sin(a), np.cos(b), np.sin(b)
        c = (ca * cb - sa * sb).astype(np.float32)
        s = (sa * cb + ca * sb).astype(np.float32)
        # Both are float64 angle computations rounded once: the direct one rounds pos * f once,
        # the factored one rounds a and b and adds them, so the two angles differ by up to 1.5
        # float64 ulp of the largest angle (1.4e5 rad here: 2^-35 = 2.9e-11 per ulp), which is an
        # absolute difference of the cosine or sine; away from zero that is far below a float32
        # ulp, so the roundings agree or differ in the last bit next to a midpoint.
        tol = 1.5 * 2.0 ** -35 + 1e-15
        for got, ref in ((c, c_dir), (s, s_dir)):
            d = np.abs(got.astype(np.float64) - ref.astype(np.float64))
            assert np.all(d <= np.spacing(np.abs(ref)).astype(np.float64) + tol)
            assert np.mean(d == 0) > 0.9999, float(np.mean(d == 0))


def test_compensated_rotation_with_midpoint_test_is_exact():
    # the factored path's bf16 rotation: t = fl(s x1), e = s x1 - t (exact), y = fl(fl(c x0 - t) - e)
    # is within one float32 ulp of the exact value, so rounded once to bf16 it is within one bf16
    # ulp of the correctly rounded rotation, and wherever y is more than eight float32 ulps from a
    # bf16 rounding midpoint (the kernel's test; the rest goes to float64) it is that value exactly;
    # plain float32 (no e) is not within one bf16 ulp under cancellation
    rng = np.random.default_rng(0)
    n = 400000

    def bf16(x):  # float32 -> bf16 (nearest, ties to even), as float64
        b = np.asarray(x, np.float32).view(np.uint32).astype(np.uint64)
        r = ((b + 0x7FFF + ((b >> 16) & 1)) >> 16) << 16
        return r.astype(np.uint32).view(np.float32).astype(np.float64)

    def bf16_exact(v):  # float64 -> bf16 with one rounding
        m, e = np.frexp(v)
        return np.ldexp(np.round(m * 256.0) / 256.0, e)

    def fl32(x):
        return np.asarray(x, np.float64).astype(np.float32).astype(np.float64)

    ang = rng.uniform(0.1, 1.4, n)
    c, s = fl32(np.cos(ang)), fl32(np.sin(ang))
    x0 = bf16(rng.standard_normal(n))
    # half the pairs random, half chosen so that c x0 - s x1 nearly cancels (x1 ~ c x0 / s)
    x1 = np.where(np.arange(n) % 2 == 0, bf16(rng.standard_normal(n)), bf16(c * x0 / s))
    exact = bf16_exact(c * x0 - s * x1)          # float64 holds the bf16 x float32 products exactly
    t = fl32(s * x1)
    e = s * x1 - t
    faithful = bf16(fl32(fl32(c * x0 - t) - e))
    plain = bf16(fl32(c * x0 - t))
    ulp = np.ldexp(1.0, np.frexp(np.maximum(np.abs(exact), 1e-30))[1] - 8)
    assert np.max(np.abs(faithful - exact) / ulp) <= 1.0
    assert np.mean(faithful == exact) > 0.9999
    yb = fl32(fl32(c * x0 - t) - e).astype(np.float32).view(np.uint32).astype(np.int64)
    far = ((yb + 8) & 0xFFF0) != 0x8000
    assert np.mean(far) > 0.999
    assert np.all(faithful[far] == exact[far])          # the test never passes a wrong rounding
    assert np.max(np.abs(plain - exact) / ulp) > 1.0   # the compensation is what keeps one ulp
