"""Host emulation of the quantizers' reciprocal-multiply rounding rules:
the codes they produce must equal those of one IEEE binary32 division
rounded half to even (the definition the oracle follows).  numpy float32
arithmetic is IEEE round-to-nearest, so r = x * inv is the kernels' product;
inv is taken as RN(1/s) and as either neighbour (the hardware reciprocal is
within one ulp).  A fused multiply-add a b + c rounded once is emulated in
80-bit long double: for the operands below the product is exact there, and
the one rounding to binary32 happens on a value that no 64-bit rounding
moved onto a binary32 rounding boundary."""
import numpy as np
import pytest

import oracle

F32 = np.float32


def invs(s):
    inv = F32(1.0) / s
    return [inv, np.nextafter(inv, F32(np.inf)), np.nextafter(inv, F32(-np.inf))]


LD = np.longdouble
MAGIC = F32(12582912.0)  # 1.5 * 2^23


def fma32(a, b, c):
    """binary32 a * b + c with one rounding (long double emulation)."""
    return (LD(a) * LD(b) + LD(c)).astype(F32)


def int4_rule(x, s, inv):
    """The 16-bit INT4 route: q0 = x inv, the exact residual r = x - q0 s,
    q = q0 + r inv rounded once (this is fl(x / s) itself), and the code
    from the pattern of q + 1.5 2^23."""
    q0 = (x * inv).astype(F32)
    r = fma32(-q0, s, x)
    q = fma32(r, inv, q0)
    return ((q + MAGIC).astype(F32) - MAGIC).astype(F32)


def sixteen_bit_values(kind):
    if kind == "bf16":
        return (np.arange(0, 0x7F80, dtype=np.uint32) << 16).view(np.float32)
    return np.arange(0, 0x7C00, dtype=np.uint16).view(np.float16).astype(F32)


@pytest.mark.parametrize("kind", ["bf16", "f16"])
def test_int4_rule_equals_division(kind):
    """Every 16-bit x against a sample of fp16 scales (all binades, subnormal
    scales included), |x/s| <= 24.5 (beyond it the code saturates)."""
    pos = sixteen_bit_values(kind)
    xs = np.sort(np.concatenate([pos, -pos[1:]]))
    s_all = np.arange(1, 0x7C00, dtype=np.uint16).view(np.float16).astype(F32)
    rng = np.random.default_rng(0)
    scales = np.concatenate([s_all[:64], rng.choice(s_all, 400, replace=False),
                             np.array([0.0625, 0.25, 1.0, 2.0 ** -24], F32)])
    ties = 0
    for s in scales.astype(F32):
        lo, hi = np.searchsorted(xs, -24.5 * s), np.searchsorted(xs, 24.5 * s, side="right")
        x = xs[lo:hi]
        ref = np.rint((x / s).astype(F32))
        for inv in invs(s):
            np.testing.assert_array_equal(int4_rule(x, s, inv), ref)
        ties += int(np.count_nonzero(np.abs(x / s - np.rint(x / s)) == 0.5))
    assert ties > 100  # exact half-way quotients were among the cases


def i8_rule(x, s, inv):
    """t = fl(x inv + 1.5 2^23) and its residual d; near-half-way elements
    (|d| >= 1/2 - 2^-14) are decided against h = k + sign(d) / 2 from the
    exact e = x - h s and half an ulp of h, as the kernels do."""
    t = fma32(x, inv, MAGIC)
    d = fma32(x, inv, (MAGIC - t).astype(F32))
    k = (t - MAGIC).astype(F32)
    near = np.abs(d) >= F32(0.5 - 2.0 ** -14)
    sg = np.where(d >= 0, F32(1), F32(-1))
    h = (k + F32(0.5) * sg).astype(F32)
    e = fma32(-h, s, x)
    hexp = (h.view(np.uint32) & np.uint32(0x7F800000)) - np.uint32(24 << 23)
    tol = (F32(s) * hexp.view(np.float32)).astype(F32)
    tie = np.abs(e) <= tol
    odd = (k.astype(np.int64) & 1) == 1
    beyond = (e > 0) == (sg > 0)
    fixed = np.where(tie, np.where(odd, k + sg, k), np.where(beyond, k + sg, k))
    return np.where(near, fixed, k), near


def test_int8_rule_equals_division():
    rng = np.random.default_rng(1)
    hits = 0
    for _ in range(200):
        x = rng.standard_normal(20000).astype(F32) * F32(rng.uniform(0.01, 100.0))
        amax = np.abs(x).max()
        s = F32(max(F32(amax) / F32(127.0), F32(1e-8)))
        ref = np.rint((x / s).astype(F32))
        for inv in invs(s):
            got, near = i8_rule(x, s, inv)
            np.testing.assert_array_equal(got, ref)
            hits += int(near.sum())
    # exact half-way quotients of a power-of-two scale take the exact path
    s = F32(2.0 ** -7)
    x = ((np.arange(-127, 127) + 0.5) * 2.0 ** -7).astype(F32)
    got, near = i8_rule(x, s, F32(1.0) / s)
    assert near.all()
    np.testing.assert_array_equal(got, np.rint(x / s))
    assert hits > 0


@pytest.mark.parametrize("kind", ["bf16", "f16"])
def test_int8_rule_every_16bit_x(kind):
    """Every 16-bit x with |x| <= amax against a sample of 16-bit row maxima
    (s = max(amax / 127, 1e-8)): x = amax / 2 puts x / s within 2^-18 of 63.5,
    the near-half-way case that dominates real rows."""
    pos = sixteen_bit_values(kind)
    rng = np.random.default_rng(3)
    amaxes = np.concatenate([rng.choice(pos[1:], 120, replace=False),
                             np.array([1.0, 2.5, 0.0078125, 3.0e-6], F32)]).astype(F32)
    near_total = 0
    for amax in amaxes:
        xp = pos[pos <= amax]
        x = np.concatenate([xp, -xp]).astype(F32)
        s = F32(max(F32(amax) / F32(127.0), F32(1e-8)))
        ref = np.rint((x / s).astype(F32))
        for inv in invs(s):
            got, near = i8_rule(x, s, inv)
            np.testing.assert_array_equal(got, ref)
            near_total += int(near.sum())
    assert near_total > 0


def e4m3_rule(x, s, inv):
    """r = x * inv, unless r is in the E4M3 subnormal range or its low 20
    mantissa bits are within 4 units of a half-way pattern: then x / s."""
    r = (x * inv).astype(F32)
    m20 = (r.view(np.uint32) & 0xFFFFF).astype(np.int64) - 0x80000
    near = ((r != 0) & (np.abs(r) < 2.0 ** -6)) | ((m20 >= -4) & (m20 <= 4))
    return np.where(near, (x / s).astype(F32), r), near


def test_e4m3_rule_equals_division():
    rng = np.random.default_rng(2)
    x = np.concatenate([rng.standard_normal(3000), rng.standard_normal(300) * 1e-3,
                        [0.0, -0.0]]).astype(F32)
    for s in (F32(0.0123), F32(2.0 ** -6), F32(np.abs(x).max() / 448.0)):
        ref = oracle.f32_to_e4m3((x / s).astype(F32))
        for inv in invs(s):
            got, _ = e4m3_rule(x, s, inv)
            np.testing.assert_array_equal(oracle.f32_to_e4m3(got), ref)
    # E4M3 half-way points in the normal range, and subnormal values
    e = rng.integers(-6, 8, 2000).astype(np.float64)
    m = rng.integers(8, 16, 2000).astype(np.float64)
    v = ((m + 0.5) * 2.0 ** (e - 3)).astype(F32)
    sub = ((rng.integers(0, 16, 200) + 0.5) * 2.0 ** -10).astype(F32)
    s = F32(2.0 ** -6)
    x = (np.concatenate([v, sub]) * s).astype(F32)
    got, near = e4m3_rule(x, s, F32(1.0) / s)
    assert near.all()
    np.testing.assert_array_equal(oracle.f32_to_e4m3(got), oracle.f32_to_e4m3((x / s).astype(F32)))
