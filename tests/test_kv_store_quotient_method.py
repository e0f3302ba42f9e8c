"""The KV-store kernel divides by the per-token scale with one correction of the reciprocal
product (Markstein 1990): y0 = RN(x * r), r = RN(1 / s), y = RN(y0 + (x - y0 * s) * r), both steps
single-rounding fmas, the remainder formed as -(y0 * s - x).  This CPU test checks that method in
exact arithmetic (float64 with error-free transformations, ties decided exactly) on the quantiser's
domain: bf16 x, s = RN(amax / 448) >= 2^-90, |x| <= amax.  It pins the kernel's method, not the
oracle (which divides directly).
"""
import numpy as np
import torch


def _bf16(v):
    u = np.asarray(v, dtype=np.float32).view(np.uint32).astype(np.uint64)
    return (((u + 0x7FFF + ((u >> 16) & 1)) >> 16) << 16).astype(np.uint32).view(np.float32)


def _rn32_sum(a, b):
    """RN32(a + b) of float64 a, b exactly (TwoSum; the error term decides at float32 midpoints)."""
    s = a + b
    bb = s - a
    e = (a - (s - bb)) + (b - bb)
    f = s.astype(np.float32)
    f64 = f.astype(np.float64)
    lo = np.nextafter(f, np.float32(-np.inf)).astype(np.float64)
    hi = np.nextafter(f, np.float32(np.inf)).astype(np.float64)
    f = np.where((s == (f64 + hi) / 2) & (e > 0), hi.astype(np.float32), f)
    f = np.where((s == (f64 + lo) / 2) & (e < 0), lo.astype(np.float32), f)
    return f


def _rn32_div(x, s):
    """Correctly rounded float32 x / s (near a float32 midpoint, decided by the exact sign of x - m s)."""
    q = x / s
    f = q.astype(np.float32)
    for nb in (np.nextafter(f, np.float32(-np.inf)), np.nextafter(f, np.float32(np.inf))):
        m = (f.astype(np.float64) + nb.astype(np.float64)) / 2
        near = np.abs(q - m) <= np.abs(m) * 2.0 ** -50
        side = np.sign(x - m * s) * np.sign(s)                  # m * s exact (25 x 24 bits)
        nb_up = nb.astype(np.float64) > f.astype(np.float64)
        pick = np.where(nb_up, side > 0, side < 0) | ((side == 0) & ((f.view(np.uint32) & 1) == 1))
        f = np.where(near & pick, nb, f)
    return f


def _method(x, s):
    r = _rn32_div(np.ones_like(s), s).astype(np.float64)
    y0 = (x * r).astype(np.float32).astype(np.float64)          # x * r exact in float64 (8 x 24 bits)
    t = (y0 * s - x).astype(np.float32).astype(np.float64)      # exact difference, one rounding
    return _rn32_sum(y0, -t * r)                                 # -t * r exact (48 bits)


def _codes(y):
    y = np.clip(y.astype(np.float32), -448, 448)
    return torch.from_numpy(y).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def _draw(rng, n, e_lo):
    amax = _bf16(np.ldexp(1 + rng.random(n), rng.integers(e_lo, 127, n)))
    s = (amax / np.float32(448)).astype(np.float32)
    x = _bf16(amax * np.ldexp(1 + rng.random(n), -rng.integers(1, 60, n)).astype(np.float32))
    x = np.where(rng.random(n) < 0.1, amax, x)
    x = np.where(rng.random(n) < 0.02, np.float32(0), x)
    x = np.where(rng.random(n) < 0.5, -x, x).astype(np.float32)
    return x.astype(np.float64), s.astype(np.float64)


def test_quotient_bit_exact_for_normal_inputs():
    rng = np.random.default_rng(2024)
    x, s = _draw(rng, 1_000_000, -80)
    keep = (np.abs(x) >= 2.0 ** -100) & (s >= 2.0 ** -90)
    y = _method(x[keep], s[keep])
    want = _rn32_div(x[keep], s[keep])
    assert keep.sum() > 500_000
    assert np.array_equal(y.view(np.uint32), want.view(np.uint32))


def test_codes_equal_for_every_scale_above_the_switch():
    rng = np.random.default_rng(7)
    x, s = _draw(rng, 1_000_000, -80)
    keep = s >= 2.0 ** -90
    y = _method(x[keep], s[keep])
    assert np.array_equal(_codes(y), _codes(_rn32_div(x[keep], s[keep])))
    # negative zero keeps its sign (code 0x80)
    z = _method(np.array([-0.0, 0.0]), np.array([0.5, 0.5]))
    assert np.signbit(z[0]) and not np.signbit(z[1])


def test_a_planted_plain_reciprocal_product_is_caught():
    """Without the correction the codes differ somewhere on the same sample."""
    rng = np.random.default_rng(7)
    x, s = _draw(rng, 1_000_000, -80)
    keep = s >= 2.0 ** -90
    r = _rn32_div(np.ones_like(s[keep]), s[keep]).astype(np.float64)
    plain = (x[keep] * r).astype(np.float32)
    assert not np.array_equal(_codes(plain), _codes(_rn32_div(x[keep], s[keep])))
