"""Pins for the oracle's KV-store step (quantise new tokens to e4m3 and scatter them into pages).

The encoder is tied to the format itself (every finite code round-trips, brute-force nearest code
with ties to the even mantissa), to two library casts (ml_dtypes and torch float8_e4m3fn) and to
saturation cases; the per-token quantiser to closed forms (an all-zero row, the row maximum maps
to +-448) and an error bound; the scatter to a brute-force contiguous layout.  The last tests plant
plausible mistakes and check that a pin catches each.
"""
import ml_dtypes
import numpy as np
import pytest
import torch

from oracle import mla_oracle as O

FINITE = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)


def _torch_e4m3(y):
    return torch.from_numpy(np.asarray(y, dtype=np.float32).copy()).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def _brute_nearest(y):
    """Nearest finite e4m3 code to each y (|y| <= 448) by scanning all codes; ties to even mantissa."""
    vals = O.e4m3_decode(FINITE)
    out = np.empty(len(y), dtype=np.uint8)
    for k, v in enumerate(np.asarray(y, dtype=np.float64)):
        d = np.abs(vals - v)
        best = np.flatnonzero(d == d.min())
        cand = FINITE[best]
        if len(cand) > 1:                                   # a tie: keep the even mantissa
            cand = cand[(cand & 1) == 0]
            if len(cand) > 1:                               # +0 / -0: keep the sign of y
                cand = cand[((cand >> 7) & 1) == (1 if np.signbit(v) else 0)]
        out[k] = cand[0]
    return out


# --------------------------------------------------------------------------- encoder
def test_every_finite_code_round_trips():
    v = O.e4m3_decode(FINITE).astype(np.float32)
    assert np.array_equal(O.e4m3_encode_rn_sat(v), FINITE)


def test_encoder_matches_library_casts_on_random_and_ties():
    rng = np.random.default_rng(11)
    y = rng.standard_normal(300_000) * rng.choice([1e-5, 1e-3, 0.1, 1.0, 17.0, 300.0], 300_000)
    vals = np.sort(np.unique(O.e4m3_decode(FINITE)))
    mids = (vals[1:] + vals[:-1]) / 2                       # exact ties (representable in fp32)
    y = np.concatenate([y, mids, np.nextafter(mids.astype(np.float32), np.float32(np.inf)),
                        np.nextafter(mids.astype(np.float32), np.float32(-np.inf))])
    y = np.clip(y, -448, 448).astype(np.float32)
    ours = O.e4m3_encode_rn_sat(y)
    assert np.array_equal(ours, _torch_e4m3(y))
    ml = y.astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    assert np.array_equal(ours, ml)


def test_encoder_matches_brute_force_nearest():
    rng = np.random.default_rng(12)
    y = (rng.standard_normal(3000) * rng.choice([1e-3, 0.05, 2.0, 100.0], 3000)).astype(np.float32)
    y = np.clip(y, -448, 448).astype(np.float32)
    vals = np.sort(np.unique(O.e4m3_decode(FINITE)))
    y = np.concatenate([y, ((vals[1:] + vals[:-1]) / 2)[::7].astype(np.float32)])
    assert np.array_equal(O.e4m3_encode_rn_sat(y), _brute_nearest(y))


def test_encoder_saturates():
    y = np.array([448.0, 449.0, 464.0, 1e6, -448.0, -470.0, -3e38], dtype=np.float32)
    assert list(O.e4m3_encode_rn_sat(y)) == [0x7E, 0x7E, 0x7E, 0x7E, 0xFE, 0xFE, 0xFE]


# --------------------------------------------------------------------------- per-token quantiser
def _bf16_bits(x):
    return torch.from_numpy(np.asarray(x, dtype=np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def test_zero_row_has_unit_scale_and_zero_codes():
    codes, s = O.quantize_token(np.zeros(576, dtype=np.uint16))
    assert s == np.float32(1.0) and not codes.any()


def test_row_maximum_maps_to_448_and_error_is_bounded():
    rng = np.random.default_rng(13)
    for trial in range(50):
        x = rng.standard_normal(576) * (10.0 ** rng.uniform(-3, 3))
        bits = _bf16_bits(x)
        xv = O.bf16_bits_to_f64(bits)
        codes, s = O.quantize_token(bits)
        assert s == np.float32(np.float32(np.max(np.abs(xv))) / np.float32(448))
        k = int(np.argmax(np.abs(xv)))
        assert codes[k] & 0x7F == 0x7E
        back = O.e4m3_decode(codes) * np.float64(s)
        # half a step of the format: 2^-4 relative in the normal range, 2^-10 * s below it
        assert np.all(np.abs(back - xv) <= np.abs(xv) * 2.0 ** -4 + 2.0 ** -10 * np.float64(s) * 1.0000001)


def _discriminating_rows():
    """40 random rows plus seeded rows on which x / f32(amax/448) and x * f32(448/amax) round to
    different e4m3 codes (found by a vectorised search; ~1 row in 200 has such an element)."""
    rng = np.random.default_rng(16)
    x = torch.from_numpy(rng.standard_normal((4000, 576)) * 3.0).to(torch.bfloat16)
    xf = x.float().numpy()
    amax = np.abs(xf).max(1).astype(np.float32)
    s = (amax / np.float32(448)).astype(np.float32)
    inv = (np.float32(448) / amax).astype(np.float32)
    differ = (_torch_e4m3((xf / s[:, None]).clip(-448, 448)) != _torch_e4m3((xf * inv[:, None]).clip(-448, 448))).any(1)
    rows = np.flatnonzero(differ)[:8]
    assert len(rows) >= 4
    return torch.cat([x[:40], x[torch.from_numpy(rows)]])


def test_quantiser_matches_torch_quantiser():
    """Same definition written with torch ops (fp32 division, clamp, library cast)."""
    x = _discriminating_rows()
    xf = x.float()
    amax = xf.abs().amax(-1)
    s = amax / 448.0
    ref = (xf / s[:, None]).clamp(-448, 448).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    for r in range(x.shape[0]):
        codes, sc = O.quantize_token(x[r].view(torch.int16).numpy().view(np.uint16))
        assert sc == s[r].item()
        assert np.array_equal(codes, ref[r])


# --------------------------------------------------------------------------- scatter
@pytest.mark.parametrize("P,separate", [(16, False), (48, True), (64, False)])
def test_store_lands_at_logical_positions(P, separate):
    rng = np.random.default_rng(15)
    B, T, NL, layer = 3, 5, 2, 1
    L = np.array([0, P - 2, 3 * P + 7])
    pages = (L + T + P - 1) // P
    maxp = int(pages.max())
    NB = int(pages.sum()) + 4
    perm = rng.permutation(NB)
    lut = np.full((B, maxp), 0xFFFFFFFF, dtype=np.uint32)
    k = 0
    for b in range(B):
        for pg in range(pages[b]):
            lut[b, pg] = perm[k]
            k += 1
    slut = None
    NSB = NB
    if separate:
        NSB = NB + 3
        slut = np.full_like(lut, 0xFFFFFFFF)
        sperm = rng.permutation(NSB)
        k = 0
        for b in range(B):
            for pg in range(pages[b]):
                slut[b, pg] = sperm[k]
                k += 1
    blocks = np.full((NB, 1, NL, P, 1, 576), 0x7F, dtype=np.uint8)    # NaN codes everywhere
    scales = np.full((NSB, 1, NL, P, 1, 1), np.nan, dtype=np.float32)
    lat = _bf16_bits(rng.standard_normal((B, T, 576)) * 2.0)
    nb, ns = O.kv_store(lat, L, lut, slut, layer, blocks, scales)
    written = 0
    for b in range(B):
        codes, sc = O.gather_request(nb, ns, lut, slut, b, int(L[b]) + T, layer)
        for i in range(T):
            c, s = O.quantize_token(lat[b, i])
            assert np.array_equal(codes[L[b] + i], c) and sc[L[b] + i, 0] == s
            written += 1
    # nothing else changed
    changed = (nb != blocks).any(axis=-1).sum()
    assert changed <= written and np.isnan(ns).sum() == np.isnan(scales).sum() - written


# --------------------------------------------------------------------------- planted mistakes
def _encode_round_half_away(y):
    y = np.asarray(y, dtype=np.float32).astype(np.float64)
    a = np.minimum(np.abs(y), 448.0)
    out = []
    vals = O.e4m3_decode(FINITE)
    for v, s in zip(a, np.signbit(y)):
        d = np.abs(vals - (-v if s else v))
        best = FINITE[np.flatnonzero(d == d.min())]
        out.append(max(best, key=lambda c: abs(O.e4m3_decode(np.uint8(c)))))
    return np.array(out, dtype=np.uint8)


def test_planted_round_half_away_is_caught(monkeypatch):
    monkeypatch.setattr(O, "e4m3_encode_rn_sat", _encode_round_half_away)
    with pytest.raises(AssertionError):
        test_encoder_matches_library_casts_on_random_and_ties()


def test_planted_missing_saturation_is_caught(monkeypatch):
    real = O.e4m3_encode_rn_sat

    def no_sat(y):
        y = np.asarray(y, dtype=np.float32)
        out = real(y)
        return np.where(np.abs(y) > 448, np.uint8(0x7F) | (out & 0x80), out).astype(np.uint8)

    monkeypatch.setattr(O, "e4m3_encode_rn_sat", no_sat)
    with pytest.raises(AssertionError):
        test_encoder_saturates()


def test_planted_reciprocal_scale_is_caught(monkeypatch):
    """Quantising with x * f32(448 / amax) instead of x / f32(amax / 448) differs in rare ties."""
    def quant_recip(x_bits):
        x = O.bf16_bits_to_f64(x_bits).astype(np.float32)
        amax = np.float32(np.max(np.abs(x)))
        inv = np.float32(np.float32(448.0) / amax) if amax > 0 else np.float32(1.0)
        s = np.float32(amax / np.float32(448.0)) if amax > 0 else np.float32(1.0)
        return O.e4m3_encode_rn_sat((x * inv).astype(np.float32)), s

    monkeypatch.setattr(O, "quantize_token", quant_recip)
    with pytest.raises(AssertionError):
        test_quantiser_matches_torch_quantiser()
