"""Pins of the oracle's E4M3 index-key storage (haiqwa "DeepSeek-V4"
§FP4精度加速: the indexer's key/query path runs in low precision; the format
and scale are this library's reading: one power-of-two scale per entry, the
smallest 2^e, -126 <= e <= 127, with 448 * 2^e >= max |key dim|, codes
E4M3(key / scale) rounded to nearest even).

Pinned against: the closed form of the scale at and just past every
power-of-two boundary; a second transcription (oracle/twin.py: frexp for the
scale, ml_dtypes for the codes); exact round trips of keys that are E4M3
values times a power of two; the decoded keys of a cache view."""
import ml_dtypes
import numpy as np
import pytest

import oracle
from oracle import twin

E4M3 = np.arange(256, dtype=np.uint8).view(ml_dtypes.float8_e4m3fn).astype(np.float64)


# 448 * 2^j is an fp32 value for -126 <= j <= 119 (the keys are fp32)
@pytest.mark.parametrize("j", list(range(-126, 120, 7)) + [119])
def test_scale_closed_form_at_power_of_two_boundaries(j):
    a = 448.0 * 2.0 ** j
    assert float(np.float32(a)) == a
    assert oracle.key_scale_e4m3(a) == 2.0 ** j
    above = float(np.nextafter(np.float32(a), np.float32(np.inf)))
    assert oracle.key_scale_e4m3(above) == 2.0 ** (j + 1)
    if j > -126:
        below = float(np.nextafter(np.float32(a), np.float32(0)))
        assert oracle.key_scale_e4m3(below) == 2.0 ** j


def test_scale_of_zero_and_extremes():
    assert oracle.key_scale_e4m3(0.0) == 2.0 ** -126
    assert oracle.key_scale_e4m3(1e-45) == 2.0 ** -126
    # the largest fp32 value needs 2^120 (448 * 2^119 < 3.4e38 <= 448 * 2^120)
    assert oracle.key_scale_e4m3(float(np.finfo(np.float32).max)) == 2.0 ** 120


def _keys(rng, m, dI, mag):
    xs = rng.standard_normal((m, dI)) * mag
    w = rng.standard_normal(dI) / np.sqrt(dI)
    b = rng.standard_normal(m)
    return xs, w, b


@pytest.mark.parametrize("mag", [1e-30, 1e-3, 1.0, 37.0, 1e5])
def test_codes_and_scale_match_the_twin(mag):
    rng = np.random.default_rng(11)
    for _ in range(20):
        xs, w, b = _keys(rng, 4, 128, mag)
        codes, s = oracle.index_key_e4m3(xs, w, b)
        tc, ts = twin.index_key_e4m3(xs, w, b)
        assert s == ts
        assert np.array_equal(codes, tc)
        # the largest dim lands in the top binade of E4M3: its value / scale
        # is in (224, 448], rounded to 224 .. 448 (unless the scale is clamped)
        vals = E4M3[codes]
        assert np.max(np.abs(vals)) <= 448.0
        if s > 2.0 ** -126:
            assert np.max(np.abs(vals)) >= 224.0


def test_exact_round_trip_of_representable_keys():
    """A block whose pooled key is an E4M3 value times 2^j in every dim
    (one token, zero gate) is stored losslessly."""
    rng = np.random.default_rng(3)
    finite = np.nonzero(np.isfinite(E4M3))[0]
    for j in (-20, -5, 0, 7):
        codes_in = rng.choice(finite, size=128)
        codes_in[0] = 0x7E   # 448: the largest magnitude, so the scale is exactly 2^j
        key = E4M3[codes_in] * 2.0 ** j
        codes, s = oracle.index_key_e4m3(key[None, :], np.zeros(128), np.zeros(1))
        assert s == 2.0 ** j
        assert np.array_equal(E4M3[codes] * s, key)


def test_cache_view_decodes_codes_times_scale():
    rng = np.random.default_rng(5)
    n_pages, epp, dI = 3, 32, 64
    codes = rng.integers(0, 0x7F, size=(n_pages, epp, dI)).astype(np.uint8)
    codes |= (rng.integers(0, 2, size=codes.shape) << 7).astype(np.uint8)
    kscale = (2.0 ** rng.integers(-20, 5, size=(n_pages, epp))).astype(np.float32)
    bt = np.array([[2, 0, 1]], np.int32)
    cv = oracle.CacheView(4, 128, np.zeros((n_pages, epp, 192), np.uint8), np.ones((n_pages, epp), np.float32),
                          bt, np.zeros((1, 128, 192), np.uint8), np.ones((1, 128), np.float32), codes, dI,
                          kscale=kscale)
    keys = cv.gather_keys(0, 96)
    for e in range(96):
        pg = bt[0, e // epp]
        want = codes[pg, e % epp].view(ml_dtypes.float8_e4m3fn).astype(np.float64) * float(kscale[pg, e % epp])
        assert np.array_equal(keys[e], want)
