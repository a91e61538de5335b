"""Pins for the oracle's number formats (E4M3, bf16) against the OCP OFP8
definition, exhaustive enumeration and ml_dtypes' conversions."""
import math

import ml_dtypes
import numpy as np
import pytest

from conftest import read_table


def test_e4m3_ocp_table(oracle_lib):
    for code, val in read_table("e4m3_ocp.txt"):
        got = oracle_lib.e4m3_value(int(code, 16))
        if val == "nan":
            assert math.isnan(got), code
        else:
            assert got == float(val), (code, got, val)
            assert math.copysign(1.0, got) == math.copysign(1.0, float(val))


def test_e4m3_all_codes_match_library(oracle_lib):
    lib_vals = np.arange(256, dtype=np.uint8).view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    for c in range(256):
        got = oracle_lib.e4m3_value(c)
        if math.isnan(lib_vals[c]):
            assert math.isnan(got)
        else:
            assert got == lib_vals[c], c


def test_e4m3_roundtrip_every_finite_code(oracle_lib):
    for c in range(256):
        v = oracle_lib.e4m3_value(c)
        if math.isnan(v):
            continue
        assert oracle_lib.e4m3_from_f32(v) == c, hex(c)


def test_e4m3_rne_brute_force(oracle_lib):
    """Nearest representable value, ties to the code with even mantissa LSB,
    clamp beyond +-448: checked by exhaustive nearest search on a dense set
    of fp32 probes including every midpoint."""
    lib_codes = np.arange(256, dtype=np.uint8)
    lib_vals = lib_codes.view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    finite = [(v, c) for v, c in zip(lib_vals, lib_codes) if not math.isnan(v) and c < 0x80]
    finite.sort()
    probes = []
    for (a, _), (b, _) in zip(finite[:-1], finite[1:]):
        mid = 0.5 * (a + b)
        probes += [mid, np.nextafter(np.float32(mid), np.float32(0)), np.nextafter(np.float32(mid), np.float32(1e9)),
                   a + 0.25 * (b - a), a + 0.75 * (b - a)]
    probes += [449.0, 463.9, 464.0, 500.0, 1e6, 1e-12, 2.0 ** -10, 3 * 2.0 ** -11]
    for p in probes:
        p32 = float(np.float32(p))
        dist = [abs(v - p32) for v, _ in finite]
        cands = [c for (v, c), d in zip(finite, dist) if d == min(dist)]
        if len(cands) == 2:          # exact midpoint: the even mantissa wins
            cands = [c for c in cands if (c & 1) == 0]
        want = cands[0] if p32 < 448.0 else 0x7E
        assert oracle_lib.e4m3_from_f32(p32) == want, (p32, hex(want))
        assert oracle_lib.e4m3_from_f32(-p32) == (want | 0x80 if want else 0x80), p32


def test_e4m3_matches_library_cast_on_random_values(oracle_lib):
    rng = np.random.default_rng(1)
    x = np.concatenate([rng.standard_normal(3000) * 100, rng.standard_normal(3000) * 0.01]).astype(np.float32)
    x = np.clip(x, -448, 448)
    want = x.astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    for v, w in zip(x, want):
        assert oracle_lib.e4m3_from_f32(v) == w, v


def test_bf16_exhaustive_roundtrip(oracle_lib):
    pats = np.arange(65536, dtype=np.uint32)
    f = (pats << np.uint32(16)).view(np.float32)
    for h in range(0, 65536, 7):
        v = oracle_lib.bf16_value(h)
        if math.isnan(f[h]):
            assert math.isnan(v)
            continue
        assert v == float(f[h])
        assert oracle_lib.bf16_from_f32(v) == h


def test_bf16_rne_against_library(oracle_lib):
    rng = np.random.default_rng(2)
    x = rng.standard_normal(5000).astype(np.float32)
    # exact ties: low 16 bits == 0x8000
    ties = ((rng.integers(0, 2 ** 15, 500).astype(np.uint32) << 16) | 0x8000).view(np.float32)
    x = np.concatenate([x, ties[np.isfinite(ties)]])
    want = x.astype(ml_dtypes.bfloat16).view(np.uint16)
    for v, w in zip(x, want):
        assert oracle_lib.bf16_from_f32(v) == w, v
